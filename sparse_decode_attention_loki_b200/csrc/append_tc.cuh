// Bulk rotate-and-append on the 5th-generation tensor cores (sm_100a).
//
// A prompt appended in one call is a contraction per KV head g:
//   K_hat[n, :] = K_new[n, :] . P_g        (n = the B*n_new new vectors)
// ("PCA-project ... keys", "Loki: Low-rank Keys for Efficient Sparse
// Attention", atlas.scime.ai summary, section "Approach"), i.e. a GEMM of
// [n x D] by [D x D].  Here it runs on tcgen05.mma: tiles of M = 128 vectors,
// N = D output columns, the fp32 accumulator in tensor memory (TMEM).
//
// Precision.  The cache keys are bf16 (exact in the bf16 operand); P is fp32,
// so it is split into three bf16 terms P = P0 + P1 + P2 (each the bf16
// rounding of what the previous terms leave), whose sum equals P to about
// 2^-24 relative.  The 3 * D products per output are accumulated in fp32 by
// the tensor core and the result is rounded once to bf16 (round to nearest
// even).
//
// The grid is persistent: one CTA per SM, each taking a contiguous range of
// the (head, tile) units, so that every SM has the same number of tiles.  A
// CTA splits P_g into shared memory when its range enters head g.  Per tile
// j one thread issues the 3 * D/16 MMAs (K = 16 each) into one of two TMEM
// accumulators and commits them to that accumulator's mbarrier; meanwhile
// all sixteen warps read back tile j-1's accumulator (tcgen05.ld; warp w:
// TMEM lanes 32*(w%4) .., columns of quarter w/4), round it into tile j-1's
// key stage (free once its MMAs are done) and store it from there row by
// row, coalesced, and copy tile j's values.  Key tiles are staged three deep (cp.async), so two tiles
// of keys are in flight while one is being multiplied.
//
// Shared-memory operand layout (no swizzle, "K-major"): 8x16-byte core
// matrices, row r of an operand and its 16-byte K chunk c at byte
//   (r % 8) * 16 + (r / 8) * 128 + c * (rows / 8) * 128,
// i.e. stride between 8-row groups SBO = 128 B and between K chunks
// LBO = rows * 16 B.
//
// Every wait on the mbarrier is bounded: on a timeout the CTA counts an error
// in g_loki_device_errors, releases its TMEM and returns.
#pragma once

#include "append.cuh"
#include "errors.cuh"

namespace loki {

constexpr int kTcM = 128;            // vectors per tile (the MMA's M)
constexpr int kTcTerms = 3;          // bf16 terms of P
constexpr int kTcMinVectors = 256;   // below this many vectors per head the CUDA-core kernel is used
constexpr uint32_t kTcWaitLimit = 1u << 20;

constexpr int kTcStages = 3;         // key tiles staged in shared memory

template <int D>
struct TcLayout {
  static constexpr int kA = kTcM * D * 2;  // bytes of one key tile
  static constexpr int kB = D * D * 2;     // bytes of one bf16 term of P
  static constexpr int kBoff = kTcStages * kA;
  static constexpr int kBar = kBoff + kTcTerms * kB;  // two mbarriers, then the TMEM address
  static constexpr int kBytes = kBar + 64;
  static constexpr uint32_t kTmemCols = 2 * D;  // two accumulators of D fp32 columns
};

// Byte offset of (row r, 16-byte K chunk c) in an operand of `rows` rows.
__host__ __device__ constexpr int tc_off(int r, int c, int rows) { return (r & 7) * 16 + (r >> 3) * 128 + c * rows * 16; }

// tcgen05 shared-memory matrix descriptor: no swizzle, K-major, the layout of
// tc_off (LBO = K-chunk stride, SBO = 8-row-group stride), Blackwell version 1.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)((lbo >> 4) & 0x3fffu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3fffu) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, both
// operands K-major, M = 128, N = D.
template <int D>
__host__ __device__ constexpr uint32_t tc_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kTcM >> 4) << 24);
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < kTcWaitLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

constexpr int kTcThreads = 512;  // 16 warps: four per TMEM lane quarter

// P_g as three bf16 terms into the B operand (row j = output column, K = i).
// Thread unit (j, 8-wide K chunk c): eight loads down column j of P, one
// 16-byte store per term; a warp's stores cover 32 consecutive rows of one
// chunk, 512 contiguous bytes.
template <int D>
__device__ __forceinline__ void split_basis(const float *__restrict__ Pg, unsigned char *Bs) {
  using Lay = TcLayout<D>;
  constexpr int U = D * D / 8 / kTcThreads;  // units per thread
  static_assert((D * D / 8) % kTcThreads == 0, "P is split in whole units per thread");
  float pv[U][8];
#pragma unroll
  for (int x = 0; x < U; ++x) {
    const int e = x * kTcThreads + threadIdx.x, j = e % D, c = e / D;
#pragma unroll
    for (int y = 0; y < 8; ++y) pv[x][y] = __ldg(Pg + (size_t)(c * 8 + y) * D + j);
  }
#pragma unroll
  for (int x = 0; x < U; ++x) {
    const int e = x * kTcThreads + threadIdx.x, j = e % D, c = e / D;
    uint32_t w[kTcTerms][4];
#pragma unroll
    for (int y = 0; y < 8; y += 2) {
      float r0 = pv[x][y], r1 = pv[x][y + 1];
#pragma unroll
      for (int term = 0; term < kTcTerms; ++term) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(r0, r1);
        w[term][y / 2] = *reinterpret_cast<const uint32_t *>(&h);
        r0 -= __low2float(h);
        r1 -= __high2float(h);
      }
    }
#pragma unroll
    for (int term = 0; term < kTcTerms; ++term)
      *reinterpret_cast<uint4 *>(Bs + term * Lay::kB + tc_off(j, c, D)) =
          make_uint4(w[term][0], w[term][1], w[term][2], w[term][3]);
  }
  fence_async_smem();
}

// Batch and position of row r of the tile whose first row (b0, t0): rows of
// a tile are consecutive vectors f = b * n_new + t.
__device__ __forceinline__ void tile_row(int n_new, int b0, int t0, int r, int &b, int &t) {
  t = t0 + r;
  b = b0;
  if (t >= n_new) {
    if (n_new >= kTcM) {  // at most one wrap in a tile
      t -= n_new;
      ++b;
    } else {
      b += t / n_new;
      t %= n_new;
    }
  }
}

template <int D, bool PAGED>
__global__ void __launch_bounds__(kTcThreads, 1) append_tc_kernel(const __grid_constant__ AppendArgs<__nv_bfloat16> a) {
  using Lay = TcLayout<D>;
  constexpr int CH = D / 8;                 // 16-byte chunks per vector
  constexpr int RS = kTcThreads / CH;       // rows per pass of all threads
  constexpr int NV = kTcM / RS;             // rows (one chunk each) per thread per tile
  constexpr int QC = D / 4;                 // accumulator columns per warp in the epilogue
  static_assert(kTcM % RS == 0 && QC % 16 == 0, "tile shape");
  extern __shared__ __align__(1024) unsigned char tsm[];
  unsigned char *As = tsm;  // kTcStages key tiles
  unsigned char *Bs = tsm + Lay::kBoff;
  uint64_t *bar = reinterpret_cast<uint64_t *>(tsm + Lay::kBar);  // bar[0], bar[1]: one per accumulator
  uint32_t *tslot = reinterpret_cast<uint32_t *>(tsm + Lay::kBar + 16);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tiles = (a.n_vec + kTcM - 1) / kTcM;
  const long long units = (long long)a.n_kv_heads * tiles;
  const int lo = (int)((long long)blockIdx.x * units / gridDim.x);
  const int hi = (int)((long long)(blockIdx.x + 1) * units / gridDim.x);
  const int n = hi - lo;
  if (n <= 0) return;  // uniform: nothing allocated yet
  const int crow = tid / CH, cch = tid % CH;  // copy role: rows crow + RS*x, chunk cch

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                 "r"(Lay::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar + 1)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  // offsets (in elements) of vector (b, t) of head g in the new-vector
  // arrays and in the cache
  auto src_off = [&](int g, int b, int t) { return (((size_t)b * a.n_kv_heads + g) * a.n_new + t) * D; };
  auto dst_off = [&](int g, int b, int t) { return append_dst<__nv_bfloat16, D, PAGED>(a, b, g, t); };

  // keys of unit u into stage `st` (rows past n_vec are zero); always one
  // commit group, empty when u is past the range
  auto load_keys = [&](int u, int st) {
    if (u < hi) {
      const int g = u / tiles, f0 = (u - g * tiles) * kTcM;
      const int b0 = f0 / a.n_new, t0 = f0 - b0 * a.n_new;
      unsigned char *dstA = As + st * Lay::kA;
#pragma unroll
      for (int x = 0; x < NV; ++x) {
        const int r = crow + RS * x;
        const bool valid = f0 + r < a.n_vec;
        int b, t;
        tile_row(a.n_new, b0, t0, r, b, t);
        const __nv_bfloat16 *src = valid ? a.k_new + src_off(g, b, t) + cch * 8 : a.k_new;
        cp_async16_zfill(dstA + tc_off(r, cch, kTcM), src, valid);
      }
    }
    cp_async_commit();
  };

  int g_cur = lo / tiles;
  split_basis<D>(a.P + (size_t)g_cur * D * D, Bs);
  load_keys(lo, 0);
  load_keys(lo + 1, 1);
  __syncthreads();
  const uint32_t tbase = *tslot;
  const uint32_t a_base = smem_u32(As), b_base = smem_u32(Bs), bar0 = smem_u32(bar);
  constexpr uint32_t idesc = tc_idesc<D>();
  bool failed = false;

  // the accumulator of local tile j: wait for its MMAs, round, store.  Warp
  // w reads TMEM lanes 32*(w%4) .. (tile rows) and columns [QC*(w/4), +QC).
  auto epilogue = [&](int j) -> bool {
    const bool ok = mbar_wait_bounded(bar0 + 8u * (uint32_t)(j & 1), (uint32_t)((j >> 1) & 1));
    if (__syncthreads_or(!ok)) return false;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const int u = lo + j, g = u / tiles, f0 = (u - g * tiles) * kTcM;
    // the accumulator, rounded, into tile j's key stage (its MMAs are done),
    // rows of D*2 bytes with 16-byte chunk c of row r at chunk c ^ (r % CH):
    // a warp's 32 rows then spread over all banks
    unsigned char *stg = As + (j % kTcStages) * Lay::kA;
    {
      const int r = 32 * (warp & 3) + lane;
      const int col0 = QC * (warp >> 2);
      const uint32_t tacc = tbase + (uint32_t)((j & 1) * D) + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)col0;
#pragma unroll
      for (int cb = 0; cb < QC / 16; ++cb) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(tacc + (uint32_t)(16 * cb)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          uint32_t w4[4];
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const __nv_bfloat162 h =
                __floats2bfloat162_rn(__uint_as_float(v[8 * x + 2 * y]), __uint_as_float(v[8 * x + 2 * y + 1]));
            w4[y] = *reinterpret_cast<const uint32_t *>(&h);
          }
          const int c = (col0 + 16 * cb) / 8 + x;
          *reinterpret_cast<uint4 *>(stg + r * (D * 2) + ((c ^ (r & (CH - 1))) * 16)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    // out to the cache, two whole rows per warp instruction
    const int b0 = f0 / a.n_new, t0 = f0 - b0 * a.n_new;
#pragma unroll
    for (int x = 0; x < NV; ++x) {
      const int r = crow + RS * x;
      if (f0 + r < a.n_vec) {
        int b, t;
        tile_row(a.n_new, b0, t0, r, b, t);
        const long long off = dst_off(g, b, t);
        const uint4 w = *reinterpret_cast<const uint4 *>(stg + r * (D * 2) + ((cch ^ (r & (CH - 1))) * 16));
        if (off >= 0) {
          reinterpret_cast<uint4 *>(a.k_hat + off)[cch] = w;
          // the low-rank plane (d_lr a multiple of 8: whole 16-byte chunks)
          if (a.k_lr != nullptr && cch * 8 < a.d_lr)
            reinterpret_cast<uint4 *>(a.k_lr + append_lr_dst<__nv_bfloat16, D>(a, off))[cch] = w;
        }
      }
    }
    __syncthreads();  // the stage is read before it is refilled
    return true;
  };

  bool pending = false;  // tile j-1's accumulator not yet stored
  for (int j = 0; j < n; ++j) {
    const int u = lo + j, g = u / tiles, f0 = (u - g * tiles) * kTcM;
    const int b0 = f0 / a.n_new, t0 = f0 - b0 * a.n_new;
    if (g != g_cur) {
      // the range enters the next head: drain, then split its basis
      if (pending && !epilogue(j - 1)) {
        failed = true;
        break;
      }
      pending = false;
      __syncthreads();
      g_cur = g;
      split_basis<D>(a.P + (size_t)g * D * D, Bs);
    }
    // this tile's values: loads now, stores after the epilogue
    uint4 vv[NV];
#pragma unroll
    for (int x = 0; x < NV; ++x) {
      const int r = crow + RS * x;
      vv[x] = make_uint4(0u, 0u, 0u, 0u);
      if (f0 + r < a.n_vec) {
        int b, t;
        tile_row(a.n_new, b0, t0, r, b, t);
        vv[x] = __ldg(reinterpret_cast<const uint4 *>(a.v_new + src_off(g, b, t)) + cch);
      }
    }
    cp_async_wait<1>();
    fence_async_smem();
    __syncthreads();  // key tile j is in shared memory (and the basis, after a split)

    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a_tile = a_base + (uint32_t)((j % kTcStages) * Lay::kA);
      const uint32_t tacc = tbase + (uint32_t)((j & 1) * D);
#pragma unroll 1
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t ad = tc_desc(a_tile + (uint32_t)(2 * ks * kTcM * 16), kTcM * 16, 128);
#pragma unroll
        for (int term = 0; term < kTcTerms; ++term) {
          const uint64_t bd = tc_desc(b_base + (uint32_t)(term * Lay::kB + 2 * ks * D * 16), D * 16, 128);
          const uint32_t acc = (ks | term) != 0 ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
              ::"r"(tacc), "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
              : "memory");
        }
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       bar0 + 8u * (uint32_t)(j & 1))
                   : "memory");
    }
    // tile j-1's MMAs done: its accumulator is stored and its key stage is free
    if (pending && !epilogue(j - 1)) {
      failed = true;
      break;
    }
    load_keys(u + 2, (j + 2) % kTcStages);
#pragma unroll
    for (int x = 0; x < NV; ++x) {
      const int r = crow + RS * x;
      if (f0 + r < a.n_vec) {
        int b, t;
        tile_row(a.n_new, b0, t0, r, b, t);
        const long long off = dst_off(g, b, t);
        if (off >= 0) reinterpret_cast<uint4 *>(a.v + off)[cch] = vv[x];
      }
    }
    pending = true;
  }
  if (!failed && pending && !epilogue(n - 1)) failed = true;
  cp_async_wait<0>();  // prefetches left in flight (past the range, or by an early exit)

  if (failed && tid == 0) atomicAdd(&g_loki_device_errors, 1u);
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(Lay::kTmemCols)
                 : "memory");
}

}  // namespace loki
