// The Loki decode step for short rows ("Loki: Low-rank Keys for Efficient
// Sparse Attention", atlas.scime.ai summary, section "Approach": rank the
// tokens on the top-d principal dimensions of the keys, attend exactly to the
// top-k), for rows of at most kShortMaxTokens tokens, whose keys all fit in
// every CTA's shared memory.
// One thread-block cluster of ncta CTAs per (batch, KV head) row; CTA r owns
// tokens [r*chunk, (r+1)*chunk):
//
//   1. q_hat and u (in the kernel for query groups of up to 4 heads, from the
//      rotate grid for 8) while the first stages of its low-rank key stream
//      are in flight; then one order-preserving uint32 key per token into
//      its own shared memory (an appended token is stored and scored by the
//      CTA that owns its position);
//   2. each CTA pushes its keys into every other CTA's shared memory, then
//      one cluster barrier: every CTA holds the whole row's keys and runs the
//      same exact radix select on them (11/11/10-bit digits, ties at the
//      threshold to the lower index), so that no CTA waits for another's
//      result;
//   3. each CTA writes its even share [r*k/ncta, (r+1)*k/ncta) of the
//      ascending list of selected indices and gathers those K_hat and V rows
//      for the exact attention (online softmax per query head);
//   4. each CTA pushes its (max, sum, acc) state into the owners' receive
//      buffers; after the second and last cluster barrier every owner merges
//      its output elements from its own shared memory.
//
// Against loki_decode_kernel this spends a few microseconds of redundant
// select work per CTA on rows of a few thousand tokens, and saves the
// histogram reduction, the leader's select with its two barriers and the
// distribution of the list: the chain of dependent steps of a short row.
#pragma once

#include "loki_step.cuh"

namespace loki {

#ifndef LOKI_SHORT_MAX_TOKENS
#define LOKI_SHORT_MAX_TOKENS 8192
#endif
// Rows of at most this many tokens take the short kernel.
constexpr int kShortMaxTokens = LOKI_SHORT_MAX_TOKENS;
static_assert(kShortMaxTokens <= 32 * kThreads,
              "the share's masks hold at most 32 tokens per thread (and its scan packs counts into 16 bits)");

// Shared-memory layout (4-byte words, 16-byte aligned regions).  `scratch`
// holds the rotation's staging and partial sums, then the bf16 query tiles of
// the tensor-core attention; `recv` receives the other CTAs' merge states and
// nothing else, since a CTA may push into it while the owner still selects;
// the ring carries the key stream, then the select's histogram, then the
// gathered rows; `all` holds the row's keys (round4(seq_len) words: this
// CTA's from its stream, the others' as they push them); `ids` holds the
// CTA's share of the selected indices (at most chunk).
struct ShortSmem {
  int u, qhat, pm, pl, pacc, ctl, scratch, recv, ring, all, ids, words;
};

__host__ __device__ inline ShortSmem short_smem(int G, int D, int chunk, int ncta, int seq_len) {
  ShortSmem L;
  int o = 0;
  L.u = o;       o += round4(D);
  L.qhat = o;    o += G * D;
  L.pm = o;      o += 16;
  L.pl = o;      o += 16;
  L.pacc = o;    o += G * D;
  L.ctl = o;     o += 128;
  L.scratch = o; o += round4(rot_words(G, D) > 8 * D ? rot_words(G, D) : 8 * D);
  L.recv = o;    o += ncta > 1 ? round4(ncta * push_slot_words(G, D, ncta)) : 0;
  L.ring = o;    o += kRingWords;
  L.all = o;     o += round4(seq_len);
  L.ids = o;     o += round4(chunk);
  L.words = o;
  return L;
}

// Positions [s0, s1) of the ascending list of the row's selected tokens into
// ids[p - s0] and idx_row[p].  all[0, S) are the row's keys; the selected
// tokens are those whose masked key is above `prefix`, then the first `take`
// (in token order) whose masked key equals it.  Thread t takes the tokens
// [t*tpt, (t+1)*tpt) (tpt a multiple of 4, at most 32): bit masks of its
// tokens above and at the threshold, one block-wide exclusive scan of their
// counts (16-bit halves, S < 65536), the ties it still takes (the lowest set
// bits of its tie mask), then its selected tokens in order from the selected
// count before it.  Ends with __syncthreads().
__device__ __forceinline__ void write_share(const uint32_t *all, int S, uint32_t prefix, uint32_t mask,
                                            uint32_t take, int s0, int s1, uint32_t *ctl, int32_t *ids,
                                            int32_t *idx_row) {
  const int tpt = round4((S + kThreads - 1) / kThreads);
  const int j0 = min(S, (int)threadIdx.x * tpt), j1 = min(S, j0 + tpt);
  uint32_t gm = 0u, tm = 0u;  // bit i: token j0 + i is above / at the threshold
  for (int j = j0; j < j1; j += 4) {
    const uint4 v = *reinterpret_cast<const uint4 *>(all + j);
    const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t km = kk[e] & mask;
      const uint32_t bit = (j + e < j1) ? 1u << (j - j0 + e) : 0u;
      gm |= km > prefix ? bit : 0u;
      tm |= km == prefix ? bit : 0u;
    }
  }
  const uint32_t eq = (uint32_t)__popc(tm);
  const uint32_t before = block_excl_prefix_sum(((uint32_t)__popc(gm) << 16) | eq, ctl + kSelWtot);
  const uint32_t eq_before = before & 0xffffu;
  const uint32_t tk = take > eq_before ? min(eq, take - eq_before) : 0u;  // ties this thread takes
  uint32_t tsel = tm;  // its lowest tk ties: drop the highest set bits
  for (uint32_t drop = eq - tk; drop > 0u; --drop) tsel &= ~(0x80000000u >> __clz(tsel));
  uint32_t sel = gm | tsel;
  uint32_t p = (before >> 16) + min(eq_before, take);  // selected tokens before this thread's
  if (p < (uint32_t)s1 && p + (uint32_t)__popc(sel) > (uint32_t)s0) {
    while (sel != 0u && p < (uint32_t)s1) {
      const int i = __ffs(sel) - 1;
      sel &= sel - 1u;
      if (p >= (uint32_t)s0) {
        ids[p - s0] = j0 + i;
        idx_row[p] = j0 + i;
      }
      ++p;
    }
  }
  __syncthreads();
}

// One histogram pass over all[0, S): the keys with (key & mask) == prefix add
// one to bin (key >> shift) & (nb - 1) of the skewed histogram.  Eight keys
// per thread are loaded before their atomics, so the loads overlap.
__device__ __forceinline__ void short_hist_pass(const uint32_t *all, int S, uint32_t prefix, uint32_t mask,
                                                int shift, int nb, uint32_t *hist) {
  const int tid = threadIdx.x;
  for (int base = 0; base < S; base += 8 * kThreads) {
    uint32_t kk[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int i = base + x * kThreads + tid;
      kk[x] = i < S ? all[i] : 0u;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x)
      if (base + x * kThreads + tid < S && (kk[x] & mask) == prefix)
        atomicAdd(&hist[hskew((int)((kk[x] >> shift) & (uint32_t)(nb - 1)))], 1u);
  }
}

// The select's two block-wide steps as single out-of-line copies: each runs
// two or three times per call, and a second call then executes from the
// instruction cache instead of fetching another inlined copy from memory
// (measured: llama2-7b-decode 27.3 -> 26.6 us).
static __device__ __noinline__ void short_find_bucket(const uint32_t *hist, int nb, uint32_t remaining,
                                                      uint32_t *ctl) {
  find_bucket(hist, nb, remaining, ctl);
}
static __device__ __noinline__ void short_hist(const uint32_t *all, int S, uint32_t prefix, uint32_t mask, int shift,
                                               int nb, uint32_t *hist) {
  short_hist_pass(all, S, prefix, mask, shift, nb, hist);
}

template <typename T, int D, int G, bool PAGED>
__global__ void __launch_bounds__(kThreads, (G >= 8) ? 1 : 2) loki_short_kernel(const __grid_constant__ StepArgs<T> a) {
  extern __shared__ __align__(16) uint32_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int ncta = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / ncta;
  const int b = row / a.da.n_kv_heads, g = row - b * a.da.n_kv_heads;
  const ShortSmem L = short_smem(G, D, a.da.chunk, ncta, a.da.seq_len);
  float *u = reinterpret_cast<float *>(smem + L.u);
  float *qhat = reinterpret_cast<float *>(smem + L.qhat);
  float *pm = reinterpret_cast<float *>(smem + L.pm);
  float *pl = reinterpret_cast<float *>(smem + L.pl);
  float *pacc = reinterpret_cast<float *>(smem + L.pacc);
  uint32_t *ctl = smem + L.ctl;
  uint32_t *scratch = smem + L.scratch;
  float *recv = reinterpret_cast<float *>(smem + L.recv);
  unsigned char *ring = reinterpret_cast<unsigned char *>(smem + L.ring);
  uint32_t *rw = smem + L.ring;
  uint32_t *all = smem + L.all;
  int32_t *ids = reinterpret_cast<int32_t *>(smem + L.ids);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = a.da.chunk;
  const int S = row_seq_len(a.da, b);
  const uint32_t k = (uint32_t)row_k(a.da, b, S);
  const int t0 = min(S, rank * chunk);
  const int len = min(S, t0 + chunk) - t0;
  const Rows<T, D, PAGED> rows = make_rows<T, D, PAGED>(a.da, b, g);
  constexpr int MAXL = D / VecN<T>::value;
  LOKI_PHASE(0);
  cluster_arrive_relaxed();  // this CTA runs: the others may write into its shared memory

  // 1. the queries and the key stream (as in loki_decode_kernel, without the
  // histogram)
  const bool own = kRotateInKernel<G> && a.da.k_new != nullptr && len > 0 && S - 1 < t0 + len;
  const int slen = own ? len - 1 : len;
  float *xkh = pacc;  // D floats, free until the attention
  if constexpr (kRotateInKernel<G>) {
    rotate_queries<T, D, G>(
        a.da, b, g, qhat, u, reinterpret_cast<float *>(scratch), true,
        [&] {
          LOKI_LPT_DISPATCH(a.da.lpt, MAXL,
                            (score_prologue<T, D, L_, kScoreStageBytes, kScoreStages>(rows, t0, slen, a.da.nck, ring)));
        },
        own ? a.da.k_new + ((size_t)b * a.da.n_kv_heads + g) * D : nullptr, xkh);
    if (own) store_appended<T, D, PAGED>(a.da, rows, b, g, S - 1, xkh);
  } else {
    LOKI_LPT_DISPATCH(a.da.lpt, MAXL,
                      (score_prologue<T, D, L_, kScoreStageBytes, kScoreStages>(rows, t0, len, a.da.nck, ring)));
    griddep_wait();
    if (tid < D) u[tid] = __ldcg(a.u + (size_t)row * D + tid);
    for (int e = tid; e < G * D; e += kThreads) qhat[e] = __ldcg(a.qhat + (size_t)row * G * D + e);
    __syncthreads();
  }
  LOKI_PHASE(1);
  LOKI_LPT_DISPATCH(a.da.lpt, MAXL,
                    (score_keys_loop<T, D, L_, kScoreStageBytes, kScoreStages, 32>(rows, t0, slen, a.da.nck, ring, u,
                                                                                    all + t0, nullptr)));
  if (own) {
    // the appended token's key, from its stored (rounded) values
    if (warp == 0) {
      float sc = 0.f;
      for (int i = lane; i < a.da.d; i += 32) sc = fmaf(u[i], xkh[i], sc);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sc += __shfl_xor_sync(kFull, sc, off);
      if (lane == 0) all[t0 + len - 1] = score_key(sc);
    }
    __syncthreads();
  }
  LOKI_PHASE(2);

  // 2. this CTA's keys into every other CTA's `all` (t0 is a multiple of 4;
  // the last non-empty CTA's final word group runs past S into words nobody
  // reads), then the barrier after which every CTA holds the row's keys
  uint32_t *href = rw + kHref;
  cluster_wait();  // every CTA of the cluster runs
  if (ncta > 1) {
    // (destination, word group) pairs over the CTA's threads, every store in flight at once
    const int n4 = (len + 3) >> 2;
    const uint4 *src = reinterpret_cast<const uint4 *>(all + t0);
    for (int it = tid; it < (ncta - 1) * n4; it += kThreads) {
      const int r = it / n4, j4 = it - r * n4;
      dsmem_st_v4(dsmem_addr(all + t0 + 4 * j4, (uint32_t)((rank + 1 + r) % ncta)), src[j4]);
    }
  }
  for (int e = tid; e < skewed_words(kDig1Bins); e += kThreads) href[e] = 0u;
  cluster.sync();  // every CTA's keys are in every CTA, an appended token stored
  LOKI_PHASE(3);

  // 3. the select, the same in every CTA: the first digit's bucket of the
  // k-th largest key, then up to two refinement passes over the keys in it
  short_hist(all, S, 0u, 0u, 32 - kDig1Bits, kDig1Bins, href);
  __syncthreads();
  short_find_bucket(href, kDig1Bins, k, ctl);
  uint32_t rem = k - ctl[kSelBucket + 1], inb = ctl[kSelBucket + 2];
  uint32_t pre = ctl[kSelBucket + 0] << (32 - kDig1Bits), msk = ~0u << (32 - kDig1Bits);
#pragma unroll 1
  for (int pass = 0; pass < 2 && inb != rem; ++pass) {
    const int shift = pass == 0 ? 32 - kDig1Bits - kDig2Bits : 0;
    const int nb = pass == 0 ? (1 << kDig2Bits) : (1 << kDig3Bits);
    // every thread read ctl above; find_bucket's reads of href ended at its
    // closing barrier
    for (int e = tid; e < skewed_words(nb); e += kThreads) href[e] = 0u;
    __syncthreads();
    short_hist(all, S, pre, msk, shift, nb, href);
    __syncthreads();
    short_find_bucket(href, nb, rem, ctl);
    rem -= ctl[kSelBucket + 1];
    inb = ctl[kSelBucket + 2];
    pre |= ctl[kSelBucket + 0] << shift;
    msk |= (uint32_t)(nb - 1) << shift;
  }
  const int s0 = (int)(((long long)rank * k) / ncta);  // this CTA's even share of the selection
  const int s1 = (int)(((long long)(rank + 1) * k) / ncta);
  int32_t *idx_row = a.da.idx + (size_t)row * a.da.k_stride;
  write_share(all, S, pre, msk, rem, s0, s1, ctl, ids, idx_row);
  // a row shorter than the longest one: the rest of its idx row is -1
  for (int i = (int)k + rank * kThreads + tid; i < a.da.k_stride; i += ncta * kThreads) idx_row[i] = -1;
  LOKI_PHASE(4);

  // 4. attention over the share (the ring's histogram is dead: write_share
  // ended with a barrier)
  if constexpr (PAGED) {
    for (int i = tid; i < s1 - s0; i += kThreads) ids[i] = rows.phys(ids[i]);
    __syncthreads();
    const Rows<T, D, false> pool = pool_rows<T, D>(a.da);
    attend_prologue_any<T, D, G, true>(pool, ids, 0, s1 - s0, ring);
    attend_loop_any<T, D, G, true>(pool, ids, 0, s1 - s0, qhat, reinterpret_cast<unsigned char *>(scratch), ring,
                                   pm, pl, pacc);
  } else {
    attend_prologue_any<T, D, G, true>(rows, ids, 0, s1 - s0, ring);
    attend_loop_any<T, D, G, true>(rows, ids, 0, s1 - s0, qhat, reinterpret_cast<unsigned char *>(scratch), ring,
                                   pm, pl, pacc);
  }
  LOKI_PHASE(5);

  // 5. log-sum-exp merge: states pushed into the owners' receive buffers,
  // one barrier (after which no CTA reads another's shared memory)
  const int Hq = a.da.n_kv_heads * G;
  float *out = a.da.out + ((size_t)b * Hq + (size_t)g * G) * D;
  __syncthreads();  // the CTA's state is complete
  if (ncta == 1) {
    local_combine<D, G>(pl, pacc, out);
  } else {
    push_state<D, G>(ncta, rank, pm, pl, pacc, recv);
    cluster.sync();
    push_combine<D, G>(ncta, rank, recv, out);
  }
  LOKI_PHASE(6);
#ifdef LOKI_PHASE_STAMPS
  if (tid == 0 && blockIdx.x < kMaxStampCtas) {
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    g_phase_stamps[blockIdx.x][7] = sm;
    g_phase_stamps[blockIdx.x][8] = (unsigned long long)rank | ((unsigned long long)ncta << 8) | (1ull << 16) |
                                    (1ull << 17);
    g_phase_stamps[blockIdx.x][9] = (unsigned long long)row;
  }
#endif
}

}  // namespace loki
