// Rotate-and-append kernel for sm_100a.
//
// "PCA-project ... keys" ("Loki: Low-rank Keys for Efficient Sparse
// Attention", atlas.scime.ai summary, section "Approach"); the cache holds
// every token, nothing is evicted (same page, "Limitations").
//
// k_hat[b][g][pos+t][j] = round( sum_i k_new[b][g][t][i] * P[g][i][j] ), fp32
// accumulation in increasing i, round to nearest even into the cache dtype;
// v_new is copied unchanged.  Grid (Hkv, D/32, chunks): a CTA holds a 32-column
// slice of P_g in shared memory (16 KB for D = 128) and produces those 32
// output columns for a chunk of the B*n_new vectors of KV head g, 8 vectors at
// a time (one vector per warp, one column per lane).  CTAs of column block 0
// also copy the values.
#pragma once

#include "common.cuh"

namespace loki {

template <typename T>
struct AppendArgs {
  T *k_hat;          // [B, Hkv, S_cap, D]
  T *v;              // [B, Hkv, S_cap, D]
  const T *k_new;    // [B, Hkv, n_new, D]
  const T *v_new;    // [B, Hkv, n_new, D]
  const float *P;    // [Hkv, D, D]
  // the cache's low-rank key plane (null: none), laid out like k_hat with
  // rows of d_lr: it receives the first d_lr dims of every appended key
  T *k_lr;
  int32_t d_lr;
  int32_t n_kv_heads;
  int32_t capacity;
  int32_t pos;
  int32_t n_new;
  int32_t n_vec;     // B * n_new vectors per KV head
  int32_t per_cta;   // vectors per CTA (multiple of kAppendBatch)
  // paged cache (PAGED instantiations): pools [num_pages, Hkv, page, D], new
  // vector t of sequence b goes to token pos_arr[b] + t of its page table
  const int32_t *pos_arr;  // [B]
  const int32_t *table;    // [B, pages_per_seq]
  int32_t pages_per_seq;
  int32_t page_shift;      // page size = 1 << page_shift tokens
  int32_t num_pages;
};

// Element offset in the cache of new vector t of sequence b, head g; -1 when
// a paged sequence's position falls outside its page table (not written).
// Page ids are clamped into the pool.
template <typename T, int D, bool PAGED>
__device__ __forceinline__ long long append_dst(const AppendArgs<T> &a, int b, int g, int t) {
  if constexpr (!PAGED) {
    return (((long long)b * a.n_kv_heads + g) * a.capacity + a.pos + t) * D;
  } else {
    const int tok = __ldg(a.pos_arr + b) + t;
    if (tok < 0 || (tok >> a.page_shift) >= a.pages_per_seq) return -1;
    const int p =
        min(max(__ldg(a.table + (size_t)b * a.pages_per_seq + (tok >> a.page_shift)), 0), a.num_pages - 1);
    return ((((long long)p * a.n_kv_heads + g) << a.page_shift) + (tok & ((1 << a.page_shift) - 1))) * D;
  }
}

// Element offset in the low-rank plane of the row whose k_hat offset is off
// (>= 0): the same row index, rows of d_lr.
template <typename T, int D>
__device__ __forceinline__ long long append_lr_dst(const AppendArgs<T> &a, long long off) {
  return off / D * a.d_lr;
}

constexpr int kAppendBatch = kWarps;   // vectors per batch: one per warp
constexpr int kAppendCols = 32;        // output columns per CTA: one per lane

__host__ __device__ inline int append_smem_words(int D) { return D * kAppendCols + kAppendBatch * D; }

template <typename T, int D, bool PAGED>
__global__ void __launch_bounds__(kThreads) append_kernel(const __grid_constant__ AppendArgs<T> a) {
  extern __shared__ __align__(16) float asmem[];
  float *Ps = asmem;                   // [D][32]: columns cb*32 .. cb*32+31 of P_g
  float *ks = asmem + D * kAppendCols; // [8][D]
  const int g = blockIdx.x, cb = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int f_begin = blockIdx.z * a.per_cta;
  const int f_end = min(a.n_vec, f_begin + a.per_cta);
  if (f_begin >= f_end) return;  // uniform over the CTA; no barrier has been reached

  {
    // P_g[i][cb*32 .. +32): 8 float4 per row, all issued before any is stored
    constexpr int N4 = D * kAppendCols / 4;
    const float *src = a.P + (size_t)g * D * D + cb * kAppendCols;
    float4 r[N4 / kThreads];
#pragma unroll
    for (int x = 0; x < N4 / kThreads; ++x) {
      const int q = x * kThreads + tid;
      r[x] = __ldg(reinterpret_cast<const float4 *>(src + (size_t)(q / 8) * D) + (q % 8));
    }
#pragma unroll
    for (int x = 0; x < N4 / kThreads; ++x) reinterpret_cast<float4 *>(Ps)[x * kThreads + tid] = r[x];
  }

  const int j = cb * kAppendCols + lane;
  for (int f0 = f_begin; f0 < f_end; f0 += kAppendBatch) {
    __syncthreads();  // P staged / previous batch consumed
    for (int e = tid; e < kAppendBatch * D; e += kThreads) {
      const int f = f0 + e / D;
      float x = 0.f;
      if (f < f_end) {
        const int b = f / a.n_new, t = f % a.n_new;
        x = to_f32(a.k_new[(((size_t)b * a.n_kv_heads + g) * a.n_new + t) * D + (e % D)]);
      }
      ks[e] = x;
    }
    __syncthreads();
    const float *kv = ks + warp * D;
    float acc = 0.f;
#pragma unroll 16
    for (int i = 0; i < D; ++i) acc = fmaf(kv[i], Ps[i * kAppendCols + lane], acc);
    const int f = f0 + warp;
    if (f < f_end) {
      const int b = f / a.n_new, t = f % a.n_new;
      const long long off = append_dst<T, D, PAGED>(a, b, g, t);
      if (off >= 0) {
        from_f32(acc, a.k_hat + off + j);
        if (a.k_lr != nullptr && j < a.d_lr) from_f32(acc, a.k_lr + append_lr_dst<T, D>(a, off) + j);
      }
    }
  }

  if (cb != 0) return;
  // values: straight 16-byte copies
  constexpr int VEC = VecN<T>::value;
  constexpr int VPR = D / VEC;  // vectors per row
  const int rows = f_end - f_begin;
  for (int e = tid; e < rows * VPR; e += kThreads) {
    const int f = f_begin + e / VPR, c = e % VPR;
    const int b = f / a.n_new, t = f % a.n_new;
    const uint4 *src = reinterpret_cast<const uint4 *>(
        a.v_new + (((size_t)b * a.n_kv_heads + g) * a.n_new + t) * D) + c;
    const long long off = append_dst<T, D, PAGED>(a, b, g, t);
    if (off >= 0) reinterpret_cast<uint4 *>(a.v + off)[c] = __ldg(src);
  }
}

}  // namespace loki
