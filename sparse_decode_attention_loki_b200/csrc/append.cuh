// Rotate-and-append kernel for sm_100a.
//
// "PCA-project ... keys" ("Loki: Low-rank Keys for Efficient Sparse
// Attention", atlas.scime.ai summary, section "Approach"); the cache holds
// every token, nothing is evicted (same page, "Limitations").
//
// k_hat[b][g][pos+t][j] = round( sum_i k_new[b][g][t][i] * P[g][i][j] ), fp32
// accumulation in increasing i, round to nearest even into the cache dtype;
// v_new is copied unchanged.  Grid (Hkv, chunks): a CTA holds P_g in shared
// memory (64 KB for D = 128) and rotates a chunk of the B*n_new vectors of
// KV head g, 8 at a time.
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
  int32_t n_kv_heads;
  int32_t capacity;
  int32_t pos;
  int32_t n_new;
  int32_t n_vec;     // B * n_new vectors per KV head
  int32_t per_cta;   // vectors per CTA (multiple of kAppendBatch)
};

constexpr int kAppendBatch = 8;

__host__ __device__ inline int append_smem_words(int D) { return D * D + kAppendBatch * D; }

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) append_kernel(const __grid_constant__ AppendArgs<T> a) {
  extern __shared__ __align__(16) float asmem[];
  float *Ps = asmem;               // [D][D]
  float *ks = asmem + D * D;       // [kAppendBatch][D]
  const int g = blockIdx.x;
  const int tid = threadIdx.x;
  const int f_begin = blockIdx.y * a.per_cta;
  const int f_end = min(a.n_vec, f_begin + a.per_cta);
  if (f_begin >= f_end) return;  // uniform over the CTA; no barrier has been reached

  {
    const float4 *src = reinterpret_cast<const float4 *>(a.P + (size_t)g * D * D);
    float4 *dst = reinterpret_cast<float4 *>(Ps);
    for (int i = tid; i < D * D / 4; i += kThreads) dst[i] = __ldg(src + i);
  }

  constexpr int GROUPS = kThreads / D;                 // 2 (D=128) or 4 (D=64)
  constexpr int VPT = kAppendBatch / GROUPS;           // vectors per thread per batch
  const int j = tid % D, grp = tid / D;
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
    float acc[VPT];
#pragma unroll
    for (int x = 0; x < VPT; ++x) acc[x] = 0.f;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float p = Ps[i * D + j];
#pragma unroll
      for (int x = 0; x < VPT; ++x) acc[x] = fmaf(ks[(grp + x * GROUPS) * D + i], p, acc[x]);
    }
#pragma unroll
    for (int x = 0; x < VPT; ++x) {
      const int f = f0 + grp + x * GROUPS;
      if (f < f_end) {
        const int b = f / a.n_new, t = f % a.n_new;
        from_f32(acc[x], a.k_hat + (((size_t)b * a.n_kv_heads + g) * a.capacity + a.pos + t) * D + j);
      }
    }
  }

  // values: straight 16-byte copies
  constexpr int VEC = VecN<T>::value;
  constexpr int VPR = D / VEC;  // vectors per row
  const int rows = f_end - f_begin;
  for (int e = tid; e < rows * VPR; e += kThreads) {
    const int f = f_begin + e / VPR, c = e % VPR;
    const int b = f / a.n_new, t = f % a.n_new;
    const uint4 *src = reinterpret_cast<const uint4 *>(
        a.v_new + (((size_t)b * a.n_kv_heads + g) * a.n_new + t) * D) + c;
    uint4 *dst = reinterpret_cast<uint4 *>(
        a.v + (((size_t)b * a.n_kv_heads + g) * a.capacity + a.pos + t) * D) + c;
    *dst = __ldg(src);
  }
}

}  // namespace loki
