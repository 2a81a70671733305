// Device helpers shared by the Loki kernels (sm_100a).
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace loki {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;            // every kernel runs 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

// Elements per 16-byte vector.
template <typename T> struct VecN;
template <> struct VecN<float> { static constexpr int value = 4; };
template <> struct VecN<__nv_bfloat16> { static constexpr int value = 8; };

// 16-byte streaming load that does not allocate in L1 (cache rows are read
// once per call).  Only used on data no thread writes during the kernel.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// 16-byte asynchronous copy global -> shared (L2 only), completed by
// cp.async.wait_group.  Both addresses must be 16-byte aligned.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem_src) : "memory");
}
// Same, but copies `valid ? 16 : 0` bytes and zero-fills the rest (the source
// is not read when invalid; it must still be a mapped address).
__device__ __forceinline__ void cp_async16_zfill(void *smem_dst, const void *gmem_src, bool valid) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem_dst);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem_src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Widen a 16-byte vector to fp32 (exact for both dtypes).
__device__ __forceinline__ void unpack16(const uint4 &r, float (&f)[4]) {
  f[0] = __uint_as_float(r.x);
  f[1] = __uint_as_float(r.y);
  f[2] = __uint_as_float(r.z);
  f[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void unpack16(const uint4 &r, float (&f)[8]) {
  // bf16 is the upper half of an fp32; element 2i sits in the low 16 bits.
  f[0] = __uint_as_float(r.x << 16);
  f[1] = __uint_as_float(r.x & 0xffff0000u);
  f[2] = __uint_as_float(r.y << 16);
  f[3] = __uint_as_float(r.y & 0xffff0000u);
  f[4] = __uint_as_float(r.z << 16);
  f[5] = __uint_as_float(r.z & 0xffff0000u);
  f[6] = __uint_as_float(r.w << 16);
  f[7] = __uint_as_float(r.w & 0xffff0000u);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void from_f32(float x, float *dst) { *dst = x; }
__device__ __forceinline__ void from_f32(float x, __nv_bfloat16 *dst) {
  *dst = __float2bfloat16_rn(x);  // round to nearest even
}

// ---- warp-level tensor-core helpers (bf16 operands, fp32 accumulation) ----
// Four 8x8 b16 matrices from shared memory; lane l supplies the address of row
// l%8 of matrix l/8.  Thread (g = lane/4, t = lane%4) receives row g, columns
// 2t and 2t+1 of each matrix (.trans: row 2t and 2t+1, column g).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                              uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D[16x8] += A[16x16] . B[16x8]
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D[16x8] += A[16x8] . B[8x8]
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// (x0, x1) as two bf16 pairs hi + lo with x ~= hi + lo to about 2^-17 relative:
// hi = RNE(x), lo = RNE(x - hi); element 0 in the low half of each word.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Skewed index of bin b in a shared-memory histogram (one spare word per 32
// bins): the consecutive bins one thread scans fall into distinct banks
// across a warp.
__host__ __device__ inline int hskew(int b) { return b + (b >> 5); }
__host__ __device__ inline constexpr int skewed_words(int bins) { return bins + bins / 32; }

// Order-preserving map fp32 -> uint32: a > b  <=>  key(a) > key(b) for finite
// a, b.  -0 and +0 map to the same key so that equal scores tie (and the lower
// index wins) regardless of the sign of zero.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b << 1) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Programmatic dependent launch.  griddep_wait(): block until every grid this
// one depends on has completed and its memory operations are visible (returns
// at once when the kernel was not launched as a dependent).
// griddep_launch_dependents(): allow the dependent grid to be scheduled once
// every CTA of this grid has executed it or exited.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte global load and store at L2 (not cached in L1): for data written by
// other CTAs of the same grid and published through a fence + atomic.
__device__ __forceinline__ uint4 ld_cg16(const void *p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_cg16(void *p, const uint4 &v) {
  asm volatile("st.global.cg.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Distributed shared memory: the shared::cluster address of `local` (this
// CTA's shared memory) in CTA `rank` of the cluster, and accesses through it.
__device__ __forceinline__ uint32_t dsmem_addr(const void *local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ void dsmem_red_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void dsmem_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void dsmem_st_v4(uint32_t addr, const uint4 &v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 dsmem_ld_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float dsmem_ld_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Split cluster barrier (arrive with release, wait with acquire).  Every thread
// of every CTA in the cluster must execute each of them the same number of times.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Sum of v over all threads with a larger threadIdx.x (exclusive suffix sum).
// wtot: kWarps words of shared memory.  Contains two __syncthreads().
__device__ __forceinline__ uint32_t block_excl_suffix_sum(uint32_t v, uint32_t *wtot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t s = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t t = __shfl_down_sync(kFull, s, off);
    if (lane + off < 32) s += t;
  }
  if (lane == 0) wtot[warp] = s;
  __syncthreads();
  uint32_t higher = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w > warp) higher += wtot[w];
  __syncthreads();
  return higher + (s - v);
}

// Sum of v over all threads with a smaller threadIdx.x (exclusive prefix sum).
// wtot: kWarps words of shared memory.  Contains two __syncthreads().
__device__ __forceinline__ uint32_t block_excl_prefix_sum(uint32_t v, uint32_t *wtot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t s = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t t = __shfl_up_sync(kFull, s, off);
    if (lane >= off) s += t;
  }
  if (lane == 31) wtot[warp] = s;
  __syncthreads();
  uint32_t lower = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w < warp) lower += wtot[w];
  __syncthreads();
  return lower + (s - v);
}

// Sum over the CTA; the result is returned to every thread.
// wtot: kWarps words of shared memory.  Contains two __syncthreads().
__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t *wtot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  if (lane == 0) wtot[warp] = v;
  __syncthreads();
  uint32_t s = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) s += wtot[w];
  __syncthreads();
  return s;
}

}  // namespace loki
