// Host-side pieces shared by the translation units of libloki.so: error
// reporting, per-device attributes, launch helpers and the decode dispatch
// that each (dtype, head dim) unit compiles on its own (decode_inst.cu).
#pragma once

#include <atomic>
#include <mutex>
#include <vector>

#include "loki.h"
#include "decode.cuh"

namespace loki {

// Sets the calling thread's last-error message and returns s.
loki_status fail(loki_status s, const char *fmt, ...);
loki_status cuda_fail(cudaError_t e, const char *what);

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device attributes, read once per device.
struct DevInfo {
  int sms;
  int smem_optin;
};
constexpr int kMaxDevices = 64;
loki_status device_info(DevInfo *out);

// The launch-shape override of loki_set_launch_override (0: none).
int forced_cluster();

// A validated decode call.
struct DecodeShape {
  int B, Hkv, D, Scap, S, Hq, G;
  size_t esize;
  int d_lr;  // width of the cache's low-rank key plane, 0 without one
};

// Launch shape a decode call took (or would take).
struct Plan {
  int ncta;    // CTAs per (batch, KV head) row: the cluster size
  int chunk;   // tokens per CTA
  int smem;    // dynamic shared memory per CTA
  int grid;    // CTAs of the decode kernel
  int rot;     // Loki: CTAs of the rotate kernel (query groups of 8), else 0
  int spare;   // Loki: 1 when the short-row kernel runs, else 0
};

// Per-sequence lengths and paging of a decode call (all null: a contiguous
// cache where every row has seq_len tokens and takes k).
struct VarPage {
  const int32_t *seq_lens = nullptr, *ks = nullptr, *table = nullptr;
  int32_t pages_per_seq = 0, page_shift = 0, num_pages = 0;
  const void *k_new = nullptr, *v_new = nullptr;  // a token appended by the call, [B, Hkv, D]
};

inline void set_cluster(cudaLaunchAttribute *attr, int ncta) {
  attr->id = cudaLaunchAttributeClusterDimension;
  attr->val.clusterDim.x = (unsigned)ncta;
  attr->val.clusterDim.y = 1;
  attr->val.clusterDim.z = 1;
}
inline void set_pdl(cudaLaunchAttribute *attr) {
  attr->id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr->val.programmaticStreamSerializationAllowed = 1;
}

// Launch `kern` on `grid` CTAs of `threads` threads, as a cluster of `ncta`
// CTAs when ncta > 0 and as a programmatic dependent of the previous kernel on
// the stream when pdl is set.
template <typename Kern, typename Args>
loki_status launch_ex(Kern kern, long long grid, int smem, int ncta, bool pdl, const Args &args, void *stream,
                      const char *what, int threads = kThreads) {
  if (grid < 1 || grid > 0x7fffffffLL) return fail(LOKI_ERR_UNSUPPORTED, "%s: grid of %lld CTAs", what, grid);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 0;
  if (ncta > 0) set_cluster(&attr[cfg.numAttrs++], ncta);
  if (pdl) set_pdl(&attr[cfg.numAttrs++]);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return LOKI_OK;
}

// Occupancy figures, cached per device, kernel, cluster size and 4 KB
// shared-memory bucket (the cache lives in loki_api.cu).
struct OccEntry {
  const void *kern;
  int dev, ncta, smem_q, n;
};
bool occ_lookup(const void *kern, int dev, int ncta, int smem_q, int *n);
void occ_store(const void *kern, int dev, int ncta, int smem_q, int n);

// Co-resident clusters of `ncta` CTAs (ncta > 0) or co-resident CTAs per SM
// (ncta == 0) of a kernel with `smem` bytes of dynamic shared memory; 0 if
// the device cannot schedule it.
template <typename Kern>
int max_active(Kern kern, int dev, int ncta, int smem, int smem_limit) {
  int smem_q = (smem + 4095) & ~4095;
  if (smem_q > smem_limit) smem_q = smem;
  int n = 0;
  if (occ_lookup((const void *)kern, dev, ncta, smem_q, &n)) return n;
  if (ncta > 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)ncta, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem_q;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    set_cluster(&attr[0], ncta);
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
  } else if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kThreads, (size_t)smem_q) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  occ_store((const void *)kern, dev, ncta, smem_q, n);
  return n;
}

// Per-kernel, per-device record of the dynamic shared memory already allowed.
struct SmemGate {
  std::atomic<int> bytes[kMaxDevices];
};

// Raise a kernel's dynamic shared-memory limit to the device's opt-in maximum
// (once per device and kernel: `gate` belongs to exactly one kernel) and, for
// cluster kernels, allow clusters of up to 16 CTAs.  Launches then pass their
// own smaller sizes.
template <typename Kern>
loki_status allow_smem(Kern kern, const DevInfo &di, SmemGate &gate, bool cluster) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (gate.bytes[dev].load(std::memory_order_acquire) >= di.smem_optin) return LOKI_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, di.smem_optin);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(MaxDynamicSharedMemorySize)");
  if (cluster) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(NonPortableClusterSizeAllowed)");
  }
  gate.bytes[dev].store(di.smem_optin, std::memory_order_release);
  return LOKI_OK;
}

// One token per row, rotated and written at position pos of a contiguous
// cache (the append kernel of loki_append, in loki_api.cu): the generation
// step of query groups of 8, whose decode kernel does not append.
loki_status append_token(int dtype, int D, void *k_hat, void *v, void *k_lr, int d_lr, int Hkv, int capacity, int pos,
                         int B, const void *k_new, const void *v_new, const float *P, void *stream);

// The decode calls of one (dtype, head dim), compiled in decode_inst.cu once
// per pair: dense == true runs the dense kernel, else the Loki step (ws:
// the caller's workspace).  used != nullptr: plan only, launch nothing.
template <typename T, int D>
loki_status decode_td(bool dense, const DevInfo &di, const DecodeShape &sh, const DecodeArgs<T> &a, void *ws,
                      void *stream, Plan *used);
// Phase stamps of that unit's last Loki decode (instrumented builds only).
template <typename T, int D>
loki_status decode_phase_stamps(unsigned long long *host, int32_t capacity, int32_t *n);

extern template loki_status decode_phase_stamps<float, 64>(unsigned long long *, int32_t, int32_t *);
extern template loki_status decode_phase_stamps<float, 128>(unsigned long long *, int32_t, int32_t *);
extern template loki_status decode_phase_stamps<__nv_bfloat16, 64>(unsigned long long *, int32_t, int32_t *);
extern template loki_status decode_phase_stamps<__nv_bfloat16, 128>(unsigned long long *, int32_t, int32_t *);
extern template loki_status decode_td<float, 64>(bool, const DevInfo &, const DecodeShape &, const DecodeArgs<float> &,
                                                 void *, void *, Plan *);
extern template loki_status decode_td<float, 128>(bool, const DevInfo &, const DecodeShape &,
                                                  const DecodeArgs<float> &, void *, void *, Plan *);
extern template loki_status decode_td<__nv_bfloat16, 64>(bool, const DevInfo &, const DecodeShape &,
                                                         const DecodeArgs<__nv_bfloat16> &, void *, void *, Plan *);
extern template loki_status decode_td<__nv_bfloat16, 128>(bool, const DevInfo &, const DecodeShape &,
                                                          const DecodeArgs<__nv_bfloat16> &, void *, void *, Plan *);

}  // namespace loki
