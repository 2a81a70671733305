// Host side of libloki.so: argument validation, launch planning and launches
// for the C ABI declared in include/loki.h.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "loki.h"
#include "append.cuh"
#include "decode.cuh"

namespace {

using namespace loki;

thread_local char g_err[512];

loki_status fail(loki_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

loki_status cuda_fail(cudaError_t e, const char *what) {
  return fail(LOKI_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device attributes, read once per device.
struct DevInfo {
  int sms;
  int smem_optin;
};
constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ready[kMaxDevices];
DevInfo g_dev[kMaxDevices];

loki_status device_info(DevInfo *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LOKI_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  if (!g_dev_ready[dev].load(std::memory_order_acquire)) {
    DevInfo di;
    e = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    e = cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(smem opt-in)");
    g_dev[dev] = di;
    g_dev_ready[dev].store(1, std::memory_order_release);
  }
  *out = g_dev[dev];
  return LOKI_OK;
}

// Tuning override (development only): LOKI_CLUSTER forces the CTAs per row.
int env_int(const char *name, int dflt) {
  const char *s = std::getenv(name);
  if (!s || !*s) return dflt;
  return std::atoi(s);
}

// Raise a kernel's dynamic shared-memory limit (per device, remembered) and
// allow 16-CTA clusters.
template <typename Kern>
loki_status prepare(Kern kern, int smem_bytes, std::atomic<int> *done_smem) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (done_smem[dev].load(std::memory_order_acquire) >= smem_bytes) return LOKI_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(MaxDynamicSharedMemorySize)");
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(NonPortableClusterSizeAllowed)");
  int prev = done_smem[dev].load();
  while (prev < smem_bytes && !done_smem[dev].compare_exchange_weak(prev, smem_bytes)) {
  }
  return LOKI_OK;
}

// ---------------------------------------------------------------------------
// validation shared by the two decode entry points
struct DecodeShape {
  int B, Hkv, D, Scap, S, Hq, G;
  size_t esize;
};

loki_status check_cache(const loki_cache *c, DecodeShape *sh) {
  if (!c) return fail(LOKI_ERR_INVALID_ARG, "cache descriptor is NULL");
  if (c->dtype != LOKI_F32 && c->dtype != LOKI_BF16)
    return fail(LOKI_ERR_INVALID_ARG, "cache dtype %d is not LOKI_F32 or LOKI_BF16", c->dtype);
  if (c->batch < 1 || c->n_kv_heads < 1 || c->capacity < 1 || c->head_dim < 1)
    return fail(LOKI_ERR_INVALID_ARG, "cache sizes must be >= 1 (B=%d Hkv=%d D=%d S_cap=%d)", c->batch,
                c->n_kv_heads, c->head_dim, c->capacity);
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(LOKI_ERR_UNSUPPORTED, "head_dim %d not supported (64 or 128)", c->head_dim);
  if (!c->k_hat || !c->v) return fail(LOKI_ERR_INVALID_ARG, "cache k_hat or v is NULL");
  if (!aligned(c->k_hat, 16) || !aligned(c->v, 16))
    return fail(LOKI_ERR_INVALID_ARG, "cache k_hat and v must be 16-byte aligned");
  if ((long long)c->batch * c->n_kv_heads > (1LL << 26))
    return fail(LOKI_ERR_UNSUPPORTED, "batch * n_kv_heads too large");
  sh->B = c->batch;
  sh->Hkv = c->n_kv_heads;
  sh->D = c->head_dim;
  sh->Scap = c->capacity;
  sh->esize = c->dtype == LOKI_F32 ? 4 : 2;
  return LOKI_OK;
}

loki_status check_decode(const loki_cache *c, int32_t seq_len, int32_t n_q_heads, const void *q,
                         const float *P, float *out, DecodeShape *sh) {
  loki_status s = check_cache(c, sh);
  if (s != LOKI_OK) return s;
  if (seq_len < 1 || seq_len > sh->Scap)
    return fail(LOKI_ERR_INVALID_ARG, "seq_len %d outside [1, capacity=%d]", seq_len, sh->Scap);
  if (n_q_heads < sh->Hkv || n_q_heads % sh->Hkv != 0)
    return fail(LOKI_ERR_INVALID_ARG, "n_q_heads %d is not a positive multiple of n_kv_heads %d", n_q_heads,
                sh->Hkv);
  const int G = n_q_heads / sh->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(LOKI_ERR_UNSUPPORTED, "query group size %d not supported (1, 2, 4 or 8)", G);
  if (!q || !P || !out) return fail(LOKI_ERR_INVALID_ARG, "q, P or out is NULL");
  if (!aligned(q, 16)) return fail(LOKI_ERR_INVALID_ARG, "q must be 16-byte aligned");
  if (!aligned(P, 16)) return fail(LOKI_ERR_INVALID_ARG, "P must be 16-byte aligned");
  if (!aligned(out, 4)) return fail(LOKI_ERR_INVALID_ARG, "out must be 4-byte aligned");
  sh->S = seq_len;
  sh->Hq = n_q_heads;
  sh->G = G;
  return LOKI_OK;
}

float resolve_scale(float scale, int D) {
  const float s = (scale > 0.f && std::isfinite(scale)) ? scale : 1.0f / std::sqrt((float)D);
  return s * 1.4426950408889634f;  // log2(e)
}

// ---------------------------------------------------------------------------
// launch planning: CTAs per row (cluster size) and tokens per CTA
struct Plan {
  int ncta;
  int chunk;
  int smem;
};

int smem_bytes(int G, int D, int chunk, int ncta, bool loki) {
  return decode_layout(G, D, chunk, ncta, loki).words * 4;
}

void fill_config(cudaLaunchConfig_t *cfg, cudaLaunchAttribute *attr, const Plan &pl, int rows, void *stream) {
  *cfg = cudaLaunchConfig_t{};
  cfg->gridDim = dim3((unsigned)(rows * pl.ncta), 1, 1);
  cfg->blockDim = dim3(kThreads, 1, 1);
  cfg->dynamicSmemBytes = (size_t)pl.smem;
  cfg->stream = static_cast<cudaStream_t>(stream);
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)pl.ncta;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

// Co-resident clusters of `ncta` CTAs for a kernel with `smem` bytes of
// dynamic shared memory (cached per device, kernel, cluster size and 4 KB
// shared-memory bucket).  0 if the device cannot schedule such a cluster.
struct OccEntry {
  const void *kern;
  int dev, ncta, smem_q, clusters;
};
std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;

template <typename Kern>
int max_active_clusters(Kern kern, int dev, int ncta, int smem, int smem_limit) {
  int smem_q = (smem + 4095) & ~4095;
  if (smem_q > smem_limit) smem_q = smem;
  {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    for (const OccEntry &e : g_occ)
      if (e.kern == (const void *)kern && e.dev == dev && e.ncta == ncta && e.smem_q == smem_q) return e.clusters;
  }
  Plan pl{ncta, 0, smem_q};
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  fill_config(&cfg, attr, pl, 1, nullptr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(g_occ_mu);
  g_occ.push_back(OccEntry{(const void *)kern, dev, ncta, smem_q, n});
  return n;
}

// Launch plan: CTAs per row (cluster size) and tokens per CTA.  Among cluster
// sizes whose per-CTA share is at least kMinTokens tokens and whose shared
// memory fits, take the one that keeps the most CTAs busy per wave of
// co-resident clusters (rows*n / waves); ties go to the smaller cluster, which
// spends less on the cross-CTA steps.  LOKI_CLUSTER (tuning only) forces n.
template <typename Kern>
loki_status plan_for(Kern kern, const DevInfo &di, const DecodeShape &sh, bool dense, Plan *p) {
  constexpr int kMinTokens = 256;
  const int rows = sh.B * sh.Hkv;
  int dev = 0;
  cudaGetDevice(&dev);
  const int forced = env_int("LOKI_CLUSTER", 0);
  double best = -1.0;
  Plan bp{0, 0, 0};
  int last_smem = 0;
  for (int n = 1; n <= 16; n *= 2) {
    if (forced && n != forced) continue;
    const int chunk = (sh.S + n - 1) / n;
    if (!forced && n > 1 && chunk < kMinTokens) continue;
    const int smem = smem_bytes(sh.G, sh.D, chunk, n, !dense);
    last_smem = smem;
    if (smem > di.smem_optin) continue;
    const int mc = max_active_clusters(kern, dev, n, smem, di.smem_optin);
    if (mc <= 0) continue;
    const long long waves = (rows + mc - 1) / mc;
    const double per_wave = (double)rows * n / (double)waves;
    if (per_wave > best * 1.0001) {
      best = per_wave;
      bp = Plan{n, chunk, smem};
    }
  }
  if (bp.ncta == 0 && forced) {
    setenv("LOKI_CLUSTER", "", 1);  // a forced size that cannot run: plan normally
    loki_status s = plan_for(kern, di, sh, dense, p);
    setenv("LOKI_CLUSTER", std::to_string(forced).c_str(), 1);
    return s;
  }
  if (bp.ncta == 0)
    return fail(LOKI_ERR_UNSUPPORTED,
                "no launch shape fits: seq_len %d needs %d B of shared memory per CTA (limit %d) or an "
                "unschedulable cluster",
                sh.S, last_smem, di.smem_optin);
  *p = bp;
  return LOKI_OK;
}

template <typename Kern, typename Args>
loki_status launch(Kern kern, const Plan &pl, int rows, const Args &args, void *stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  fill_config(&cfg, attr, pl, rows, stream);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args);
  if (e != cudaSuccess) return cuda_fail(e, "cudaLaunchKernelEx");
  return LOKI_OK;
}

template <typename T, int D, int G>
struct DecodeKernels {
  static std::atomic<int> smem_loki[kMaxDevices];
  static std::atomic<int> smem_dense[kMaxDevices];
};
template <typename T, int D, int G>
std::atomic<int> DecodeKernels<T, D, G>::smem_loki[kMaxDevices];
template <typename T, int D, int G>
std::atomic<int> DecodeKernels<T, D, G>::smem_dense[kMaxDevices];

template <typename Kern, typename T>
loki_status prepare_and_launch(Kern kern, std::atomic<int> *done_smem, const DevInfo &di, const DecodeShape &sh,
                               bool dense, int rows, DecodeArgs<T> args, void *stream, Plan *used) {
  // the attribute covers every plan this device can take
  loki_status s = prepare(kern, di.smem_optin, done_smem);
  if (s != LOKI_OK) return s;
  Plan pl;
  s = plan_for(kern, di, sh, dense, &pl);
  if (s != LOKI_OK) return s;
  args.chunk = pl.chunk;
  if (used) *used = pl;
  if (!stream && used) return LOKI_OK;  // shape query only
  return launch(kern, pl, rows, args, stream);
}

template <typename T, int D, int G>
loki_status run_decode(bool dense, const DevInfo &di, const DecodeShape &sh, int rows, const DecodeArgs<T> &args,
                       void *stream, Plan *used) {
  if (dense)
    return prepare_and_launch(dense_decode_kernel<T, D, G>, DecodeKernels<T, D, G>::smem_dense, di, sh, true, rows,
                              args, stream, used);
  return prepare_and_launch(loki_decode_kernel<T, D, G>, DecodeKernels<T, D, G>::smem_loki, di, sh, false, rows,
                            args, stream, used);
}

template <typename T, int D>
loki_status run_decode_g(const DevInfo &di, const DecodeShape &sh, bool dense, int rows, const DecodeArgs<T> &args,
                         void *stream, Plan *used) {
  switch (sh.G) {
    case 1: return run_decode<T, D, 1>(dense, di, sh, rows, args, stream, used);
    case 2: return run_decode<T, D, 2>(dense, di, sh, rows, args, stream, used);
    case 4: return run_decode<T, D, 4>(dense, di, sh, rows, args, stream, used);
    case 8: return run_decode<T, D, 8>(dense, di, sh, rows, args, stream, used);
  }
  return fail(LOKI_ERR_UNSUPPORTED, "group size %d", sh.G);
}

template <typename T>
loki_status decode_common(const loki_cache *c, const DecodeShape &sh, bool dense, const void *q, const float *P,
                          int32_t d, int32_t k, float scale, float *out, int32_t *idx, void *stream,
                          Plan *used = nullptr) {
  DevInfo di;
  loki_status s = device_info(&di);
  if (s != LOKI_OK) return s;
  constexpr int VEC = VecN<T>::value;
  DecodeArgs<T> a;
  a.k_hat = static_cast<const T *>(c->k_hat);
  a.v = static_cast<const T *>(c->v);
  a.q = static_cast<const T *>(q);
  a.P = P;
  a.out = out;
  a.idx = idx;
  a.n_kv_heads = sh.Hkv;
  a.capacity = sh.Scap;
  a.seq_len = sh.S;
  a.d = d;
  a.k = k;
  a.chunk = 0;  // set by the plan
  a.nck = (d + VEC - 1) / VEC;
  int lpt = 1;
  while (lpt < a.nck) lpt *= 2;
  a.lpt = lpt;
  a.scale_log2 = resolve_scale(scale, sh.D);
  const int rows = sh.B * sh.Hkv;
  if (sh.D == 64) return run_decode_g<T, 64>(di, sh, dense, rows, a, stream, used);
  return run_decode_g<T, 128>(di, sh, dense, rows, a, stream, used);
}

template <typename T, int D>
struct AppendKernel {
  static std::atomic<int> smem[kMaxDevices];
};
template <typename T, int D>
std::atomic<int> AppendKernel<T, D>::smem[kMaxDevices];

template <typename T, int D>
loki_status run_append(const loki_cache *c, int32_t pos, int32_t n_new, const void *k_new, const void *v_new,
                       const float *P, void *stream) {
  DevInfo di;
  loki_status s = device_info(&di);
  if (s != LOKI_OK) return s;
  AppendArgs<T> a;
  a.k_hat = static_cast<T *>(c->k_hat);
  a.v = static_cast<T *>(c->v);
  a.k_new = static_cast<const T *>(k_new);
  a.v_new = static_cast<const T *>(v_new);
  a.P = P;
  a.n_kv_heads = c->n_kv_heads;
  a.capacity = c->capacity;
  a.pos = pos;
  a.n_new = n_new;
  a.n_vec = c->batch * n_new;
  // enough CTAs to cover the SMs twice (heads x column blocks x chunks), at
  // least one 8-vector batch each
  const int col_blocks = D / kAppendCols;
  const long long base = (long long)c->n_kv_heads * col_blocks;
  const long long want = (2LL * di.sms + base - 1) / base;
  long long per = (a.n_vec + want - 1) / want;
  per = ((per + kAppendBatch - 1) / kAppendBatch) * kAppendBatch;
  if (per < kAppendBatch) per = kAppendBatch;
  a.per_cta = (int)per;
  const long long chunks = (a.n_vec + per - 1) / per;
  if (chunks > 65535 || c->n_kv_heads > 65535)
    return fail(LOKI_ERR_UNSUPPORTED, "append of %d vectors per head is too large", a.n_vec);
  const int smem = append_smem_words(D) * 4;
  s = prepare(append_kernel<T, D>, smem, AppendKernel<T, D>::smem);
  if (s != LOKI_OK) return s;
  dim3 grid((unsigned)c->n_kv_heads, (unsigned)col_blocks, (unsigned)chunks);
  append_kernel<T, D><<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "append_kernel launch");
  return LOKI_OK;
}

}  // namespace

extern "C" {

loki_status loki_append(const loki_cache *cache, int32_t pos, int32_t n_new, const void *k_new, const void *v_new,
                        const float *P, void *stream) {
  DecodeShape sh;
  loki_status s = check_cache(cache, &sh);
  if (s != LOKI_OK) return s;
  if (pos < 0 || n_new < 1 || (long long)pos + n_new > sh.Scap)
    return fail(LOKI_ERR_INVALID_ARG, "append range [%d, %d+%d) outside [0, capacity=%d)", pos, pos, n_new, sh.Scap);
  if ((long long)sh.B * n_new > (1LL << 30)) return fail(LOKI_ERR_UNSUPPORTED, "append too large");
  if (!k_new || !v_new || !P) return fail(LOKI_ERR_INVALID_ARG, "k_new, v_new or P is NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(P, 16))
    return fail(LOKI_ERR_INVALID_ARG, "k_new, v_new and P must be 16-byte aligned");
  if (cache->dtype == LOKI_F32)
    return sh.D == 64 ? run_append<float, 64>(cache, pos, n_new, k_new, v_new, P, stream)
                      : run_append<float, 128>(cache, pos, n_new, k_new, v_new, P, stream);
  return sh.D == 64 ? run_append<__nv_bfloat16, 64>(cache, pos, n_new, k_new, v_new, P, stream)
                    : run_append<__nv_bfloat16, 128>(cache, pos, n_new, k_new, v_new, P, stream);
}

loki_status loki_decode_attention(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads, const void *q,
                                  const float *P, int32_t d, int32_t k, float scale, float *out, int32_t *idx,
                                  void *stream) {
  DecodeShape sh;
  loki_status s = check_decode(cache, seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  if (d < 1 || d > sh.D) return fail(LOKI_ERR_INVALID_ARG, "d=%d outside [1, D=%d]", d, sh.D);
  if (k < 1 || k > seq_len) return fail(LOKI_ERR_INVALID_ARG, "k=%d outside [1, seq_len=%d]", k, seq_len);
  if (!idx) return fail(LOKI_ERR_INVALID_ARG, "idx is NULL");
  if (!aligned(idx, 4)) return fail(LOKI_ERR_INVALID_ARG, "idx must be 4-byte aligned");
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(cache, sh, false, q, P, d, k, scale, out, idx, stream);
  return decode_common<__nv_bfloat16>(cache, sh, false, q, P, d, k, scale, out, idx, stream);
}

loki_status dense_decode_attention(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads, const void *q,
                                   const float *P, float scale, float *out, void *stream) {
  DecodeShape sh;
  loki_status s = check_decode(cache, seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(cache, sh, true, q, P, 1, 1, scale, out, nullptr, stream);
  return decode_common<__nv_bfloat16>(cache, sh, true, q, P, 1, 1, scale, out, nullptr, stream);
}

loki_status loki_decode_launch_shape(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads, int32_t dense,
                                     int32_t *cluster_ctas, int32_t *ctas) {
  DecodeShape sh;
  loki_status s = check_cache(cache, &sh);
  if (s != LOKI_OK) return s;
  if (seq_len < 1 || seq_len > sh.Scap) return fail(LOKI_ERR_INVALID_ARG, "seq_len %d outside [1, capacity]", seq_len);
  if (n_q_heads < sh.Hkv || n_q_heads % sh.Hkv != 0) return fail(LOKI_ERR_INVALID_ARG, "bad n_q_heads");
  sh.S = seq_len;
  sh.Hq = n_q_heads;
  sh.G = n_q_heads / sh.Hkv;
  if (!cluster_ctas || !ctas) return fail(LOKI_ERR_INVALID_ARG, "output pointers are NULL");
  if (sh.G != 1 && sh.G != 2 && sh.G != 4 && sh.G != 8)
    return fail(LOKI_ERR_UNSUPPORTED, "query group size %d not supported (1, 2, 4 or 8)", sh.G);
  Plan pl;
  if (cache->dtype == LOKI_F32)
    s = decode_common<float>(cache, sh, dense != 0, nullptr, nullptr, 1, 1, 0.f, nullptr, nullptr, nullptr, &pl);
  else
    s = decode_common<__nv_bfloat16>(cache, sh, dense != 0, nullptr, nullptr, 1, 1, 0.f, nullptr, nullptr, nullptr,
                                     &pl);
  if (s != LOKI_OK) return s;
  *cluster_ctas = pl.ncta;
  *ctas = pl.ncta * sh.B * sh.Hkv;
  return LOKI_OK;
}

const char *loki_status_string(loki_status s) {
  switch (s) {
    case LOKI_OK: return "LOKI_OK";
    case LOKI_ERR_INVALID_ARG: return "LOKI_ERR_INVALID_ARG: invalid argument";
    case LOKI_ERR_UNSUPPORTED: return "LOKI_ERR_UNSUPPORTED: valid request not implemented by this build";
    case LOKI_ERR_CUDA: return "LOKI_ERR_CUDA: the CUDA runtime reported an error";
  }
  return "unknown loki_status";
}

const char *loki_last_error(void) { return g_err; }

int32_t loki_version(void) { return LOKI_VERSION; }

}  // extern "C"
