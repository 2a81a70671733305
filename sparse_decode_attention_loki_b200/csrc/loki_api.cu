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
#include "append_tc.cuh"
#include "host.h"
#include "pca.cuh"
#include "loki_step.cuh"
#include "topk_stats.cuh"

namespace loki {

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

// Launch-shape override for tests and tuning (loki_set_launch_override):
// the CTAs per row of the next launches, 0 for the planner's own choice.
// Starts from LOKI_CLUSTER, read once; the library never writes the process
// environment.
std::atomic<int> g_override{-1};
int forced_cluster() {
  int v = g_override.load(std::memory_order_relaxed);
  if (v < 0) {
    const char *s = std::getenv("LOKI_CLUSTER");
    int e = (s && *s) ? std::atoi(s) : 0;
    if (e < 0) e = 0;
    g_override.compare_exchange_strong(v, e, std::memory_order_relaxed);
    v = g_override.load(std::memory_order_relaxed);
  }
  return v;
}

std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;

bool occ_lookup(const void *kern, int dev, int ncta, int smem_q, int *n) {
  std::lock_guard<std::mutex> lk(g_occ_mu);
  for (const OccEntry &e : g_occ)
    if (e.kern == kern && e.dev == dev && e.ncta == ncta && e.smem_q == smem_q) {
      *n = e.n;
      return true;
    }
  return false;
}

void occ_store(const void *kern, int dev, int ncta, int smem_q, int n) {
  std::lock_guard<std::mutex> lk(g_occ_mu);
  g_occ.push_back(OccEntry{kern, dev, ncta, smem_q, n});
}


}  // namespace loki

namespace {

using namespace loki;

// ---------------------------------------------------------------------------
// validation shared by the decode entry points
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
  const int es = c->dtype == LOKI_F32 ? 4 : 2;
  sh->d_lr = 0;
  if (c->k_lr) {
    if (c->d_lr < 1 || c->d_lr > c->head_dim || (c->d_lr * es) % 16 != 0)
      return fail(LOKI_ERR_INVALID_ARG, "low-rank plane width d_lr=%d must be in [1, D=%d] with d_lr * %d bytes a "
                  "multiple of 16", c->d_lr, c->head_dim, es);
    if (!aligned(c->k_lr, 16)) return fail(LOKI_ERR_INVALID_ARG, "low-rank plane k_lr must be 16-byte aligned");
    sh->d_lr = c->d_lr;
  }
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

template <typename T>
loki_status decode_common(const loki_cache *c, const DecodeShape &sh, bool dense, const void *q, const float *P,
                          int32_t d, int32_t k, float scale, float *out, int32_t *idx, void *ws, void *stream,
                          Plan *used = nullptr, const VarPage &vp = VarPage()) {
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
  a.seq_lens = vp.seq_lens;
  a.ks = vp.ks;
  a.k_stride = k;
  a.table = vp.table;
  a.pages_per_seq = vp.pages_per_seq;
  a.page_shift = vp.page_shift;
  a.num_pages = vp.num_pages;
  a.k_new = static_cast<const T *>(vp.k_new);
  a.v_new = static_cast<const T *>(vp.v_new);
  a.k_lr = sh.d_lr > 0 ? static_cast<const T *>(c->k_lr) : nullptr;
  a.d_lr = sh.d_lr;
  a.lr_read = a.k_lr != nullptr && d <= sh.d_lr;
  if (sh.D == 64) return decode_td<T, 64>(dense, di, sh, a, ws, stream, used);
  return decode_td<T, 128>(dense, di, sh, a, ws, stream, used);
}

template <int D, bool PAGED>
struct AppendTcGate {
  static SmemGate gate;
};
template <int D, bool PAGED>
SmemGate AppendTcGate<D, PAGED>::gate;

template <typename T, int D, bool PAGED>
struct AppendGate {
  static SmemGate gate;
};
template <typename T, int D, bool PAGED>
SmemGate AppendGate<T, D, PAGED>::gate;

// Launch the append of a.n_vec = B * n_new vectors per KV head (a filled in
// except per_cta).
template <typename T, int D, bool PAGED>
loki_status launch_append(AppendArgs<T> a, void *stream) {
  DevInfo di;
  loki_status s = device_info(&di);
  if (s != LOKI_OK) return s;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (a.n_vec >= kTcMinVectors) {
      // a bulk append: the rotation is a GEMM per head, on the tensor cores
      auto kern = append_tc_kernel<D, PAGED>;
      s = allow_smem(kern, di, AppendTcGate<D, PAGED>::gate, false);
      if (s != LOKI_OK) return s;
      // persistent: one CTA per SM over the (head, tile) units
      const long long units = (long long)a.n_kv_heads * ((a.n_vec + kTcM - 1) / kTcM);
      if (units > INT32_MAX) return fail(LOKI_ERR_UNSUPPORTED, "bulk append of %d vectors per head is too large", a.n_vec);
      a.per_cta = 0;
      dim3 grid((unsigned)(units < di.sms ? units : di.sms), 1, 1);
      kern<<<grid, kTcThreads, TcLayout<D>::kBytes, static_cast<cudaStream_t>(stream)>>>(a);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail(e, "append_tc_kernel launch");
      return LOKI_OK;
    }
  }
  // enough CTAs to cover the SMs twice (heads x column blocks x chunks), at
  // least one 8-vector batch each
  const int col_blocks = D / kAppendCols;
  const long long base = (long long)a.n_kv_heads * col_blocks;
  const long long want = (2LL * di.sms + base - 1) / base;
  long long per = (a.n_vec + want - 1) / want;
  per = ((per + kAppendBatch - 1) / kAppendBatch) * kAppendBatch;
  if (per < kAppendBatch) per = kAppendBatch;
  a.per_cta = (int)per;
  const long long chunks = (a.n_vec + per - 1) / per;
  if (chunks > 65535 || a.n_kv_heads > 65535)
    return fail(LOKI_ERR_UNSUPPORTED, "append of %d vectors per head is too large", a.n_vec);
  const int smem = append_smem_words(D) * 4;
  s = allow_smem(append_kernel<T, D, PAGED>, di, AppendGate<T, D, PAGED>::gate, false);
  if (s != LOKI_OK) return s;
  dim3 grid((unsigned)a.n_kv_heads, (unsigned)col_blocks, (unsigned)chunks);
  append_kernel<T, D, PAGED><<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "append_kernel launch");
  return LOKI_OK;
}

template <typename T, int D>
loki_status run_append(const loki_cache *c, int32_t pos, int32_t n_new, const void *k_new, const void *v_new,
                       const float *P, void *stream) {
  AppendArgs<T> a{};
  a.k_hat = static_cast<T *>(c->k_hat);
  a.v = static_cast<T *>(c->v);
  a.k_new = static_cast<const T *>(k_new);
  a.v_new = static_cast<const T *>(v_new);
  a.P = P;
  if (c->k_lr) {
    a.k_lr = static_cast<T *>(c->k_lr);
    a.d_lr = c->d_lr;
  }
  a.n_kv_heads = c->n_kv_heads;
  a.capacity = c->capacity;
  a.pos = pos;
  a.n_new = n_new;
  a.n_vec = c->batch * n_new;
  return launch_append<T, D, false>(a, stream);
}

}  // namespace

namespace loki {

loki_status append_token(int dtype, int D, void *k_hat, void *v, void *k_lr, int d_lr, int Hkv, int capacity, int pos,
                         int B, const void *k_new, const void *v_new, const float *P, void *stream) {
  auto go = [&](auto *tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    AppendArgs<T> ap{};
    ap.k_hat = static_cast<T *>(k_hat);
    ap.v = static_cast<T *>(v);
    ap.k_new = static_cast<const T *>(k_new);
    ap.v_new = static_cast<const T *>(v_new);
    ap.P = P;
    ap.k_lr = static_cast<T *>(k_lr);
    ap.d_lr = k_lr ? d_lr : 0;
    ap.n_kv_heads = Hkv;
    ap.capacity = capacity;
    ap.pos = pos;
    ap.n_new = 1;
    ap.n_vec = B;
    return D == 64 ? launch_append<T, 64, false>(ap, stream) : launch_append<T, 128, false>(ap, stream);
  };
  return dtype == LOKI_F32 ? go(static_cast<float *>(nullptr)) : go(static_cast<__nv_bfloat16 *>(nullptr));
}

}  // namespace loki

namespace {

// ---------------------------------------------------------------------------
// Fixed scratch of loki_decode_attention_noalloc: a file-scope device array
// that every device loading this library holds until the process exits.  In
// host code its name is only a host-side stand-in; the device address comes
// from cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
std::atomic<int> g_noalloc_ready[kMaxDevices];
void *g_noalloc_addr[kMaxDevices];

loki_status noalloc_scratch(void **addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LOKI_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  if (!g_noalloc_ready[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ready[dev].load(std::memory_order_relaxed)) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
      g_noalloc_addr[dev] = p;
      g_noalloc_ready[dev].store(1, std::memory_order_release);
    }
  }
  *addr = g_noalloc_addr[dev];
  return LOKI_OK;
}

// A paged cache and its sequence table, checked and described as the
// contiguous cache the decode planner knows: B = batch, capacity =
// pages_per_seq * page_size (kernels use the pages, not the capacity).
loki_status check_paged(const loki_paged_cache *c, const loki_seq_table *q, loki_cache *flat, DecodeShape *sh,
                        int *shift) {
  if (!c || !q) return fail(LOKI_ERR_INVALID_ARG, "paged cache or sequence table is NULL");
  if (c->page_size < 1 || c->page_size > 65536 || (c->page_size & (c->page_size - 1)) != 0)
    return fail(LOKI_ERR_INVALID_ARG, "page_size %d is not a power of two in [1, 65536]", c->page_size);
  if (c->num_pages < 1) return fail(LOKI_ERR_INVALID_ARG, "num_pages %d must be >= 1", c->num_pages);
  if (q->batch < 1 || q->pages_per_seq < 1)
    return fail(LOKI_ERR_INVALID_ARG, "batch %d and pages_per_seq %d must be >= 1", q->batch, q->pages_per_seq);
  if (!q->block_table || !aligned(q->block_table, 4))
    return fail(LOKI_ERR_INVALID_ARG, "block_table must be a non-NULL 4-byte aligned device array");
  if (q->seq_lens && !aligned(q->seq_lens, 4)) return fail(LOKI_ERR_INVALID_ARG, "seq_lens must be 4-byte aligned");
  const long long cap = (long long)q->pages_per_seq * c->page_size;
  if (cap > (1LL << 30)) return fail(LOKI_ERR_UNSUPPORTED, "pages_per_seq * page_size = %lld tokens", cap);
  if (q->max_seq_len < 1 || q->max_seq_len > cap)
    return fail(LOKI_ERR_INVALID_ARG, "max_seq_len %d outside [1, pages_per_seq * page_size = %lld]", q->max_seq_len,
                cap);
  if ((long long)c->num_pages * c->n_kv_heads * c->page_size > (1LL << 31) - 1)
    return fail(LOKI_ERR_UNSUPPORTED, "page pool of more than 2^31 - 1 rows (num_pages * n_kv_heads * page_size)");
  flat->dtype = c->dtype;
  flat->batch = q->batch;
  flat->n_kv_heads = c->n_kv_heads;
  flat->head_dim = c->head_dim;
  flat->capacity = (int32_t)cap;
  flat->k_hat = c->k_hat;
  flat->v = c->v;
  flat->k_lr = c->k_lr;
  flat->d_lr = c->d_lr;
  loki_status s = check_cache(flat, sh);
  if (s != LOKI_OK) return s;
  int sft = 0;
  while ((1 << sft) < c->page_size) ++sft;
  *shift = sft;
  return LOKI_OK;
}

VarPage paging_of(const loki_paged_cache *c, const loki_seq_table *q, int shift, const int32_t *ks) {
  VarPage vp;
  vp.seq_lens = q->seq_lens;
  vp.ks = ks;
  vp.table = q->block_table;
  vp.pages_per_seq = q->pages_per_seq;
  vp.page_shift = shift;
  vp.num_pages = c->num_pages;
  return vp;
}

// PCA workspace: per-head means [H, D] then covariances [H, D, D], fp64,
// each region 256-byte aligned.
struct PcaWs {
  size_t mean, cov, total;
};
PcaWs pca_ws(long long heads, int D) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  PcaWs w;
  w.mean = 0;
  w.cov = up((size_t)heads * D * sizeof(double));
  w.total = w.cov + up((size_t)heads * D * D * sizeof(double));
  return w;
}

template <int D>
struct PcaGate {
  static SmemGate gate;
};
template <int D>
SmemGate PcaGate<D>::gate;

template <typename T, int D>
loki_status run_pca(const T *keys, int32_t H, int32_t N, float *P, double *eigvals, void *ws, void *stream) {
  DevInfo di;
  loki_status s = device_info(&di);
  if (s != LOKI_OK) return s;
  const PcaWs w = pca_ws(H, D);
  PcaArgs<T> a;
  a.keys = keys;
  a.n_heads = H;
  a.n_keys = N;
  a.mean = reinterpret_cast<double *>(static_cast<unsigned char *>(ws) + w.mean);
  a.cov = reinterpret_cast<double *>(static_cast<unsigned char *>(ws) + w.cov);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  constexpr int NT = D / kPcaTile;
  pca_mean_kernel<T, D><<<dim3((unsigned)H, NT), 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pca_mean_kernel launch");
  pca_cov_kernel<T, D><<<dim3((unsigned)H, NT * (NT + 1) / 2), 256, 0, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pca_cov_kernel launch");
  auto kern = pca_jacobi_kernel<D>;
  s = allow_smem(kern, di, PcaGate<D>::gate, false);
  if (s != LOKI_OK) return s;
  PcaEigArgs ea;
  ea.cov = a.cov;
  ea.P = P;
  ea.eigvals = eigvals;
  kern<<<(unsigned)H, kPcaThreads, PcaSmem<D>::kBytes, st>>>(ea);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pca_jacobi_kernel launch");
  return LOKI_OK;
}

}  // namespace

using namespace loki;

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

loki_status loki_decode_workspace_size(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads,
                                       size_t *bytes) {
  DecodeShape sh;
  loki_status s = check_cache(cache, &sh);
  if (s != LOKI_OK) return s;
  if (!bytes) return fail(LOKI_ERR_INVALID_ARG, "bytes is NULL");
  if (seq_len < 1 || seq_len > sh.Scap)
    return fail(LOKI_ERR_INVALID_ARG, "seq_len %d outside [1, capacity=%d]", seq_len, sh.Scap);
  if (n_q_heads < sh.Hkv || n_q_heads % sh.Hkv != 0)
    return fail(LOKI_ERR_INVALID_ARG, "n_q_heads %d is not a positive multiple of n_kv_heads %d", n_q_heads, sh.Hkv);
  *bytes = ws_layout((long long)sh.B * sh.Hkv, n_q_heads / sh.Hkv, sh.D).total;
  return LOKI_OK;
}

loki_status loki_decode_attention(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads, const void *q,
                                  const float *P, int32_t d, int32_t k, float scale, float *out, int32_t *idx,
                                  void *workspace, size_t workspace_bytes, void *stream) {
  DecodeShape sh;
  loki_status s = check_decode(cache, seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  if (d < 1 || d > sh.D) return fail(LOKI_ERR_INVALID_ARG, "d=%d outside [1, D=%d]", d, sh.D);
  if (k < 1 || k > seq_len) return fail(LOKI_ERR_INVALID_ARG, "k=%d outside [1, seq_len=%d]", k, seq_len);
  if (!idx) return fail(LOKI_ERR_INVALID_ARG, "idx is NULL");
  if (!aligned(idx, 4)) return fail(LOKI_ERR_INVALID_ARG, "idx must be 4-byte aligned");
  if (!workspace) return fail(LOKI_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(LOKI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = ws_layout((long long)sh.B * sh.Hkv, sh.G, sh.D).total;
  if (workspace_bytes < need)
    return fail(LOKI_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes this call needs",
                workspace_bytes, need);
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(cache, sh, false, q, P, d, k, scale, out, idx, workspace, stream);
  return decode_common<__nv_bfloat16>(cache, sh, false, q, P, d, k, scale, out, idx, workspace, stream);
}

loki_status loki_decode_attention_noalloc(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads,
                                          const void *q, const float *P, int32_t d, int32_t k, float scale,
                                          float *out, int32_t *idx, void *stream) {
  size_t need = 0;
  loki_status s = loki_decode_workspace_size(cache, seq_len, n_q_heads, &need);
  if (s != LOKI_OK) return s;
  // query groups of up to 4 heads rotate their queries on chip and use no
  // scratch: only groups of 8 need the array to hold their workspace
  const bool small_group = n_q_heads / cache->n_kv_heads <= 4;
  if (!small_group && need > kNoAllocScratchBytes)
    return fail(LOKI_ERR_UNSUPPORTED,
                "this call needs %zu bytes of scratch; the fixed scratch of loki_decode_attention_noalloc holds "
                "%zu (use loki_decode_attention with a workspace)",
                need, kNoAllocScratchBytes);
  void *scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != LOKI_OK) return s;
  // small groups: the decode never reads or writes the workspace, whatever
  // size loki_decode_attention would ask of a caller's one
  return loki_decode_attention(cache, seq_len, n_q_heads, q, P, d, k, scale, out, idx, scratch,
                               small_group ? need : kNoAllocScratchBytes, stream);
}

loki_status loki_device_error_count(uint32_t *count) {
  if (!count) return fail(LOKI_ERR_INVALID_ARG, "count is NULL");
  cudaError_t e = cudaMemcpyFromSymbol(count, g_loki_device_errors, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(device error count)");
  return LOKI_OK;
}

loki_status loki_topk_jaccard(const int32_t *idx_a, const int32_t *idx_b, int32_t rows, int32_t k, float *jaccard,
                              void *stream) {
  if (rows < 1 || k < 1) return fail(LOKI_ERR_INVALID_ARG, "rows=%d and k=%d must be >= 1", rows, k);
  if (!idx_a || !idx_b || !jaccard) return fail(LOKI_ERR_INVALID_ARG, "idx_a, idx_b or jaccard is NULL");
  if (!aligned(idx_a, 4) || !aligned(idx_b, 4) || !aligned(jaccard, 4))
    return fail(LOKI_ERR_INVALID_ARG, "idx_a, idx_b and jaccard must be 4-byte aligned");
  JaccardArgs a;
  a.a = idx_a;
  a.b = idx_b;
  a.out = jaccard;
  a.k = k;
  topk_jaccard_kernel<<<(unsigned)rows, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "topk_jaccard_kernel launch");
  return LOKI_OK;
}

loki_status dense_decode_attention(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads, const void *q,
                                   const float *P, float scale, float *out, void *stream) {
  DecodeShape sh;
  loki_status s = check_decode(cache, seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(cache, sh, true, q, P, 1, 1, scale, out, nullptr, nullptr, stream);
  return decode_common<__nv_bfloat16>(cache, sh, true, q, P, 1, 1, scale, out, nullptr, nullptr, stream);
}

static loki_status check_new_token(const void *k_new, const void *v_new) {
  if (!k_new || !v_new) return fail(LOKI_ERR_INVALID_ARG, "k_new or v_new is NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(LOKI_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
  return LOKI_OK;
}

loki_status loki_decode_attention_append(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads,
                                         const void *k_new, const void *v_new, const void *q, const float *P,
                                         int32_t d, int32_t k, float scale, float *out, int32_t *idx, void *workspace,
                                         size_t workspace_bytes, void *stream) {
  DecodeShape sh;
  loki_status s = check_decode(cache, seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  s = check_new_token(k_new, v_new);
  if (s != LOKI_OK) return s;
  if (d < 1 || d > sh.D) return fail(LOKI_ERR_INVALID_ARG, "d=%d outside [1, D=%d]", d, sh.D);
  if (k < 1 || k > seq_len) return fail(LOKI_ERR_INVALID_ARG, "k=%d outside [1, seq_len=%d]", k, seq_len);
  if (!idx) return fail(LOKI_ERR_INVALID_ARG, "idx is NULL");
  if (!aligned(idx, 4)) return fail(LOKI_ERR_INVALID_ARG, "idx must be 4-byte aligned");
  if (!workspace) return fail(LOKI_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(LOKI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = ws_layout((long long)sh.B * sh.Hkv, sh.G, sh.D).total;
  if (workspace_bytes < need)
    return fail(LOKI_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes this call needs",
                workspace_bytes, need);
  VarPage vp;
  vp.k_new = k_new;
  vp.v_new = v_new;
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(cache, sh, false, q, P, d, k, scale, out, idx, workspace, stream, nullptr, vp);
  return decode_common<__nv_bfloat16>(cache, sh, false, q, P, d, k, scale, out, idx, workspace, stream, nullptr, vp);
}

loki_status dense_decode_attention_append(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads,
                                          const void *k_new, const void *v_new, const void *q, const float *P,
                                          float scale, float *out, void *stream) {
  DecodeShape sh;
  loki_status s = check_decode(cache, seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  s = check_new_token(k_new, v_new);
  if (s != LOKI_OK) return s;
  VarPage vp;
  vp.k_new = k_new;
  vp.v_new = v_new;
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(cache, sh, true, q, P, 1, 1, scale, out, nullptr, nullptr, stream, nullptr, vp);
  return decode_common<__nv_bfloat16>(cache, sh, true, q, P, 1, 1, scale, out, nullptr, nullptr, stream, nullptr, vp);
}

loki_status loki_decode_launch_shape(const loki_cache *cache, int32_t seq_len, int32_t n_q_heads, int32_t k,
                                     int32_t dense, int32_t *shape) {
  DecodeShape sh;
  loki_status s = check_cache(cache, &sh);
  if (s != LOKI_OK) return s;
  if (seq_len < 1 || seq_len > sh.Scap) return fail(LOKI_ERR_INVALID_ARG, "seq_len %d outside [1, capacity]", seq_len);
  if (n_q_heads < sh.Hkv || n_q_heads % sh.Hkv != 0) return fail(LOKI_ERR_INVALID_ARG, "bad n_q_heads");
  if (!dense && (k < 1 || k > seq_len)) return fail(LOKI_ERR_INVALID_ARG, "k=%d outside [1, seq_len=%d]", k, seq_len);
  if (!shape) return fail(LOKI_ERR_INVALID_ARG, "shape is NULL");
  sh.S = seq_len;
  sh.Hq = n_q_heads;
  sh.G = n_q_heads / sh.Hkv;
  if (sh.G != 1 && sh.G != 2 && sh.G != 4 && sh.G != 8)
    return fail(LOKI_ERR_UNSUPPORTED, "query group size %d not supported (1, 2, 4 or 8)", sh.G);
  const long long rows = (long long)sh.B * sh.Hkv;
  Plan pl;
  if (cache->dtype == LOKI_F32)
    s = decode_common<float>(cache, sh, dense != 0, nullptr, nullptr, 1, 1, 0.f, nullptr, nullptr, nullptr, nullptr,
                             &pl);
  else
    s = decode_common<__nv_bfloat16>(cache, sh, dense != 0, nullptr, nullptr, 1, 1, 0.f, nullptr, nullptr, nullptr,
                                     nullptr, &pl);
  if (s != LOKI_OK) return s;
  shape[0] = dense ? 0 : pl.rot;
  shape[1] = pl.ncta;
  shape[2] = (int32_t)(rows * pl.ncta);
  shape[3] = dense ? 0 : pl.spare;
  return LOKI_OK;
}

loki_status loki_paged_append(const loki_paged_cache *cache, const loki_seq_table *seqs, const int32_t *pos,
                              int32_t n_new, const void *k_new, const void *v_new, const float *P, void *stream) {
  loki_cache flat;
  DecodeShape sh;
  int shift = 0;
  loki_status s = check_paged(cache, seqs, &flat, &sh, &shift);
  if (s != LOKI_OK) return s;
  if (!pos || !aligned(pos, 4)) return fail(LOKI_ERR_INVALID_ARG, "pos must be a non-NULL 4-byte aligned device array");
  if (n_new < 1) return fail(LOKI_ERR_INVALID_ARG, "n_new %d must be >= 1", n_new);
  if ((long long)sh.B * n_new > (1LL << 30)) return fail(LOKI_ERR_UNSUPPORTED, "append too large");
  if (!k_new || !v_new || !P) return fail(LOKI_ERR_INVALID_ARG, "k_new, v_new or P is NULL");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(P, 16))
    return fail(LOKI_ERR_INVALID_ARG, "k_new, v_new and P must be 16-byte aligned");
  auto fill = [&](auto *tag) {
    using T = std::remove_pointer_t<decltype(tag)>;
    AppendArgs<T> a{};
    a.k_hat = static_cast<T *>(cache->k_hat);
    a.v = static_cast<T *>(cache->v);
    a.k_new = static_cast<const T *>(k_new);
    a.v_new = static_cast<const T *>(v_new);
    a.P = P;
    a.n_kv_heads = sh.Hkv;
    a.capacity = flat.capacity;
    a.pos = 0;
    a.n_new = n_new;
    a.n_vec = sh.B * n_new;
    a.pos_arr = pos;
    if (cache->k_lr) {
      a.k_lr = static_cast<T *>(cache->k_lr);
      a.d_lr = cache->d_lr;
    }
    a.table = seqs->block_table;
    a.pages_per_seq = seqs->pages_per_seq;
    a.page_shift = shift;
    a.num_pages = cache->num_pages;
    return a;
  };
  if (cache->dtype == LOKI_F32) {
    const AppendArgs<float> a = fill(static_cast<float *>(nullptr));
    return sh.D == 64 ? launch_append<float, 64, true>(a, stream) : launch_append<float, 128, true>(a, stream);
  }
  const AppendArgs<__nv_bfloat16> a = fill(static_cast<__nv_bfloat16 *>(nullptr));
  return sh.D == 64 ? launch_append<__nv_bfloat16, 64, true>(a, stream)
                    : launch_append<__nv_bfloat16, 128, true>(a, stream);
}

loki_status loki_paged_decode_workspace_size(const loki_paged_cache *cache, const loki_seq_table *seqs,
                                             int32_t n_q_heads, size_t *bytes) {
  loki_cache flat;
  DecodeShape sh;
  int shift = 0;
  loki_status s = check_paged(cache, seqs, &flat, &sh, &shift);
  if (s != LOKI_OK) return s;
  return loki_decode_workspace_size(&flat, seqs->max_seq_len, n_q_heads, bytes);
}

loki_status loki_paged_decode_attention(const loki_paged_cache *cache, const loki_seq_table *seqs, int32_t n_q_heads,
                                        const void *q, const float *P, int32_t d, const int32_t *ks, int32_t k_max,
                                        float scale, float *out, int32_t *idx, void *workspace,
                                        size_t workspace_bytes, void *stream) {
  loki_cache flat;
  DecodeShape sh;
  int shift = 0;
  loki_status s = check_paged(cache, seqs, &flat, &sh, &shift);
  if (s != LOKI_OK) return s;
  s = check_decode(&flat, seqs->max_seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  if (d < 1 || d > sh.D) return fail(LOKI_ERR_INVALID_ARG, "d=%d outside [1, D=%d]", d, sh.D);
  if (k_max < 1 || k_max > sh.S) return fail(LOKI_ERR_INVALID_ARG, "k_max=%d outside [1, max_seq_len=%d]", k_max, sh.S);
  if (ks && !aligned(ks, 4)) return fail(LOKI_ERR_INVALID_ARG, "ks must be 4-byte aligned");
  if (!idx) return fail(LOKI_ERR_INVALID_ARG, "idx is NULL");
  if (!aligned(idx, 4)) return fail(LOKI_ERR_INVALID_ARG, "idx must be 4-byte aligned");
  if (!workspace) return fail(LOKI_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(LOKI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = ws_layout((long long)sh.B * sh.Hkv, sh.G, sh.D).total;
  if (workspace_bytes < need)
    return fail(LOKI_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes this call needs",
                workspace_bytes, need);
  const VarPage vp = paging_of(cache, seqs, shift, ks);
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(&flat, sh, false, q, P, d, k_max, scale, out, idx, workspace, stream, nullptr, vp);
  return decode_common<__nv_bfloat16>(&flat, sh, false, q, P, d, k_max, scale, out, idx, workspace, stream, nullptr,
                                      vp);
}

loki_status loki_paged_decode_attention_append(const loki_paged_cache *cache, const loki_seq_table *seqs,
                                               int32_t n_q_heads, const void *k_new, const void *v_new, const void *q,
                                               const float *P, int32_t d, const int32_t *ks, int32_t k_max,
                                               float scale, float *out, int32_t *idx, void *workspace,
                                               size_t workspace_bytes, void *stream) {
  loki_cache flat;
  DecodeShape sh;
  int shift = 0;
  loki_status s = check_paged(cache, seqs, &flat, &sh, &shift);
  if (s != LOKI_OK) return s;
  s = check_decode(&flat, seqs->max_seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  s = check_new_token(k_new, v_new);
  if (s != LOKI_OK) return s;
  if (sh.G > 4)
    return fail(LOKI_ERR_UNSUPPORTED, "appending in a paged Loki decode needs query groups of up to 4 heads");
  if (d < 1 || d > sh.D) return fail(LOKI_ERR_INVALID_ARG, "d=%d outside [1, D=%d]", d, sh.D);
  if (k_max < 1 || k_max > sh.S) return fail(LOKI_ERR_INVALID_ARG, "k_max=%d outside [1, max_seq_len=%d]", k_max, sh.S);
  if (ks && !aligned(ks, 4)) return fail(LOKI_ERR_INVALID_ARG, "ks must be 4-byte aligned");
  if (!idx) return fail(LOKI_ERR_INVALID_ARG, "idx is NULL");
  if (!aligned(idx, 4)) return fail(LOKI_ERR_INVALID_ARG, "idx must be 4-byte aligned");
  if (!workspace) return fail(LOKI_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(LOKI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = ws_layout((long long)sh.B * sh.Hkv, sh.G, sh.D).total;
  if (workspace_bytes < need)
    return fail(LOKI_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes this call needs",
                workspace_bytes, need);
  VarPage vp = paging_of(cache, seqs, shift, ks);
  vp.k_new = k_new;
  vp.v_new = v_new;
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(&flat, sh, false, q, P, d, k_max, scale, out, idx, workspace, stream, nullptr, vp);
  return decode_common<__nv_bfloat16>(&flat, sh, false, q, P, d, k_max, scale, out, idx, workspace, stream, nullptr,
                                      vp);
}

loki_status dense_paged_decode_attention(const loki_paged_cache *cache, const loki_seq_table *seqs,
                                         int32_t n_q_heads, const void *q, const float *P, float scale, float *out,
                                         void *stream) {
  loki_cache flat;
  DecodeShape sh;
  int shift = 0;
  loki_status s = check_paged(cache, seqs, &flat, &sh, &shift);
  if (s != LOKI_OK) return s;
  s = check_decode(&flat, seqs->max_seq_len, n_q_heads, q, P, out, &sh);
  if (s != LOKI_OK) return s;
  const VarPage vp = paging_of(cache, seqs, shift, nullptr);
  if (cache->dtype == LOKI_F32)
    return decode_common<float>(&flat, sh, true, q, P, 1, 1, scale, out, nullptr, nullptr, stream, nullptr, vp);
  return decode_common<__nv_bfloat16>(&flat, sh, true, q, P, 1, 1, scale, out, nullptr, nullptr, stream, nullptr, vp);
}

loki_status loki_pca_workspace_size(int32_t n_heads, int32_t head_dim, size_t *bytes) {
  if (!bytes) return fail(LOKI_ERR_INVALID_ARG, "bytes is NULL");
  if (n_heads < 1 || n_heads > 65535) return fail(LOKI_ERR_INVALID_ARG, "n_heads=%d outside [1, 65535]", n_heads);
  if (head_dim != 64 && head_dim != 128) return fail(LOKI_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", head_dim);
  *bytes = pca_ws(n_heads, head_dim).total;
  return LOKI_OK;
}

loki_status loki_pca_calibrate(const void *keys, int32_t dtype, int32_t n_heads, int32_t n_keys, int32_t head_dim,
                               float *P, double *eigvals, void *workspace, size_t workspace_bytes, void *stream) {
  size_t need = 0;
  loki_status s = loki_pca_workspace_size(n_heads, head_dim, &need);
  if (s != LOKI_OK) return s;
  if (dtype != LOKI_F32 && dtype != LOKI_BF16) return fail(LOKI_ERR_INVALID_ARG, "dtype %d", dtype);
  if (n_keys < 1) return fail(LOKI_ERR_INVALID_ARG, "n_keys=%d must be >= 1", n_keys);
  if ((long long)n_keys * head_dim > INT32_MAX) return fail(LOKI_ERR_UNSUPPORTED, "n_keys=%d too large", n_keys);
  if (!keys || !P || !workspace) return fail(LOKI_ERR_INVALID_ARG, "keys, P or workspace is NULL");
  if (!aligned(keys, 16) || !aligned(P, 16) || (eigvals && !aligned(eigvals, 8)))
    return fail(LOKI_ERR_INVALID_ARG, "keys and P must be 16-byte aligned, eigvals 8-byte aligned");
  if (!aligned(workspace, 256)) return fail(LOKI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < need)
    return fail(LOKI_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes this call needs",
                workspace_bytes, need);
  if (dtype == LOKI_F32)
    return head_dim == 64 ? run_pca<float, 64>(static_cast<const float *>(keys), n_heads, n_keys, P, eigvals,
                                               workspace, stream)
                          : run_pca<float, 128>(static_cast<const float *>(keys), n_heads, n_keys, P, eigvals,
                                                workspace, stream);
  return head_dim == 64 ? run_pca<__nv_bfloat16, 64>(static_cast<const __nv_bfloat16 *>(keys), n_heads, n_keys, P,
                                                     eigvals, workspace, stream)
                        : run_pca<__nv_bfloat16, 128>(static_cast<const __nv_bfloat16 *>(keys), n_heads, n_keys, P,
                                                      eigvals, workspace, stream);
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

loki_status loki_phase_stamps(int32_t dtype, int32_t head_dim, uint64_t *host, int32_t capacity, int32_t *n) {
  if (!host || !n || capacity < 1) return fail(LOKI_ERR_INVALID_ARG, "host, n and capacity >= 1 are required");
  if (head_dim != 64 && head_dim != 128) return fail(LOKI_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", head_dim);
  unsigned long long *h = reinterpret_cast<unsigned long long *>(host);
  if (dtype == LOKI_F32)
    return head_dim == 64 ? decode_phase_stamps<float, 64>(h, capacity, n)
                          : decode_phase_stamps<float, 128>(h, capacity, n);
  if (dtype == LOKI_BF16)
    return head_dim == 64 ? decode_phase_stamps<__nv_bfloat16, 64>(h, capacity, n)
                          : decode_phase_stamps<__nv_bfloat16, 128>(h, capacity, n);
  return fail(LOKI_ERR_INVALID_ARG, "dtype %d", dtype);
}

loki_status loki_set_launch_override(int32_t per_row) {
  if (per_row < 0) return fail(LOKI_ERR_INVALID_ARG, "per_row %d must be >= 0", per_row);
  g_override.store(per_row, std::memory_order_relaxed);
  return LOKI_OK;
}

const char *loki_last_error(void) { return g_err; }

int32_t loki_version(void) { return LOKI_VERSION; }

}  // extern "C"
