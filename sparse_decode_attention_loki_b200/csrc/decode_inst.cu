// Planning and launches of the decode calls for one (cache dtype, head dim)
// pair, chosen at compile time (LOKI_T_BF16 or not, LOKI_D = 64 or 128): the
// library compiles this file once per pair so that the four units build in
// parallel.  loki_api.cu validates the arguments and calls decode_td.
#include <type_traits>

#include "host.h"
#include "short_step.cuh"

#ifndef LOKI_D
#error "LOKI_D (64 or 128) must be defined"
#endif
#ifdef LOKI_T_BF16
#define LOKI_T __nv_bfloat16
#else
#define LOKI_T float
#endif

namespace loki {
namespace {

// ---------------------------------------------------------------------------
// dense decode: one cluster of ncta CTAs per (batch, KV head) row.  Among
// cluster sizes whose per-CTA share is at least kDenseMinTokens tokens and
// whose shared memory fits, take the one that keeps the most CTAs busy per
// wave of co-resident clusters (rows*n / waves); ties go to the smaller
// cluster, which spends less on the cross-CTA merge.  `forced` (the launch
// override) fixes n where it can run.
constexpr int kDenseMinTokens = 256;

template <typename Kern>
loki_status plan_dense(Kern kern, const DevInfo &di, const DecodeShape &sh, Plan *p, int forced) {
  const int rows = sh.B * sh.Hkv;
  int dev = 0;
  cudaGetDevice(&dev);
  double best = -1.0;
  Plan bp{};
  int last_smem = 0;
  for (int n = 1; n <= 16; n *= 2) {
    if (forced && n != forced) continue;
    const int chunk = (sh.S + n - 1) / n;
    if (!forced && n > 1 && chunk < kDenseMinTokens) continue;
    const int smem = decode_layout(sh.G, sh.D, chunk, false).words * 4;
    last_smem = smem;
    if (smem > di.smem_optin) continue;
    const int mc = max_active(kern, dev, n, smem, di.smem_optin);
    if (mc <= 0) continue;
    const long long waves = (rows + mc - 1) / mc;
    const double per_wave = (double)rows * n / (double)waves;
    if (per_wave > best * 1.0001) {
      best = per_wave;
      bp = Plan{n, chunk, smem, rows * n, 0, 0};
    }
  }
  if (bp.ncta == 0 && forced) return plan_dense(kern, di, sh, p, 0);  // a forced size that cannot run
  if (bp.ncta == 0)
    return fail(LOKI_ERR_UNSUPPORTED,
                "no dense launch shape fits: %d B of shared memory per CTA (limit %d) or an unschedulable cluster",
                last_smem, di.smem_optin);
  *p = bp;
  return LOKI_OK;
}

template <typename T, int D, int G, bool PAGED>
struct DenseGate {
  static SmemGate gate;
};
template <typename T, int D, int G, bool PAGED>
SmemGate DenseGate<T, D, G, PAGED>::gate;

template <typename T, int D, int G, bool PAGED>
loki_status run_dense(const DevInfo &di, const DecodeShape &sh, DecodeArgs<T> a, void *stream, Plan *used) {
  auto kern = dense_decode_kernel<T, D, G, PAGED>;
  loki_status s = allow_smem(kern, di, DenseGate<T, D, G, PAGED>::gate, true);
  if (s != LOKI_OK) return s;
  Plan pl;
  s = plan_dense(kern, di, sh, &pl, forced_cluster());
  if (s != LOKI_OK) return s;
  if (used) {  // shape query only: launch nothing
    *used = pl;
    return LOKI_OK;
  }
  a.chunk = pl.chunk;
  return launch_ex(kern, (long long)sh.B * sh.Hkv * pl.ncta, pl.smem, pl.ncta, false, a, stream,
                   "dense_decode_kernel launch");
}

// ---------------------------------------------------------------------------
// Loki step: rotate grid (query groups of 8), then the decode grid as its
// programmatic dependent: loki_short_kernel for rows of at most
// kShortMaxTokens tokens when it keeps as many CTAs per SM as the long-row
// kernel, else loki_decode_kernel.  CTAs per row (cluster
// size) of the decode kernel:
// start from the fewest CTAs whose share is at most kTargetChunk tokens (two
// CTAs then fit on an SM; more only when a share would exceed kMaxChunk), and
// take the first power of two up to 16 whose grid covers at least 80% of the
// device's co-resident CTAs, else the largest schedulable one: fewer, longer
// CTAs spend less on the cross-CTA steps.  `forced` (the launch override)
// fixes the size where it can run.
constexpr int kTargetChunk = 8192;

template <typename Kern>
loki_status plan_step(Kern kern, const DevInfo &di, const DecodeShape &sh, Plan *p, int forced, bool short_row) {
  const long long rows = (long long)sh.B * sh.Hkv;
  const int S = sh.S;
  int dev = 0;
  cudaGetDevice(&dev);
  int need = 1;
  while (need < kMaxCluster && (S + need - 1) / need > kTargetChunk) need *= 2;
  while (need > 1 && (S + need - 1) / need > kMaxChunk) need *= 2;
  if ((S + kMaxCluster - 1) / kMaxCluster > kMaxChunk)
    return fail(LOKI_ERR_UNSUPPORTED, "seq_len %d exceeds %d tokens", S, kMaxChunk * kMaxCluster);
  if (need > kMaxCluster) need = kMaxCluster;
  Plan best{};
  for (int n = 1; n <= kMaxCluster; n *= 2) {
    if (forced ? n != forced : n < need) continue;
    const int chunk = round4((S + n - 1) / n);
    if (chunk > kMaxChunk) continue;
    const int smem = (short_row ? short_smem(sh.G, sh.D, chunk, n, sh.S).words : fused_smem(sh.G, sh.D, chunk).words) * 4;
    if (smem > di.smem_optin) continue;
    const int mc = max_active(kern, dev, n, smem, di.smem_optin);
    if (mc <= 0) continue;
    best = Plan{n, chunk, smem, (int)(rows * n), sh.G > 4 ? (int)(rows * (sh.D / kRotCols)) : 0, short_row ? 1 : 0};
    if (forced || rows * 5 >= 4LL * mc) break;  // covers 80% of a wave
  }
  if (best.ncta == 0 && forced) return plan_step(kern, di, sh, p, 0, short_row);  // a forced size that cannot run
  if (best.ncta == 0)
    return fail(LOKI_ERR_UNSUPPORTED, "seq_len %d: no schedulable cluster fits the keys in shared memory", S);
  *p = best;
  return LOKI_OK;
}

template <typename T, int D, int G, bool PAGED, bool SHORT>
struct StepGate {
  static SmemGate gate;
};
template <typename T, int D, int G, bool PAGED, bool SHORT>
SmemGate StepGate<T, D, G, PAGED, SHORT>::gate;

template <typename T, int D, int G, bool PAGED>
loki_status run_step(const DevInfo &di, const DecodeShape &sh, DecodeArgs<T> da, void *ws, void *stream,
                     Plan *used) {
  auto kshort = loki_short_kernel<T, D, G, PAGED>;
  auto klong = loki_decode_kernel<T, D, G, PAGED>;
  loki_status s = allow_smem(klong, di, StepGate<T, D, G, PAGED, false>::gate, true);
  if (s != LOKI_OK) return s;
  Plan pl;
  bool short_row = sh.S <= kShortMaxTokens;
  if (short_row) {
    // the short-row kernel holds the whole row's keys in every CTA: it runs
    // only where that leaves as many CTAs per SM as the long-row kernel has
    // with the same cluster shape (measured: fewer loses to the long kernel)
    s = allow_smem(kshort, di, StepGate<T, D, G, PAGED, true>::gate, true);
    if (s != LOKI_OK) return s;
    s = plan_step(kshort, di, sh, &pl, forced_cluster(), true);
    if (s != LOKI_OK) return s;
    int dev = 0;
    cudaGetDevice(&dev);
    const int occ_short = max_active(kshort, dev, 0, pl.smem, di.smem_optin);
    const int occ_long = max_active(klong, dev, 0, fused_smem(sh.G, sh.D, pl.chunk).words * 4, di.smem_optin);
    short_row = occ_short >= occ_long;
  }
  if (!short_row) {
    s = plan_step(klong, di, sh, &pl, forced_cluster(), false);
    if (s != LOKI_OK) return s;
  }
  auto kern = short_row ? kshort : klong;
  if (used) {  // shape query only: launch nothing
    *used = pl;
    return LOKI_OK;
  }
  const long long rows = (long long)sh.B * sh.Hkv;
  const WsLayout W = ws_layout(rows, G, D);
  unsigned char *w = static_cast<unsigned char *>(ws);
  da.chunk = pl.chunk;
  StepArgs<T> a;
  a.da = da;
  a.qhat = reinterpret_cast<float *>(w + W.qhat);
  a.u = reinterpret_cast<float *>(w + W.u);
  if (!kRotateInKernel<G>) {
    s = launch_ex(loki_rotate_kernel<T, D, G>, rows * (D / kRotCols), 0, 0, false, a, stream,
                  "loki_rotate_kernel launch");
    if (s != LOKI_OK) return s;
  }
  return launch_ex(kern, rows * pl.ncta, pl.smem, pl.ncta, !kRotateInKernel<G>, a, stream,
                   "loki_decode_kernel launch");
}

// ---------------------------------------------------------------------------
template <typename T, int D, int G, bool PAGED>
loki_status dispatch_p(bool dense, const DevInfo &di, const DecodeShape &sh, const DecodeArgs<T> &a, void *ws,
                       void *stream, Plan *used) {
  if (dense) return run_dense<T, D, G, PAGED>(di, sh, a, stream, used);
  return run_step<T, D, G, PAGED>(di, sh, a, ws, stream, used);
}

template <typename T, int D, int G>
loki_status dispatch(bool dense, const DevInfo &di, const DecodeShape &sh, const DecodeArgs<T> &a, void *ws,
                     void *stream, Plan *used) {
  if (!dense && a.k_new != nullptr && !kRotateInKernel<G>) {
    // the decode kernel appends only for query groups of up to 4 heads: for
    // 8, the append kernel writes the new token first (contiguous caches)
    if (a.table != nullptr)
      return fail(LOKI_ERR_UNSUPPORTED, "appending in a paged Loki decode needs query groups of up to 4 heads");
    if (used == nullptr) {
      loki_status s = append_token(std::is_same<T, float>::value ? LOKI_F32 : LOKI_BF16, D,
                                   const_cast<T *>(a.k_hat), const_cast<T *>(a.v), const_cast<T *>(a.k_lr), a.d_lr,
                                   a.n_kv_heads, a.capacity, sh.S - 1, sh.B, a.k_new, a.v_new, a.P, stream);
      if (s != LOKI_OK) return s;
    }
    DecodeArgs<T> rest = a;
    rest.k_new = rest.v_new = nullptr;
    return dispatch_p<T, D, G, false>(dense, di, sh, rest, ws, stream, used);
  }
  if (a.table != nullptr) return dispatch_p<T, D, G, true>(dense, di, sh, a, ws, stream, used);
  return dispatch_p<T, D, G, false>(dense, di, sh, a, ws, stream, used);
}

}  // namespace

template <typename T, int D>
loki_status decode_td(bool dense, const DevInfo &di, const DecodeShape &sh, const DecodeArgs<T> &a, void *ws,
                      void *stream, Plan *used) {
  switch (sh.G) {
    case 1: return dispatch<T, D, 1>(dense, di, sh, a, ws, stream, used);
    case 2: return dispatch<T, D, 2>(dense, di, sh, a, ws, stream, used);
    case 4: return dispatch<T, D, 4>(dense, di, sh, a, ws, stream, used);
    case 8: return dispatch<T, D, 8>(dense, di, sh, a, ws, stream, used);
  }
  return fail(LOKI_ERR_UNSUPPORTED, "group size %d", sh.G);
}

template <typename T, int D>
loki_status decode_phase_stamps(unsigned long long *host, int32_t capacity, int32_t *n) {
#ifdef LOKI_PHASE_STAMPS
  const int m = capacity < kMaxStampCtas ? capacity : kMaxStampCtas;
  cudaError_t e = cudaMemcpyFromSymbol(host, g_phase_stamps, (size_t)m * sizeof(g_phase_stamps[0]));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(phase stamps)");
  *n = m;
  return LOKI_OK;
#else
  (void)host;
  (void)capacity;
  *n = 0;
  return fail(LOKI_ERR_UNSUPPORTED, "this library was built without LOKI_PHASE_STAMPS");
#endif
}

template loki_status decode_phase_stamps<LOKI_T, LOKI_D>(unsigned long long *, int32_t, int32_t *);
template loki_status decode_td<LOKI_T, LOKI_D>(bool, const DevInfo &, const DecodeShape &,
                                               const DecodeArgs<LOKI_T> &, void *, void *, Plan *);

}  // namespace loki
