// Building blocks of the Loki decode step and the dense decode kernel (sm_100a).
//
// Method ("Loki: Low-rank Keys for Efficient Sparse Attention", atlas.scime.ai
// summary, section "Approach"): rotate the query into the PCA basis, rank every
// cached token on the first d principal dimensions, keep the top k tokens and
// compute exact softmax attention over them.  The dense kernel is the "Full
// Attention" baseline (same page, "Experimental setup").
//
// This file holds the pieces: token addressing (contiguous or paged caches),
// the query rotation, the low-rank score stream, the gather/stream attention
// loops (CUDA cores, or warp-level tensor cores for query groups of 4+), the
// cluster log-sum-exp combine and the dense decode kernel.  loki_step.cuh
// chains them, with the cluster top-k select, into the two kernels of one
// Loki step.
//
// Dense decode: one thread-block cluster of `ncta` CTAs owns one (batch, KV
// head) row; CTA r streams the contiguous token range [r*chunk, (r+1)*chunk)
// of K_hat and V through a per-warp cp.async ring with an online softmax per
// query head, and the cluster merges the CTAs' (max, sum, acc) states through
// distributed shared memory.  No workspace and no global atomics.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace loki {

template <typename T>
struct DecodeArgs {
  const T *k_hat;      // [B, Hkv, S_cap, D]; paged: [num_pages, Hkv, page_size, D]
  const T *v;          // same layout as k_hat
  const T *q;          // [B, Hq, D]
  const float *P;      // [Hkv, D, D]
  float *out;          // [B, Hq, D]
  int32_t *idx;        // [B, Hkv, k]
  int32_t n_kv_heads;
  int32_t capacity;
  int32_t seq_len;
  int32_t d;
  int32_t k;
  int32_t chunk;       // tokens per CTA
  int32_t lpt;         // 16-byte chunks per token in the score stream (power of two)
  int32_t nck;         // chunks that hold the first d dims: ceil(d / elements per chunk)
  float scale_log2;    // softmax scale * log2(e)
  // per-sequence lengths (null: every row has seq_len tokens and k picks);
  // seq_len and k are then the largest values, and idx rows are k_stride long
  const int32_t *seq_lens;  // [B] or null
  const int32_t *ks;        // [B] or null
  int32_t k_stride;         // entries per idx row (= k without per-sequence k)
  // paged cache (used by the PAGED instantiations only)
  const int32_t *table;     // [B, pages_per_seq] page ids
  int32_t pages_per_seq;
  int32_t page_shift;       // page size = 1 << page_shift tokens
  int32_t num_pages;
  // a new token of every row, appended by the decode call itself at the
  // row's last attended position (null: no append)
  const T *k_new;           // [B, Hkv, D], not rotated
  const T *v_new;           // [B, Hkv, D]
  // the cache's low-rank key plane (null: none), a copy of k_hat[..., :d_lr]
  // in the layout of k_hat with rows of d_lr: [B, Hkv, S_cap, d_lr], or
  // [num_pages, Hkv, page_size, d_lr] for paged pools.  Written with every
  // appended key; the score stream reads it when lr_read (d <= d_lr).
  const T *k_lr;
  int32_t d_lr;
  bool lr_read;
};

// Tokens of one (batch, KV head) row, by position.  Contiguous caches: rows
// of [B, Hkv, S_cap, D].  Paged caches: token t lives in page
// table[t >> shift] (clamped into the pool) at slot t & (page - 1), the pool
// laid out [num_pages, Hkv, page, D].
template <typename T, int D, bool PAGED>
struct Rows {
  const T *k, *v;        // contiguous: the row's token 0; paged: the pools
  const T *s;            // the same for the rows the score stream reads (k or the plane)
  T *lr;                 // the same for the low-rank plane, or null
  int32_t sstride;       // elements per score row (D, or d_lr for the plane)
  int32_t d_lr;          // width of the low-rank plane
  const int32_t *table;  // paged: this sequence's page ids
  int32_t shift, hkv, g, last_page;
  __device__ __forceinline__ size_t off(int t) const {
    if constexpr (!PAGED) {
      return (size_t)t * D;
    } else {
      const int p = min(max(__ldg(table + (t >> shift)), 0), last_page);
      return ((((size_t)p * hkv + g) << shift) + (size_t)(t & ((1 << shift) - 1))) * D;
    }
  }
  __device__ __forceinline__ const T *key(int t) const { return k + off(t); }
  __device__ __forceinline__ const T *val(int t) const { return v + off(t); }
  // paged: the row of the pools that holds token t (off(t) / D)
  __device__ __forceinline__ int phys(int t) const {
    const int p = min(max(__ldg(table + (t >> shift)), 0), last_page);
    return ((p * hkv + g) << shift) + (t & ((1 << shift) - 1));
  }
  // token t's row index from the bases k, v, s and lr: t (contiguous) or
  // its pool row (paged)
  __device__ __forceinline__ int row_of(int t) const {
    if constexpr (!PAGED) return t;
    else return phys(t);
  }
  // the first dims of token t's key as the score stream reads them: the
  // low-rank plane's row when the call reads the plane, else the k_hat row
  __device__ __forceinline__ const T *skey(int t) const { return s + (size_t)row_of(t) * sstride; }
};

template <typename T, int D, bool PAGED>
__device__ __forceinline__ Rows<T, D, PAGED> make_rows(const DecodeArgs<T> &a, int b, int g) {
  Rows<T, D, PAGED> r;
  if constexpr (PAGED) {
    r.k = a.k_hat;
    r.v = a.v;
    r.table = a.table + (size_t)b * a.pages_per_seq;
    r.shift = a.page_shift;
    r.hkv = a.n_kv_heads;
    r.g = g;
    r.last_page = a.num_pages - 1;
    r.lr = const_cast<T *>(a.k_lr);
    r.d_lr = a.k_lr ? a.d_lr : 0;
    r.s = a.lr_read ? r.lr : r.k;
    r.sstride = a.lr_read ? a.d_lr : D;
  } else {
    const size_t row = (size_t)b * a.n_kv_heads + g;
    const size_t off = row * a.capacity * D;
    r.k = a.k_hat + off;
    r.v = a.v + off;
    r.lr = a.k_lr ? const_cast<T *>(a.k_lr) + row * a.capacity * a.d_lr : nullptr;
    r.d_lr = a.k_lr ? a.d_lr : 0;
    r.s = a.lr_read ? r.lr : r.k;
    r.sstride = a.lr_read ? a.d_lr : D;
    r.table = nullptr;
    r.shift = r.hkv = r.g = r.last_page = 0;
  }
  return r;
}

// The page pools seen as one contiguous row array (row r at r * D): the
// gather of a paged cache addresses physical rows (Rows::phys) through it.
template <typename T, int D>
__device__ __forceinline__ Rows<T, D, false> pool_rows(const DecodeArgs<T> &a) {
  Rows<T, D, false> r;
  r.k = a.k_hat;
  r.v = a.v;
  r.s = a.k_hat;
  r.lr = nullptr;
  r.sstride = D;
  r.d_lr = 0;
  r.table = nullptr;
  r.shift = r.hkv = r.g = r.last_page = 0;
  return r;
}

// Tokens attended by batch entry b: its own length when lengths are given
// (clamped into [1, seq_len]), else seq_len.
template <typename T>
__device__ __forceinline__ int row_seq_len(const DecodeArgs<T> &a, int b) {
  return a.seq_lens ? min(max(__ldg(a.seq_lens + b), 1), a.seq_len) : a.seq_len;
}
// Tokens selected for batch entry b: its own k when given, else k; clamped
// into [1, min(S_b, k)].
template <typename T>
__device__ __forceinline__ int row_k(const DecodeArgs<T> &a, int b, int S_b) {
  return a.ks ? min(max(__ldg(a.ks + b), 1), min(S_b, a.k)) : min(S_b, a.k);
}

// ---------------------------------------------------------------------------
// shared memory
// Every warp streams through its own slice of the ring: kStages stages of
// kWarpStageBytes, kStages-1 of them in flight while it computes on one.
// Warps synchronise only with __syncwarp() inside the streams.
constexpr int kStages = 4;
constexpr int kWarpStageBytes = 2048;
constexpr int kWarpRingBytes = kStages * kWarpStageBytes;
constexpr int kRingWords = kWarps * kWarpRingBytes / 4;

__host__ __device__ inline int round4(int x) { return (x + 3) & ~3; }

// Words of the receive buffer of the pushed cluster merge (push_state).
constexpr int kPushRecvWords = 1088;

// rotation scratch: q staging + partial dot products
// rotation scratch: G query heads and one appended key, then per-part sums
__host__ __device__ constexpr int rot_words(int G, int D) { return (G + 1) * D * (1 + kThreads / D); }

struct SmemLayout {
  int qhat, u, pm, pl, pacc, ctl, slots, ring, keys, recv, words;
};

// Layout in 4-byte words, identical on host and device.  `slots` serves as
// the rotation scratch and then as the bf16 query tiles of the tensor-core
// attention; the ring also holds the per-warp softmax states after the
// attention loop.  `ids`: the attention kernel of the Loki step keeps its
// share of the selected indices in the `keys` region (chunk words).
__host__ __device__ inline SmemLayout decode_layout(int G, int D, int chunk, bool ids) {
  SmemLayout L;
  int o = 0;
  L.qhat = o;  o += G * D;
  L.u = o;     o += round4(D);
  L.pm = o;    o += 16;
  L.pl = o;    o += 16;
  L.pacc = o;  o += G * D;
  L.ctl = o;   o += 128;
  L.slots = o;
  {
    const int r = rot_words(G, D);
    const int q = 8 * D;  // bf16 query tiles of the tensor-core attention: 2 x 8 rows x D
    o += round4(r > q ? r : q);
  }
  L.ring = o;  o += kRingWords;
  L.keys = o;  o += ids ? round4(chunk) : 0;
  L.recv = o;  o += kPushRecvWords;
  L.words = o;
  return L;
}

// ctl word offsets (per CTA)
constexpr int kCtlWarpGt = 48;    // [48..55]
constexpr int kCtlWarpEq = 56;    // [56..63]
static_assert(kWarps == 8, "ctl layout assumes 8 warps");

// ---------------------------------------------------------------------------
// 1. query rotation: q_hat_h = q_h . P_g for the G heads of KV head g, and
//    u = sum_h q_hat_h[:d] (zero beyond d).  q_hat is then pre-scaled by
//    scale*log2(e) for the log2-domain softmax.  The loads of P are issued
//    first; `after_loads()` runs while they are in flight (the caller puts its
//    first stream stages in flight there).  Ends with __syncthreads().
template <typename T, int D, int G, typename F>
__device__ __forceinline__ void rotate_queries(const DecodeArgs<T> &a, int b, int g,
                                               float *qhat, float *u, float *scratch,
                                               bool want_u, F &&after_loads, const T *xk = nullptr,
                                               float *xk_hat = nullptr) {
  const int tid = threadIdx.x;
  const int Hq = a.n_kv_heads * G;
  const T *qg = a.q + ((size_t)b * Hq + (size_t)g * G) * D;
  constexpr int PARTS = kThreads / D;
  constexpr int IPP = D / PARTS;
  constexpr int NH = G + 1;  // query heads, then the appended key (when xk)
  const int j = tid % D, part = tid / D;
  const float *Pg = a.P + (size_t)g * D * D + (size_t)part * IPP * D + j;
  float pv[IPP];
#pragma unroll
  for (int ii = 0; ii < IPP; ++ii) pv[ii] = __ldg(Pg + (size_t)ii * D);
  float *qs = scratch;  // [NH][D]
  for (int i = tid; i < G * D; i += kThreads) qs[i] = to_f32(qg[i]);
  if (xk != nullptr)
    for (int i = tid; i < D; i += kThreads) qs[G * D + i] = to_f32(xk[i]);
  after_loads();
  __syncthreads();
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
  float accx = 0.f;
#pragma unroll
  for (int ii = 0; ii < IPP; ++ii) {
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = fmaf(qs[h * D + part * IPP + ii], pv[ii], acc[h]);
  }
  if (xk != nullptr) {
#pragma unroll
    for (int ii = 0; ii < IPP; ++ii) accx = fmaf(qs[G * D + part * IPP + ii], pv[ii], accx);
  }
  float *red = scratch + NH * D;  // [PARTS][NH][D]
#pragma unroll
  for (int h = 0; h < G; ++h) red[(part * NH + h) * D + j] = acc[h];
  if (xk != nullptr) red[(part * NH + G) * D + j] = accx;
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D, jj = e % D;
    float s = 0.f;
#pragma unroll
    for (int p = 0; p < PARTS; ++p) s += red[(p * NH + h) * D + jj];
    qhat[e] = s;
  }
  if (xk != nullptr) {
    for (int jj = tid; jj < D; jj += kThreads) {
      float s = 0.f;
#pragma unroll
      for (int p = 0; p < PARTS; ++p) s += red[(p * NH + G) * D + jj];
      xk_hat[jj] = s;
    }
  }
  __syncthreads();
  if (want_u) {
    for (int jj = tid; jj < D; jj += kThreads) {
      float s = 0.f;
      if (jj < a.d) {
#pragma unroll
        for (int h = 0; h < G; ++h) s += qhat[h * D + jj];
      }
      u[jj] = s;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) qhat[e] *= a.scale_log2;
  __syncthreads();
}

// Write the appended token of row (b, g) into the cache at position t: its
// rotated key xk_hat rounded to the cache dtype (xk_hat then holds the
// rounded values, as fp32), the first d_lr of them into the low-rank plane
// when the cache has one, and its value.  The cache is the caller's
// writable memory; Rows hands out read pointers.  Ends with __syncthreads().
template <typename T, int D, bool PAGED>
__device__ __forceinline__ void store_appended(const DecodeArgs<T> &a, const Rows<T, D, PAGED> &rows, int b, int g,
                                               int t, float *xk_hat) {
  T *kd = const_cast<T *>(rows.key(t));
  T *vd = const_cast<T *>(rows.val(t));
  T *ld = rows.lr ? rows.lr + (size_t)rows.row_of(t) * rows.d_lr : nullptr;
  const T *vs = a.v_new + ((size_t)b * a.n_kv_heads + g) * D;
  for (int i = threadIdx.x; i < D; i += kThreads) {
    T r;
    from_f32(xk_hat[i], &r);
    kd[i] = r;
    if (ld != nullptr && i < rows.d_lr) ld[i] = r;
    xk_hat[i] = to_f32(r);
    vd[i] = vs[i];
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// 2. low-rank score stream.  The CTA's tokens are cut into blocks of
//    TS = SB/(16*LPT) tokens; warp w streams blocks w, w+8, ... through its
//    own ring slice of NS stages of SB bytes.  Token t of a block keeps its
//    LPT 16-byte chunks at byte (t*LPT + c)*16 of the stage; chunks c >= nck
//    (beyond the first d dims) are neither copied nor used.  Each score
//    becomes an order-preserving key in keys[].
template <typename T, int D, int LPT, int SB = kWarpStageBytes, int NS = kStages>
struct ScoreStream {
  static constexpr int VEC = VecN<T>::value;
  static constexpr int TS = SB / (16 * LPT);  // tokens per warp stage
  static constexpr int TPW = 32 / LPT;        // tokens per warp instruction
  static_assert(TS >= TPW && TS % TPW == 0, "a stage must hold whole warp steps");

  template <class R>
  __device__ __forceinline__ static void issue(const R &rows, int t0, int len, int nck, int s,
                                               unsigned char *wring) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char *st = wring + (s % NS) * SB;
    const int base = (s * kWarps + warp) * TS;
#pragma unroll
    for (int it = 0; it < TS * LPT / 32; ++it) {
      const int q = it * 32 + lane;
      const int t = q / LPT, c = q % LPT;
      if (base + t < len && c < nck) cp_async16(st + q * 16, rows.skey(t0 + base + t) + c * VEC);
    }
  }

  // Score of token t of a stage: its nck chunks dotted with u, summed over the
  // LPT lanes that share the token (every lane of the group gets the sum).
  __device__ __forceinline__ static float dot_chunk(const unsigned char *st, int t, int c, int nck,
                                                    const float (&uv)[VEC]) {
    float sc = 0.f;
    if (c < nck) {
      const uint4 r = *reinterpret_cast<const uint4 *>(st + (t * LPT + c) * 16);
      float f[VEC];
      unpack16(r, f);
#pragma unroll
      for (int y = 0; y < VEC; ++y) sc = fmaf(uv[y], f[y], sc);
    }
#pragma unroll
    for (int off = LPT / 2; off > 0; off >>= 1) sc += __shfl_xor_sync(kFull, sc, off);
    return sc;
  }

  // keys[token] = score_key(score) for the tokens of stage s, and bin
  // key >> HSHIFT of the skewed histogram hist (see hskew) += 1 for each
  // (no histogram when HSHIFT is 32).
  template <int HSHIFT>
  __device__ __forceinline__ static void consume_keys(int len, int nck, int s, const unsigned char *wring,
                                                      const float (&uv)[VEC], uint32_t *keys, uint32_t *hist) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned char *st = wring + (s % NS) * SB;
    const int c = lane % LPT;
    const int base = (s * kWarps + warp) * TS;
#pragma unroll
    for (int step = 0; step < TS / TPW; ++step) {
      const int t = step * TPW + lane / LPT;
      const float sc = dot_chunk(st, t, c, nck, uv);
      if (c == 0 && base + t < len) {
        const uint32_t key = score_key(sc);
        keys[base + t] = key;
        if constexpr (HSHIFT < 32) atomicAdd(&hist[hskew((int)(key >> HSHIFT))], 1u);
      }
    }
  }

  __device__ __forceinline__ static int warp_stages(int len) {
    const int warp = threadIdx.x >> 5;
    const int blocks = (len + TS - 1) / TS;
    return blocks > warp ? (blocks - warp + kWarps - 1) / kWarps : 0;
  }
};

// Prologue: put the first NS-1 stages of this warp in flight.
template <typename T, int D, int LPT, int SB = kWarpStageBytes, int NS = kStages, class R>
__device__ __forceinline__ void score_prologue(const R &rows, int t0, int len, int nck, unsigned char *ring) {
  using SS = ScoreStream<T, D, LPT, SB, NS>;
  unsigned char *wring = ring + (threadIdx.x >> 5) * (SB * NS);
#pragma unroll
  for (int s = 0; s < NS - 1; ++s) {
    SS::issue(rows, t0, len, nck, s, wring);
    cp_async_commit();
  }
}

// The key stream: leaves score_key(score) of every token of [t0, t0+len) in
// keys[] and counts each key's top bits in the skewed histogram hist.  Ends
// with __syncthreads().
template <typename T, int D, int LPT, int SB, int NS, int HSHIFT, class R>
__device__ __forceinline__ void score_keys_loop(const R &rows, int t0, int len, int nck, unsigned char *ring,
                                                const float *u, uint32_t *keys, uint32_t *hist) {
  using SS = ScoreStream<T, D, LPT, SB, NS>;
  constexpr int VEC = VecN<T>::value;
  unsigned char *wring = ring + (threadIdx.x >> 5) * (SB * NS);
  const int c = (threadIdx.x & 31) % LPT;
  float uv[VEC];
#pragma unroll
  for (int y = 0; y < VEC; ++y) uv[y] = u[(c * VEC + y) % D];
  const int ns = SS::warp_stages(len);
  for (int s = 0; s < ns; ++s) {
    // NS-1 stages in flight while stage s lands (refilling the slot of stage
    // s-1 before this wait, NS in flight, measured slower on the long rows)
    cp_async_wait<NS - 2>();
    __syncwarp();
    SS::issue(rows, t0, len, nck, s + NS - 1, wring);
    cp_async_commit();
    SS::template consume_keys<HSHIFT>(len, nck, s, wring, uv, keys, hist);
  }
  cp_async_wait<0>();
  __syncthreads();
}

#define LOKI_LPT_DISPATCH(lpt, MAXL, CALL)                 \
  switch (lpt) {                                           \
    case 1: { constexpr int L_ = 1; CALL; } break;         \
    case 2: { constexpr int L_ = 2; CALL; } break;         \
    case 4: { constexpr int L_ = 4; CALL; } break;         \
    case 8: { constexpr int L_ = 8; CALL; } break;         \
    case 16:                                               \
      if constexpr (MAXL >= 16) { constexpr int L_ = 16; CALL; } \
      break;                                               \
    default:                                               \
      if constexpr (MAXL >= 32) { constexpr int L_ = 32; CALL; } \
      break;                                               \
  }

// ---------------------------------------------------------------------------
// 3. the outcome of a radix select, as seen by one CTA: its selected set is
//    {key : key & mask > prefix} plus its first `take` keys (in token order)
//    with key & mask == prefix, written from position `offset` of the row.
struct SelectState {
  uint32_t prefix, mask, take, offset;
};

// ---------------------------------------------------------------------------
// 4. exact attention over `cnt` rows -- gathered through ids[] (shared memory,
//    already clamped into the row) or the contiguous rows tok0 .. tok0+cnt-1.
//    Rows are cut into blocks of TA = kWarpStageBytes/(2*row bytes); warp w
//    streams blocks w, w+8, ... through its ring slice, each row as its K row
//    followed by its V row.  D/VEC lanes share a row; each lane keeps an online
//    softmax (max, sum, acc over its VEC dims) per query head.  Leaves the
//    CTA's merged state in pm/pl/pacc (not normalised).
template <typename T, int D, bool GATHER>
struct RowStream {
  static constexpr int VEC = VecN<T>::value;
  static constexpr int RB = D * (int)sizeof(T);  // bytes per row
  static constexpr int CPR = RB / 16;            // chunks per row
  static constexpr int TA = kWarpStageBytes / (2 * RB);

  template <class R>
  __device__ __forceinline__ static void issue(const R &rows, const int32_t *ids, int tok0, int cnt, int s,
                                               unsigned char *wring) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char *st = wring + (s % kStages) * kWarpStageBytes;
    const int base = (s * kWarps + warp) * TA;
#pragma unroll
    for (int it = 0; it < TA * 2 * CPR / 32; ++it) {
      const int q = it * 32 + lane;
      const int t = q / (2 * CPR), c = q % (2 * CPR);
      const int i = base + t;
      if (i < cnt) {
        const int tok = GATHER ? ids[i] : tok0 + i;
        const T *src = (c < CPR ? rows.k : rows.v) + rows.off(tok) + (c % CPR) * VEC;
        cp_async16(st + q * 16, src);
      }
    }
  }

  __device__ __forceinline__ static int warp_stages(int cnt) {
    const int warp = threadIdx.x >> 5;
    const int blocks = (cnt + TA - 1) / TA;
    return blocks > warp ? (blocks - warp + kWarps - 1) / kWarps : 0;
  }
};

template <typename T, int D, bool GATHER, class R>
__device__ __forceinline__ void attend_prologue(const R &rows, const int32_t *ids, int tok0, int cnt,
                                                unsigned char *ring) {
  unsigned char *wring = ring + (threadIdx.x >> 5) * kWarpRingBytes;
  // a share that fits the ring goes in flight whole: one memory round trip
  const bool whole = cnt <= kStages * kWarps * RowStream<T, D, GATHER>::TA;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    RowStream<T, D, GATHER>::issue(rows, ids, tok0, cnt, s, wring);
    cp_async_commit();
  }
  if (whole) {
    RowStream<T, D, GATHER>::issue(rows, ids, tok0, cnt, kStages - 1, wring);
    cp_async_commit();
  }
}

template <typename T, int D, int G, bool GATHER, class R>
__device__ __forceinline__ void attend_loop(const R &rows, const int32_t *ids, int tok0, int cnt,
                                            const float *qhat, unsigned char *ring, float *pm, float *pl,
                                            float *pacc) {
  using RS = RowStream<T, D, GATHER>;
  constexpr int VEC = RS::VEC;
  constexpr int LPR = D / VEC;
  constexpr int RG = 32 / LPR;                  // rows per warp instruction
  constexpr int U = RS::TA / RG;                // rows per lane group per stage
  static_assert(RS::TA % RG == 0, "a stage must be a whole number of warp steps");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % LPR, grp = lane / LPR;
  unsigned char *wring = ring + warp * kWarpRingBytes;

  float qv[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int x = 0; x < VEC; ++x) qv[h][x] = qhat[h * D + sub * VEC + x];
  float m[G], l[G], acc[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int x = 0; x < VEC; ++x) acc[h][x] = 0.f;
  }

  const int ns = RS::warp_stages(cnt);
  const bool whole = cnt <= kStages * kWarps * RS::TA;  // the prologue issued every stage
  for (int s = 0; s < ns; ++s) {
    if (whole) {
      if (s == 0) cp_async_wait<0>();
      __syncwarp();
    } else {
      __syncwarp();  // stage s-1's slot is consumed: refill it before waiting for stage s
      RS::issue(rows, ids, tok0, cnt, s + kStages - 1, wring);
      cp_async_commit();
      cp_async_wait<kStages - 1>();
      __syncwarp();
    }
    const unsigned char *st = wring + (s % kStages) * kWarpStageBytes;
    const int base = (s * kWarps + warp) * RS::TA;
    float lg[U][G];
    bool ok[U];
#pragma unroll
    for (int x = 0; x < U; ++x) {
      const int t = x * RG + grp;
      ok[x] = base + t < cnt;
      // rows past cnt were never copied: read zeros instead of stale memory
      const uint4 kr = ok[x] ? *reinterpret_cast<const uint4 *>(st + t * 2 * RS::RB + sub * 16)
                             : make_uint4(0u, 0u, 0u, 0u);
      float f[VEC];
      unpack16(kr, f);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float a = 0.f;
#pragma unroll
        for (int y = 0; y < VEC; ++y) a = fmaf(qv[h][y], f[y], a);
        lg[x][h] = a;
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
      for (int x = 0; x < U; ++x)
#pragma unroll
        for (int h = 0; h < G; ++h) lg[x][h] += __shfl_xor_sync(kFull, lg[x][h], off);
    float p[U][G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = m[h];
#pragma unroll
      for (int x = 0; x < U; ++x)
        if (ok[x]) mx = fmaxf(mx, lg[x][h]);
      const float mref = (mx == -INFINITY) ? 0.f : mx;
      const float corr = exp2f(m[h] - mref);
      l[h] *= corr;
#pragma unroll
      for (int y = 0; y < VEC; ++y) acc[h][y] *= corr;
#pragma unroll
      for (int x = 0; x < U; ++x) {
        p[x][h] = ok[x] ? exp2f(lg[x][h] - mref) : 0.f;
        l[h] += p[x][h];
      }
      m[h] = mx;
    }
#pragma unroll
    for (int x = 0; x < U; ++x) {
      const int t = x * RG + grp;
      const uint4 vr = ok[x] ? *reinterpret_cast<const uint4 *>(st + t * 2 * RS::RB + RS::RB + sub * 16)
                             : make_uint4(0u, 0u, 0u, 0u);
      float f[VEC];
      unpack16(vr, f);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int y = 0; y < VEC; ++y) acc[h][y] = fmaf(p[x][h], f[y], acc[h][y]);
    }
  }
  cp_async_wait<0>();

  // merge the row groups of the warp (lanes that share `sub`)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mo = __shfl_xor_sync(kFull, m[h], off);
      const float lo = __shfl_xor_sync(kFull, l[h], off);
      const float mx = fmaxf(m[h], mo);
      const float mref = (mx == -INFINITY) ? 0.f : mx;
      const float c1 = exp2f(m[h] - mref), c2 = exp2f(mo - mref);
      l[h] = l[h] * c1 + lo * c2;
#pragma unroll
      for (int y = 0; y < VEC; ++y) {
        const float ao = __shfl_xor_sync(kFull, acc[h][y], off);
        acc[h][y] = acc[h][y] * c1 + ao * c2;
      }
      m[h] = mx;
    }
  }
  __syncthreads();  // every warp is done with the ring: it now holds the per-warp states
  float *wpart = reinterpret_cast<float *>(ring);  // [kWarps][G][D+2]
  if (grp == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float *wp = wpart + (warp * G + h) * (D + 2);
#pragma unroll
      for (int y = 0; y < VEC; ++y) wp[sub * VEC + y] = acc[h][y];
      if (sub == 0) {
        wp[D] = m[h];
        wp[D + 1] = l[h];
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D, dim = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wpart[(w * G + h) * (D + 2) + D]);
    const float mref = (M == -INFINITY) ? 0.f : M;
    float A = 0.f, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float *wp = wpart + (w * G + h) * (D + 2);
      const float c = exp2f(wp[D] - mref);
      A = fmaf(c, wp[dim], A);
      Ls = fmaf(c, wp[D + 1], Ls);
    }
    pacc[e] = A;
    if (dim == 0) {
      pm[h] = M;
      pl[h] = Ls;
    }
  }
}

// ---------------------------------------------------------------------------
// 5'. exact attention for bf16 caches on the tensor cores (warp-level mma.sync,
//    bf16 operands, fp32 accumulation).  Rows are cut into tiles of 8 tokens;
//    warp w streams tiles w, w+8, ... through its ring slice (cp.async, zero
//    fill past cnt).  In a tile, token r's record is its K row then its V row,
//    16-byte chunk c stored at chunk (c & ~7) | ((c ^ r) & 7) so that the eight
//    rows an ldmatrix reads fall in distinct bank groups.  Per tile:
//      logits  S[16 x 8] = Q[16 x D] . K^T   (rows: query heads, zero-padded
//              to 16; columns: the 8 tokens; q_hat split into bf16 hi + lo);
//      output  O^T[D x 8] += V^T[D x 8] . P^T[8 x 8]  (rows: dims; columns:
//              query heads, padded to 8; P split into bf16 hi + lo), where the
//              P fragment is exactly the S accumulator of the same lane.
//    Thread (g = lane/4, t = lane%4) owns head g's logits for tokens 2t, 2t+1
//    and the output of heads 2t, 2t+1 at dims 16j+g, 16j+g+8.
template <int D, int G, bool GATHER>
struct MmaRowStream {
  static constexpr int RB = D * 2;            // bytes per row
  static constexpr int REC = 2 * RB;          // K row + V row
  static constexpr int CPT = REC / 16;        // chunks per token record
  static constexpr int TILE = 8;
  static constexpr int TB = TILE * REC;       // bytes per tile
  static constexpr int NST = kWarpRingBytes / TB;
  static_assert(NST >= 2, "ring slice must hold two tiles");

  __device__ __forceinline__ static int swz(int c, int r) { return (c & ~7) | ((c ^ r) & 7); }

  template <class R>
  __device__ __forceinline__ static void issue(const R &rows, const int32_t *ids, int tok0, int cnt, int s,
                                               unsigned char *wring) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char *st = wring + (s % NST) * TB;
    const int base = (s * kWarps + warp) * TILE;
#pragma unroll
    for (int x = 0; x < TILE * CPT / 32; ++x) {
      const int q = x * 32 + lane;
      const int r = q / CPT, c = q % CPT;
      const int i = base + r;
      const bool valid = i < cnt;
      const int tok = valid ? (GATHER ? ids[i] : tok0 + i) : 0;
      const __nv_bfloat16 *src = (c < CPT / 2 ? rows.k : rows.v) + rows.off(tok) + (c % (CPT / 2)) * 8;
      cp_async16_zfill(st + r * REC + swz(c, r) * 16, src, valid);
    }
  }

  __device__ __forceinline__ static int warp_tiles(int cnt) {
    const int warp = threadIdx.x >> 5;
    const int tiles = (cnt + TILE - 1) / TILE;
    return tiles > warp ? (tiles - warp + kWarps - 1) / kWarps : 0;
  }
};

template <int D, int G, bool GATHER, class R>
__device__ __forceinline__ void attend_mma_prologue(const R &rows, const int32_t *ids, int tok0, int cnt,
                                                    unsigned char *ring) {
  using RS = MmaRowStream<D, G, GATHER>;
  unsigned char *wring = ring + (threadIdx.x >> 5) * kWarpRingBytes;
  // a share that fits the ring goes in flight whole: one memory round trip
  const bool whole = cnt <= RS::NST * kWarps * RS::TILE;
#pragma unroll
  for (int s = 0; s < RS::NST - 1; ++s) {
    RS::issue(rows, ids, tok0, cnt, s, wring);
    cp_async_commit();
  }
  if (whole) {
    RS::issue(rows, ids, tok0, cnt, RS::NST - 1, wring);
    cp_async_commit();
  }
}

// The query operand: q_hat (pre-scaled, fp32) as two bf16 tiles hi and lo of
// 8 rows x D (row h = head h, zero for h >= G), swizzled like the ring so
// that ldmatrix reads them without bank conflicts.  Ends with __syncthreads().
template <int D, int G>
__device__ __forceinline__ void build_query_tiles(const float *qhat, unsigned char *qt) {
  constexpr int RB = D * 2;
  for (int e = threadIdx.x; e < 8 * D / 2; e += kThreads) {
    const int r = e / (D / 2), c2 = e % (D / 2);  // row, pair of columns
    float x0 = 0.f, x1 = 0.f;
    if (r < G) {
      x0 = qhat[r * D + 2 * c2];
      x1 = qhat[r * D + 2 * c2 + 1];
    }
    uint32_t hi, lo;
    split_bf16x2(x0, x1, hi, lo);
    const int chunk = (2 * c2) / 8, within = (2 * c2) % 8;
    const int off = r * RB + (((chunk & ~7) | ((chunk ^ r) & 7)) * 16) + within * 2;
    *reinterpret_cast<uint32_t *>(qt + off) = hi;
    *reinterpret_cast<uint32_t *>(qt + 8 * RB + off) = lo;
  }
  __syncthreads();
}

template <int D, int G, bool GATHER, class R>
__device__ __forceinline__ void attend_mma_loop(const R &rows, const int32_t *ids, int tok0, int cnt,
                                                const unsigned char *qt, unsigned char *ring, float *pm, float *pl,
                                                float *pacc) {
  using RS = MmaRowStream<D, G, GATHER>;
  constexpr int KS = D / 16;  // k-steps of the logit product
  constexpr int MT = D / 16;  // 16-dim tiles of the output product
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  unsigned char *wring = ring + warp * kWarpRingBytes;

  float o[MT][4];
#pragma unroll
  for (int j = 0; j < MT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m = -INFINITY, lsum = 0.f;  // head g

  const int nt = RS::warp_tiles(cnt);
  const int r8 = lane & 7, mi = lane >> 3;
  const bool whole = cnt <= RS::NST * kWarps * RS::TILE;  // the prologue issued every tile
  for (int s = 0; s < nt; ++s) {
    if (whole) {
      if (s == 0) cp_async_wait<0>();
      __syncwarp();
    } else {
      __syncwarp();  // tile s-1's slot is consumed: refill it before waiting for tile s
      RS::issue(rows, ids, tok0, cnt, s + RS::NST - 1, wring);
      cp_async_commit();
      cp_async_wait<RS::NST - 1>();
      __syncwarp();
    }
    const unsigned char *st = wring + (s % RS::NST) * RS::TB;
    const int base = (s * kWarps + warp) * RS::TILE;

    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int jj = 0; jj < KS / 2; ++jj) {
      // rows 0-7 of the query tiles; rows 8-15 of the A operand are zero
      const int qoff = r8 * (2 * D) + RS::swz(4 * jj + mi, r8) * 16;
      uint32_t h0, h1, h2, h3, l0, l1, l2, l3, b0, b1, b2, b3;
      ldsm_x4(smem_u32(qt + qoff), h0, h1, h2, h3);
      ldsm_x4(smem_u32(qt + 8 * (2 * D) + qoff), l0, l1, l2, l3);
      ldsm_x4(smem_u32(st + r8 * RS::REC + RS::swz(4 * jj + mi, r8) * 16), b0, b1, b2, b3);
      mma_16816(sc, h0, 0u, h1, 0u, b0, b1);
      mma_16816(sc, l0, 0u, l1, 0u, b0, b1);
      mma_16816(sc, h2, 0u, h3, 0u, b2, b3);
      mma_16816(sc, l2, 0u, l3, 0u, b2, b3);
    }
    const float s0 = (base + 2 * t < cnt) ? sc[0] : -INFINITY;
    const float s1 = (base + 2 * t + 1 < cnt) ? sc[1] : -INFINITY;
    float tmax = fmaxf(s0, s1);
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 2));
    const float mnew = fmaxf(m, tmax);
    const float mref = (mnew == -INFINITY) ? 0.f : mnew;
    const float corr = exp2f(m - mref);
    const float p0 = exp2f(s0 - mref), p1 = exp2f(s1 - mref);
    lsum = lsum * corr + p0 + p1;
    m = mnew;
    // this lane's output columns are heads 2t and 2t+1: their factors live in
    // lanes 8t and 8t+4
    const float ca = __shfl_sync(kFull, corr, 8 * t);
    const float cb = __shfl_sync(kFull, corr, 8 * t + 4);
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      o[j][0] *= ca;
      o[j][1] *= cb;
      o[j][2] *= ca;
      o[j][3] *= cb;
    }
    uint32_t ph, plo;
    split_bf16x2(p0, p1, ph, plo);
#pragma unroll
    for (int jj = 0; jj < MT / 2; ++jj) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(smem_u32(st + r8 * RS::REC + RS::swz(RS::CPT / 2 + 4 * jj + mi, r8) * 16), a0, a1, a2, a3);
      mma_1688(o[2 * jj], a0, a1, ph);
      mma_1688(o[2 * jj], a0, a1, plo);
      mma_1688(o[2 * jj + 1], a2, a3, ph);
      mma_1688(o[2 * jj + 1], a2, a3, plo);
    }
  }
  cp_async_wait<0>();
  lsum += __shfl_xor_sync(kFull, lsum, 1);
  lsum += __shfl_xor_sync(kFull, lsum, 2);

  __syncthreads();  // every warp is done with the ring: it now holds the per-warp states
  float *wpart = reinterpret_cast<float *>(ring);  // [kWarps][G][D+2]
  const int h0 = 2 * t, h1 = 2 * t + 1;
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    if (h0 < G) {
      wpart[(warp * G + h0) * (D + 2) + 16 * j + g] = o[j][0];
      wpart[(warp * G + h0) * (D + 2) + 16 * j + g + 8] = o[j][2];
    }
    if (h1 < G) {
      wpart[(warp * G + h1) * (D + 2) + 16 * j + g] = o[j][1];
      wpart[(warp * G + h1) * (D + 2) + 16 * j + g + 8] = o[j][3];
    }
  }
  if (t == 0 && g < G) {
    wpart[(warp * G + g) * (D + 2) + D] = m;
    wpart[(warp * G + g) * (D + 2) + D + 1] = lsum;
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D, dim = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wpart[(w * G + h) * (D + 2) + D]);
    const float mref = (M == -INFINITY) ? 0.f : M;
    float A = 0.f, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float *wp = wpart + (w * G + h) * (D + 2);
      const float c = exp2f(wp[D] - mref);
      A = fmaf(c, wp[dim], A);
      Ls = fmaf(c, wp[D + 1], Ls);
    }
    pacc[e] = A;
    if (dim == 0) {
      pm[h] = M;
      pl[h] = Ls;
    }
  }
}

// Dispatch: tensor cores for bf16 caches whose query group has G >= 4 heads
// (there the CUDA-core loop, at 2G+1 instructions per cache element, can no
// longer keep up with HBM); CUDA cores for smaller groups and for fp32 caches
// (whose 1e-4 tolerance rules out bf16 operands).
template <typename T, int D, int G, bool GATHER, class R>
__device__ __forceinline__ void attend_prologue_any(const R &rows, const int32_t *ids, int tok0, int cnt,
                                                    unsigned char *ring) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value && G >= 4)
    attend_mma_prologue<D, G, GATHER>(rows, ids, tok0, cnt, ring);
  else
    attend_prologue<T, D, GATHER>(rows, ids, tok0, cnt, ring);
}

// qtiles: 8*D words of shared memory that nothing else uses during the call.
template <typename T, int D, int G, bool GATHER, class R>
__device__ __forceinline__ void attend_loop_any(const R &rows, const int32_t *ids, int tok0, int cnt,
                                                const float *qhat, unsigned char *qtiles, unsigned char *ring,
                                                float *pm, float *pl, float *pacc) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value && G >= 4) {
    build_query_tiles<D, G>(qhat, qtiles);
    attend_mma_loop<D, G, GATHER>(rows, ids, tok0, cnt, qtiles, ring, pm, pl, pacc);
  } else {
    attend_loop<T, D, G, GATHER>(rows, ids, tok0, cnt, qhat, ring, pm, pl, pacc);
  }
}

// Fold one more token into the CTA's merged attention state (pm, pl, pacc,
// log2 domain with q_hat pre-scaled): kr holds its key as the fp32 values of
// the stored cache entry, vs its value.  lg: G floats of scratch.  Starts and
// ends with __syncthreads().
template <typename T, int D, int G>
__device__ __forceinline__ void fold_token(const float *qhat, const float *kr, const T *vs, float *pm, float *pl,
                                           float *pacc, float *lg) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __syncthreads();
  if (warp < G) {
    float s = 0.f;
    for (int i = lane; i < D; i += 32) s = fmaf(qhat[warp * D + i], kr[i], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
    if (lane == 0) lg[warp] = s;
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int h = e / D;
    const float m0 = pm[h], x = lg[h], M = fmaxf(m0, x);
    pacc[e] = fmaf(pacc[e], exp2f(m0 - M), exp2f(x - M) * to_f32(vs[e - h * D]));
  }
  __syncthreads();  // every pm read before it changes
  if (tid < G) {
    const float m0 = pm[tid], x = lg[tid], M = fmaxf(m0, x);
    pl[tid] = fmaf(pl[tid], exp2f(m0 - M), exp2f(x - M));
    pm[tid] = M;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// 5. log-sum-exp combine of the cluster's partial states: CTA r writes the
//    output elements r*256 + t (stride ncta*256); each reads the (max, sum,
//    acc) of its head from every CTA through distributed shared memory, all
//    loads issued before the first use.  Must follow a cluster barrier that
//    orders every CTA's pm/pl/pacc writes, and be followed by one before any
//    CTA exits.
template <int D, int G>
__device__ __forceinline__ void cluster_combine(int ncta, int rank, const float *pm, const float *pl,
                                                const float *pacc, float *out) {
  constexpr int R = 16;  // the largest cluster
  for (int e = rank * kThreads + (int)threadIdx.x; e < G * D; e += ncta * kThreads) {
    const int h = e / D;
    float m[R], l[R], v[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      m[r] = r < ncta ? dsmem_ld_f32(dsmem_addr(pm + h, (uint32_t)r)) : -INFINITY;
      l[r] = r < ncta ? dsmem_ld_f32(dsmem_addr(pl + h, (uint32_t)r)) : 0.f;
      v[r] = r < ncta ? dsmem_ld_f32(dsmem_addr(pacc + e, (uint32_t)r)) : 0.f;
    }
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < R; ++r) M = fmaxf(M, m[r]);
    const float mref = (M == -INFINITY) ? 0.f : M;
    float A = 0.f, Ls = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r < ncta) {
        const float c = exp2f(m[r] - mref);
        A = fmaf(c, v[r], A);
        Ls = fmaf(c, l[r], Ls);
      }
    }
    out[e] = A / Ls;
  }
}

// 5'. the same merge by pushing: output elements are owned in blocks of
//    kThreads (block i by CTA i % ncta); right after its attention each CTA
//    stores its accumulator for each owner's elements, and its max and sum of
//    every head, into that owner's receive buffer (`recv`: push_slot_words per
//    sender, in shared memory the owner no longer uses), so that after one
//    cluster barrier every owner merges from its own shared memory and no CTA
//    reads another's afterwards (no second barrier).  Used when the buffers
//    fit in kPushRecvWords.
__host__ __device__ inline int push_slot_words(int G, int D, int ncta) {
  const int blocks = (G * D + kThreads - 1) / kThreads;
  const int per = (blocks + ncta - 1) / ncta;
  const int elems = per * kThreads < G * D ? per * kThreads : G * D;
  return elems + 2 * G;
}
__host__ __device__ inline bool push_merge_fits(int G, int D, int ncta) {
  return ncta > 1 && ncta * push_slot_words(G, D, ncta) <= kPushRecvWords;
}

// The CTA's state (pm, pl, pacc, final) into the owners' receive buffers.
template <int D, int G>
__device__ __forceinline__ void push_state(int ncta, int rank, const float *pm, const float *pl, const float *pacc,
                                           float *recv) {
  const int slot = push_slot_words(G, D, ncta);
  const int elems = slot - 2 * G;
  const int blocks = (G * D + kThreads - 1) / kThreads;
  for (int e = threadIdx.x; e < G * D; e += kThreads) {
    const int bi = e / kThreads;
    const int local = (bi / ncta) * kThreads + (e - bi * kThreads);
    dsmem_st(dsmem_addr(recv + rank * slot + local, (uint32_t)(bi % ncta)), __float_as_uint(pacc[e]));
  }
  if ((int)threadIdx.x < G) {
    const int h = threadIdx.x;
    for (int r = 0; r < ncta && r < blocks; ++r) {
      dsmem_st(dsmem_addr(recv + rank * slot + elems + h, (uint32_t)r), __float_as_uint(pm[h]));
      dsmem_st(dsmem_addr(recv + rank * slot + elems + G + h, (uint32_t)r), __float_as_uint(pl[h]));
    }
  }
}

// After the cluster barrier that follows every push_state: this CTA's owned
// output elements from its receive buffer.
template <int D, int G>
__device__ __forceinline__ void push_combine(int ncta, int rank, const float *recv, float *out) {
  const int slot = push_slot_words(G, D, ncta);
  const int elems = slot - 2 * G;
  const int blocks = (G * D + kThreads - 1) / kThreads;
  for (int bi = rank; bi < blocks; bi += ncta) {
    const int e = bi * kThreads + (int)threadIdx.x;
    if (e < G * D) {
      const int local = (bi / ncta) * kThreads + (int)threadIdx.x;
      const int h = e / D;
      float M = -INFINITY;
      for (int s = 0; s < ncta; ++s) M = fmaxf(M, recv[s * slot + elems + h]);
      const float mref = (M == -INFINITY) ? 0.f : M;
      float A = 0.f, Ls = 0.f;
      for (int s = 0; s < ncta; ++s) {
        const float c = exp2f(recv[s * slot + elems + h] - mref);
        A = fmaf(c, recv[s * slot + local], A);
        Ls = fmaf(c, recv[s * slot + elems + G + h], Ls);
      }
      out[e] = A / Ls;
    }
  }
}

// The CTA's own state as the output (clusters of one CTA).
template <int D, int G>
__device__ __forceinline__ void local_combine(const float *pl, const float *pacc, float *out) {
  for (int e = threadIdx.x; e < G * D; e += kThreads) out[e] = pacc[e] / pl[e / D];
}

template <typename T, int D, int G, bool PAGED>
__global__ void __launch_bounds__(kThreads, (G >= 8) ? 1 : 2) dense_decode_kernel(const __grid_constant__ DecodeArgs<T> a) {
  extern __shared__ __align__(16) uint32_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int ncta = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / ncta;
  const int b = row / a.n_kv_heads, g = row % a.n_kv_heads;
  const SmemLayout L = decode_layout(G, D, a.chunk, false);
  float *qhat = reinterpret_cast<float *>(smem + L.qhat);
  float *u = reinterpret_cast<float *>(smem + L.u);
  float *pm = reinterpret_cast<float *>(smem + L.pm);
  float *pl = reinterpret_cast<float *>(smem + L.pl);
  float *pacc = reinterpret_cast<float *>(smem + L.pacc);
  float *scratch = reinterpret_cast<float *>(smem + L.slots);
  unsigned char *ring = reinterpret_cast<unsigned char *>(smem + L.ring);

  const int S = row_seq_len(a, b);
  const int t0 = min(S, rank * a.chunk);
  const int len = min(S, t0 + a.chunk) - t0;
  const Rows<T, D, PAGED> rows = make_rows<T, D, PAGED>(a, b, g);
  // an appended token sits at the row's last position: the CTA that owns it
  // rotates and stores it, streams the rest and folds it in at the end
  const bool own = a.k_new != nullptr && len > 0 && S - 1 < t0 + len;
  const int slen = own ? len - 1 : len;
  const size_t nv = ((size_t)b * a.n_kv_heads + g) * D;
  float *xkh = u;  // the dense kernel has no low-rank query
  rotate_queries<T, D, G>(
      a, b, g, qhat, u, scratch, false, [&] { attend_prologue_any<T, D, G, false>(rows, nullptr, t0, slen, ring); },
      own ? a.k_new + nv : nullptr, xkh);
  if (own) store_appended<T, D, PAGED>(a, rows, b, g, S - 1, xkh);
  attend_loop_any<T, D, G, false>(rows, nullptr, t0, slen, qhat, reinterpret_cast<unsigned char *>(scratch), ring,
                                  pm, pl, pacc);
  if (own) fold_token<T, D, G>(qhat, xkh, a.v_new + nv, pm, pl, pacc, scratch);
  const int Hq = a.n_kv_heads * G;
  float *out = a.out + ((size_t)b * Hq + (size_t)g * G) * D;
  __syncthreads();  // the CTA's state is complete
  if (ncta == 1) {
    local_combine<D, G>(pl, pacc, out);
  } else if (push_merge_fits(G, D, ncta)) {
    float *recv = reinterpret_cast<float *>(smem + L.recv);
    push_state<D, G>(ncta, rank, pm, pl, pacc, recv);
    cluster.sync();
    push_combine<D, G>(ncta, rank, recv, out);
  } else {
    cluster.sync();
    cluster_combine<D, G>(ncta, rank, pm, pl, pacc, out);
    cluster.sync();
  }
}

}  // namespace loki
