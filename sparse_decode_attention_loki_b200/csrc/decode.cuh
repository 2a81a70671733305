// Loki decode-step kernels for sm_100a.
//
// Method ("Loki: Low-rank Keys for Efficient Sparse Attention", atlas.scime.ai
// summary, section "Approach"): rotate the query into the PCA basis, rank every
// cached token on the first d principal dimensions, keep the top k tokens and
// compute exact softmax attention over them.  The dense kernel is the "Full
// Attention" baseline (same page, "Experimental setup").
//
// B200 design.  One thread-block cluster of `ncta` CTAs owns one (batch, KV
// head) row.  CTA r of the cluster owns the contiguous token range
// [r*chunk, (r+1)*chunk).  The whole decode step is one kernel:
//   1. every CTA rotates the G queries of its KV group (q . P, fp32) and forms
//      the group's low-rank query u = sum_h q_hat_h[:d];
//   2. it streams K_hat[i, :d] of its range with 16-byte loads, one score per
//      token, and keeps the scores as order-preserving uint32 keys in shared
//      memory -- scores never go to HBM;
//   3. the cluster finds the k-th largest key by an 11/11/10-bit radix select:
//      each CTA histograms its keys and adds the histogram into the leader
//      CTA's shared memory through distributed shared memory (DSMEM);
//   4. each CTA writes its selected token indices, ascending, at its offset in
//      idx (ties at the threshold go to the lower index);
//   5. the k selected tokens are split evenly over the cluster; each CTA
//      gathers full K_hat and V rows and keeps an online softmax per query
//      head (log2 domain, fp32);
//   6. the CTAs' partial (max, sum, acc) states are merged through DSMEM with
//      the log-sum-exp rule and the leader-free combine writes out.
// No workspace, no atomics in global memory, no spin-waits: every cross-CTA
// step is a hardware cluster barrier.
#pragma once

#include "common.cuh"

namespace loki {

template <typename T>
struct DecodeArgs {
  const T *k_hat;      // [B, Hkv, S_cap, D]
  const T *v;          // [B, Hkv, S_cap, D]
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
  int32_t lpt;         // lanes per token in the score loop (power of two)
  int32_t dpad;        // d rounded up to a whole 16-byte vector
  float scale_log2;    // softmax scale * log2(e)
};

// Shared-memory layout, in 4-byte words.  Identical on host and device.
struct SmemLayout {
  int qhat, u, pm, pl, pacc, ctl, scratch, keys, words;
};

__host__ __device__ inline int scratch_words(int G, int D) {
  int a = 4 * 2048;                          // local histogram + 3 cluster histograms
  int b = G * D + (kThreads / D) * G * D;    // query staging + partial dot products
  int c = kWarps * G * (D + 2);              // per-warp softmax states
  int m = a > b ? a : b;
  return m > c ? m : c;
}

__host__ __device__ inline SmemLayout decode_layout(int G, int D, int chunk, bool with_keys) {
  SmemLayout L;
  int o = 0;
  L.qhat = o;    o += G * D;
  L.u = o;       o += D;
  L.pm = o;      o += 16;
  L.pl = o;      o += 16;
  L.pacc = o;    o += G * D;
  L.ctl = o;     o += 128;
  L.scratch = o; o += scratch_words(G, D);
  L.keys = o;    o += with_keys ? chunk : 0;
  L.words = (o + 3) & ~3;
  return L;
}

// ctl word offsets
constexpr int kCtlBucket = 0;    // [0..2]: bucket, count above it, count in it
constexpr int kCtlWtot = 4;      // [4..11]: warp totals for block scans
constexpr int kCtlMine = 12;     // [12..13]: this CTA's (#above, #in bucket)
constexpr int kCtlGt = 16;       // [16..31]: #above per CTA of the cluster
constexpr int kCtlEq = 32;       // [32..47]: #in bucket per CTA of the cluster
constexpr int kCtlWarpGt = 48;   // [48..55]
constexpr int kCtlWarpEq = 56;   // [56..63]

// ---------------------------------------------------------------------------
// 1. query rotation: q_hat_h = q_h . P_g for the G heads of KV head g, and
//    u = sum_h q_hat_h[:d] (zero beyond d).  q_hat is then pre-scaled by
//    scale*log2(e) for the log2-domain softmax.  Ends with __syncthreads().
template <typename T, int D, int G>
__device__ __forceinline__ void rotate_queries(const DecodeArgs<T> &a, int b, int g,
                                               float *qhat, float *u, float *scratch,
                                               bool want_u) {
  const int tid = threadIdx.x;
  const int Hq = a.n_kv_heads * G;
  const T *qg = a.q + ((size_t)b * Hq + (size_t)g * G) * D;
  float *qs = scratch;  // [G][D]
  for (int i = tid; i < G * D; i += kThreads) qs[i] = to_f32(qg[i]);
  __syncthreads();

  constexpr int PARTS = kThreads / D;
  constexpr int IPP = D / PARTS;
  const int j = tid % D, part = tid / D;
  const float *Pg = a.P + (size_t)g * D * D + (size_t)part * IPP * D + j;
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
  float pv[IPP];
#pragma unroll
  for (int ii = 0; ii < IPP; ++ii) pv[ii] = __ldg(Pg + (size_t)ii * D);
#pragma unroll
  for (int ii = 0; ii < IPP; ++ii) {
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = fmaf(qs[h * D + part * IPP + ii], pv[ii], acc[h]);
  }
  float *red = scratch + G * D;  // [PARTS][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h) red[(part * G + h) * D + j] = acc[h];
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    float s = 0.f;
#pragma unroll
    for (int p = 0; p < PARTS; ++p) s += red[p * G * D + e];
    qhat[e] = s;
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

// ---------------------------------------------------------------------------
// 2. low-rank scores of tokens [t0, t0+len): key = score_key(u . K_hat[i, :d]).
//    LPT lanes cooperate on one token (16 bytes each); a warp load instruction
//    covers 32/LPT consecutive tokens.
template <typename T, int D, int LPT>
__device__ __forceinline__ void score_tokens(const T *__restrict__ Krow, int t0, int len,
                                             int dpad, const float *u, uint32_t *keys) {
  constexpr int VEC = VecN<T>::value;
  constexpr int TPW = 32 / LPT;
  constexpr int TPB = TPW * kWarps;
  constexpr int UNR = (LPT >= 8) ? 4 : 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPT;
  const int slot = warp * TPW + lane / LPT;
  const bool active = sub * VEC < dpad;
  float uv[VEC];
#pragma unroll
  for (int x = 0; x < VEC; ++x) uv[x] = u[sub * VEC + x];
  const T *base = Krow + (size_t)t0 * D + sub * VEC;
  for (int s0 = 0; s0 < len; s0 += TPB * UNR) {
    uint4 r[UNR];
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
      const int j = s0 + x * TPB + slot;
      r[x] = (active && j < len) ? ld_stream16(base + (size_t)j * D) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int x = 0; x < UNR; ++x) {
      float f[VEC];
      unpack16(r[x], f);
      float s = 0.f;
#pragma unroll
      for (int y = 0; y < VEC; ++y) s = fmaf(uv[y], f[y], s);
#pragma unroll
      for (int off = LPT / 2; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
      const int j = s0 + x * TPB + slot;
      if (sub == 0 && j < len) keys[j] = score_key(s);
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void score_dispatch(int lpt, const T *Krow, int t0, int len, int dpad,
                                               const float *u, uint32_t *keys) {
  constexpr int MAXL = D / VecN<T>::value;
  switch (lpt) {
    case 1: score_tokens<T, D, 1>(Krow, t0, len, dpad, u, keys); break;
    case 2: score_tokens<T, D, 2>(Krow, t0, len, dpad, u, keys); break;
    case 4: score_tokens<T, D, 4>(Krow, t0, len, dpad, u, keys); break;
    case 8: score_tokens<T, D, 8>(Krow, t0, len, dpad, u, keys); break;
    case 16:
      if constexpr (MAXL >= 16) score_tokens<T, D, 16>(Krow, t0, len, dpad, u, keys);
      break;
    default:
      if constexpr (MAXL >= 32) score_tokens<T, D, 32>(Krow, t0, len, dpad, u, keys);
      break;
  }
}

// ---------------------------------------------------------------------------
// 3. cluster radix select.  Finds (prefix, mask, remaining) such that the
//    selected set is {key: key&mask > prefix} plus the first `remaining` (by
//    token index) of {key: key&mask == prefix}.  merged: the three cluster
//    histograms (local address; the leader's copy is the one used), zeroed by
//    the leader before its cluster_arrive().  Pass 0 performs the matching
//    cluster_wait().
struct SelectState {
  uint32_t prefix, mask, remaining;
};

__device__ __forceinline__ SelectState radix_select(cg::cluster_group &cluster, const uint32_t *keys,
                                                    int len, uint32_t k, uint32_t *hist,
                                                    uint32_t *merged, uint32_t *ctl) {
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t prefix = 0u, mask = 0u, remaining = k;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nbits = pass == 2 ? 10 : 11;
    const uint32_t nb = 1u << nbits;
    for (uint32_t i = tid; i < nb; i += kThreads) hist[i] = 0u;
    __syncthreads();
    // warp-aggregated shared atomics: lanes with the same bin add once
    for (int j0 = 0; j0 < len; j0 += kThreads) {
      const int j = j0 + tid;
      uint32_t bin = 0xffffffffu;
      if (j < len) {
        const uint32_t key = keys[j];
        if ((key & mask) == prefix) bin = (key >> shift) & (nb - 1u);
      }
      const uint32_t peers = __match_any_sync(kFull, bin);
      if (bin != 0xffffffffu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (pass == 0) cluster_wait();  // leader histograms zeroed; all CTAs running
    uint32_t *dst = cluster.map_shared_rank(merged + pass * 2048, 0);
    for (uint32_t i = tid; i < nb; i += kThreads) {
      const uint32_t c = hist[i];
      if (c) atomicAdd(dst + i, c);
    }
    cluster.sync();
    // every CTA scans the merged histogram from the top bin down
    const int bpt = (int)(nb / kThreads);  // 8 or 4
    uint32_t c[8];
    uint32_t sum = 0u;
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      c[x] = (x < bpt) ? dst[tid * bpt + x] : 0u;
      sum += c[x];
    }
    const uint32_t above = block_excl_suffix_sum(sum, ctl + kCtlWtot);
    if (above < remaining && above + sum >= remaining) {
      uint32_t cum = above;
      bool found = false;
#pragma unroll
      for (int x = 7; x >= 0; --x) {
        if (!found && x < bpt) {
          if (cum + c[x] >= remaining) {
            ctl[kCtlBucket + 0] = (uint32_t)(tid * bpt + x);
            ctl[kCtlBucket + 1] = cum;
            ctl[kCtlBucket + 2] = c[x];
            found = true;
          } else {
            cum += c[x];
          }
        }
      }
    }
    __syncthreads();
    const uint32_t bucket = ctl[kCtlBucket + 0];
    const uint32_t cnt_above = ctl[kCtlBucket + 1];
    const uint32_t cnt_in = ctl[kCtlBucket + 2];
    __syncthreads();
    remaining -= cnt_above;
    prefix |= bucket << shift;
    mask |= (nb - 1u) << shift;
    if (cnt_in == remaining) break;  // the whole bucket is taken: done
  }
  return SelectState{prefix, mask, remaining};
}

// ---------------------------------------------------------------------------
// 4. write this CTA's selected indices, ascending, at its offset in the row of
//    idx.  Ends with a cluster barrier after which the whole row of idx is
//    written and visible to every CTA of the cluster.
__device__ __forceinline__ void write_selection(cg::cluster_group &cluster, int ncta, int rank,
                                                const uint32_t *keys, int len, int t0,
                                                const SelectState &st, uint32_t k, uint32_t *ctl,
                                                int32_t *idx_row) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t my_gt = 0u, my_eq = 0u;
  for (int j = tid; j < len; j += kThreads) {
    const uint32_t km = keys[j] & st.mask;
    my_gt += km > st.prefix;
    my_eq += km == st.prefix;
  }
  my_gt = block_sum(my_gt, ctl + kCtlWtot);
  my_eq = block_sum(my_eq, ctl + kCtlWtot);
  if (tid == 0) {
    ctl[kCtlMine + 0] = my_gt;
    ctl[kCtlMine + 1] = my_eq;
  }
  cluster.sync();
  if (tid < ncta) {
    const uint32_t *rc = cluster.map_shared_rank(ctl + kCtlMine, tid);
    ctl[kCtlGt + tid] = rc[0];
    ctl[kCtlEq + tid] = rc[1];
  }
  __syncthreads();
  // ties at the threshold are taken in token order: lower CTAs first
  uint32_t eq_before = 0u, offset = 0u;
  for (int r = 0; r < rank; ++r) {
    const uint32_t want = st.remaining > eq_before ? st.remaining - eq_before : 0u;
    offset += ctl[kCtlGt + r] + min(ctl[kCtlEq + r], want);
    eq_before += ctl[kCtlEq + r];
  }
  const uint32_t take = min(ctl[kCtlEq + rank], st.remaining > eq_before ? st.remaining - eq_before : 0u);

  // each warp owns a contiguous segment of the CTA's tokens
  const int seg = (((len + kWarps - 1) / kWarps) + 31) & ~31;
  const int sbeg = min(len, warp * seg), send = min(len, sbeg + seg);
  uint32_t wg = 0u, we = 0u;
  for (int j0 = sbeg; j0 < send; j0 += 32) {
    const int j = j0 + lane;
    const bool in = j < send;
    const uint32_t km = in ? (keys[j] & st.mask) : 0u;
    wg += __popc(__ballot_sync(kFull, in && km > st.prefix));
    we += __popc(__ballot_sync(kFull, in && km == st.prefix));
  }
  if (lane == 0) {
    ctl[kCtlWarpGt + warp] = wg;
    ctl[kCtlWarpEq + warp] = we;
  }
  __syncthreads();
  uint32_t eq_base = 0u, sel_base = 0u;
  for (int w = 0; w < warp; ++w) {
    const uint32_t want = take > eq_base ? take - eq_base : 0u;
    sel_base += ctl[kCtlWarpGt + w] + min(ctl[kCtlWarpEq + w], want);
    eq_base += ctl[kCtlWarpEq + w];
  }
  int32_t *dst = idx_row + offset;
  uint32_t run_eq = eq_base, run_sel = sel_base;
  const uint32_t lt = lanemask_lt();
  for (int j0 = sbeg; j0 < send; j0 += 32) {
    const int j = j0 + lane;
    const bool in = j < send;
    const uint32_t km = in ? (keys[j] & st.mask) : 0u;
    const bool gt = in && km > st.prefix;
    const bool eq = in && km == st.prefix;
    const uint32_t eb = __ballot_sync(kFull, eq);
    const uint32_t eq_rank = run_eq + __popc(eb & lt);
    const bool sel = gt || (eq && eq_rank < take);
    const uint32_t sb = __ballot_sync(kFull, sel);
    const uint32_t p = run_sel + __popc(sb & lt);
    if (sel && offset + p < k) dst[p] = t0 + j;  // bound: the row holds k entries
    run_eq += __popc(eb);
    run_sel += __popc(sb);
  }
  cluster.sync();
}

// ---------------------------------------------------------------------------
// 5. exact attention over `cnt` rows (gathered through ids[], or the
//    contiguous rows tok0 .. tok0+cnt-1).  D/VEC lanes share one row; each
//    lane keeps an online softmax (max, sum, acc over its VEC dims) per query
//    head.  Leaves the CTA's merged state in pm/pl/pacc (not normalised).
template <typename T, int D, int G, bool GATHER>
__device__ __forceinline__ void attend_rows(const T *__restrict__ Kb, const T *__restrict__ Vb,
                                            const int32_t *ids, int tok0, int cnt, int seq_len,
                                            const float *qhat, float *wpart, float *pm,
                                            float *pl, float *pacc) {
  constexpr int VEC = VecN<T>::value;
  constexpr int LPR = D / VEC;
  constexpr int RG = 32 / LPR;
  constexpr int U = (G >= 8) ? 2 : 4;
  constexpr int STRIDE = kWarps * RG;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane % LPR, grp = lane / LPR;
  const int slot = warp * RG + grp;

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

  for (int base = 0; base < cnt; base += STRIDE * U) {
    int tok[U];
    bool ok[U];
#pragma unroll
    for (int x = 0; x < U; ++x) {
      const int i = base + x * STRIDE + slot;
      ok[x] = i < cnt;
      if constexpr (GATHER) {
        // indices come from this kernel's own selection; clamp them into the
        // row so that no load can leave the cache even if they were wrong
        tok[x] = ok[x] ? min(max(__ldcg(ids + i), 0), seq_len - 1) : 0;
      } else {
        tok[x] = tok0 + i;
      }
    }
    uint4 kr[U], vr[U];
#pragma unroll
    for (int x = 0; x < U; ++x) {
      if (ok[x]) {
        kr[x] = ld_stream16(Kb + (size_t)tok[x] * D + sub * VEC);
        vr[x] = ld_stream16(Vb + (size_t)tok[x] * D + sub * VEC);
      } else {
        kr[x] = make_uint4(0u, 0u, 0u, 0u);
        vr[x] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float lg[U][G];
#pragma unroll
    for (int x = 0; x < U; ++x) {
      float f[VEC];
      unpack16(kr[x], f);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float s = 0.f;
#pragma unroll
        for (int y = 0; y < VEC; ++y) s = fmaf(qv[h][y], f[y], s);
        lg[x][h] = s;
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
      for (int x = 0; x < U; ++x)
#pragma unroll
        for (int h = 0; h < G; ++h) lg[x][h] += __shfl_xor_sync(kFull, lg[x][h], off);
    float vf[U][VEC];
#pragma unroll
    for (int x = 0; x < U; ++x) unpack16(vr[x], vf[x]);
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
        const float p = ok[x] ? exp2f(lg[x][h] - mref) : 0.f;
        l[h] += p;
#pragma unroll
        for (int y = 0; y < VEC; ++y) acc[h][y] = fmaf(p, vf[x][y], acc[h][y]);
      }
      m[h] = mx;
    }
  }

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
// 6. log-sum-exp combine of the cluster's partial states; CTA r writes the
//    output elements r*256 + t (stride ncta*256).  Must follow a cluster
//    barrier that orders every CTA's pm/pl/pacc writes.
template <int D, int G>
__device__ __forceinline__ void cluster_combine(cg::cluster_group &cluster, int ncta, int rank,
                                                const float *pm, const float *pl, const float *pacc,
                                                float *out) {
  for (int e = rank * kThreads + (int)threadIdx.x; e < G * D; e += ncta * kThreads) {
    const int h = e / D;
    float M = -INFINITY;
    for (int r = 0; r < ncta; ++r) M = fmaxf(M, *cluster.map_shared_rank(pm + h, r));
    float A = 0.f, Ls = 0.f;
    for (int r = 0; r < ncta; ++r) {
      const float c = exp2f(*cluster.map_shared_rank(pm + h, r) - M);
      A = fmaf(c, *cluster.map_shared_rank(pacc + e, r), A);
      Ls = fmaf(c, *cluster.map_shared_rank(pl + h, r), Ls);
    }
    out[e] = A / Ls;
  }
}

// ---------------------------------------------------------------------------
template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) loki_decode_kernel(const __grid_constant__ DecodeArgs<T> a) {
  extern __shared__ __align__(16) uint32_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int ncta = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / ncta;
  const int b = row / a.n_kv_heads, g = row % a.n_kv_heads;
  const SmemLayout L = decode_layout(G, D, a.chunk, true);
  float *qhat = reinterpret_cast<float *>(smem + L.qhat);
  float *u = reinterpret_cast<float *>(smem + L.u);
  float *pm = reinterpret_cast<float *>(smem + L.pm);
  float *pl = reinterpret_cast<float *>(smem + L.pl);
  float *pacc = reinterpret_cast<float *>(smem + L.pacc);
  uint32_t *ctl = smem + L.ctl;
  uint32_t *scratch = smem + L.scratch;
  uint32_t *keys = smem + L.keys;

  const int t0 = min(a.seq_len, rank * a.chunk);
  const int len = min(a.seq_len, t0 + a.chunk) - t0;

  rotate_queries<T, D, G>(a, b, g, qhat, u, reinterpret_cast<float *>(scratch), true);
  if (rank == 0)
    for (int i = threadIdx.x; i < 3 * 2048; i += kThreads) scratch[2048 + i] = 0u;
  cluster_arrive();

  const size_t row_off = (size_t)row * a.capacity * D;
  score_dispatch<T, D>(a.lpt, a.k_hat + row_off, t0, len, a.dpad, u, keys);
  __syncthreads();

  const SelectState st = radix_select(cluster, keys, len, (uint32_t)a.k, scratch, scratch + 2048, ctl);
  int32_t *idx_row = a.idx + (size_t)row * a.k;
  write_selection(cluster, ncta, rank, keys, len, t0, st, (uint32_t)a.k, ctl, idx_row);

  const int s0 = (int)(((long long)rank * a.k) / ncta);
  const int s1 = (int)(((long long)(rank + 1) * a.k) / ncta);
  attend_rows<T, D, G, true>(a.k_hat + row_off, a.v + row_off, idx_row + s0, 0, s1 - s0, a.seq_len, qhat,
                             reinterpret_cast<float *>(scratch), pm, pl, pacc);
  cluster.sync();
  const int Hq = a.n_kv_heads * G;
  cluster_combine<D, G>(cluster, ncta, rank, pm, pl, pacc, a.out + ((size_t)b * Hq + (size_t)g * G) * D);
  cluster.sync();
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) dense_decode_kernel(const __grid_constant__ DecodeArgs<T> a) {
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
  float *scratch = reinterpret_cast<float *>(smem + L.scratch);

  const int t0 = min(a.seq_len, rank * a.chunk);
  const int len = min(a.seq_len, t0 + a.chunk) - t0;
  rotate_queries<T, D, G>(a, b, g, qhat, u, scratch, false);
  const size_t row_off = (size_t)row * a.capacity * D;
  attend_rows<T, D, G, false>(a.k_hat + row_off, a.v + row_off, nullptr, t0, len, a.seq_len, qhat, scratch,
                              pm, pl, pacc);
  cluster.sync();
  const int Hq = a.n_kv_heads * G;
  cluster_combine<D, G>(cluster, ncta, rank, pm, pl, pacc, a.out + ((size_t)b * Hq + (size_t)g * G) * D);
  cluster.sync();
}

}  // namespace loki
