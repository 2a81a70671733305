// One Loki decode step ("Loki: Low-rank Keys for Efficient Sparse
// Attention", atlas.scime.ai summary, section "Approach": PCA-project
// queries and keys, rank tokens on the top-d principal dimensions, exact
// attention over the top-k tokens), one kernel for query groups of up to 4
// heads, two for 8.  This file holds the rotate kernel and the decode kernel
// of rows longer than kShortMaxTokens; short_step.cuh holds the short-row
// decode kernel, which reuses the pieces here.
//
//   rotate  (groups of 8 only) D/32 CTAs per (batch, KV head) row: q_hat_h =
//           q_h . P_g for the G query heads of the row (fp32, pre-scaled for
//           the softmax) and the group's low-rank query u = sum_h
//           q_hat_h[:d], into the workspace.
//   decode  one thread-block cluster of ncta CTAs per row, about one wave of
//           CTAs in all; CTA r owns tokens [r*chunk, (r+1)*chunk):
//     1. the first stages of its low-rank key stream go in flight (cp.async
//        ring) while it forms q_hat and u from q and P_g (or, for groups of
//        8, waits for the rotate grid and reads them); then it streams
//        K_hat[i, :d], keeps one order-preserving uint32 key per token in
//        shared memory and histograms the keys' top 11 bits on the way;
//     2. cluster radix select over 11/11/10-bit digits: every CTA adds the
//        non-zero bins of its histogram into the leader CTA's (distributed
//        shared memory reductions).  A row with S + k within the leader's
//        ring is then selected by the leader alone on all its keys, read
//        from the cluster's shared memory, into an ascending list of k
//        indices.  On a longer row the leader finds the bucket of the k-th
//        largest key and tells every CTA; each CTA sends the leader its keys
//        in that bucket (the candidates, a few percent) and its count above
//        it; the leader finishes the threshold on the candidates, derives
//        every CTA's share of the selection (ties at the threshold go to the
//        lower index) and hands each CTA its (threshold, ties to take,
//        offset); each CTA writes its indices in ascending order (should a
//        CTA's candidates overflow its slot at the leader, the cluster
//        refines with distributed histogram passes instead).  Once the
//        first digit's bucket is known, both paths keep per-warp lists of
//        the tokens at or above it and run their later passes and the
//        ordered write over the lists;
//     3. the k selected rows are split evenly over the cluster: gather K_hat
//        and V rows through the ring, online softmax per query head;
//     4. the CTAs' (max, sum, acc) states are merged through distributed
//        shared memory with the log-sum-exp rule into out.
// Scores never leave the chip; the workspace holds only q_hat and u (groups
// of 8).
#pragma once

#include "decode.cuh"

namespace loki {

// Phase stamps of the decode kernel (builds with -DLOKI_PHASE_STAMPS only):
// per CTA, the global timer at eight points of the step, then its SM, rank
// and row.  Read by loki_phase_stamps.
constexpr int kMaxStampCtas = 1 << 16;
constexpr int kStampWords = 10;
#ifdef LOKI_PHASE_STAMPS
static __device__ unsigned long long g_phase_stamps[kMaxStampCtas][kStampWords];
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define LOKI_PHASE(i)                                                               \
  do {                                                                              \
    if (threadIdx.x == 0 && blockIdx.x < kMaxStampCtas) g_phase_stamps[blockIdx.x][i] = global_ns(); \
  } while (0)
#else
#define LOKI_PHASE(i) \
  do {                \
  } while (0)
#endif

// Geometry of the low-rank key stream's per-warp ring slice: stages of
// kScoreStageBytes, kScoreStages of them (kScoreStages - 1 in flight).  The
// slice is the same 8 KB per warp as the attention's.
#ifndef LOKI_SCORE_STAGE_BYTES
#define LOKI_SCORE_STAGE_BYTES 2048
#endif
#ifndef LOKI_SCORE_STAGES
#define LOKI_SCORE_STAGES 4
#endif
constexpr int kScoreStageBytes = LOKI_SCORE_STAGE_BYTES;
constexpr int kScoreStages = LOKI_SCORE_STAGES;
static_assert(kScoreStageBytes * kScoreStages <= kWarpRingBytes, "the key stream fits the ring slice");

constexpr int kDig1Bits = 11;                   // first radix digit: key bits 31..21
constexpr int kDig1Bins = 1 << kDig1Bits;       // 2048
constexpr int kDig2Bits = 11;                   // second digit: bits 20..10
constexpr int kDig3Bits = 10;                   // third digit: bits 9..0
constexpr int kMaxCluster = 16;
constexpr int kMaxChunk = 24576;                // tokens per decode CTA, at most

// Workspace layout (bytes, each region 256-byte aligned).
struct WsLayout {
  size_t qhat, u, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

__host__ __device__ inline WsLayout ws_layout(long long rows, int G, int D) {
  WsLayout w;
  size_t o = 0;
  w.qhat = o; o = align256(o + (size_t)rows * G * D * 4);
  w.u = o;    o = align256(o + (size_t)rows * D * 4);
  w.total = o;
  return w;
}

template <typename T>
struct StepArgs {
  DecodeArgs<T> da;  // cache, q, P, out, idx, sizes, d, k, scale; da.chunk = tokens per decode CTA
  float *qhat;       // [rows, G, D], pre-scaled by scale * log2(e)
  float *u;          // [rows, D], zero beyond d
};

// The decode kernel rotates its own queries (and an appended key) when the
// rotation's scratch (rot_words) fits in the histogram words; larger query
// groups take q_hat and u from the rotate grid below.
template <int G>
constexpr bool kRotateInKernel = G <= 4;
static_assert(rot_words(4, 64) <= skewed_words(kDig1Bins) && rot_words(4, 128) <= skewed_words(kDig1Bins),
              "the in-kernel rotation's scratch (queries and an appended key) fits in the histogram words");

// ---------------------------------------------------------------------------
// rotate: CTA (row, cb) computes columns [32cb, 32cb + 32) of q_hat for the G
// query heads of the row from a 32-column slice of P_g held in shared memory,
// and those columns of u that lie below d.
constexpr int kRotCols = 32;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) loki_rotate_kernel(const __grid_constant__ StepArgs<T> a) {
  constexpr int NB = D / kRotCols;        // column blocks per row
  constexpr int PARTS = kThreads / kRotCols;  // 8 partial sums per column
  constexpr int RPP = D / PARTS;          // rows of P per part
  __shared__ __align__(16) float Ps[D][kRotCols];
  __shared__ float qs[G][D];
  __shared__ float red[PARTS][G][kRotCols];
  griddep_launch_dependents();
  const int tid = threadIdx.x;
  const int row = blockIdx.x / NB, cb = blockIdx.x - row * NB;
  const int b = row / a.da.n_kv_heads, g = row - b * a.da.n_kv_heads;

  // P_g[:, 32cb .. 32cb+32): eight float4 per row of P, all loads issued first
  const float *Pg = a.da.P + (size_t)g * D * D + cb * kRotCols;
  float4 pv[D / 32];
#pragma unroll
  for (int r = 0; r < D / 32; ++r) {
    const int i = r * 32 + tid / 8;
    pv[r] = __ldg(reinterpret_cast<const float4 *>(Pg + (size_t)i * D) + (tid % 8));
  }
  const int Hq = a.da.n_kv_heads * G;
  const T *qg = a.da.q + ((size_t)b * Hq + (size_t)g * G) * D;
  for (int e = tid; e < G * D; e += kThreads) qs[e / D][e % D] = to_f32(qg[e]);
#pragma unroll
  for (int r = 0; r < D / 32; ++r) reinterpret_cast<float4 *>(&Ps[r * 32 + tid / 8][0])[tid % 8] = pv[r];
  __syncthreads();

  const int j = tid % kRotCols, part = tid / kRotCols;
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 8
  for (int i = part * RPP; i < (part + 1) * RPP; ++i) {
    const float p = Ps[i][j];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = fmaf(qs[h][i], p, acc[h]);
  }
#pragma unroll
  for (int h = 0; h < G; ++h) red[part][h][j] = acc[h];
  __syncthreads();

  const int col = cb * kRotCols + j;
  if (tid < G * kRotCols) {
    const int h = tid / kRotCols;
    float s = 0.f;
#pragma unroll
    for (int p = 0; p < PARTS; ++p) s += red[p][h][j];
    a.qhat[((size_t)row * G + h) * D + col] = s * a.da.scale_log2;
  }
  if (tid < kRotCols) {
    float s = 0.f;
    if (col < a.da.d) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float t = 0.f;
#pragma unroll
        for (int p = 0; p < PARTS; ++p) t += red[p][h][j];
        s += t;
      }
    }
    a.u[(size_t)row * D + col] = s;
  }
}

// ---------------------------------------------------------------------------
// decode: shared-memory layout (4-byte words).  The select phase keeps its
// histograms and candidate list in the ring (idle between the key stream and
// the gather); the tensor-core query tiles reuse the first-digit histogram.
struct FusedSmem {
  int u, qhat, pm, pl, pacc, ctl, tbl, hist, ring, keys, words;
};

__host__ __device__ inline FusedSmem fused_smem(int G, int D, int chunk) {
  FusedSmem L;
  int o = 0;
  L.u = o;    o += round4(D);
  L.qhat = o; o += G * D;
  L.pm = o;   o += 16;
  L.pl = o;   o += 16;
  L.pacc = o; o += G * D;
  L.ctl = o;  o += 128;
  L.tbl = o;  o += 2 * kMaxCluster;
  L.hist = o; o += round4(skewed_words(kDig1Bins) > 8 * D ? skewed_words(kDig1Bins) : 8 * D);

  L.ring = o; o += kRingWords;
  L.keys = o; o += round4(chunk);
  L.words = o;
  return L;
}


static_assert(skewed_words(kDig1Bins) - 8 * 128 >= kPushRecvWords && skewed_words(kDig1Bins) - 8 * 64 >= kPushRecvWords,
              "the pushed merge's receive buffer fits in the histogram words above the query tiles");

// select buffers inside the ring (word offsets).  The leader (rank 0) keeps
// the candidate slots of every CTA and its own refinement histogram; the
// distributed fallback reuses the same words once the slots are dead.
constexpr int kHref = 0;                                       // leader's refinement histogram
constexpr int kHdr = kHref + skewed_words(1 << kDig2Bits);     // [kMaxCluster][2]: candidates, count above
constexpr int kSlots = kHdr + 2 * kMaxCluster;                 // candidate keys, one slot per CTA
constexpr int kRecv2 = 0;
constexpr int kRecv3 = kRecv2 + skewed_words(1 << kDig2Bits);
constexpr int kHloc = kRecv3 + skewed_words(1 << kDig3Bits);
static_assert(kHloc + (1 << kDig2Bits) <= kRingWords, "select buffers must fit in the ring");
static_assert(kSlots + kMaxCluster * 256 <= kRingWords, "candidate slots must fit in the ring");
// Rows with S + k <= kGatherWords take the gather path: the leader reads
// every CTA's keys into its ring at kAllKeys, selects alone and writes the k
// indices after them (kAllKeys + round4(S) + 4).
constexpr int kAllKeys = skewed_words(1 << kDig2Bits);
constexpr int kGatherWords = kRingWords - kAllKeys - 8;
static_assert(kAllKeys % 4 == 0, "the gathered keys are stored 16 bytes at a time");

// ctl words (write_selection_bal uses 48..63)
constexpr int kSelWtot = 0;     // [0..7] block-scan scratch
constexpr int kSelBucket = 8;   // [8..10] bucket, count above it, count in it (this CTA's search)
constexpr int kSelFirst = 16;   // [16..18] the leader's first-digit result
constexpr int kSelOut = 20;     // [20..24] from the leader: prefix, mask, take, offset, fallback

// Among nb bins (skewed layout), find the one in which the count taken from
// the top reaches `remaining` (1 <= remaining <= total).  Result in
// ctl[kSelBucket..+2]: (bin, count in the bins above it, count in it).  Ends
// with __syncthreads().
__device__ __forceinline__ void find_bucket(const uint32_t *hist, int nb, uint32_t remaining, uint32_t *ctl) {
  const int per = nb / kThreads;
  const int lo = (int)threadIdx.x * per;
  uint32_t mine = 0u;
  for (int e = 0; e < per; ++e) mine += hist[hskew(lo + e)];
  uint32_t above = block_excl_suffix_sum(mine, ctl + kSelWtot);
  for (int e = per - 1; e >= 0; --e) {
    const uint32_t c = hist[hskew(lo + e)];
    if (above < remaining && above + c >= remaining) {
      ctl[kSelBucket + 0] = (uint32_t)(lo + e);
      ctl[kSelBucket + 1] = above;
      ctl[kSelBucket + 2] = c;
    }
    above += c;
  }
  __syncthreads();
}

// Add the non-zero bins of this CTA's histogram (nb bins, plain layout) into
// the skewed receive histogram of every CTA of the cluster (DSMEM reductions).
__device__ __forceinline__ void push_bins(int ncta, const uint32_t *local, int nb, uint32_t *recv) {
  uint32_t base[kMaxCluster];
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) base[r] = r < ncta ? dsmem_addr(recv, (uint32_t)r) : 0u;
  for (int e = threadIdx.x; e < nb; e += kThreads) {
    const uint32_t c = local[e];
    if (c) {
      const uint32_t off = 4u * (uint32_t)hskew(e);
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r)
        if (r < ncta) dsmem_red_add(base[r] + off, c);
    }
  }
}

// Add the non-zero bins of this CTA's skewed histogram into the skewed
// histogram at `dst` (a shared::cluster address, another CTA's).
__device__ __forceinline__ void push_skewed(const uint32_t *local, int nb, uint32_t dst) {
  for (int e = threadIdx.x; e < nb; e += kThreads) {
    const uint32_t c = local[hskew(e)];
    if (c) dsmem_red_add(dst + 4u * (uint32_t)hskew(e), c);
  }
}

// Warp-inclusive scan of a 32-bit value.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t t = __shfl_up_sync(kFull, v, off);
    if (lane >= off) v += t;
  }
  return v;
}

// One cluster refinement pass: keys of set[0, n) with (key & mask) == prefix
// add to bin (key >> shift) & (nb - 1); the cluster's sum lands in every CTA's
// recv (zeroed before the cluster's first barrier) and each CTA finds the
// bucket of rank `remaining` in it.
__device__ __forceinline__ void refine_pass(cg::cluster_group &cluster, int ncta, const uint32_t *set, int n,
                                            uint32_t prefix, uint32_t mask, int shift, int nb, uint32_t remaining,
                                            uint32_t *hloc, uint32_t *recv, uint32_t *ctl) {
  const int tid = threadIdx.x;
  for (int e = tid; e < nb; e += kThreads) hloc[e] = 0u;
  __syncthreads();
  for (int i = tid; i < n; i += kThreads) {
    const uint32_t key = set[i];
    if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (uint32_t)(nb - 1)], 1u);
  }
  __syncthreads();
  push_bins(ncta, hloc, nb, recv);
  cluster.sync();
  find_bucket(recv, nb, remaining, ctl);
}

// Write the CTA's selection, ascending: keys whose masked value is above
// `prefix`, and the first `take` keys (in token order) whose masked value
// equals it, from position `offset` of the row.  Warp w owns a contiguous
// segment of the CTA's tokens (a multiple of 128).  A counting sweep (four
// keys per lane and load) gives each warp its offset; the writing sweep takes
// 32 tokens per ballot, four ballots in flight: lane l's position is the
// selected count before it, popc of the above-mask below l plus the ties
// below l that are still taken, min(popc(tie-mask below l), ties left).
__device__ __forceinline__ void write_selection_bal(const uint32_t *keys, int len, int t0, const SelectState &st,
                                                    uint32_t k, uint32_t *ctl, int32_t *idx_row) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (((len + kWarps - 1) / kWarps) + 127) & ~127;
  const int sbeg = min(len, warp * seg), send = min(len, sbeg + seg);
  uint32_t gt = 0u, eq = 0u;
  for (int j0 = sbeg; j0 < send; j0 += 128) {
    const int j = j0 + 4 * lane;
    if (j < send) {
      const uint4 v = *reinterpret_cast<const uint4 *>(keys + j);
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (j + e < send) {
          const uint32_t km = kk[e] & st.mask;
          gt += km > st.prefix;
          eq += km == st.prefix;
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    gt += __shfl_xor_sync(kFull, gt, off);
    eq += __shfl_xor_sync(kFull, eq, off);
  }
  if (lane == 0) {
    ctl[kCtlWarpGt + warp] = gt;
    ctl[kCtlWarpEq + warp] = eq;
  }
  __syncthreads();
  const uint32_t take = st.take;
  uint32_t run_eq = 0u, run_sel = 0u;
  for (int w = 0; w < warp; ++w) {
    const uint32_t want = take > run_eq ? take - run_eq : 0u;
    run_sel += ctl[kCtlWarpGt + w] + min(ctl[kCtlWarpEq + w], want);
    run_eq += ctl[kCtlWarpEq + w];
  }
  int32_t *dst = idx_row + st.offset;
  const uint32_t lt = lanemask_lt();
  for (int j0 = sbeg; j0 < send; j0 += 128) {
    uint32_t gb[4], eb[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int j = j0 + 32 * x + lane;
      const bool in = j < send;
      const uint32_t km = in ? (keys[j] & st.mask) : 0u;
      gb[x] = __ballot_sync(kFull, in && km > st.prefix);
      eb[x] = __ballot_sync(kFull, in && km == st.prefix);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const uint32_t left = take > run_eq ? take - run_eq : 0u;  // ties still taken
      const uint32_t me = 1u << lane;
      const uint32_t ties_below = __popc(eb[x] & lt);
      const bool sel = (gb[x] & me) != 0u || ((eb[x] & me) != 0u && ties_below < left);
      const uint32_t p = run_sel + __popc(gb[x] & lt) + min(ties_below, left);
      if (sel && st.offset + p < k) dst[p] = t0 + j0 + 32 * x + lane;  // bound: the row holds k entries
      run_sel += __popc(gb[x]) + min((uint32_t)__popc(eb[x]), left);
      run_eq += __popc(eb[x]);
    }
  }
}

// Per-warp token lists.  Once the first digit's bucket is known, every token
// that can still be selected has key & mask >= prefix (above the bucket or in
// it): a few times k/S of the tokens.  One ballot sweep compacts them, per
// warp and in token order, into lists in the first-digit histogram's words
// (free from then until the attention): warp w owns the same segment of the
// tokens as in write_selection_bal and its list holds up to kListCap token
// offsets (16 bits).  The refinement passes and the ordered write then visit
// the lists instead of every token.
constexpr int kCtlWarpN = 64;   // [64..71] entries of warp w's list
constexpr int kCtlWarpAb = 72;  // [72..79] its tokens above the bucket
constexpr int kCtlWarpCd = 80;  // [80..87] its tokens in the bucket
constexpr int kListCap = 2 * skewed_words(kDig1Bins) / kWarps;  // 16-bit entries per warp
static_assert(kListCap % 2 == 0 && kMaxChunk < 65536 && kGatherWords < 65536,
              "list entries are 16-bit token offsets; each warp's list starts on a 4-byte boundary");

// The lists of keys[0, len) for (prefix, mask).  Returns true (uniform over
// the CTA) when every warp's list fit; the counts are in ctl either way.
// Ends with __syncthreads().
__device__ __forceinline__ bool list_sweep(const uint32_t *keys, int len, uint32_t prefix, uint32_t mask,
                                           uint16_t *lists, uint32_t *ctl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = (((len + kWarps - 1) / kWarps) + 127) & ~127;
  const int sbeg = min(len, warp * seg), send = min(len, sbeg + seg);
  uint16_t *wl = lists + warp * kListCap;
  const uint32_t lt = lanemask_lt();
  uint32_t n = 0u, ab = 0u, cd = 0u;
  for (int j0 = sbeg; j0 < send; j0 += 128) {
    uint32_t gb[4], eb[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int j = j0 + 32 * x + lane;
      const bool in = j < send;
      const uint32_t km = in ? (keys[j] & mask) : 0u;
      gb[x] = __ballot_sync(kFull, in && km > prefix);
      eb[x] = __ballot_sync(kFull, in && km == prefix);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const uint32_t bx = gb[x] | eb[x];
      const uint32_t p = n + __popc(bx & lt);
      if (((bx >> lane) & 1u) != 0u && p < (uint32_t)kListCap) wl[p] = (uint16_t)(j0 + 32 * x + lane);
      n += __popc(bx);
      ab += __popc(gb[x]);
      cd += __popc(eb[x]);
    }
  }
  if (lane == 0) {
    ctl[kCtlWarpN + warp] = n;
    ctl[kCtlWarpAb + warp] = ab;
    ctl[kCtlWarpCd + warp] = cd;
  }
  __syncthreads();
  bool fit = true;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) fit &= ctl[kCtlWarpN + w] <= (uint32_t)kListCap;
  return fit;
}

// write_selection_bal over the lists of list_sweep (which hold every token
// the final (prefix, mask) can select, in token order).
__device__ __forceinline__ void write_selection_list(const uint32_t *keys, const uint16_t *lists, int t0,
                                                     const SelectState &st, uint32_t k, uint32_t *ctl,
                                                     int32_t *idx_row) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint16_t *wl = lists + warp * kListCap;
  const int n = (int)ctl[kCtlWarpN + warp];
  uint32_t gt = 0u, eq = 0u;
  for (int i = lane; i < n; i += 32) {
    const uint32_t km = keys[wl[i]] & st.mask;
    gt += km > st.prefix;
    eq += km == st.prefix;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    gt += __shfl_xor_sync(kFull, gt, off);
    eq += __shfl_xor_sync(kFull, eq, off);
  }
  if (lane == 0) {
    ctl[kCtlWarpGt + warp] = gt;
    ctl[kCtlWarpEq + warp] = eq;
  }
  __syncthreads();
  const uint32_t take = st.take;
  uint32_t run_eq = 0u, run_sel = 0u;
  for (int w = 0; w < warp; ++w) {
    const uint32_t want = take > run_eq ? take - run_eq : 0u;
    run_sel += ctl[kCtlWarpGt + w] + min(ctl[kCtlWarpEq + w], want);
    run_eq += ctl[kCtlWarpEq + w];
  }
  int32_t *dst = idx_row + st.offset;
  const uint32_t lt = lanemask_lt(), me = 1u << lane;
  for (int i0 = 0; i0 < n; i0 += 64) {
    // two ballots of 32 list entries in flight
    uint32_t gb[2], eb[2];
    int tok[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int i = i0 + 32 * x + lane;
      const bool in = i < n;
      tok[x] = in ? (int)wl[i] : 0;
      const uint32_t km = in ? (keys[tok[x]] & st.mask) : 0u;
      gb[x] = __ballot_sync(kFull, in && km > st.prefix);
      eb[x] = __ballot_sync(kFull, in && km == st.prefix);
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const uint32_t left = take > run_eq ? take - run_eq : 0u;  // ties still taken
      const uint32_t ties_below = __popc(eb[x] & lt);
      const bool sel = (gb[x] & me) != 0u || ((eb[x] & me) != 0u && ties_below < left);
      const uint32_t p = run_sel + __popc(gb[x] & lt) + min(ties_below, left);
      if (sel && st.offset + p < k) dst[p] = t0 + tok[x];  // bound: the row holds k entries
      run_sel += __popc(gb[x]) + min((uint32_t)__popc(eb[x]), left);
      run_eq += __popc(eb[x]);
    }
  }
}

// ---------------------------------------------------------------------------
template <typename T, int D, int G, bool PAGED>
__global__ void __launch_bounds__(kThreads, (G >= 8) ? 1 : 2) loki_decode_kernel(const __grid_constant__ StepArgs<T> a) {
  extern __shared__ __align__(16) uint32_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int ncta = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / ncta;
  const int b = row / a.da.n_kv_heads, g = row - b * a.da.n_kv_heads;
  const FusedSmem L = fused_smem(G, D, a.da.chunk);
  float *u = reinterpret_cast<float *>(smem + L.u);
  float *qhat = reinterpret_cast<float *>(smem + L.qhat);
  float *pm = reinterpret_cast<float *>(smem + L.pm);
  float *pl = reinterpret_cast<float *>(smem + L.pl);
  float *pacc = reinterpret_cast<float *>(smem + L.pacc);
  uint32_t *ctl = smem + L.ctl;
  uint32_t *tbl = smem + L.tbl;
  uint32_t *hist = smem + L.hist;
  unsigned char *ring = reinterpret_cast<unsigned char *>(smem + L.ring);
  uint32_t *rw = smem + L.ring;  // the ring as words, for the select buffers
  uint32_t *keys = smem + L.keys;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int S = row_seq_len(a.da, b);
  const uint32_t k = (uint32_t)row_k(a.da, b, S);
  const int t0 = min(S, rank * a.da.chunk);
  const int len = min(S, t0 + a.da.chunk) - t0;
  const Rows<T, D, PAGED> rows = make_rows<T, D, PAGED>(a.da, b, g);
  constexpr int MAXL = D / VecN<T>::value;
  LOKI_PHASE(0);

  // 1. the queries (q_hat, u) and the key stream; the stream's first stages
  // go in flight before u is needed.  An appended token sits at the row's
  // last position: the CTA that owns it rotates and stores it, streams the
  // rest and scores it from the stored values (query groups of up to 4 heads;
  // the host appends first for 8)
  const bool own = kRotateInKernel<G> && a.da.k_new != nullptr && len > 0 && S - 1 < t0 + len;
  const int slen = own ? len - 1 : len;
  float *xkh = pacc;  // D floats, free until the attention
  if constexpr (kRotateInKernel<G>) {
    // q_hat and u from q and P_g here (the histogram words are scratch until
    // zeroed), with the stream's first stages in flight behind the loads
    rotate_queries<T, D, G>(
        a.da, b, g, qhat, u, reinterpret_cast<float *>(hist), true,
        [&] {
          LOKI_LPT_DISPATCH(a.da.lpt, MAXL,
                            (score_prologue<T, D, L_, kScoreStageBytes, kScoreStages>(rows, t0, slen, a.da.nck, ring)));
        },
        own ? a.da.k_new + ((size_t)b * a.da.n_kv_heads + g) * D : nullptr, xkh);
    if (own) store_appended<T, D, PAGED>(a.da, rows, b, g, S - 1, xkh);
  } else {
    // q_hat and u from the rotate grid (a programmatic dependency)
    LOKI_LPT_DISPATCH(a.da.lpt, MAXL,
                      (score_prologue<T, D, L_, kScoreStageBytes, kScoreStages>(rows, t0, len, a.da.nck, ring)));
    griddep_wait();
    if (tid < D) u[tid] = __ldcg(a.u + (size_t)row * D + tid);
    for (int e = tid; e < G * D; e += kThreads) qhat[e] = __ldcg(a.qhat + (size_t)row * G * D + e);
  }
  for (int e = tid; e < skewed_words(kDig1Bins); e += kThreads) hist[e] = 0u;
  __syncthreads();
  LOKI_PHASE(1);
  cluster_arrive();  // this CTA's histogram is zero (the leader's receives the others')
  LOKI_LPT_DISPATCH(a.da.lpt, MAXL,
                    (score_keys_loop<T, D, L_, kScoreStageBytes, kScoreStages, 32 - kDig1Bits>(
                        rows, t0, slen, a.da.nck, ring, u, keys, hist)));
  if (own) {
    // the appended token's key, from its stored (rounded) values
    if (warp == 0) {
      float sc = 0.f;
      for (int i = lane; i < a.da.d; i += 32) sc = fmaf(u[i], xkh[i], sc);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sc += __shfl_xor_sync(kFull, sc, off);
      if (lane == 0) {
        const uint32_t key = score_key(sc);
        keys[len - 1] = key;
        atomicAdd(&hist[hskew((int)(key >> (32 - kDig1Bits)))], 1u);
      }
    }
    __syncthreads();
  }

  LOKI_PHASE(2);
  // 2. cluster radix select; the ring is idle until the gather
  const bool leader = rank == 0;
  int32_t *idx_row = a.da.idx + (size_t)row * a.da.k_stride;
  const int s0 = (int)(((long long)rank * k) / ncta);  // this CTA's even share of the selection
  const int s1 = (int)(((long long)(rank + 1) * k) / ncta);
  int32_t *ids = reinterpret_cast<int32_t *>(keys);  // the share's indices, where the keys were
  const bool gather = S + (int)k <= kGatherWords;    // uniform over the cluster
  cluster_wait();  // every CTA, the leader in particular, zeroed its histogram before its stream
  if (gather) {
    // S + k within the leader's ring: the leader collects the histogram, then reads every CTA's
    // keys (distributed shared memory; CTA r holds tokens [r*chunk, ..),
    // chunk a multiple of 4) into its ring and selects alone
    if (!leader) push_skewed(hist, kDig1Bins, dsmem_addr(hist, 0u));
    cluster.sync();  // every stream is done; the leader's histogram holds the row's
    LOKI_PHASE(3);
    uint32_t *all = rw + kAllKeys;
    if (leader) {
      const int n4 = (S + 3) >> 2;
      for (int j0 = tid; j0 < n4; j0 += 4 * kThreads) {
        uint4 v[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int j4 = j0 + x * kThreads;
          if (j4 < n4) {
            const int r = (4 * j4) / a.da.chunk;
            v[x] = dsmem_ld_v4(dsmem_addr(keys + (4 * j4 - r * a.da.chunk), (uint32_t)r));
          }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
          if (j0 + x * kThreads < n4) reinterpret_cast<uint4 *>(all)[j0 + x * kThreads] = v[x];
      }
      __syncthreads();
    }
    int32_t *list = reinterpret_cast<int32_t *>(all + round4(S) + 4);
    if (leader) {
      constexpr int SH2 = 32 - kDig1Bits - kDig2Bits;
      uint32_t *href = rw + kHref;
      find_bucket(hist, kDig1Bins, k, ctl);
      uint32_t rem = k - ctl[kSelBucket + 1], inb = ctl[kSelBucket + 2];
      uint32_t pre = ctl[kSelBucket + 0] << (32 - kDig1Bits), msk = ~0u << (32 - kDig1Bits);
      // lists when they are likely to fit (tokens at or above the bucket: k - rem + inb)
      const bool try_lists = k - rem + inb <= (uint32_t)(kWarps * kListCap * 3 / 4);
      __syncthreads();  // ctl and the histogram read before they are reused
      uint16_t *lists = reinterpret_cast<uint16_t *>(hist);
      const bool listed = try_lists && list_sweep(all, S, pre, msk, lists, ctl);
      for (int pass = 0; pass < 2 && inb != rem; ++pass) {
        const int shift = pass == 0 ? SH2 : 0;
        const int nb = pass == 0 ? (1 << kDig2Bits) : (1 << kDig3Bits);
        for (int e = tid; e < skewed_words(1 << kDig2Bits); e += kThreads) href[e] = 0u;
        __syncthreads();
        if (listed) {
          const uint16_t *wl = lists + warp * kListCap;
          const int n = (int)ctl[kCtlWarpN + warp];
          for (int i = lane; i < n; i += 32) {
            const uint32_t key = all[wl[i]];
            if ((key & msk) == pre) atomicAdd(&href[hskew((int)((key >> shift) & (uint32_t)(nb - 1)))], 1u);
          }
        } else {
          for (int i = tid; i < S; i += kThreads) {
            const uint32_t key = all[i];
            if ((key & msk) == pre) atomicAdd(&href[hskew((int)((key >> shift) & (uint32_t)(nb - 1)))], 1u);
          }
        }
        __syncthreads();
        find_bucket(href, nb, rem, ctl);
        rem -= ctl[kSelBucket + 1];
        inb = ctl[kSelBucket + 2];
        pre |= ctl[kSelBucket + 0] << shift;
        msk |= (uint32_t)(nb - 1) << shift;
        __syncthreads();  // ctl read before it is reused
      }
      if (listed)
        write_selection_list(all, lists, 0, SelectState{pre, msk, rem, 0u}, k, ctl, list);
      else
        write_selection_bal(all, S, 0, SelectState{pre, msk, rem, 0u}, k, ctl, list);
    }
    cluster.sync();  // the leader's list of the k indices is complete (and it read every CTA's keys)
    const uint32_t src = dsmem_addr(list + s0, 0u);
    for (int i = tid; i < s1 - s0; i += kThreads) {
      const int v = (int)dsmem_ld_u32(src + 4u * (uint32_t)i);
      idx_row[s0 + i] = v;
      ids[i] = min(max(v, 0), S - 1);
    }
    // a row shorter than the longest one: the rest of its idx row is -1
    for (int i = (int)k + rank * kThreads + tid; i < a.da.k_stride; i += ncta * kThreads) idx_row[i] = -1;
    cluster_arrive();  // done reading the leader's ring
    if (leader) cluster_wait();  // its ring is about to carry the gather
  } else {
  if (!leader) push_skewed(hist, kDig1Bins, dsmem_addr(hist, 0u));
  cluster.sync();  // the leader's histogram holds the cluster's sum
  if (leader) {
    find_bucket(hist, kDig1Bins, k, ctl);
    if (tid < ncta) {
      const uint32_t dst = dsmem_addr(ctl + kSelFirst, (uint32_t)tid);
      dsmem_st(dst, ctl[kSelBucket + 0]);
      dsmem_st(dst + 4u, ctl[kSelBucket + 1]);
      dsmem_st(dst + 8u, ctl[kSelBucket + 2]);
    }
  }
  cluster.sync();
  LOKI_PHASE(3);
  uint32_t remaining = k - ctl[kSelFirst + 1];
  const bool refine = ctl[kSelFirst + 2] != remaining;  // else the whole bucket is taken
  uint32_t prefix = ctl[kSelFirst + 0] << (32 - kDig1Bits);
  uint32_t mask = ~0u << (32 - kDig1Bits);
  const int cap = ((kRingWords - kSlots) / ncta) & ~3;  // candidate slot per CTA, at the leader
  uint32_t *href = rw + kHref, *hdr = rw + kHdr;

  // this CTA's candidates (its keys in the bucket) into its slot at the
  // leader, with its count of candidates and of keys above the bucket: from
  // the per-warp lists, or (when a list overflows) from sweeps of every key
  uint16_t *lists = reinterpret_cast<uint16_t *>(hist);  // every histogram is dead from here to the attention
  // lists when they are likely to fit: the cluster's tokens at or above the
  // bucket number ctl[kSelFirst + 1] + ctl[kSelFirst + 2] (uniform decision)
  const bool try_lists =
      ctl[kSelFirst + 1] + ctl[kSelFirst + 2] <= (uint32_t)(ncta * kWarps * kListCap * 3 / 4);
  const bool listed = try_lists && list_sweep(keys, len, prefix, mask, lists, ctl);
  if (listed) {
    uint32_t total = 0u, above = 0u, before = 0u;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t c = ctl[kCtlWarpCd + w];
      total += c;
      above += ctl[kCtlWarpAb + w];
      before += w < warp ? c : 0u;
    }
    if (refine && total <= (uint32_t)cap) {
      // warp w's candidates at [before, before + its count) of the slot
      const uint32_t slot = dsmem_addr(rw + kSlots + rank * cap, 0u);
      const uint16_t *wl = lists + warp * kListCap;
      const int n = (int)ctl[kCtlWarpN + warp];
      const uint32_t lt = lanemask_lt();
      uint32_t pos = before;
      for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < n ? keys[wl[i]] : 0u;
        const bool c = i < n && (key & mask) == prefix;
        const uint32_t bc = __ballot_sync(kFull, c);
        if (c) dsmem_st(slot + 4u * (pos + __popc(bc & lt)), key);
        pos += __popc(bc);
      }
    }
    if (tid == 0) {
      const uint32_t h = dsmem_addr(hdr + 2 * rank, 0u);
      dsmem_st(h, total);
      dsmem_st(h + 4u, above);
    }
  } else {
    const int n4 = (len + 3) >> 2;
    uint32_t mine = 0u, above = 0u;
    for (int j4 = tid; j4 < n4; j4 += kThreads) {
      const uint4 v = reinterpret_cast<const uint4 *>(keys)[j4];
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (4 * j4 + e < len) {
          const uint32_t km = kk[e] & mask;
          mine += km == prefix;
          above += km > prefix;
        }
      }
    }
    const uint32_t after = block_excl_suffix_sum(mine, ctl + kSelWtot);
    const uint32_t total = block_sum(mine, ctl + kSelWtot);
    above = block_sum(above, ctl + kSelWtot);
    if (refine && total <= (uint32_t)cap) {
      const uint32_t slot = dsmem_addr(rw + kSlots + rank * cap, 0u);
      uint32_t pos = total - after - mine;
      for (int j4 = tid; j4 < n4; j4 += kThreads) {
        const uint4 v = reinterpret_cast<const uint4 *>(keys)[j4];
        const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (4 * j4 + e < len && (kk[e] & mask) == prefix) {
            dsmem_st(slot + 4u * pos, kk[e]);
            ++pos;
          }
        }
      }
    }
    if (tid == 0) {
      const uint32_t h = dsmem_addr(hdr + 2 * rank, 0u);
      dsmem_st(h, total);
      dsmem_st(h + 4u, above);
    }
  }
  cluster.sync();  // the leader holds every CTA's candidates and counts

  // the leader finishes the threshold on the union of the candidates, then
  // gives every CTA its (prefix, mask, take, offset)
  if (leader) {
    bool overflow = false;
    for (int r = 0; r < ncta; ++r) overflow |= hdr[2 * r] > (uint32_t)cap;
    uint32_t pre = prefix, msk = mask, rem = remaining;
    if (refine && !overflow) {
      constexpr int SH2 = 32 - kDig1Bits - kDig2Bits;
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? SH2 : 0;
        const int nb = pass == 0 ? (1 << kDig2Bits) : (1 << kDig3Bits);
        for (int e = tid; e < skewed_words(1 << kDig2Bits); e += kThreads) href[e] = 0u;
        __syncthreads();
        for (int r = 0; r < ncta; ++r) {
          const uint32_t *sl = rw + kSlots + r * cap;
          for (int i = tid; i < (int)hdr[2 * r]; i += kThreads) {
            const uint32_t key = sl[i];
            if ((key & msk) == pre) atomicAdd(&href[hskew((int)((key >> shift) & (uint32_t)(nb - 1)))], 1u);
          }
        }
        __syncthreads();
        find_bucket(href, nb, rem, ctl);
        rem -= ctl[kSelBucket + 1];
        const uint32_t inb = ctl[kSelBucket + 2];
        pre |= ctl[kSelBucket + 0] << shift;
        msk |= (uint32_t)(nb - 1) << shift;
        __syncthreads();  // ctl read before it is reused
        if (inb == rem) break;
      }
      // every CTA's counts above and at the threshold (warp w: CTAs w, w+8)
      for (int r = warp; r < ncta; r += kWarps) {
        const uint32_t *sl = rw + kSlots + r * cap;
        uint32_t gtc = 0u, eqc = 0u;
        for (int i = lane; i < (int)hdr[2 * r]; i += 32) {
          const uint32_t km = sl[i] & msk;
          gtc += km > pre;
          eqc += km == pre;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          gtc += __shfl_xor_sync(kFull, gtc, off);
          eqc += __shfl_xor_sync(kFull, eqc, off);
        }
        if (lane == 0) {
          tbl[r] = gtc + hdr[2 * r + 1];
          tbl[kMaxCluster + r] = eqc;
        }
      }
    } else if (!refine) {
      if (tid < ncta) {
        tbl[tid] = hdr[2 * tid + 1];
        tbl[kMaxCluster + tid] = hdr[2 * tid];
      }
    }
    __syncthreads();
    if (tid == 0) {
      // ties at the threshold go to the lower index: lower CTAs first
      const uint32_t fallback = (refine && overflow) ? 1u : 0u;
      uint32_t eq_before = 0u, off = 0u;
      for (int r = 0; r < ncta; ++r) {
        const uint32_t eqr = tbl[kMaxCluster + r];
        const uint32_t take_r = fallback ? 0u : min(eqr, rem > eq_before ? rem - eq_before : 0u);
        const uint32_t dst = dsmem_addr(ctl + kSelOut, (uint32_t)r);
        dsmem_st(dst, pre);
        dsmem_st(dst + 4u, msk);
        dsmem_st(dst + 8u, take_r);
        dsmem_st(dst + 12u, off);
        dsmem_st(dst + 16u, fallback);
        off += tbl[r] + take_r;
        eq_before += eqr;
      }
    }
  }
  cluster.sync();
  uint32_t take, offset;
  if (ctl[kSelOut + 4] == 0u) {
    prefix = ctl[kSelOut + 0];
    mask = ctl[kSelOut + 1];
    take = ctl[kSelOut + 2];
    offset = ctl[kSelOut + 3];
  } else {
    // a candidate slot overflowed (uniform over the cluster): distributed
    // refinement passes over every CTA's own keys
    uint32_t *recv2 = rw + kRecv2, *recv3 = rw + kRecv3, *hloc = rw + kHloc;
    for (int e = tid; e < kHloc - kRecv2; e += kThreads) recv2[e] = 0u;  // recv2 and recv3
    cluster.sync();  // every CTA's receive histograms are zero
    constexpr int SH2 = 32 - kDig1Bits - kDig2Bits;
    refine_pass(cluster, ncta, keys, len, prefix, mask, SH2, 1 << kDig2Bits, remaining, hloc, recv2, ctl);
    remaining -= ctl[kSelBucket + 1];
    prefix |= ctl[kSelBucket + 0] << SH2;
    mask |= (uint32_t)((1 << kDig2Bits) - 1) << SH2;
    if (ctl[kSelBucket + 2] != remaining) {  // uniform over the cluster
      refine_pass(cluster, ncta, keys, len, prefix, mask, 0, 1 << kDig3Bits, remaining, hloc, recv3, ctl);
      remaining -= ctl[kSelBucket + 1];
      prefix |= ctl[kSelBucket + 0];
      mask = ~0u;
    }
    uint32_t gt = 0u, eq = 0u;
    for (int j4 = tid; j4 < (len + 3) >> 2; j4 += kThreads) {
      const uint4 v = reinterpret_cast<const uint4 *>(keys)[j4];
      const uint32_t kk[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (4 * j4 + e < len) {
          const uint32_t km = kk[e] & mask;
          gt += km > prefix;
          eq += km == prefix;
        }
      }
    }
    gt = block_sum(gt, ctl + kSelWtot);
    eq = block_sum(eq, ctl + kSelWtot);
    if (tid < ncta) {
      dsmem_st(dsmem_addr(tbl + rank, (uint32_t)tid), gt);
      dsmem_st(dsmem_addr(tbl + kMaxCluster + rank, (uint32_t)tid), eq);
    }
    cluster.sync();
    // ties at the threshold go to the lower index: lower CTAs first
    uint32_t eq_before = 0u;
    offset = 0u;
    for (int r = 0; r < rank; ++r) {
      const uint32_t want = remaining > eq_before ? remaining - eq_before : 0u;
      offset += tbl[r] + min(tbl[kMaxCluster + r], want);
      eq_before += tbl[kMaxCluster + r];
    }
    take = min(eq, remaining > eq_before ? remaining - eq_before : 0u);
  }
  if (listed)
    write_selection_list(keys, lists, t0, SelectState{prefix, mask, take, offset}, k, ctl, idx_row);
  else
    write_selection_bal(keys, len, t0, SelectState{prefix, mask, take, offset}, k, ctl, idx_row);
  // a row shorter than the longest one: the rest of its idx row is -1
  for (int i = (int)k + rank * kThreads + tid; i < a.da.k_stride; i += ncta * kThreads) idx_row[i] = -1;
  cluster.sync();  // the whole row of idx is written and visible to the cluster
  // the share's indices, clamped into the row so that no load can leave the
  // cache even if wrong
  for (int i = tid; i < s1 - s0; i += kThreads) ids[i] = min(max(__ldcg(idx_row + s0 + i), 0), S - 1);
  }  // gather / candidate paths

  // 3. attention over this CTA's even share of the k selected rows (the
  // share is at most chunk)
  __syncthreads();
  LOKI_PHASE(4);
  if constexpr (PAGED) {
    // the share's token positions become rows of the page pools first (one
    // page-table load each, all in flight at once), so that the gather loop
    // computes no page addresses of its own
    for (int i = tid; i < s1 - s0; i += kThreads) ids[i] = rows.phys(ids[i]);
    __syncthreads();
    const Rows<T, D, false> pool = pool_rows<T, D>(a.da);
    attend_prologue_any<T, D, G, true>(pool, ids, 0, s1 - s0, ring);
    attend_loop_any<T, D, G, true>(pool, ids, 0, s1 - s0, qhat, reinterpret_cast<unsigned char *>(hist), ring,
                                   pm, pl, pacc);
  } else {
    attend_prologue_any<T, D, G, true>(rows, ids, 0, s1 - s0, ring);
    attend_loop_any<T, D, G, true>(rows, ids, 0, s1 - s0, qhat, reinterpret_cast<unsigned char *>(hist), ring,
                                   pm, pl, pacc);
  }

  LOKI_PHASE(5);
  // 4. log-sum-exp merge of the cluster's states: pushed into the owners'
  // receive buffers (above the tensor-core query tiles in the histogram words,
  // dead since the select) when they fit, else read from every CTA
  const int Hq = a.da.n_kv_heads * G;
  float *out = a.da.out + ((size_t)b * Hq + (size_t)g * G) * D;
  __syncthreads();  // the CTA's state is complete
  const bool push = push_merge_fits(G, D, ncta);
  float *recv = reinterpret_cast<float *>(hist) + 8 * D;
  if (push) push_state<D, G>(ncta, rank, pm, pl, pacc, recv);
  if (gather && !leader) cluster_wait();
  if (ncta == 1) {
    local_combine<D, G>(pl, pacc, out);
  } else if (push) {
    cluster.sync();
    push_combine<D, G>(ncta, rank, recv, out);
  } else {
    cluster.sync();
    cluster_combine<D, G>(ncta, rank, pm, pl, pacc, out);
    cluster.sync();
  }
  LOKI_PHASE(6);
#ifdef LOKI_PHASE_STAMPS
  if (tid == 0 && blockIdx.x < kMaxStampCtas) {
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    g_phase_stamps[blockIdx.x][7] = sm;
    g_phase_stamps[blockIdx.x][8] = (unsigned long long)rank | ((unsigned long long)ncta << 8) |
                                    ((unsigned long long)(gather ? 1 : 0) << 16);
    g_phase_stamps[blockIdx.x][9] = (unsigned long long)row;
  }
#endif
}

}  // namespace loki
