/*
 * loki.h -- C ABI of libloki.so: Loki sparse decode-step attention on one
 * NVIDIA B200 (sm_100a).
 *
 * The method ("Loki: Low-rank Keys for Efficient Sparse Attention",
 * atlas.scime.ai summary, sections "Approach" and the summary paragraph;
 * mlsanity.com arXiv record 2406.02542, "Abstract"):  keys and queries are
 * projected into a PCA basis P calibrated offline; every cached token is ranked
 * by its attention score computed on the first d principal dimensions only; the
 * k best tokens are kept and exact softmax attention is computed over them.
 * No cache entry is ever deleted.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All pointers are DEVICE pointers of the current CUDA device unless stated,
 *    owned by the caller.  The library never allocates, frees or synchronises;
 *    it keeps no state between calls except per-device attribute caches.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream) and runs asynchronously.  A call returns after the
 *    launch is enqueued; results are ready when the stream reaches that point.
 *  - Tensors are dense, row-major (last index fastest), with no padding.
 *  - dtype LOKI_F32 (fp32) or LOKI_BF16 (bfloat16) applies to the cache and to
 *    q, k_new and v_new.  P is always fp32.  Outputs `out` are always fp32.
 *  - Validation happens on the host before anything is launched.  On invalid
 *    arguments the call returns LOKI_ERR_INVALID_ARG (or LOKI_ERR_UNSUPPORTED
 *    for a valid but unimplemented shape) and enqueues nothing.  A failed launch
 *    returns LOKI_ERR_CUDA.  loki_last_error() gives a one-line message for the
 *    calling thread's last failure.  Kernels never trap or assert.
 *  - Inputs must be finite (no NaN or Inf); this precondition is not checked.
 *
 * Sizes:  B batch, Hq query heads, Hkv KV heads (Hq % Hkv == 0, G = Hq / Hkv
 * query heads share KV head g = h / G), D head dimension (64 or 128), S_cap
 * cache capacity in tokens, seq_len tokens currently attended.
 */
#ifndef LOKI_H
#define LOKI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LOKI_VERSION 13

/* Symbols are exported from the shared object; everything else is hidden. */
#if defined(LOKI_BUILD) && defined(__GNUC__)
#define LOKI_API __attribute__((visibility("default")))
#else
#define LOKI_API
#endif

typedef enum {
  LOKI_OK = 0,
  LOKI_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or range           */
  LOKI_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement     */
  LOKI_ERR_CUDA = 3          /* the CUDA runtime refused a launch or attribute  */
} loki_status;

typedef enum { LOKI_F32 = 0, LOKI_BF16 = 1 } loki_dtype;

/* A rotated-key KV cache in caller-owned device memory.
 *   k_hat : [B, Hkv, S_cap, D] keys already rotated into the PCA basis
 *           (k_hat = k . P_g), in `dtype`; 16-byte aligned.
 *   v     : [B, Hkv, S_cap, D] values, unrotated, in `dtype`; 16-byte aligned.
 *   k_lr  : optional low-rank key plane, [B, Hkv, S_cap, d_lr] in `dtype`,
 *           16-byte aligned, or NULL.  It holds a copy of the first d_lr
 *           dimensions of every key row, k_lr[b][g][t][j] = k_hat[b][g][t][j]
 *           for j < d_lr, kept by every call that writes keys (loki_append,
 *           loki_paged_append and the *_append decode calls).  A Loki decode with d <= d_lr streams
 *           the low-rank scores from it instead of from k_hat: HBM serves
 *           reads in whole 128-byte lines, so reading d < 64 bf16 dimensions
 *           of each 256-byte k_hat row costs a full line per token, while the
 *           plane's rows are contiguous.  Results are bit-identical with and
 *           without the plane.  Costs d_lr / D of the key cache in memory.
 *   d_lr  : the plane's width, with d_lr * sizeof(dtype) a multiple of 16
 *           bytes and d_lr <= D; ignored when k_lr is NULL.
 * The cache holds every token ever appended: entries are never evicted, so its
 * footprint equals a dense cache ("Limitations" section of the summary page),
 * plus the plane when there is one. */
typedef struct {
  int32_t dtype;       /* loki_dtype                                          */
  int32_t batch;       /* B >= 1                                              */
  int32_t n_kv_heads;  /* Hkv >= 1                                            */
  int32_t head_dim;    /* D: 64 or 128                                        */
  int32_t capacity;    /* S_cap >= 1                                          */
  void *k_hat;
  void *v;
  void *k_lr;          /* optional low-rank key plane, or NULL                */
  int32_t d_lr;        /* its width (elements per token)                      */
} loki_cache;

/* loki_append -- rotate new keys into the PCA basis and append them, with
 * their values, at token positions [pos, pos + n_new) of every (batch, KV head)
 * row.  Source: summary page, section "Approach" ("PCA-project ... keys") and
 * "Surprising findings" (appending KV-cache entries is a large share of
 * inference time).
 *   k_new, v_new : [B, Hkv, n_new, D] in the cache dtype, 16-byte aligned.
 *   P            : [Hkv, D, D] fp32; P[g][i][j] is component i of the j-th
 *                  principal direction of KV head g (column j = direction j,
 *                  sorted by descending eigenvalue).  16-byte aligned.
 * Computes k_hat[b][g][pos+t][j] = round_to_dtype( sum_i k_new[b][g][t][i] *
 * P[g][i][j] ) with fp32 accumulation and round-to-nearest-even, writes the
 * same values for j < d_lr into the low-rank plane when the cache has one, and
 * copies v_new unchanged.  Entries outside [pos, pos + n_new) are not touched.
 * bf16 caches with B * n_new >= 256 take the tensor-core path: P is split into
 * three bf16 terms (summing to P within 2^-27 relative) and the 3*D products
 * are accumulated in fp32 by tcgen05.mma before the single rounding.
 * Requires 0 <= pos, 1 <= n_new, pos + n_new <= S_cap. */
LOKI_API loki_status loki_append(const loki_cache *cache, int32_t pos, int32_t n_new,
                        const void *k_new, const void *v_new, const float *P,
                        void *stream);

/* loki_decode_workspace_size -- bytes of device workspace that
 * loki_decode_attention needs for a cache of this shape with n_q_heads query
 * heads: room for the rotated queries and the low-rank group queries of every
 * (batch, KV head) row, B * Hkv * (G + 1) * D * 4 bytes plus alignment (the
 * call writes them there when its query groups have 8 heads; smaller groups
 * rotate their queries on chip and leave it untouched).  *bytes is a host
 * pointer. */
LOKI_API loki_status loki_decode_workspace_size(const loki_cache *cache, int32_t seq_len,
                                       int32_t n_q_heads, size_t *bytes);

/* loki_decode_attention -- one Loki decode step over tokens [0, seq_len).
 * Source: summary page, summary paragraph and section "Approach"; arXiv
 * record "Abstract".
 *   q     : [B, Hq, D] queries in the cache dtype (NOT rotated), 16-byte aligned.
 *   P     : [Hkv, D, D] fp32, the basis the cache keys were rotated with;
 *           16-byte aligned.
 *   d     : reduced dimension, 1 <= d <= D (the first d principal dims).
 *   k     : key budget, 1 <= k <= seq_len.
 *   scale : softmax scale of the exact attention; <= 0 selects 1/sqrt(D).
 *   out   : [B, Hq, D] fp32 output (written).
 *   idx   : [B, Hkv, k] int32 selected token indices (written), ascending.
 *   workspace, workspace_bytes : caller-owned device scratch of at least
 *           loki_decode_workspace_size() bytes, 256-byte aligned.  Its contents
 *           need no initialisation and are undefined after the call.  Calls
 *           that may run at the same time (other streams) must not share a
 *           workspace.
 * Per (b, g): q_hat_h = q_h . P_g (fp32, never rounded to the cache dtype);
 * score_i = sum over the G query heads h of group g of q_hat_h[:d] . k_hat_i[:d];
 * the k tokens with the largest scores are selected, ties going to the lower
 * index; out_h = softmax(scale * q_hat_h . k_hat_i over the selected i, full D)
 * weighted sum of v_i.  The scores read the cache's low-rank plane when it has
 * one at least d wide, else k_hat; the gathered rows always come from k_hat.
 * Requires seq_len <= S_cap and G in {1, 2, 4, 8}; otherwise
 * LOKI_ERR_INVALID_ARG or LOKI_ERR_UNSUPPORTED (also for seq_len above 393216
 * tokens, whose scores would not fit on chip).  Enqueues one kernel on the
 * stream (query rotation, scores, selection, attention); for query groups of
 * 8 heads, two: the query rotation, then the decode kernel as its
 * programmatic dependent. */
LOKI_API loki_status loki_decode_attention(const loki_cache *cache, int32_t seq_len,
                                  int32_t n_q_heads, const void *q, const float *P,
                                  int32_t d, int32_t k, float scale, float *out,
                                  int32_t *idx, void *workspace, size_t workspace_bytes,
                                  void *stream);

/* loki_decode_attention_noalloc -- loki_decode_attention without a caller
 * workspace, for callers that cannot allocate device memory on the decode
 * path: for example a host runtime whose device memory plan is fixed at
 * start-up, or one for which the implicit device synchronisation of
 * cudaMalloc is not acceptable between decode steps.  The pages have no
 * counterpart; this is an interface convenience of this library.
 * Arguments and results are those of loki_decode_attention, minus the
 * workspace.  The scratch is instead a fixed 4 MiB array in the library's
 * device code, which every GPU that loads the library holds until the process
 * exits; the call allocates and frees nothing.  Query groups of up to 4 heads
 * use none of it; for groups of 8, a call whose loki_decode_workspace_size
 * exceeds 4 MiB returns LOKI_ERR_UNSUPPORTED with a message, and enqueues
 * nothing.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture.  Every call on a device
 * shares the one array and leaves its contents behind (nothing in it needs to
 * start at zero): calls that may overlap on the GPU, from other streams or
 * threads, race on it and must not be issued. */
LOKI_API loki_status loki_decode_attention_noalloc(const loki_cache *cache, int32_t seq_len,
                                          int32_t n_q_heads, const void *q, const float *P,
                                          int32_t d, int32_t k, float scale, float *out,
                                          int32_t *idx, void *stream);

/* dense_decode_attention -- full softmax attention over every token
 * [0, seq_len) of the same rotated cache: the "Full Attention" baseline of the
 * summary page, section "Experimental setup".  Arguments as above; q is rotated
 * by P so that q_hat . k_hat = q . k.  out: [B, Hq, D] fp32. */
LOKI_API loki_status dense_decode_attention(const loki_cache *cache, int32_t seq_len,
                                   int32_t n_q_heads, const void *q,
                                   const float *P, float scale, float *out,
                                   void *stream);

/* loki_decode_attention_append -- one generation step: append the step's
 * token to every row, then the Loki step of loki_decode_attention over
 * tokens [0, seq_len), the new token being token seq_len - 1.  The pages
 * time the cache append apart from attention (summary page, "Key results")
 * and find it dominates inference time in a Hugging Face setup ("Surprising
 * findings"); here it happens inside the decode kernel.
 *   k_new : [B, Hkv, D] the new keys, NOT rotated, in the cache dtype;
 *   v_new : [B, Hkv, D] the new values; both 16-byte aligned.
 * Position seq_len - 1 of k_hat receives k_new . P_g rounded to the cache
 * dtype (the arithmetic of loki_append up to the fp32 summation order) and
 * of v receives v_new; the new token is scored, selected and attended like
 * any other.  Other arguments as loki_decode_attention.  One kernel for query
 * groups of up to 4 heads (the CTA that owns the last position rotates and
 * stores the token); for 8, the append kernel and then the two decode
 * kernels. */
LOKI_API loki_status loki_decode_attention_append(const loki_cache *cache, int32_t seq_len,
                                         int32_t n_q_heads, const void *k_new,
                                         const void *v_new, const void *q, const float *P,
                                         int32_t d, int32_t k, float scale, float *out,
                                         int32_t *idx, void *workspace,
                                         size_t workspace_bytes, void *stream);

/* dense_decode_attention_append -- the same generation step for the full
 * attention baseline: append the token at position seq_len - 1 of every row,
 * then dense_decode_attention over [0, seq_len).  One kernel. */
LOKI_API loki_status dense_decode_attention_append(const loki_cache *cache, int32_t seq_len,
                                          int32_t n_q_heads, const void *k_new,
                                          const void *v_new, const void *q, const float *P,
                                          float scale, float *out, void *stream);

/* loki_device_error_count -- the number of bounded device-side waits that
 * have timed out in this process on the current device since the library was
 * loaded (a kernel that times out records it here, releases what it holds and
 * returns; its outputs are then incomplete).  Synchronous: copies a counter
 * from device memory.  *count is a host pointer. */
LOKI_API loki_status loki_device_error_count(uint32_t *count);

/* loki_topk_jaccard -- agreement of two top-k selections: for every row r,
 * jaccard[r] = |A_r n B_r| / |A_r u B_r| of the index sets A_r = idx_a[r, :k]
 * and B_r = idx_b[r, :k].  This is the selection-agreement measure the summary
 * page reports between Loki and the exact top-k (sections "Key results" and
 * "Experimental setup"); the exact top-k is loki_decode_attention with
 * d = D (the ranking on all principal dimensions equals the ranking on the
 * unrotated keys, since P is orthonormal).
 *   idx_a, idx_b : [rows, k] int32 device arrays; each row holds k distinct
 *                  indices in ascending order (as loki_decode_attention
 *                  writes them).  Rows that are not ascending give an
 *                  unspecified value, never an out-of-bounds access.
 *   jaccard      : [rows] float device array (written).
 * Requires rows >= 1 and k >= 1.  One kernel on `stream`. */
LOKI_API loki_status loki_topk_jaccard(const int32_t *idx_a, const int32_t *idx_b, int32_t rows,
                              int32_t k, float *jaccard, void *stream);

/* ------------------------------------------------------------------------
 * Paged caches and per-sequence lengths
 * ------------------------------------------------------------------------
 * The pages name the missing integration with paged serving kernels as a
 * limitation (summary page, section "Limitations": not yet integrated with
 * FlashAttention; PagedAttention is among its references).  These calls run
 * the same Loki step on a paged cache whose sequences have their own lengths;
 * the per-row computation is exactly that of loki_decode_attention on the
 * sequence's tokens 0 .. seq_lens[b]-1 in order.
 *
 * A paged rotated-key cache: fixed-size pages from one pool.
 *   k_hat : [num_pages, Hkv, page_size, D] rotated keys in `dtype`, 16-byte
 *           aligned; v : the same layout, values.
 *   k_lr, d_lr : optional low-rank key plane, as in loki_cache, in the pool
 *           layout [num_pages, Hkv, page_size, d_lr] (same page ids), or NULL.
 * page_size is a power of two, 1 .. 65536 tokens; a pool holds at most
 * 2^31 - 1 rows (num_pages * Hkv * page_size; 512 GiB of bf16 keys at D = 128),
 * else LOKI_ERR_UNSUPPORTED. */
typedef struct {
  int32_t dtype;       /* loki_dtype                                          */
  int32_t n_kv_heads;  /* Hkv >= 1                                            */
  int32_t head_dim;    /* D: 64 or 128                                        */
  int32_t page_size;   /* tokens per page, a power of two                     */
  int32_t num_pages;   /* pages in each pool, >= 1                            */
  void *k_hat;
  void *v;
  void *k_lr;          /* optional low-rank key plane pool, or NULL           */
  int32_t d_lr;        /* its width (elements per token)                      */
} loki_paged_cache;

/* The sequences of a batch in a paged cache.
 *   block_table : [batch, pages_per_seq] int32 device array: token t of
 *                 sequence b sits at slot t % page_size of page
 *                 block_table[b][t / page_size].  Ids outside
 *                 [0, num_pages) are clamped into it (never an out-of-bounds
 *                 access; the result is then unspecified).
 *   seq_lens    : [batch] int32 device array, tokens attended per sequence,
 *                 each in [1, max_seq_len] (values outside are clamped), or
 *                 NULL for max_seq_len everywhere.  Ignored by
 *                 loki_paged_append.
 *   max_seq_len : the largest length, 1 <= max_seq_len <= pages_per_seq *
 *                 page_size; launch shapes are planned for it. */
typedef struct {
  int32_t batch;          /* B >= 1                                           */
  int32_t pages_per_seq;  /* columns of block_table, >= 1                     */
  int32_t max_seq_len;
  const int32_t *block_table;
  const int32_t *seq_lens;
} loki_seq_table;

/* loki_paged_append -- loki_append for a paged cache: new vector t of
 * sequence b (k_new[b, :, t, :] rotated by P, v_new[b, :, t, :] as is) goes to
 * token pos[b] + t of sequence b.  pos: [batch] int32 device array.  Tokens
 * whose position is negative or beyond the sequence's pages_per_seq *
 * page_size are not written.  Same arithmetic and kernels as loki_append
 * (tensor cores for bf16 appends of at least 256 vectors per KV head). */
LOKI_API loki_status loki_paged_append(const loki_paged_cache *cache, const loki_seq_table *seqs,
                              const int32_t *pos, int32_t n_new, const void *k_new,
                              const void *v_new, const float *P, void *stream);

/* Workspace bytes of loki_paged_decode_attention (same rule as
 * loki_decode_workspace_size for B = seqs->batch). */
LOKI_API loki_status loki_paged_decode_workspace_size(const loki_paged_cache *cache,
                                             const loki_seq_table *seqs, int32_t n_q_heads,
                                             size_t *bytes);

/* loki_paged_decode_attention -- the Loki step of loki_decode_attention on a
 * paged cache with per-sequence lengths.
 *   ks    : [batch] int32 device array: tokens kept for sequence b, clamped
 *           into [1, min(seq_lens[b], k_max)]; or NULL for
 *           min(seq_lens[b], k_max) everywhere.
 *   k_max : 1 <= k_max <= max_seq_len; the length of each idx row.
 *   idx   : [B, Hkv, k_max] int32 (written): row (b, g) holds the k_b
 *           selected positions in ascending order, then -1 up to k_max.
 * Everything else as loki_decode_attention (out [B, Hq, D] fp32, workspace of
 * loki_paged_decode_workspace_size bytes, one kernel on `stream`, two for
 * query groups of 8; the scores read the pool's low-rank plane when it has one
 * at least d wide). */
LOKI_API loki_status loki_paged_decode_attention(const loki_paged_cache *cache,
                                        const loki_seq_table *seqs, int32_t n_q_heads,
                                        const void *q, const float *P, int32_t d,
                                        const int32_t *ks, int32_t k_max, float scale,
                                        float *out, int32_t *idx, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* loki_paged_decode_attention_append -- loki_decode_attention_append on a
 * paged cache: sequence b's new token (k_new[b], v_new[b], [B, Hkv, D]) is
 * written at its position seq_lens[b] - 1, then the step attends tokens
 * [0, seq_lens[b]).  Query groups of up to 4 heads (else
 * LOKI_ERR_UNSUPPORTED).  Other arguments as loki_paged_decode_attention. */
LOKI_API loki_status loki_paged_decode_attention_append(const loki_paged_cache *cache,
                                               const loki_seq_table *seqs, int32_t n_q_heads,
                                               const void *k_new, const void *v_new,
                                               const void *q, const float *P, int32_t d,
                                               const int32_t *ks, int32_t k_max, float scale,
                                               float *out, int32_t *idx, void *workspace,
                                               size_t workspace_bytes, void *stream);

/* dense_decode_attention on a paged cache with per-sequence lengths. */
LOKI_API loki_status dense_paged_decode_attention(const loki_paged_cache *cache,
                                         const loki_seq_table *seqs, int32_t n_q_heads,
                                         const void *q, const float *P, float scale,
                                         float *out, void *stream);

/* loki_pca_workspace_size -- bytes of device workspace loki_pca_calibrate
 * needs for n_heads heads of dimension head_dim (64 or 128): the per-head
 * means and covariances in fp64.  *bytes is a host pointer. */
LOKI_API loki_status loki_pca_workspace_size(int32_t n_heads, int32_t head_dim, size_t *bytes);

/* loki_pca_calibrate -- the offline PCA calibration of the key basis, on the
 * GPU (summary page, summary paragraph: the PCA transform is calibrated
 * offline; section "Approach": queries and keys are projected with it).  For
 * every head g, from its N calibration keys x_n:
 *   C_g = (1/N) sum_n (x_n - mean)(x_n - mean)^T          (fp64)
 *   P_g[:, j] = the unit eigenvector of C_g with the j-th largest eigenvalue,
 *               its sign chosen so that its entry of largest magnitude is
 *               positive (the first such entry on a tie), rounded to fp32.
 * Equal eigenvalues are ordered by an unspecified but deterministic rule;
 * for them only the span of their eigenvectors is defined.
 *   keys      : [n_heads, n_keys, head_dim] in dtype (LOKI_F32 or LOKI_BF16),
 *               16-byte aligned, read only.
 *   P         : [n_heads, head_dim, head_dim] fp32, 16-byte aligned (written);
 *               the layout loki_append and the decode calls take.
 *   eigvals   : [n_heads, head_dim] fp64 in descending order (written), or
 *               NULL.
 *   workspace : device scratch of at least loki_pca_workspace_size bytes,
 *               256-byte aligned; no initial contents needed.
 * Three kernels on `stream`: means, covariance tiles, and a cyclic Jacobi
 * eigensolver (one CTA per head, at most 30 sweeps).  This is a calibration
 * step, not part of the decode path; it has no counterpart in the pages'
 * kernels, which take P as given. */
LOKI_API loki_status loki_pca_calibrate(const void *keys, int32_t dtype, int32_t n_heads,
                               int32_t n_keys, int32_t head_dim, float *P, double *eigvals,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Launch shape a decode call with these sizes would use, for logging and
 * tests.  shape: host array of 4 int32.
 *   dense == 0 (loki_decode_attention): shape[0] CTAs of the separate
 *     query-rotation kernel (0 when the decode kernel rotates its own
 *     queries, query groups of up to 4 heads), shape[1] CTAs per (batch, KV
 *     head) row in one cluster of the decode kernel, shape[2] CTAs of the
 *     decode kernel, shape[3] = 1 when the decode kernel is the short-row
 *     one (each CTA of a cluster selects on the whole row's keys: rows of at
 *     most 8192 tokens whose keys leave it as many CTAs per SM as the
 *     long-row kernel) and 0 for the long-row one (cluster select through a
 *     leader CTA).
 *   dense != 0 (dense_decode_attention): shape[1] CTAs per row in one
 *     cluster, shape[2] CTAs in all, shape[0] = shape[3] = 0.
 * k is checked (1 <= k <= seq_len) for dense == 0 but does not change the
 * shape.  Reads the current device's attributes; launches nothing. */
LOKI_API loki_status loki_decode_launch_shape(const loki_cache *cache, int32_t seq_len,
                                     int32_t n_q_heads, int32_t k, int32_t dense,
                                     int32_t *shape);

/* Launch-shape override, for tests and tuning: per_row > 0 makes the
 * following decode launches in this process use that many CTAs per (batch,
 * KV head) row (the cluster size of the dense kernel; the number of key-stream
 * units per row of the Loki step) wherever that shape can run, else the
 * planner's choice; per_row == 0 restores the planner's choice.  The initial
 * value is read once from the environment variable LOKI_CLUSTER (0 when
 * unset).  Applies process-wide; an atomic, safe to call from any thread, but
 * calls already enqueued keep the shape they were planned with.
 * Returns LOKI_ERR_INVALID_ARG for per_row < 0.  Not part of the method. */
LOKI_API loki_status loki_set_launch_override(int32_t per_row);

/* Phase stamps of the last Loki decode on a cache of this dtype and head_dim
 * (for profiling; builds compiled with -DLOKI_PHASE_STAMPS only, else
 * LOKI_ERR_UNSUPPORTED).  host: host array of capacity * 10 uint64; entry c
 * (CTA c of the decode kernel, up to 65536 CTAs) holds the device global timer
 * in ns when the CTA started, when its queries were ready and its first key
 * stages in flight, when its key stream was done, when the first digit of
 * the selection was known (short-row kernel: when every key of the row had
 * arrived), when its share of the selected rows was known, when its
 * attention was done and when the cluster's merge was done; then its SM,
 * then its rank in the cluster | cluster size << 8 | (1 << 16 when the row
 * took a single-CTA select) | (1 << 17 for the short-row kernel), then its
 * (batch, KV head) row.
 * Entries of CTAs the last decode did not have hold older data.  *n receives
 * the number of entries copied.  Synchronous.  Not part of the method. */
LOKI_API loki_status loki_phase_stamps(int32_t dtype, int32_t head_dim, uint64_t *host, int32_t capacity,
                                       int32_t *n);

/* Static description of a status code (never NULL). */
LOKI_API const char *loki_status_string(loki_status s);

/* Message of the calling thread's last failed call ("" if none). */
LOKI_API const char *loki_last_error(void);

/* LOKI_VERSION of the built library. */
LOKI_API int32_t loki_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOKI_H */
