/*
 * lisa.h -- C ABI of the B200 (sm_100a) indexed sparse decode-attention library.
 *
 * One decode step for a batch of sequences, per KV head h of sequence b:
 *
 *   1. qbar  = mean of the G = Hq/Hkv query vectors of KV head h          (query head j -> KV head j / G)
 *   2. u     = P_h qbar                       (P_h: r x d basis, caller supplied)
 *   3. s_t   = scale_h * <u, c_t>   for every cached position t < n_b   (c_t: projected key, FP8 E4M3 or fp32)
 *   4. I     = the min(M, n_b) positions of largest s_t; a tie at the M-th score goes to the lower position;
 *              reported in ascending position order
 *   5. o_j   = softmax attention of query head j over the bf16 keys/values of the positions in I, read
 *              straight from the paged KV cache (no gathered copy)
 *   6. (optional) linear branch:  S += phi(k_new) v_new^T,  z += phi(k_new),  lin_j = phi(q_j)^T S / (phi(q_j).z),
 *              phi = elu + 1, and out_j = sigmoid(g_j) o_j + (1 - sigmoid(g_j)) lin_j
 *   7. (optional) cross-layer reuse: a layer may take I from an earlier layer instead of steps 1-4.
 *
 * Sources.  Steps 1-5: JSSA write-up (rit.work, "jssa-sparse-attention-long-context"; article "Joint
 * Subspace Sparse Attention for Efficient Long-Context Decoding"), section "Как JSSA сохраняет порядок
 * токенов": queries of one KV head are averaged, projected into the head's joint subspace and every
 * position is scored against an FP8 projected-key cache; attention is then exact over the original
 * full-size keys and values; each GQA group keeps its own index set and one kernel launch reads the
 * selected positions of all heads directly from the cache.  Step 6: LISA write-ups (aikraft.ru, section
 * "Архитектура LISA"; opennieuws.be, section "Hybride architectuur voor efficiëntie"): a linear-attention
 * branch beside the top-M sparse branch, fused by a gate.  Step 7: IndexCache write-up
 * (denisavetisyan.com, section "IndexCache: Совместное использование слоев ..."): Shared layers reuse
 * the indices of the preceding Full layer.  Where the pages leave a step open (scale, FP8 variant, tie
 * rule, phi, gate form) the plain reading above is used.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers (memory of the current CUDA device), allocated and owned
 *     by the caller; the library never allocates or frees, and keeps no state between calls.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and runs
 *     asynchronously; no entry point synchronises the host except lisa_check_device_error.
 *   - The decode-path kernels are launched with programmatic dependent launch, so one may start
 *     while the previous kernel of the stream drains; each waits for all earlier work of the stream
 *     before it reads or writes memory that work may touch, so stream-order semantics are unchanged.
 *   - Arguments are checked on the host before anything is enqueued.  Any return other than LISA_OK
 *     from the checks means nothing was enqueued.  A failed launch returns LISA_ERR_CUDA.
 *   - Values that can only be checked on the device (sequence lengths, page ids, indices, counts) are
 *     checked by the kernels: an out-of-range value is clamped to a safe one, the computation goes on,
 *     and a sticky bit is set in the workspace error word, read by lisa_check_device_error.
 *   - Alignment: kproj_pool 32 bytes, k_pool/v_pool 16 bytes, q and scores 4 bytes (LISA_ERR_INVALID_ARG
 *     otherwise); every allocation from cudaMalloc or torch meets this.
 *   - `ws` is a caller-owned device workspace of at least lisa_workspace_size(desc) bytes, 256-byte
 *     aligned, zeroed once with lisa_workspace_init before first use.  Its first 256 bytes hold the
 *     error word; the rest is scratch.  Calls that share one workspace must not overlap in time.
 *
 * Layouts (row-major, innermost index last):
 *   q            bf16 [B][Hq][d]
 *   P            fp32 [Hkv][r][d]
 *   kproj_pool   [num_pages][Hkv][page_size][r]  of uint8 E4M3 codes, or of fp32
 *   kproj_scale  fp32 [Hkv]
 *   k_pool/v_pool bf16 [num_pages][page_size][Hkv][d] (separate pools), or one pool
 *                bf16 [num_pages][page_size][Hkv][2][d] with K then V per row (kv_row_stride = 2d)
 *   page_table   int32 [B][max_pages_per_seq]: position t of sequence b lives in page page_table[b][t /
 *                page_size], slot t % page_size.  A contiguous cache is a pool with an identity table.
 *   seq_lens     int32 [B], 0 <= n_b <= max_seq_len
 *   scores       fp32 [B][Hkv][max_seq_len]
 *   idx          int32 [B][Hkv][M], count int32 [B][Hkv]
 *   out          bf16 [B][Hq][d],   lse fp32 [B][Hq] (natural log of the softmax denominator)
 *
 * Supported shapes (anything else returns LISA_ERR_UNSUPPORTED): d in {64, 128}; r in {16, 32};
 * 1 <= G <= 8; page_size a power of two in [16, 1024]; 1 <= M <= 16384; max_seq_len <= 262144.
 */
#ifndef LISA_H
#define LISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lisa_stream_t; /* same type as cudaStream_t */
typedef struct CUevent_st* lisa_event_t;   /* same type as cudaEvent_t */

typedef enum {
  LISA_OK = 0,
  LISA_ERR_INVALID_ARG = 1,  /* null pointer where one is required, negative size, inconsistent sizes */
  LISA_ERR_UNSUPPORTED = 2,  /* valid but outside the supported shapes listed above */
  LISA_ERR_WORKSPACE = 3,    /* ws is NULL, misaligned or smaller than lisa_workspace_size() */
  LISA_ERR_CUDA = 4,         /* a CUDA call failed (launch or attribute query) */
  LISA_ERR_DEVICE_CHECK = 5, /* lisa_check_device_error found a device-side range violation */
  LISA_ERR_TIMEOUT = 6       /* reserved: a bounded device wait ran out (no current kernel waits) */
} lisa_status;

typedef enum { LISA_KPROJ_FP32 = 0, LISA_KPROJ_FP8_E4M3 = 1 } lisa_kproj_dtype;

/* Device error word bits (lisa_check_device_error). */
#define LISA_DEVERR_SEQ_LEN 0x1u    /* seq_lens[b] < 0 or > max_seq_len (clamped)                */
#define LISA_DEVERR_PAGE_ID 0x2u    /* page id outside [0, num_pages) (row 0 of the pool used)   */
#define LISA_DEVERR_INDEX 0x4u      /* idx entry outside [0, n_b) (position 0 used)              */
#define LISA_DEVERR_COUNT 0x8u      /* count[b][h] outside [0, min(M, n_b)] (clamped)            */

/* Sizes and the two caller-owned tables of one decode step.  Plain data; no ownership taken. */
typedef struct {
  int32_t batch;             /* B >= 0 (B = 0: every entry point returns LISA_OK and does nothing) */
  int32_t num_q_heads;       /* Hq, a multiple of num_kv_heads                                     */
  int32_t num_kv_heads;      /* Hkv >= 1                                                           */
  int32_t head_dim;          /* d                                                                  */
  int32_t idx_dim;           /* r, projected-key width                                             */
  int32_t budget_m;          /* M, index-set size per (b, KV head)                                 */
  int32_t page_size;         /* tokens per page                                                    */
  int32_t max_pages_per_seq; /* columns of page_table, >= ceil(max_seq_len / page_size)            */
  int32_t max_seq_len;       /* upper bound of seq_lens; row stride of `scores`                    */
  int32_t num_pages;         /* pages in each pool (bounds for page ids)                          */
  const int32_t* seq_lens;   /* device int32 [B]                                                   */
  const int32_t* page_table; /* device int32 [B][max_pages_per_seq]                                */
  float softmax_scale;       /* attention logit scale; <= 0 selects 1/sqrt(d)                      */
  int32_t kv_row_stride;     /* elements from one (page, slot, KV head) row of k_pool / v_pool to
                                the next: 0 (or d) for separate K and V pools; 2 * d for one pool
                                holding K and V of each row side by side (v_pool = k_pool + d), the
                                faster layout: one 512-byte read per selected position at d = 128 */
} lisa_decode_desc;

/* Optional linear-attention branch (one state per (b, KV head)); S and z are updated in place. */
typedef struct {
  float* S;                 /* device fp32 [B][Hkv][d][d]                     */
  float* z;                 /* device fp32 [B][Hkv][d]                        */
  const void* k_new;        /* device bf16 [B][Hkv][d], key of the new token  */
  const void* v_new;        /* device bf16 [B][Hkv][d]                        */
  const float* gate_logit;  /* device fp32 [Hq], g_j                          */
} lisa_linear_branch;

/* Optional events recorded on `stream` between the stages of lisa_fused_decode (any may be NULL). */
typedef struct {
  lisa_event_t start;       /* before the index stage (score + top-M)         */
  lisa_event_t after_sample;/* after the threshold-sampling kernel (index stage, step 1 of 3;
                               not recorded when indices are reused)          */
  lisa_event_t after_stream;/* after the scoring stream kernel (index stage, step 2 of 3;
                               not recorded when indices are reused)          */
  lisa_event_t after_index; /* after the index stage, before attention        */
  lisa_event_t after_attn;  /* after the attention kernel (which also merges the partitions and
                               applies the linear branch and gate)            */
  lisa_event_t end;         /* end of the call                                */
} lisa_stage_events;

/* Workspace bytes any entry point needs for `desc` (0 if desc is invalid). Host only. */
size_t lisa_workspace_size(const lisa_decode_desc* desc);

/* Partial-result slots per (b, KV head) the attention step may use for `desc`: the stream-K grid
 * splits the B * Hkv * ceil(M / 64) position tiles evenly over its CTAs, and each CTA writes one
 * partial per (b, KV head) it touches (0 if desc is invalid). */
int32_t lisa_num_splits(const lisa_decode_desc* desc);

/* Zero the workspace error word (enqueued on stream). Call once after allocating ws. */
lisa_status lisa_workspace_init(void* ws, size_t ws_bytes, lisa_stream_t stream);

/* Steps 1-3: write s_t to scores[b][h][t] for t < n_b (entries t >= n_b are not written).  With
 * FP8 projected keys this is lisa_index_score_multi with one token per sequence (same kernels, same
 * use of ws); with fp32 keys one CUDA-core kernel. */
lisa_status lisa_index_score(const lisa_decode_desc* desc, const void* q, const float* P,
                             const void* kproj_pool, lisa_kproj_dtype kproj_dtype,
                             const float* kproj_scale, float* scores, void* ws, size_t ws_bytes,
                             lisa_stream_t stream);

/* Steps 1-3 for T query tokens per sequence (speculative or chunked decode; 1 <= T <= 8).  q is
 * bf16 [B][T][Hq][d], token j of sequence b seeing positions t <= n_b - T + j.  Writes
 * s_t = scale_h <P_h qbar_{b,j,h}, c_t> to scores[b][j][h][t] for those t (later entries are not
 * written); scores fp32 [B][T][Hkv][max_seq_len].  FP8 projected keys only.  The T projected queries
 * of a KV head form the N side of one tensor-core contraction per 16-position tile (E4M3 -> f16 is
 * exact; each query as an f16 hi/lo pair, fp32 accumulation), so the scores agree with an fp32 dot
 * product to rounding.  Top-M per token: lisa_topm_select on a desc with B*T sequences (b*T + j,
 * length n_b - T + j + 1) over the same scores buffer.  Two kernels on `stream`: the first forms
 * the T projected queries of each (b, KV head) into ws (the region the fused top-M keeps its
 * candidates in), the second streams the projected keys once for all T tokens. */
lisa_status lisa_index_score_multi(const lisa_decode_desc* desc, int num_tokens, const void* q, const float* P,
                                   const void* kproj_pool, lisa_kproj_dtype kproj_dtype, const float* kproj_scale,
                                   float* scores, void* ws, size_t ws_bytes, lisa_stream_t stream);

/* Workspace bytes lisa_index_topm_multi needs for `desc` and T = num_tokens (those of a desc with
 * B * T sequences; 0 if desc or num_tokens is invalid). Host only. */
size_t lisa_workspace_size_multi(const lisa_decode_desc* desc, int num_tokens);

/* Steps 1-4 fused for T query tokens per sequence (1 <= T <= 8, B * T <= 65535), FP8 projected keys
 * only: token j of sequence b (q bf16 [B][T][Hq][d]) averages its G queries per KV head, projects
 * them with P_h and keeps the min(M, n_b - T + j + 1) best of the positions t <= n_b - T + j (ties to
 * the lower position), ascending, in idx int32 [B][T][Hkv][M] (the rest -1) with count int32
 * [B][T][Hkv].  The same sets as lisa_index_score_multi followed by lisa_topm_select on a desc of
 * B * T sequences, without writing the scores: a sampled threshold per token, one stream of the
 * projected keys for all T tokens (the per-tile tensor-core contraction of lisa_index_score_multi)
 * that keeps each token's positions above its threshold, and the exact finish per token (with the
 * same exact re-scoring fallback as lisa_index_topm).  ws: lisa_workspace_size_multi bytes. */
lisa_status lisa_index_topm_multi(const lisa_decode_desc* desc, int num_tokens, const void* q, const float* P,
                                  const void* kproj_pool, lisa_kproj_dtype kproj_dtype, const float* kproj_scale,
                                  int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, lisa_stream_t stream);

/* Step 4 from caller-given fp32 scores (scores [B][Hkv][max_seq_len], entries t >= n_b never read):
 * idx[b][h][0..count) ascending, count = min(M, n_b), idx[b][h][count..M) = -1; a tie at the M-th
 * score goes to the lower position, and -0 equals +0.  Three kernels on `stream`: a threshold
 * sampled from the scores, a filter that streams the scores and keeps the positions at or above it,
 * and an exact select over those (over all n_b scores instead when fewer than M pass or the
 * candidate buffer in ws overflows), so the result is exact whatever the scores. */
lisa_status lisa_topm_select(const lisa_decode_desc* desc, const float* scores, int32_t* idx,
                             int32_t* count, void* ws, size_t ws_bytes, lisa_stream_t stream);

/* Steps 1-4 fused: the scores never leave on-chip memory. Same outputs as lisa_topm_select. */
lisa_status lisa_index_topm(const lisa_decode_desc* desc, const void* q, const float* P,
                            const void* kproj_pool, lisa_kproj_dtype kproj_dtype,
                            const float* kproj_scale, int32_t* idx, int32_t* count, void* ws,
                            size_t ws_bytes, lisa_stream_t stream);

/* Step 5 over a caller-given index set (positions idx[b][h][0..count[b][h]) of sequence b).
 * lse may be NULL. */
lisa_status lisa_sparse_decode_attn(const lisa_decode_desc* desc, const void* q, const void* k_pool,
                                    const void* v_pool, const int32_t* idx, const int32_t* count,
                                    void* out, float* lse, void* ws, size_t ws_bytes,
                                    lisa_stream_t stream);

/* Step 5 like lisa_sparse_decode_attn, for callers that cannot allocate device memory: it takes no
 * workspace.  No counterpart on the pages: the write-ups do not discuss memory management.  Its
 * scratch (partial sums of the attention partitions and their counters) is a fixed 8 MiB device
 * array inside this library that every GPU which loads the library holds until the process exits;
 * nothing is allocated or freed.  A desc whose scratch would exceed it -- about
 * B * Hkv * lisa_num_splits(desc) * G * (d + 2) * 4 bytes plus small counters -- is rejected with
 * LISA_ERR_WORKSPACE before anything is enqueued.  The first call on each device looks up the
 * array's device address (a runtime call, done once per device); make that first call before any
 * stream capture.  All calls share the one array, which keeps the last call's contents; each call
 * clears its counters on `stream` first, and calls whose work overlaps on the GPU (other streams,
 * other threads) race on it and must be serialised by the caller.  Device-side range checks still
 * clamp bad indices, counts and page ids, but their flags are not reported by this entry point. */
lisa_status lisa_sparse_decode_attn_noalloc(const lisa_decode_desc* desc, const void* q, const void* k_pool,
                                            const void* v_pool, const int32_t* idx, const int32_t* count,
                                            void* out, float* lse, lisa_stream_t stream);

/* Steps 1-7 in one call.  reuse_idx/reuse_count (both or neither): take the index set from an
 * earlier layer and skip steps 1-4 (kproj_pool, P, kproj_scale may then be NULL).  idx_out/count_out
 * (both or neither, only without reuse): also return the index set.  lin may be NULL (no linear
 * branch).  lse and events may be NULL. */
lisa_status lisa_fused_decode(const lisa_decode_desc* desc, const void* q, const float* P,
                              const void* kproj_pool, lisa_kproj_dtype kproj_dtype,
                              const float* kproj_scale, const void* k_pool, const void* v_pool,
                              const int32_t* reuse_idx, const int32_t* reuse_count, int32_t* idx_out,
                              int32_t* count_out, const lisa_linear_branch* lin, void* out,
                              float* lse, void* ws, size_t ws_bytes,
                              const lisa_stage_events* events, lisa_stream_t stream);

/* ---- Comparators (not on the decode path) --------------------------------------------------
 * The JSSA write-up states its gain against full attention and against "gather, then attend"
 * (section "Как JSSA сохраняет порядок токенов").  These two calls make those baselines on the same
 * GPU with the same kernels, so that the ratios can be measured: */

/* Full attention: every query head over all n_b cached positions (no index).  Same layouts as
 * lisa_sparse_decode_attn; lse may be NULL.  ws: lisa_dense_workspace_size(desc) bytes, 256-byte
 * aligned (initialised by lisa_workspace_init).  LISA_ERR_UNSUPPORTED when a (b, KV head) would
 * need more than 256 partial results (max_seq_len above about 261,000 positions). */
size_t lisa_dense_workspace_size(const lisa_decode_desc* desc);
lisa_status lisa_dense_decode_attn(const lisa_decode_desc* desc, const void* q, const void* k_pool,
                                   const void* v_pool, void* out, float* lse, void* ws, size_t ws_bytes,
                                   lisa_stream_t stream);

/* Gather of the selected rows into a contiguous buffer: gathered bf16 [B][Hkv][M][2][d] (16-byte
 * aligned), row i of (b, h) = (K row, V row) of position idx[b][h][i] for i < count[b][h], zeros
 * after.  Attention over it is lisa_dense_decode_attn on a desc with B*Hkv sequences of one KV head,
 * n = count, and an identity page table over the buffer.  Only the workspace error word is used
 * (ws_bytes >= 256); bad indices or page ids are flagged and give zero rows. */
lisa_status lisa_gather_kv(const lisa_decode_desc* desc, const int32_t* idx, const int32_t* count,
                           const void* k_pool, const void* v_pool, void* gathered, void* ws, size_t ws_bytes,
                           lisa_stream_t stream);

/* ---- Basis calibration (once per layer and KV head, off the decode path) -------------------------
 * JSSA write-up, "Как JSSA сохраняет порядок токенов": query and key statistics are collected once
 * and the basis is taken from eigenvectors of a matrix; the subspace is meant to preserve the
 * query-key scores.  The pages name no matrix; this library's reading: with Q = mean q q^T over the
 * averaged group queries and K = mean k k^T over the keys of head h, P_h's rows are the top-r
 * eigenvectors (largest eigenvalue first) of C = (Q K + K Q) / 2 -- the rank-r subspace that
 * maximises E[(q . k)(q . P^T P k)] = tr(P^T P K Q) -- each row signed so that its entry of largest
 * magnitude is positive.  q_samples bf16 [Hkv][nq][d], k_samples bf16 [Hkv][nk][d]; P_out fp32
 * [Hkv][r][d]; eigvals_out fp32 [Hkv][r] or NULL.  d in {64, 128}, r in {16, 32}, nq, nk >= 1.
 * ws: lisa_calibrate_workspace_size bytes, 256-byte aligned.  fp32 arithmetic (second moments,
 * then a cyclic Jacobi eigen-decomposition in shared memory). */
size_t lisa_calibrate_workspace_size(int num_kv_heads, int head_dim);
lisa_status lisa_calibrate_basis(int num_kv_heads, int head_dim, int idx_dim, const void* q_samples, int nq,
                                 const void* k_samples, int nk, float* P_out, float* eigvals_out, void* ws,
                                 size_t ws_bytes, lisa_stream_t stream);

/* Producer side of the decode step (JSSA write-up, "Как JSSA сохраняет порядок токенов": the
 * projected keys live in an FP8 cache beside the full-size K/V cache).  For every sequence b and
 * KV head h, the current token's rows are written at position t_b = positions[b] (positions may be
 * NULL: t_b = seq_lens[b] - 1), page page_table[b][t_b / page_size], slot t_b % page_size:
 *   k_pool/v_pool row  <- k_new[b][h][0..d), v_new[b][h][0..d)  (bf16, copied bit for bit)
 *   kproj_pool row     <- c = P_h k_new[b][h], where c_i = (...((P_i0 k_0) + P_i1 k_1) + ...) + P_i,d-1 k_d-1
 *                         in fp32 with every product and every sum rounded to nearest even (no
 *                         fused multiply-add), then
 *                         LISA_KPROJ_FP8_E4M3: the E4M3 code of c_i / kproj_scale[h] (fp32 division,
 *                         round to nearest even, magnitudes above 448 saturate to 448);
 *                         LISA_KPROJ_FP32: c_i.
 * The arithmetic is fixed so that the codes are reproducible bit for bit.  Layouts as in
 * lisa_fused_decode (kv_row_stride honoured); k_new, v_new bf16 [B][Hkv][d] (16-byte aligned),
 * P fp32 [Hkv][r][d].  A position outside [0, max_seq_len) or a page id outside [0, num_pages)
 * sets LISA_DEVERR_INDEX or LISA_DEVERR_PAGE_ID and that (b, h) writes nothing.  Only the error word
 * of the workspace is used (its size is lisa_workspace_size(desc) all the same). */
lisa_status lisa_append_token(const lisa_decode_desc* desc, const int32_t* positions, const void* k_new,
                              const void* v_new, const float* P, void* kproj_pool, lisa_kproj_dtype kproj_dtype,
                              const float* kproj_scale, void* k_pool, void* v_pool, void* ws, size_t ws_bytes,
                              lisa_stream_t stream);

/* Synchronise `stream`, read the workspace error word into *flags_out (may be NULL), clear it.
 * Returns LISA_ERR_DEVICE_CHECK if any bit was set, LISA_OK otherwise. */
lisa_status lisa_check_device_error(void* ws, uint32_t* flags_out, lisa_stream_t stream);

/* Static description of a status code. */
const char* lisa_status_string(lisa_status status);

#ifdef __cplusplus
}
#endif

#endif /* LISA_H */
