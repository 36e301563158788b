/*
 * qsa.h -- C ABI of the QSA sparse-decode library (libqsa.so), sm_100a.
 *
 * The library computes one decode step of Qwen Sparse Attention (QSA) as
 * described on the page "Qwen 4 QSA gets decode context parallelism: inside
 * vLLM's draft PR for Qwen3.8-Flash-Next" (orcarouter.ai), section "What the
 * pull request actually changes": a small indexer shrinks the keys four to
 * one into micro-blocks, ranks the blocks and retains the top 512 of them
 * (near 2,048 tokens); exact attention (softmax, then the weighted sum of V)
 * uses the full-precision K and V of the retained blocks only. The
 * decode-context-parallel split read of the same section (each part of the
 * main KV cache read on its own, the selector replicated, partial results
 * combined afterwards; also "Questions worth answering directly", DCP vs TP)
 * is done inside one GPU as an R-way split with a log-sum-exp merge.
 *
 * The page gives no formulas; this library fixes these readings:
 *   micro-block key   kc = bf16_rne(fp32 sum of its n keys in token order / n)
 *                     (n = 4, or L mod 4 for the trailing partial block)
 *   block score       s_b = sum_h w_h * max(0, q_idx_h . kc_b)
 *   selection         k_b = min(k, nb) blocks by (score desc, index asc),
 *                     listed in ascending block order, padded with -1
 *   slice r of R      blocks [floor(r*nb/R), floor((r+1)*nb/R))
 *   partial r         z_t = scale * q_h . K_t over tokens t < L of the
 *                     selected blocks of slice r; LSE_r = ln sum exp z_t;
 *                     O_r = sum softmax(z)_t V_t; empty slice: O_r = 0,
 *                     LSE_r = -inf
 *   merge             O = sum_r e^(LSE_r-m) O_r / sum_r e^(LSE_r-m),
 *                     LSE = m + ln sum_r e^(LSE_r-m), m = max_r LSE_r
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers owned by the caller. The library
 *     allocates no device memory and keeps no pointer after a call returns
 *     (the caller owns every cache view; nothing is kept alive behind its
 *     back).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). A returned QSA_OK means the launch was accepted.
 *   - Arrays are dense row-major with the shapes given below; bf16 arrays and
 *     pools must be 16-byte aligned.
 *   - Indices are int32. K, V, queries and indexer keys are bf16; weights,
 *     scores, partial outputs and LSEs are fp32 (LSE in natural log).
 *   - Data-dependent indices (block-table entries, sequence lengths, token
 *     positions, selected block ids) are bounds-checked on the device. A
 *     failed check skips the access and sets a bit in the device error word,
 *     which qsa_check_device_errors() reads and clears (QSA_ERR_BOUNDS).
 *     No kernel traps or asserts.
 *   - No C++ exception crosses this boundary. On a non-OK status,
 *     qsa_last_error() gives a message (thread-local).
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t qsa_status;
#define QSA_OK 0
#define QSA_ERR_INVALID_ARG 1 /* null pointer, bad size or alignment          */
#define QSA_ERR_UNSUPPORTED 2 /* dims outside the supported set               */
#define QSA_ERR_CUDA 3        /* a CUDA runtime call or a launch failed       */
#define QSA_ERR_BOUNDS 4      /* a device-side index check failed             */
#define QSA_ERR_TIMEOUT 5     /* a bounded device-side wait gave up           */

/* Same object as cudaStream_t. */
typedef struct CUstream_st *qsa_stream_t;

/* Head geometry.
 *   Hq query heads share Hkv KV heads; query head h reads KV head h / (Hq/Hkv).
 *   D   head dim of q, K and V            supported: 128
 *   Hi  indexer heads                     supported: 1..32
 *   di  indexer key width                 supported: 64, 128
 *   P   tokens per cache page             supported: multiple of 4, 4..1024
 *                                         (qsa_prefill_index_score: multiple
 *                                         of 32)
 *   G = Hq/Hkv                            supported: 1..8
 *   scale  softmax scale applied to q.K (e.g. 1/sqrt(D)). */
typedef struct qsa_dims {
  int32_t Hq, Hkv, D, Hi, di, P;
  float scale;
} qsa_dims;

/* The paged cache. ONE block table indexes all four pools, so the selector
 * state and the main KV cache can never disagree about where a token lives
 * (the page's "selector and the main KV cache are kept in one cache group").
 *   k_pool, v_pool  bf16 [num_pages, P, Hkv, D]   token (page, slot), head g
 *   kidx_pool       bf16 [num_pages, P, di]       per-token indexer key
 *   side_pool       bf16 [num_pages, P/4, di]     compressed key of each
 *                                                 complete micro-block
 *   block_table     int32 [num_seqs, max_pages_per_seq]: physical page of
 *                   tokens [j*P, (j+1)*P) of sequence b is block_table[b][j].
 * A contiguous cache is the same structure with an identity block table. */
typedef struct qsa_cache {
  void *k_pool;
  void *v_pool;
  void *kidx_pool;
  void *side_pool;
  const int32_t *block_table;
  int32_t num_seqs;
  int32_t max_pages_per_seq;
  int32_t num_pages;
} qsa_cache;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t qsa_version(void);

/* Message of the last non-OK status returned on this thread ("" if none). */
const char *qsa_last_error(void);

/* Write N new tokens into the cache (page section "What the pull request
 * actually changes": QSA keeps the main cache plus the indexer's side
 * caches; the fourth bullet: synthetic batches must not write the side
 * caches).
 *   tok_seq, tok_pos  int32 [N]: sequence row and position of each token;
 *                     an entry with tok_seq < 0 or tok_pos < 0 is padding and
 *                     writes nothing at all.
 *   k_new, v_new      bf16 [N, Hkv, D];  kidx_new  bf16 [N, di].
 * Token i goes to page block_table[seq][pos / P], slot pos % P of k/v/kidx
 * pools. After all N tokens are written, every token with pos % 4 == 3
 * stores the compressed key of its
 * micro-block (positions pos-3..pos, read back from kidx_pool) at side slot
 * (pos % P) / 4 of the same page. So a bulk prefill in any token order gives
 * the same side cache as one token per call. Two entries with the same
 * (seq, pos) in one call race (undefined which one lands). */
qsa_status qsa_append(const qsa_dims *dims, const qsa_cache *cache, int32_t N,
                      const int32_t *tok_seq, const int32_t *tok_pos,
                      const void *k_new, const void *v_new,
                      const void *kidx_new, qsa_stream_t stream);

/* Block scores of B sequences (page section "What the pull request actually
 * changes": the indexer "scores them").
 *   seq_lens  int32 [B]: L_b, context length after the current token was
 *             appended; nb_b = ceil(L_b / 4) blocks are scored. Reads
 *             block_table rows 0..B-1.
 *   q_idx     bf16 [B, Hi, di];  w  fp32 [B, Hi]
 *   scores    fp32 [B, ld_scores], ld_scores >= max_b nb_b (a longer
 *             sequence sets QSA_ERR_BOUNDS and is skipped). Entries
 *             j >= nb_b are not written.
 * Complete blocks read the side pool; the trailing partial block's key is
 * built from its L mod 4 tokens in kidx_pool by the same rule. Any page size
 * P (a multiple of 4) is scored: P a multiple of 32 by the TMA + tcgen05
 * kernel, other page sizes by a warp-level MMA kernel that gathers the
 * side-cache rows one by one. Needs q_idx 16-byte aligned. */
qsa_status qsa_index_score(const qsa_dims *dims, const qsa_cache *cache,
                           int32_t B, const int32_t *seq_lens,
                           const void *q_idx, const float *w, float *scores,
                           int32_t ld_scores, qsa_stream_t stream);

/* Scratch bytes qsa_topk_select needs (0 for this implementation). */
size_t qsa_topk_workspace_size(int32_t B, int32_t ld_scores, int32_t k);

/* Per-sequence top-k blocks (page section "What the pull request actually
 * changes": the indexer retains the top 512 blocks).
 *   scores  fp32 [B, ld_scores] (first nb_b = ceil(seq_lens[b]/4) entries
 *           used; NaN scores are not supported)
 *   sel     int32 [B, k]: the k_b = min(k, nb_b) best blocks by (score
 *           desc, block index asc), in ascending block order, then -1.
 * -0.0 ranks equal to +0.0. Supported: 1 <= k <= 4096,
 * ld_scores <= 393,216. ws may be NULL when its size is 0. */
qsa_status qsa_topk_select(int32_t B, const int32_t *seq_lens,
                           const float *scores, int32_t ld_scores, int32_t k,
                           int32_t *sel, void *ws, size_t ws_bytes,
                           qsa_stream_t stream);

/* Scratch bytes qsa_sparse_decode needs for B sequences, top-k k, R slices.
 * The scratch holds the partial results of slices that several CTAs share,
 * the list of those slices, (for qsa_decode_step's fused merge) one arrival
 * counter per sequence and group of 8 query heads and, at the end, the R + 1
 * slice starts per sequence that qsa_decode_step's top-k hands to its decode;
 * it needs no initialisation and every call writes what it later reads
 * (calls sharing one scratch buffer must be ordered on the GPU). */
size_t qsa_sparse_decode_workspace_size(const qsa_dims *dims, int32_t B,
                                        int32_t k, int32_t R);

/* Split-read sparse attention over the selected blocks (page section "What
 * the pull request actually changes": exact softmax and value aggregation on
 * the uncompressed K/V; each slice of the main cache read separately with
 * the selector replicated, results combined afterwards).
 *   q         bf16 [B, Hq, D]
 *   sel       int32 [B, k] as produced by qsa_topk_select (ascending, -1
 *             padded); the same selection serves all R slices. The list ends
 *             at its first -1 or after min(k, nb_b) entries, so a shorter
 *             selection (e.g. qsa_select_owned's) is accepted
 *   o_part    fp32 [R, B, Hq, D];  lse_part  fp32 [R, B, Hq]
 * Slice r holds the attention of each query head over the tokens t < L_b of
 * the selected blocks in [floor(r*nb/R), floor((r+1)*nb/R)); an empty slice
 * gives zeros and LSE = -inf. Supported: 1 <= R <= 64, 1 <= k <= 4096. */
qsa_status qsa_sparse_decode(const qsa_dims *dims, const qsa_cache *cache,
                             int32_t B, const int32_t *seq_lens,
                             const void *q, const int32_t *sel, int32_t k,
                             int32_t R, float *o_part, float *lse_part,
                             void *ws, size_t ws_bytes, qsa_stream_t stream);

/* Scratch bytes of qsa_sparse_decode_mq (Qn queries per sequence). */
size_t qsa_sparse_decode_mq_workspace_size(const qsa_dims *dims, int32_t B,
                                           int32_t Qn, int32_t k, int32_t R);

/* Multi-query decode: Qn decode queries per sequence share the sequence's
 * one selection and one gather of its K/V (several new tokens per step, as
 * in multi-token prediction or speculative decoding). The page names such a
 * workload (section "Why a serving PR ... is still worth your time") without
 * defining it; this library's reading: the Qn new tokens are the last Qn
 * positions of the sequence (already appended), and query j sits at position
 * L_b - Qn + j and attends to the selected tokens t <= L_b - Qn + j.
 *   q         bf16 [B, Qn, Hq, D]
 *   o_part    fp32 [R, B, Qn, Hq, D];  lse_part  fp32 [R, B, Qn, Hq]
 * Slices, selection and empty-slice rule as in qsa_sparse_decode (a slice
 * whose selected tokens all lie after a query is empty for that query);
 * qsa_merge combines the result with B * Qn rows. Queries are processed in
 * groups of two per pass over the selected K/V. Supported: 1 <= Qn <= 8;
 * qsa_sparse_decode is this call with Qn = 1. */
qsa_status qsa_sparse_decode_mq(const qsa_dims *dims, const qsa_cache *cache,
                                int32_t B, int32_t Qn, const int32_t *seq_lens,
                                const void *q, const int32_t *sel, int32_t k,
                                int32_t R, float *o_part, float *lse_part,
                                void *ws, size_t ws_bytes, qsa_stream_t stream);

/* Size of the static device scratch of qsa_sparse_decode_static (32 MiB). */
#define QSA_STATIC_SCRATCH_BYTES (32u << 20)

/* qsa_sparse_decode without a workspace argument, for callers that cannot
 * allocate device memory: a plain C host that only holds the input and
 * output buffers it was handed, a process whose device memory is entirely
 * owned by another allocator's pool (a raw cudaMalloc would fail or fragment
 * it), or a latency-critical loop where cudaMalloc / cudaFree may
 * synchronise the device. It has no counterpart on the page; it is an
 * interface convenience of this library.
 * Same arguments, results and errors as qsa_sparse_decode, except that the
 * scratch lives in a fixed device array inside the library
 * (QSA_STATIC_SCRATCH_BYTES per device, held by every device that loads the
 * library until the process exits). A call whose scratch need
 * (qsa_sparse_decode_workspace_size) exceeds that returns
 * QSA_ERR_UNSUPPORTED. The call allocates nothing.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. All calls share the one array: calls whose executions overlap on
 * the GPU race and corrupt each other. */
qsa_status qsa_sparse_decode_static(const qsa_dims *dims, const qsa_cache *cache,
                                    int32_t B, const int32_t *seq_lens,
                                    const void *q, const int32_t *sel, int32_t k,
                                    int32_t R, float *o_part, float *lse_part,
                                    qsa_stream_t stream);

/* Decode context parallelism (page section "What the pull request actually
 * changes": a rank reads just its own part of the main KV cache, the
 * selector stays replicated; "Questions worth answering directly": partial
 * attention results are merged afterwards). This library's reading of a
 * rank's slice: page p of every sequence is held by rank p mod W (balanced,
 * and stable as sequences grow). Every rank scores and selects on the
 * replicated side cache, keeps with this call the selected blocks of the
 * pages it holds (sel_out [B, k], same order, -1 padded; block j lies on page
 * 4j / P), attends over them with qsa_sparse_decode, gathers the W partials
 * from the other ranks and combines them with qsa_merge (R = W).
 * Supported: 1 <= W <= 1024, 0 <= r < W, P a positive multiple of 4. */
qsa_status qsa_select_owned(int32_t B, const int32_t *sel, int32_t k, int32_t P,
                            int32_t W, int32_t r, int32_t *sel_out,
                            qsa_stream_t stream);

/* LSE-weighted combine of R partial results (page sections "What the pull
 * request actually changes", second bullet, and "Questions worth answering
 * directly": partial attention results are merged afterwards).
 *   o_part fp32 [R, B, Hq, D], lse_part fp32 [R, B, Hq]
 *   out    [B, Hq, D], bf16 if out_is_bf16 else fp32;  lse_out fp32 [B, Hq]
 *          (lse_out may be NULL). Slices with LSE = -inf are ignored; if
 *          every slice is empty the row is 0 with LSE = -inf. */
qsa_status qsa_merge(int32_t R, int32_t B, int32_t Hq, int32_t D,
                     const float *o_part, const float *lse_part, void *out,
                     int32_t out_is_bf16, float *lse_out, qsa_stream_t stream);

/* One decode step in one call: qsa_append of the N new tokens (skipped when
 * N == 0), then qsa_index_score, qsa_topk_select (no workspace),
 * qsa_sparse_decode and qsa_merge, enqueued in that order on `stream`, with
 * the arguments documented at each of those calls (the merge writes `out`
 * [B, Hq, D] and `lse_out` [B, Hq] from o_part / lse_part, which also hold
 * the R partials afterwards). Here the merge runs inside the decode's last
 * kernel, with the arithmetic of qsa_merge, so the results are the same
 * bits; this saves a launch. The page orders the steps (section "What the pull request
 * actually changes"); the single call is an interface convenience of this
 * library that saves the caller four calls. The calls' own argument checks
 * apply; the first failing call stops the sequence and its status is
 * returned (calls before it stay enqueued). */
qsa_status qsa_decode_step(const qsa_dims *dims, const qsa_cache *cache,
                           int32_t N, const int32_t *tok_seq,
                           const int32_t *tok_pos, const void *k_new,
                           const void *v_new, const void *kidx_new, int32_t B,
                           const int32_t *seq_lens, const void *q,
                           const void *q_idx, const float *w, int32_t k,
                           int32_t R, float *scores, int32_t ld_scores,
                           int32_t *sel, float *o_part, float *lse_part,
                           void *ws, size_t ws_bytes, void *out,
                           int32_t out_is_bf16, float *lse_out,
                           qsa_stream_t stream);

/* ---------------------------------------------------------- sparse prefill
 * Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
 * "Why a serving PR about an unreleased architecture is still worth your
 * time": the engine work around the decode path includes a native sparse
 * prefill kernel for the QSA path; the page gives none of its steps. This
 * library's reading: every token of an appended chunk queries like a decode
 * step over its own causal prefix.
 * Chunks: sequence s (0 <= s < S, block-table row s) holds the query rows
 * [row_start[s], row_start[s+1]) (int32 [S + 1], non-decreasing, row_start[0]
 * = 0, row_start[S] = Nq): its T_s = row_start[s+1] - row_start[s] newest
 * tokens, already appended (qsa_append), so that seq_lens[s] = L_s >= T_s
 * counts them. Row i of sequence s is the token at position L_s - T_s + i;
 * its causal length is row_len = L_s - T_s + i + 1, and its result is the
 * decode step of a sequence of that length (score its ceil(row_len / 4)
 * blocks, keep the min(k, .) best, attend over their tokens < row_len, split
 * R ways, merge). Rows are in chunk order: q, q_idx, w, scores, sel and the
 * partials are indexed by row. Supported: as qsa_index_score, and Hi in
 * {4, 8, 16, 32}; 0 <= Nq <= 65535. A chunk whose rows overrun Nq, whose
 * T_s exceeds L_s or whose ceil(L_s / 4) blocks exceed ld_scores is skipped
 * (its rows get row_len 0 and attend to nothing) and raises device error
 * flag 16. */

/* Scratch bytes of qsa_prefill_index_score. */
size_t qsa_prefill_index_score_workspace_size(const qsa_dims *dims, int32_t S,
                                              int32_t Nq);

/* Indexer scores of every prefill row (qsa_index_score per row):
 *   q_idx   bf16 [Nq, Hi, di] (16-byte aligned);  w  fp32 [Nq, Hi]
 *   scores  fp32 [Nq, ld_scores]: row r's blocks j < ceil(row_len[r] / 4)
 *           are written, nothing else
 *   row_len int32 [Nq] (out): each row's causal length, the sequence
 *           lengths qsa_topk_select takes for the rows (0 for a row of a
 *           skipped chunk)
 *   ws      scratch of qsa_prefill_index_score_workspace_size bytes,
 *           16-byte aligned, no initialisation needed; used until the call's
 *           kernels finish.
 * Up to 256 / Hi consecutive rows of one chunk share each 128-block tile of
 * the side cache in one tensor-core MMA. */
qsa_status qsa_prefill_index_score(const qsa_dims *dims, const qsa_cache *cache,
                                   int32_t S, const int32_t *seq_lens,
                                   const int32_t *row_start, int32_t Nq,
                                   const void *q_idx, const float *w,
                                   float *scores, int32_t ld_scores,
                                   int32_t *row_len, void *ws, size_t ws_bytes,
                                   qsa_stream_t stream);

/* Split sparse attention of every prefill row over its own selection
 * (qsa_sparse_decode per row, at the row's causal length):
 *   q        bf16 [Nq, Hq, D];  sel  int32 [Nq, k] (e.g. qsa_topk_select over
 *            the rows with row_len as sequence lengths)
 *   o_part   fp32 [R, Nq, Hq, D];  lse_part  fp32 [R, Nq, Hq]
 *   ws       qsa_sparse_decode_workspace_size(dims, Nq, k, R) bytes.
 * qsa_merge with B = Nq combines the partials. */
qsa_status qsa_prefill_sparse_decode(const qsa_dims *dims, const qsa_cache *cache,
                                     int32_t S, const int32_t *seq_lens,
                                     const int32_t *row_start, int32_t Nq,
                                     const void *q, const int32_t *sel, int32_t k,
                                     int32_t R, float *o_part, float *lse_part,
                                     void *ws, size_t ws_bytes, qsa_stream_t stream);

/* Scratch bytes of qsa_sparse_prefill. */
size_t qsa_sparse_prefill_workspace_size(const qsa_dims *dims, int32_t S, int32_t Nq,
                                         int32_t k, int32_t R);

/* The whole sparse prefill of the rows: qsa_prefill_index_score,
 * qsa_topk_select (rows, row_len), qsa_prefill_sparse_decode and qsa_merge
 * (B = Nq: out [Nq, Hq, D], lse_out [Nq, Hq]) enqueued in that order, with
 * the arguments documented there; ws holds
 * qsa_sparse_prefill_workspace_size bytes (16-byte aligned). The chunk's
 * tokens must already be appended. An interface convenience of this library
 * (one call instead of four); the first failing call stops the sequence. */
qsa_status qsa_sparse_prefill(const qsa_dims *dims, const qsa_cache *cache, int32_t S,
                              const int32_t *seq_lens, const int32_t *row_start,
                              int32_t Nq, const void *q, const void *q_idx,
                              const float *w, int32_t k, int32_t R, float *scores,
                              int32_t ld_scores, int32_t *row_len, int32_t *sel,
                              float *o_part, float *lse_part, void *ws,
                              size_t ws_bytes, void *out, int32_t out_is_bf16,
                              float *lse_out, qsa_stream_t stream);

/* Wait for `stream`, then read and clear the device error word of the
 * current device. *flags receives the bits that were set (0 if none):
 *   1 sequence row out of range    2 page id out of range
 *   4 block-table column out of range   8 selected block id out of range
 *   16 sequence length out of range (negative, or nb > ld_scores)
 *   32 a bounded wait gave up
 * Returns QSA_ERR_BOUNDS if any bit below 32 was set, QSA_ERR_TIMEOUT if only
 * bit 32 was, QSA_OK otherwise. flags may be NULL. */
qsa_status qsa_check_device_errors(qsa_stream_t stream, int32_t *flags);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
