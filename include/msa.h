/*
 * msa.h - C ABI of libmsa, the routed-memory hot path of Memory Sparse Attention (MSA)
 * on one NVIDIA B200 (sm_100a).
 *
 * The method (as described on the pages about MSA):
 *  - offline "global memory encoding": each document's per-token K, V and router keys K_r
 *    are compressed by fixed-length chunk mean pooling into K̄, V̄, K̄_r, with document-wise
 *    RoPE (positions restart at 0 in every document)
 *      [news.neo-ai.one article, "全体設計 / アーキテクチャ" and "推論パイプライン" (Fig. 3);
 *       ruixiangma.github.io blog "Memory-Sparse-Attention", "方法 / 稀疏注意力机制" and
 *       "文档级RoPE"];
 *  - online routing: the router query Q_r is matched against every chunk's K̄_r by cosine
 *    similarity, averaged over heads, maximised over query tokens (and over a document's
 *    chunks), and the top-k documents are selected
 *      [news.neo-ai.one, "アーキテクチャ"; github-eval-reports "MSA 项目评测报告", "核心模块"];
 *  - context assembly: only the selected K̄/V̄ are loaded (from GPU memory or, for very large
 *    banks, from host memory, asynchronously) and concatenated with the query's local K/V
 *      [news.neo-ai.one, "推論パイプライン"; ruixiangma blog, "Memory Parallel"];
 *  - sparse generation: attention over [memory ; local] with "global RoPE" on the active
 *    context, the query's start index shifted by k, the number of retrieved blocks
 *      [news.neo-ai.one, "グローバル RoPE"; ai-papers.net summary, "MSAの提案手法"].
 *
 * Conventions (all entry points):
 *  - Every call returns an msa_status; nothing aborts, exits or prints. Arguments are
 *    validated on the host before any work is enqueued; on an error nothing is enqueued
 *    and the outputs are left untouched. msa_last_error() gives a thread-local message.
 *  - Tensors are caller-owned, dense, row-major, and DEVICE pointers unless marked "host".
 *    The library allocates nothing on the hot path: scratch space is a caller-provided
 *    workspace whose size the matching *_workspace() query returns (256-byte aligned).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). All
 *    device work is asynchronous on that stream. The only host waits are in
 *    msa_fetch_finish (bounded by timeout_ms), msa_workspace_status and the offline
 *    msa_encode_hidden (one stream synchronisation after uploading its chunk table).
 *  - dtype: MSA_FP32 (float) or MSA_BF16 (bfloat16 bit patterns); all floating tensors of
 *    one call share it, except the fp32 inverse norms and scores.
 *  - Supported shapes: d in {64, 128}; h_q % h_kv == 0; h_qr % h_kv == 0; 1 <= k <= 32;
 *    anything else returns MSA_ERR_UNSUPPORTED or MSA_ERR_INVALID_ARG.
 *  - Calls are reentrant; two calls may run concurrently on different streams as long as
 *    they do not share a workspace.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent layout */
    MSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (d, k, head counts, T) */
    MSA_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or smaller than required */
    MSA_ERR_CUDA = 4,          /* a CUDA runtime call failed (message has the CUDA error) */
    MSA_ERR_TIMEOUT = 5,       /* a bounded host wait or a bounded device wait expired */
    MSA_ERR_DEVICE = 6         /* a kernel recorded an error in its workspace status word */
} msa_status;

typedef enum { MSA_FP32 = 0, MSA_BF16 = 1 } msa_dtype;

/* Human-readable name of a status code (static string). */
const char* msa_status_string(int status);
/* Thread-local description of the last failure in this thread ("" if none). */
const char* msa_last_error(void);
/* ABI version, (major << 16) | minor. */
int msa_version(void);

/* msa_set_device_wait_limit - the limit, in SM clock cycles, after which the consumer-side
 * waits of the tensor-core routing scan (its epilogue warps waiting for the tensor cores'
 * accumulators) give up: the kernel then records MSA_ERR_DEVICE's code 1 in the workspace
 * status word, stops issuing, lets the copies and MMAs it issued land, frees its tensor memory
 * and returns (outputs undefined). Copies and MMAs in flight are always waited for with the
 * default limit. cycles <= 0 restores the default (2^31 cycles, about a second). Process-wide,
 * read when a call is enqueued; returns the previous setting (0 = default). For testing the
 * error path; the pages describing MSA have no counterpart. */
int64_t msa_set_device_wait_limit(int64_t cycles);

/* ------------------------------------------------------------------------------------
 * Bank layout helper (host only, no device work).
 * Number of chunks of a corpus whose document d owns tokens
 * [doc_tok_off_host[d], doc_tok_off_host[d+1]): sum over docs of ceil(len / chunk).
 * Chunks never cross documents; a partial last chunk counts as one chunk.
 * Returns the count, or -1 if the offsets are not non-decreasing from 0 or chunk < 1.
 */
int64_t msa_count_chunks(const int64_t* doc_tok_off_host, int64_t n_docs, int32_t chunk);

/* ------------------------------------------------------------------------------------
 * msa_encode_pool - offline memory encoding: document-wise RoPE + chunk mean pooling.
 *   [news.neo-ai.one, "アーキテクチャ": chunk-wise mean pooling compresses K/V/K_r;
 *    "並列（ドキュメント単位）RoPE": positions restart at 0 per document;
 *    ruixiangma blog, "稀疏注意力机制 / 分块压缩" and "文档级RoPE"]
 *
 * K, V, K_r        [n_tok, h_kv, d] per-token keys, values and router keys (dtype).
 * doc_tok_off_host host [n_docs+1] token offsets (validated: starts at 0, non-decreasing,
 *                  ends at n_tok, and sum of ceil(len/chunk) == n_chunks).
 * doc_tok_off      device copy of the same offsets.
 * rope_base        RoPE base (e.g. 1e6); <= 0 disables rotation. RoPE pairs element i with
 *                  element i + d/2 ("rotate half") at angle pos * base^(-2i/d), pos = the
 *                  token's index within its document. K and K_r are rotated, V is not.
 * Kbar, Vbar, Kbar_r [n_chunks, h_kv, d] outputs (dtype): mean over each chunk's valid
 *                  tokens, accumulated in fp32, stored with round-to-nearest-even.
 * kr_inv_norm      [n_chunks, h_kv] fp32 output (nullable): 1/||Kbar_r[c,h]|| of the STORED
 *                  row (0 for a zero row), consumed by msa_route_topk.
 * doc_chunk_off    [n_docs+1] int64 output: chunk offsets (doc i owns chunks
 *                  [doc_chunk_off[i], doc_chunk_off[i+1])).
 * No workspace. Errors: INVALID_ARG (layout, null), UNSUPPORTED (d, dtype, h_kv*d).
 */
msa_status msa_encode_pool(const void* K, const void* V, const void* K_r, int64_t n_tok,
                           const int64_t* doc_tok_off_host, const int64_t* doc_tok_off,
                           int64_t n_docs, int32_t chunk, int32_t h_kv, int32_t d,
                           int32_t dtype, float rope_base, void* Kbar, void* Vbar,
                           void* Kbar_r, float* kr_inv_norm, int64_t* doc_chunk_off,
                           int64_t n_chunks, void* stream);

/* msa_encode_pool_status - the status of the last msa_encode_pool call on any stream of this
 * device, read on `stream` (which it synchronises): *code = 0, or the code a bounded device
 * wait recorded when it ran out (then MSA_ERR_DEVICE; the call's outputs are not defined).
 * The bf16, d = 128 pooling streams its input through bulk copies and waits on them with a
 * bound; each msa_encode_pool call starts the word at zero. No allocation. */
msa_status msa_encode_pool_status(int32_t* code, void* stream);

/* msa_kr_inv_norm - inverse L2 norms of a pre-pooled router-key bank (bank preparation for
 * banks that were not produced by msa_encode_pool): out[c,h] = 1/||Kbar_r[c,h,:]|| (0 for a
 * zero row), fp32 [n_chunks, h_kv]. */
msa_status msa_kr_inv_norm(const void* Kbar_r, int64_t n_chunks, int32_t h_kv, int32_t d,
                           int32_t dtype, float* kr_inv_norm, void* stream);

/* msa_kr_normalize - routing-only copy of a router-key bank for the tensor-core scan:
 * out[c,h,:] = Kbar_r[c,h,:] / ||Kbar_r[c,h]|| rounded to bf16 (zero rows stay zero),
 * [n_chunks, h_kv, d] bf16. Bank preparation, made once per bank; needed by msa_route_topk
 * when T > 16 (long queries). */
msa_status msa_kr_normalize(const void* Kbar_r, int64_t n_chunks, int32_t h_kv, int32_t d,
                            int32_t dtype, void* Kbar_r_hat, void* stream);

/* ------------------------------------------------------------------------------------
 * msa_route_topk - online routing: cosine scoring of every chunk and exact top-k documents.
 *   [news.neo-ai.one, "アーキテクチャ": the routing projector computes relevance by cosine
 *    similarity (mean over attention heads, then max over tokens) and selects the Top-k
 *    documents; github-eval-reports, "核心模块 / 路由投影器"; ruixiangma blog, "Top-k检索"]
 *
 * Q_r        [B, T, h_qr, d] router queries (dtype). Router head h uses router-key head
 *            floor(h / (h_qr / h_kv)).
 * Kbar_r     [n_chunks, h_kv, d] router-key bank (dtype), 16-byte aligned (nullable with
 *            Kbar_r_hat, see below).
 * kr_inv_norm [n_chunks, h_kv] fp32 inverse norms (from msa_encode_pool / msa_kr_inv_norm;
 *            nullable with Kbar_r_hat).
 * Kbar_r_hat (nullable) [n_chunks, h_kv, d] bf16 per-head unit rows (msa_kr_normalize).
 *            With Kbar_r_hat and a bf16 bank, every query length is scored on the tensor
 *            cores as one bf16 contraction of Kbar_r_hat with the per-head normalised queries
 *            (fp32 accumulation; Kbar_r and kr_inv_norm are not read and may be NULL, so a
 *            bank prepared for this scan need not keep K̄_r resident). Without it, queries
 *            with T <= 16 are scored on CUDA cores from Kbar_r and kr_inv_norm in fp32 (B*T rows
 *            in passes of up to 16); longer queries (17 <= T <= 256) require Kbar_r_hat.
 * doc_chunk_off [n_docs+1] device int64 chunk offsets (non-decreasing, ends at n_chunks).
 * Score of doc i for query b:
 *     S[b,i] = max_{c in doc i} max_t (1/h_qr) sum_h cos(Q_r[b,t,h], Kbar_r[c, g(h)])
 *   (cosine of a zero vector = 0; a document without chunks scores -inf).
 * exclude_bits (nullable) [B, ceil(n_docs/32)] uint32: bit i set = doc i is not eligible.
 * top_ids    [B, k] int32 output: the k eligible docs with the largest S[b,.], score
 *            descending, ties to the lower doc id (-0.0 ranks as +0.0); -1 when fewer than k
 *            docs are eligible.
 * top_scores [B, k] fp32 output (S of the selected docs; -inf in unused slots).
 * doc_scores (nullable) [B, n_docs] fp32 output: every S[b,i] (for tests).
 * Requires 1 <= k <= min(32, n_docs); T <= 16 (any dtype) or 17 <= T <= 256 (bf16 with
 * Kbar_r_hat).
 * ws         workspace of msa_route_topk_workspace(...) bytes; its first word is a device
 *            status (see msa_workspace_status).
 */
size_t msa_route_topk_workspace(int32_t B, int32_t T, int32_t h_qr, int32_t h_kv, int32_t d,
                                int32_t dtype, int64_t n_docs, int64_t n_chunks, int32_t k);
msa_status msa_route_topk(const void* Q_r, int32_t B, int32_t T, int32_t h_qr,
                          const void* Kbar_r, const float* kr_inv_norm, const void* Kbar_r_hat,
                          const int64_t* doc_chunk_off, int64_t n_docs, int64_t n_chunks,
                          int32_t h_kv, int32_t d, int32_t dtype, int32_t k,
                          const uint32_t* exclude_bits, int32_t* top_ids, float* top_scores,
                          float* doc_scores, void* ws, size_t ws_bytes, void* stream);

/* msa_route_topk_noalloc - msa_route_topk without a caller workspace, for callers that
 * cannot allocate device memory where they call it: code running under another framework's
 * memory planner (which owns every device allocation), paths that must not synchronise the
 * device (cudaMalloc/cudaFree may), and serving loops that forbid allocator calls.
 * (A library service; the pages describing MSA have no counterpart.)
 *
 * Same arguments and results as msa_route_topk, minus ws/ws_bytes. The scratch is a 2 MiB
 * array inside the library, held on every GPU that loads it until the process exits; calls
 * whose msa_route_topk_workspace(...) exceeds 2 MiB return MSA_ERR_UNSUPPORTED (use
 * msa_route_topk). The first call on a device, made with that device current, looks up the
 * array's device address (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture. It allocates nothing (no cudaMalloc/cudaFree or allocating library
 * routine). All calls share the one array, which keeps the last call's contents (what must
 * start at zero is cleared by every call); calls that overlap on the GPU race and must be
 * serialised by the caller. The cached address is that of the device's primary context (the
 * CUDA runtime's): it is not valid after cudaDeviceReset or under another driver-API context.
 * Device-side failures (a bounded wait that ran out, a bad index) are recorded in the array's
 * status word as in a workspace; read it with msa_route_topk_noalloc_status. */
msa_status msa_route_topk_noalloc(const void* Q_r, int32_t B, int32_t T, int32_t h_qr,
                                  const void* Kbar_r, const float* kr_inv_norm,
                                  const void* Kbar_r_hat, const int64_t* doc_chunk_off,
                                  int64_t n_docs, int64_t n_chunks, int32_t h_kv, int32_t d,
                                  int32_t dtype, int32_t k, const uint32_t* exclude_bits,
                                  int32_t* top_ids, float* top_scores, float* doc_scores,
                                  void* stream);

/* msa_route_topk_noalloc_status - the status word of the built-in scratch of
 * msa_route_topk_noalloc on the current device, read after the work queued on `stream`
 * (synchronises `stream`; allocates nothing). *code = 0 if the last call's kernels recorded no
 * error; otherwise returns MSA_ERR_DEVICE with *code the recorded error. The word is cleared
 * by every msa_route_topk_noalloc call, so read it after the call it should describe and
 * before the next. (A library service; the pages describing MSA have no counterpart.) */
msa_status msa_route_topk_noalloc_status(int32_t* code, void* stream);

/* Read the device status word of a workspace (synchronises `stream`): *code = 0 if the
 * kernels that used it recorded no error. Returns MSA_ERR_DEVICE if *code != 0. */
msa_status msa_workspace_status(const void* ws, int32_t* code, void* stream);

/* ------------------------------------------------------------------------------------
 * msa_gather - context assembly from a bank the GPU can address (HBM, or pinned host memory
 * reached directly over the host link).
 *   [news.neo-ai.one, "推論パイプライン": only the selected K̄/V̄ are loaded and concatenated
 *    with the local context]
 *
 * top_ids    [B, k] int32 (distinct ids; -1 entries are skipped).
 * Context rows of query b: the selected docs in ascending doc id, each doc's chunks in
 * order. gather_idx [B, max_ctx] int32 output: bank chunk row of each context row, -1
 * past ctx_len[b]; ctx_len [B] int32 output.
 * ctxK, ctxV [B, max_ctx, h_kv, d] outputs (dtype): copies of Kbar/Vbar rows; rows past
 *            ctx_len[b] are not written.
 * A context longer than max_ctx is truncated to max_ctx and flagged in the status word of
 * `ws` (MSA_ERR_DEVICE via msa_workspace_status); ws must hold 256 bytes.
 */
msa_status msa_gather(const int32_t* top_ids, int32_t B, int32_t k,
                      const int64_t* doc_chunk_off, int64_t n_docs, const void* Kbar,
                      const void* Vbar, int32_t h_kv, int32_t d, int32_t dtype, int32_t max_ctx,
                      int32_t* gather_idx, int32_t* ctx_len, void* ctxK, void* ctxV, void* ws,
                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * Asynchronous fetch from a bank in pinned host memory (tiered storage: router keys on the
 * GPU, content K̄/V̄ in host DRAM, fetched on demand when selected).
 *   [ruixiangma blog, "Memory Parallel / 分层内存存储"; news.neo-ai.one, "推論パイプライン"]
 *
 * msa_fetch_create allocates a context holding a pinned staging area for max_B*max_k ids
 * and two CUDA events (set-up time, not the hot path); msa_fetch_destroy frees it.
 * msa_fetch_begin enqueues on `stream`: the device gather indices (as msa_gather) and a
 *   device-to-host copy of top_ids into the staging area, then records an event. It does
 *   not wait.
 * msa_fetch_finish waits on the host (polling, at most timeout_ms milliseconds; 0 = check
 *   once) for that event, then issues one cudaMemcpyAsync per run of consecutive selected
 *   chunks for K̄ and for V̄ from the host bank into ctxK/ctxV on `copy_stream`, records an
 *   event there and makes `stream` wait for it. Kbar_host/Vbar_host are
 *   [n_chunks, h_kv, d] pinned host arrays; doc_chunk_off_host is the host copy of the
 *   chunk offsets. Returns MSA_ERR_TIMEOUT (nothing copied) if the ids are not ready in
 *   time; the context stays usable.
 */
typedef struct msa_fetch msa_fetch;
msa_status msa_fetch_create(int32_t max_B, int32_t max_k, msa_fetch** out);
void msa_fetch_destroy(msa_fetch* f);
msa_status msa_fetch_begin(msa_fetch* f, const int32_t* top_ids, int32_t B, int32_t k,
                           const int64_t* doc_chunk_off, int64_t n_docs, int32_t max_ctx,
                           int32_t* gather_idx, int32_t* ctx_len, void* ws, size_t ws_bytes,
                           void* stream);
msa_status msa_fetch_finish(msa_fetch* f, const int64_t* doc_chunk_off_host, int64_t n_docs,
                            const void* Kbar_host, const void* Vbar_host, int32_t h_kv,
                            int32_t d, int32_t dtype, int32_t max_ctx, void* ctxK, void* ctxV,
                            void* stream, void* copy_stream, int32_t timeout_ms);

/* ------------------------------------------------------------------------------------
 * msa_sparse_attend - GQA softmax attention over [gathered memory ; causal local context]
 * with global RoPE on the active context.
 *   [news.neo-ai.one, "グローバル RoPE（アクティブコンテキスト）": the query's start index
 *    is shifted by k (the number of Top-k retrieved blocks) to keep the causal order
 *    background -> query -> generation; "推論パイプライン": sparse generation over the
 *    assembled context]
 *
 * Q          [B, T, h_q, d]; query token t is local row L_loc - T + t.
 * K_loc, V_loc [B, L_loc, h_kv, d]; K_loc before RoPE. Requires 1 <= T <= L_loc.
 * ctxK, ctxV [B, max_ctx, h_kv, d] gathered memory rows; the first ctx_len[b] are used.
 * Q and K_loc rows are rotated at position pos0 + (local row index) (pos0 = k); memory rows
 * are used as stored. Query head h reads KV head floor(h / (h_q / h_kv)).
 * O[b,t,h] = softmax over {memory rows j < ctx_len[b]} U {local rows j <= L_loc - T + t} of
 *            scale * q.k, applied to the matching V rows; scale <= 0 means 1/sqrt(d).
 * O          [B, T, h_q, d] output (dtype), fp32 accumulation and softmax.
 * ws         msa_sparse_attend_workspace(...) bytes (split partials + the RoPE table).
 */
size_t msa_sparse_attend_workspace(int32_t B, int32_t T, int32_t h_q, int32_t h_kv, int32_t d,
                                   int32_t max_ctx, int32_t L_loc);
msa_status msa_sparse_attend(const void* Q, int32_t B, int32_t T, int32_t h_q,
                             const void* K_loc, const void* V_loc, int32_t L_loc,
                             const void* ctxK, const void* ctxV, const int32_t* ctx_len,
                             int32_t max_ctx, int32_t h_kv, int32_t d, int32_t dtype,
                             int32_t pos0, float rope_base, float scale, void* O, void* ws,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * msa_sparse_attend_backward - gradients of msa_sparse_attend with respect to its inputs.
 *   [ruixiangma.github.io blog, "训练策略": MSA is trained on the generation loss plus an
 *    auxiliary routing loss; news.neo-ai.one article, "プロジェクト概要", Fig. 1: top-k
 *    selection fused with the sparse attention keeps the model differentiable end to end]
 *
 * Same forward operation and arguments as msa_sparse_attend (Q, K_loc, V_loc, ctxK, ctxV,
 * ctx_len, max_ctx, h_kv, d, dtype, pos0, rope_base, scale), plus the output gradient
 * dO [B, T, h_q, d] (dtype). Writes fp32 gradients:
 *   dQ      [B, T, h_q, d]        with respect to Q (before RoPE);
 *   dK_loc  [B, L_loc, h_kv, d]   with respect to K_loc (before RoPE);
 *   dV_loc  [B, L_loc, h_kv, d];
 *   dK_ctx, dV_ctx [B, max_ctx, h_kv, d] with respect to the gathered memory rows (rows past
 *           ctx_len[b]: 0). msa_scatter_bank_grad adds them into the bank rows.
 * The softmax is recomputed (the forward again, in the workspace); probabilities and dS enter
 * the tensor-core products in bf16, accumulation is fp32. Routing (top-k) has no gradient.
 * Supported: bf16, d = 128, h_q / h_kv dividing 64 (else MSA_ERR_UNSUPPORTED). ws:
 * msa_sparse_attend_backward_workspace(...) bytes, 256-byte aligned; its status word records
 * an expired device wait.
 */
size_t msa_sparse_attend_backward_workspace(int32_t B, int32_t T, int32_t h_q, int32_t h_kv,
                                            int32_t d, int32_t max_ctx, int32_t L_loc);
msa_status msa_sparse_attend_backward(const void* Q, int32_t B, int32_t T, int32_t h_q,
                                      const void* K_loc, const void* V_loc, int32_t L_loc,
                                      const void* ctxK, const void* ctxV, const int32_t* ctx_len,
                                      int32_t max_ctx, int32_t h_kv, int32_t d, int32_t dtype,
                                      int32_t pos0, float rope_base, float scale, const void* dO,
                                      float* dQ, float* dK_loc, float* dV_loc, float* dK_ctx,
                                      float* dV_ctx, void* ws, size_t ws_bytes, void* stream);

/* msa_scatter_bank_grad - the gathered rows' gradients flow back into the memory bank:
 * dKbar[gather_idx[b, j]] += dK_ctx[b, j] and dVbar[...] += dV_ctx[b, j] for j < ctx_len[b]
 * (fp32 [n_chunks, h_kv, d], accumulated with atomics: several queries may gather one
 * document). gather_idx, ctx_len as written by msa_gather. An index outside [0, n_chunks) is
 * skipped and recorded in the status word of ws (>= 256 bytes, 256-byte aligned). */
msa_status msa_scatter_bank_grad(const int32_t* gather_idx, const int32_t* ctx_len, int32_t B,
                                 int32_t max_ctx, int32_t h_kv, int32_t d, const float* dK_ctx,
                                 const float* dV_ctx, float* dKbar, float* dVbar,
                                 int64_t n_chunks, void* ws, size_t ws_bytes, void* stream);

/* msa_aux_routing_loss - the auxiliary routing loss of training and its gradients.
 *   [ruixiangma.github.io blog, "训练策略": the router is trained with an auxiliary loss, a
 *    supervised contrastive loss between relevant and irrelevant document chunks, next to the
 *    generation loss. The pages give no formula; this is a reading, so its agreement with the
 *    authors' loss is not pinned.]
 * Chunk scores as in routing before the document maximum:
 *   s[b, c] = max_t (1/h_qr) sum_h cos(Q_r[b, t, h], Kbar_r[c, g(h)]);
 * positives: bit c of positive_bits[b, ceil(n_chunks/32)] marks chunk c relevant to query b;
 *   loss = mean over queries with positives of -(1/|P_b|) sum_{c in P_b} log softmax_c(s[b,:]/tau)
 * written to loss (one fp32 in device memory). Gradients (fp32, nullable): dQ_r [B, T, h_qr, d]
 * and dKbar_r [n_chunks, h_kv, d]; the token maximum passes its gradient to the first maximising
 * token. fp32 or bf16 inputs, d in {64, 128}. ws: msa_aux_routing_loss_workspace(B, n_chunks)
 * bytes, 256-byte aligned. The gradient of Q_r gathers over the chunks per query row (cost
 * B*T*h_qr*n_chunks): meant for training-sized banks. */
size_t msa_aux_routing_loss_workspace(int32_t B, int64_t n_chunks);
msa_status msa_aux_routing_loss(const void* Q_r, int32_t B, int32_t T, int32_t h_qr,
                                const void* Kbar_r, int64_t n_chunks, int32_t h_kv, int32_t d,
                                int32_t dtype, const uint32_t* positive_bits, float tau,
                                float* loss, float* dQ_r, float* dKbar_r, void* ws,
                                size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * msa_assemble_local - the local context of a Memory Interleaving round: for every query b,
 * the raw per-token K/V of the documents appended so far (segment 0 .. n_seg-1, in the order
 * appended) followed by the query's own T token rows, written contiguously.
 *   [ai-papers.net summary, "MSAの提案手法"; ruixiangma.github.io blog, "Memory Interleaving":
 *    each round's retrieved documents have their original text appended to the query's
 *    context for the next round]
 *
 * seg_k, seg_v  device arrays of B * n_seg device pointers (row-major [b][segment]), each to a
 *               segment's [seg_len, h_kv, d] rows (dtype), 16-byte aligned.
 * seg_len       device int32 [B * n_seg].
 * K_q, V_q      [B, T, h_kv, d] the query tokens' own K/V (before RoPE, like K_loc).
 * K_out, V_out  [B, L_loc, h_kv, d]; caller-owned. Requires sum_q seg_len[b][q] + T == L_loc
 *               for every query; a query for which it does not hold is left unwritten and the
 *               workspace status word records the error (msa_workspace_status).
 * ws            >= 256 bytes, 256-byte aligned; 0 <= n_seg <= 1024.
 */
msa_status msa_assemble_local(int32_t B, int32_t n_seg, const void* const* seg_k,
                              const void* const* seg_v, const int32_t* seg_len, const void* K_q,
                              const void* V_q, int32_t T, int32_t h_kv, int32_t d, int32_t dtype,
                              int64_t L_loc, void* K_out, void* V_out, void* ws, size_t ws_bytes,
                              void* stream);

/* ------------------------------------------------------------------------------------
 * Sparse generation over an assembled context. Once the routed memory of a layer is fixed
 * (route -> gather, at context construction), generation proceeds token by token: each new
 * token's K/V joins the end of the local context and the token attends over
 * [gathered memory ; local context] with the routed memory unchanged
 *   [news.neo-ai.one article, "推論パイプライン"; ruixiangma.github.io blog, "三阶段推理流程":
 *    routing and context assembly are one online stage, autoregressive generation over the
 *    assembled sparse context the next].
 * The local context is a caller-owned cache K_cache, V_cache [B, cap, h_kv, d] whose
 * length len (one int32 in device memory, shared by the batch) is read and advanced by the
 * kernels, so a captured step (CUDA graph) replays unchanged while the cache grows. Cache
 * row j holds its key already rotated at its global position pos0 + j (global RoPE of the
 * active context, applied once when the row is appended), so attention over the cache
 * rotates only the query.
 */

/* msa_kv_append - rows [len, len + T_new) of every query's cache <- K_new, V_new
 * [B, T_new, h_kv, d] (K before RoPE, like K_loc); row j's key is stored rotated at
 * position pos0 + j with base rope_base (rope_base <= 0: stored as given); then
 * len += T_new. If len + T_new > cap on the device, nothing is written, len is unchanged and
 * the workspace status word records the overflow (msa_workspace_status). ws >= 256 bytes,
 * 256-byte aligned. Fills a prompt into an empty cache (len = 0) as well as appending
 * generated tokens. */
msa_status msa_kv_append(void* K_cache, void* V_cache, int32_t B, int32_t cap, int32_t* len_dev,
                         const void* K_new, const void* V_new, int32_t T_new, int32_t h_kv,
                         int32_t d, int32_t dtype, int32_t pos0, float rope_base, void* ws,
                         size_t ws_bytes, void* stream);

/* msa_decode_step - one generation step of one routed layer: msa_kv_append of the step's T
 * tokens (K_new, V_new [B, T, h_kv, d], pre-RoPE) followed by msa_sparse_attend of their
 * queries Q [B, T, h_q, d] with K_loc, V_loc = the cache's first len rows (len read on the
 * device after the append; query token t is local row len - T + t at position
 * pos0 + len - T + t). The cache must have been filled with the same pos0 and rope_base
 * (its keys are stored rotated). ctxK, ctxV, ctx_len, max_ctx, pos0, rope_base, scale and O
 * as in msa_sparse_attend.
 * Supported: bf16, d = 128, h_kv in {1, 2, 4, 8}, (h_q / h_kv) * T <= 8 (else
 * MSA_ERR_UNSUPPORTED). ws: msa_decode_step_workspace(...) bytes, 256-byte aligned; its
 * status word records a cache overflow (then O is not written and len stays) or an expired
 * device wait. The step is two launches: the attention kernel, which appends the new rows
 * itself (each in the one tile that holds it, and into the cache) and starts the status word,
 * then the merge of split queries, which advances len; ws must not be shared with a call
 * running concurrently. */
size_t msa_decode_step_workspace(int32_t B, int32_t T, int32_t h_q, int32_t h_kv, int32_t d,
                                 int32_t max_ctx, int32_t cap);
msa_status msa_decode_step(const void* Q, const void* K_new, const void* V_new, int32_t B,
                           int32_t T, int32_t h_q, void* K_cache, void* V_cache, int32_t cap,
                           int32_t* len_dev, const void* ctxK, const void* ctxV,
                           const int32_t* ctx_len, int32_t max_ctx, int32_t h_kv, int32_t d,
                           int32_t dtype, int32_t pos0, float rope_base, float scale, void* O,
                           void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * msa_encode_hidden - offline memory encoding from hidden states: for every token, the key,
 * value and router-key projections K = H W_k^T, V = H W_v^T, K_r = H W_r^T, then document-wise
 * RoPE of K and K_r and chunk mean pooling as in msa_encode_pool, in one kernel whose epilogue
 * works on the fp32 products (the per-token K, V, K_r are never written).
 *   [ruixiangma.github.io blog, "稀疏注意力机制": the router K projector produces each
 *    document's routing keys; news.neo-ai.one, "アーキテクチャ": chunk-wise mean pooling]
 *
 * H              [n_tok, D] bf16 hidden states of the documents, documents contiguous.
 * W_k, W_v, W_r  [h_kv * 128, D] bf16 projection weights (output-major rows).
 * doc_tok_off_host, n_docs, chunk, rope_base: as msa_encode_pool (chunk must be 64).
 * Kbar, Vbar, Kbar_r [n_chunks, h_kv, 128] bf16 outputs (means of fp32 values, RNE);
 * doc_chunk_off  [n_docs+1] int64 device output.
 * ws             msa_encode_hidden_workspace(n_chunks) bytes, 256-byte aligned (chunk table;
 *                the status word records an expired device wait).
 * Supported: bf16, d = 128, chunk = 64, even h_kv, D a multiple of 64 (else
 * MSA_ERR_UNSUPPORTED). Synchronises `stream` once (the chunk table is uploaded from the host).
 * Inverse norms or the normalised routing bank come from msa_kr_inv_norm / msa_kr_normalize.
 */
size_t msa_encode_hidden_workspace(int64_t n_chunks);
msa_status msa_encode_hidden(const void* H, int64_t n_tok, int32_t D, const void* W_k,
                             const void* W_v, const void* W_r, const int64_t* doc_tok_off_host,
                             int64_t n_docs, int32_t chunk, int32_t h_kv, int32_t d,
                             int32_t dtype, float rope_base, void* Kbar, void* Vbar,
                             void* Kbar_r, int64_t* doc_chunk_off, int64_t n_chunks, void* ws,
                             size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
