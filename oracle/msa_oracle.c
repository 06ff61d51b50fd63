/*
 * msa_oracle.c - CPU oracle of the Memory Sparse Attention (MSA) routed-memory path.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline (cpu_baseline / --impl reference) may load or run this code. The CUDA library
 * never calls it, includes it, or shares any source, header, table or constant with it.
 *
 * Plain and slow on purpose: every value is computed in double precision in the order the
 * method states it, one output at a time. OpenMP only splits independent outputs across
 * host threads; it does not change any result.
 *
 * Sources (the pages describing MSA; section names as printed there):
 *  [A]  news.neo-ai.one article on MSA, section "全体設計 / アーキテクチャ" (architecture)
 *       and "推論パイプライン" (inference pipeline, Fig. 3).
 *  [B]  ai-papers.net summary of MSA, section "MSAの提案手法" (the method).
 *  [C]  ruixiangma.github.io blog "Memory-Sparse-Attention", section "方法" with
 *       "稀疏注意力机制" (sparse attention), "文档级RoPE" (document-wise RoPE),
 *       "三阶段推理流程" (three-stage inference) and "Memory Interleaving".
 *  [D]  github-eval-reports "MSA 项目评测报告", section "核心模块" (core modules).
 *
 * Readings where the pages are silent (each one the plainest reading the rest supports):
 *  - RoPE pairs element i with element i + d/2 ("rotate half"), angle pos * base^(-2i/d);
 *    the backbone is Qwen3 [A, 実験設定]. rope_base <= 0 disables rotation.
 *  - Chunks never cross documents; a partial last chunk is the mean of its valid tokens.
 *  - Router head h of h_qr uses router-key head floor(h / (h_qr / h_kv)); cosine of a zero
 *    vector is 0; the head mean is over the h_qr router heads.
 *  - A document's score is the max over its chunks of (max over query tokens of the
 *    head-mean cosine); a document without chunks scores -inf.
 *  - Top-k order: score descending, ties to the lower doc id.
 *  - Gathered context: the selected docs in ascending doc id, each doc's chunks in order.
 *  - Global RoPE: query token i of T sits at local index L - T + i; local row j and the
 *    query rows are rotated at position pos0 + j (pos0 = k, the number of retrieved
 *    blocks); gathered memory rows are not rotated again; memory rows are all visible,
 *    local rows are causal; one softmax over [memory ; local] at the given scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- element access */
static double orc_bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* dtype 0: fp32, 1: bf16 stored as its upper 16 bits */
static double orc_at(const void* p, int dtype, int64_t i) {
    return dtype == 0 ? (double)((const float*)p)[i] : orc_bf16_value(((const uint16_t*)p)[i]);
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Round a double to the nearest bf16 (ties to even), returned as its bit pattern. The
 * oracle's own rounding, used to mirror the storage points of the bf16 configuration. */
uint16_t orc_round_bf16(double x) {
    if (x != x) return 0x7FC0;
    float f = (float)x; /* double -> float is exact when the bf16 decision is unaffected */
    uint32_t u;
    memcpy(&u, &f, 4);
    /* decide on the double itself: compare against the two bf16 neighbours */
    uint32_t lo = u & 0xFFFF0000u;
    float flo, fhi;
    memcpy(&flo, &lo, 4);
    uint32_t hi = lo + 0x10000u;
    memcpy(&fhi, &hi, 4);
    double dlo = flo, dhi = fhi;
    /* neighbours bracket x (toward zero / away from zero for either sign) */
    double e_lo = fabs(x - dlo), e_hi = fabs(dhi - x);
    if (e_lo < e_hi) return (uint16_t)(lo >> 16);
    if (e_hi < e_lo) return (uint16_t)(hi >> 16);
    return ((lo >> 16) & 1u) ? (uint16_t)(hi >> 16) : (uint16_t)(lo >> 16);
}

void orc_round_bf16_array(const double* x, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_round_bf16(x[i]);
}

/* ---------------------------------------------------------------- RoPE
 * Rotary position embedding of one head vector x[0..d) at position pos:
 *   for i < d/2, a = pos * base^(-2i/d):
 *     x[i]       <- x[i] cos a - x[i + d/2] sin a
 *     x[i + d/2] <- x[i + d/2] cos a + x[i] sin a
 * Document-wise RoPE restarts pos at 0 for every document [A, 並列(ドキュメント単位)RoPE];
 * [C, 文档级RoPE]. */
void orc_rope(double* x, int d, double pos, double base) {
    if (base <= 0.0) return;
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)d);
        double a = pos * theta;
        double c = cos(a), s = sin(a);
        double x1 = x[i], x2 = x[i + half];
        x[i] = x1 * c - x2 * s;
        x[i + half] = x2 * c + x1 * s;
    }
}

/* ---------------------------------------------------------------- offline encode
 * Global memory encoding [A, 推論パイプライン]; [C, 三阶段推理流程]: each document is split
 * into fixed-length chunks and the chunk's K, V and router keys K_r are mean-pooled into
 * K̄, V̄, K̄_r [A, アーキテクチャ]; [C, 稀疏注意力机制 "分块压缩"]; [D, 核心模块 "KV压缩"].
 * K and K_r carry document-wise RoPE (positions restart at 0 in every document); V does
 * not. Inputs: K, V, K_r [N_tok, h_kv, d] in `dtype`; doc_tok_off[n_docs + 1].
 * Outputs (double): Kbar, Vbar, Krbar [n_chunks, h_kv, d]; doc_chunk_off[n_docs + 1].
 * Returns n_chunks, or -1 on an invalid layout. */
int64_t orc_encode_pool(int dtype, const void* K, const void* V, const void* Kr,
                        const int64_t* doc_tok_off, int n_docs, int chunk, int h_kv, int d,
                        double rope_base, double* Kbar, double* Vbar, double* Krbar,
                        int64_t* doc_chunk_off) {
    if (chunk <= 0 || d <= 0 || (d & 1) || h_kv <= 0 || n_docs < 0) return -1;
    doc_chunk_off[0] = 0;
    for (int i = 0; i < n_docs; ++i) {
        int64_t len = doc_tok_off[i + 1] - doc_tok_off[i];
        if (len < 0) return -1;
        doc_chunk_off[i + 1] = doc_chunk_off[i] + (len + chunk - 1) / chunk;
    }
    int64_t row = (int64_t)h_kv * d;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_docs; ++i) {
        double* kx = (double*)malloc(sizeof(double) * (size_t)d);
        double* rx = (double*)malloc(sizeof(double) * (size_t)d);
        int64_t t_doc = doc_tok_off[i];
        for (int64_t c = doc_chunk_off[i]; c < doc_chunk_off[i + 1]; ++c) {
            int64_t j = c - doc_chunk_off[i];
            int64_t t0 = t_doc + j * chunk;
            int64_t t1 = t0 + chunk;
            if (t1 > doc_tok_off[i + 1]) t1 = doc_tok_off[i + 1];
            double n = (double)(t1 - t0);
            for (int h = 0; h < h_kv; ++h) {
                double* ko = Kbar + c * row + (int64_t)h * d;
                double* vo = Vbar + c * row + (int64_t)h * d;
                double* ro = Krbar + c * row + (int64_t)h * d;
                for (int e = 0; e < d; ++e) ko[e] = vo[e] = ro[e] = 0.0;
                for (int64_t t = t0; t < t1; ++t) {
                    double pos = (double)(t - t_doc); /* position within the document */
                    int64_t base = t * row + (int64_t)h * d;
                    for (int e = 0; e < d; ++e) {
                        kx[e] = orc_at(K, dtype, base + e);
                        rx[e] = orc_at(Kr, dtype, base + e);
                    }
                    orc_rope(kx, d, pos, rope_base);
                    orc_rope(rx, d, pos, rope_base);
                    for (int e = 0; e < d; ++e) {
                        ko[e] += kx[e];
                        ro[e] += rx[e];
                        vo[e] += orc_at(V, dtype, base + e);
                    }
                }
                for (int e = 0; e < d; ++e) { ko[e] /= n; vo[e] /= n; ro[e] /= n; }
            }
        }
        free(kx);
        free(rx);
    }
    return doc_chunk_off[n_docs];
}

/* ---------------------------------------------------------------- routing
 * Online routing [A, アーキテクチャ / 推論パイプライン]; [C, 稀疏注意力机制 "Top-k检索"];
 * [D, 核心模块 "路由投影器"]: the router query Q_r is compared with every chunk's K̄_r by
 * cosine similarity; the cosines are averaged over heads, then the maximum is taken over
 * query tokens; a document's score is the maximum over its chunks; the k best documents
 * are selected (score descending, ties to the lower doc id).
 *
 * Q_r [B, T, h_qr, d] and Krbar [n_chunks, h_kv, d] in `dtype`. exclude_bits (nullable)
 * [B, ceil(n_docs / 32)]: bit i set = doc i is not eligible. Outputs: doc_scores
 * [B, n_docs] (double, nullable), top_ids [B, k] (int32, -1 when fewer than k docs are
 * eligible) and top_scores [B, k] (double, -inf in unused slots). Returns 0 or -1. */
typedef struct { double s; int32_t id; } orc_cand;

static int orc_cand_cmp(const void* a, const void* b) {
    const orc_cand* x = (const orc_cand*)a;
    const orc_cand* y = (const orc_cand*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

double orc_cosine(const double* q, const double* k, int d) {
    double dot = 0.0, nq = 0.0, nk = 0.0;
    for (int e = 0; e < d; ++e) {
        dot += q[e] * k[e];
        nq += q[e] * q[e];
        nk += k[e] * k[e];
    }
    if (nq == 0.0 || nk == 0.0) return 0.0;
    return dot / (sqrt(nq) * sqrt(nk));
}

int orc_route(int dtype, const void* Qr, int B, int T, int h_qr, const void* Krbar, int h_kv,
              int d, const int64_t* doc_chunk_off, int n_docs, int k,
              const uint32_t* exclude_bits, double* doc_scores, int32_t* top_ids,
              double* top_scores) {
    if (B < 0 || T <= 0 || h_qr <= 0 || h_kv <= 0 || h_qr % h_kv || k < 0 || k > n_docs)
        return -1;
    int m = h_qr / h_kv;
    int64_t words = (n_docs + 31) / 32;
    double* S = (double*)malloc(sizeof(double) * (size_t)(n_docs > 0 ? n_docs : 1));
    orc_cand* cand = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(n_docs > 0 ? n_docs : 1));
    double* q = (double*)malloc(sizeof(double) * (size_t)T * h_qr * d);
    for (int b = 0; b < B; ++b) {
        for (int64_t e = 0; e < (int64_t)T * h_qr * d; ++e)
            q[e] = orc_at(Qr, dtype, (int64_t)b * T * h_qr * d + e);
#pragma omp parallel for schedule(dynamic, 64)
        for (int i = 0; i < n_docs; ++i) {
            double kk[512];
            double best = -INFINITY;
            for (int64_t c = doc_chunk_off[i]; c < doc_chunk_off[i + 1]; ++c) {
                double mt = -INFINITY; /* max over query tokens */
                for (int t = 0; t < T; ++t) {
                    double s = 0.0; /* mean over router heads */
                    for (int h = 0; h < h_qr; ++h) {
                        int g = h / m;
                        for (int e = 0; e < d; ++e)
                            kk[e] = orc_at(Krbar, dtype, (c * h_kv + g) * (int64_t)d + e);
                        s += orc_cosine(q + ((int64_t)t * h_qr + h) * d, kk, d);
                    }
                    s /= (double)h_qr;
                    if (s > mt) mt = s;
                }
                if (mt > best) best = mt; /* max over the document's chunks */
            }
            S[i] = best;
        }
        int n_el = 0;
        for (int i = 0; i < n_docs; ++i) {
            if (doc_scores) doc_scores[(int64_t)b * n_docs + i] = S[i];
            if (exclude_bits && ((exclude_bits[(int64_t)b * words + i / 32] >> (i % 32)) & 1u))
                continue;
            cand[n_el].s = S[i] == 0.0 ? 0.0 : S[i]; /* -0.0 ranks as +0.0 */
            cand[n_el].id = i;
            ++n_el;
        }
        qsort(cand, (size_t)n_el, sizeof(orc_cand), orc_cand_cmp);
        for (int j = 0; j < k; ++j) {
            top_ids[(int64_t)b * k + j] = j < n_el ? cand[j].id : -1;
            if (top_scores) top_scores[(int64_t)b * k + j] = j < n_el ? cand[j].s : -INFINITY;
        }
    }
    free(S);
    free(cand);
    free(q);
    return 0;
}

/* ---------------------------------------------------------------- context assembly
 * Only the selected documents' K̄/V̄ are loaded and concatenated with the query's local
 * context [A, 推論パイプライン]; [C, 三阶段推理流程 "路由与上下文组装"]. gather_idx[b, j] is
 * the bank chunk row of context row j of query b: the selected docs in ascending doc id,
 * each doc's chunks in order; rows past ctx_len[b] are -1. Returns 0, -1 if a context
 * would exceed max_ctx, -2 on a repeated or out-of-range doc id. */
static int orc_int_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

int orc_gather(const int32_t* top_ids, int B, int k, const int64_t* doc_chunk_off, int n_docs,
               int max_ctx, int32_t* gather_idx, int32_t* ctx_len) {
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    int rc = 0;
    for (int b = 0; b < B && rc == 0; ++b) {
        int n = 0;
        for (int j = 0; j < k; ++j) {
            int32_t id = top_ids[(int64_t)b * k + j];
            if (id < 0) continue;
            if (id >= n_docs) { rc = -2; break; }
            ids[n++] = id;
        }
        if (rc) break;
        qsort(ids, (size_t)n, sizeof(int32_t), orc_int_cmp);
        for (int j = 1; j < n; ++j) if (ids[j] == ids[j - 1]) rc = -2;
        if (rc) break;
        int64_t len = 0;
        for (int j = 0; j < n; ++j) {
            for (int64_t c = doc_chunk_off[ids[j]]; c < doc_chunk_off[ids[j] + 1]; ++c) {
                if (len >= max_ctx) { rc = -1; break; }
                gather_idx[(int64_t)b * max_ctx + len++] = (int32_t)c;
            }
            if (rc) break;
        }
        if (rc) break;
        ctx_len[b] = (int32_t)len;
        for (int64_t j = len; j < max_ctx; ++j) gather_idx[(int64_t)b * max_ctx + j] = -1;
    }
    free(ids);
    return rc;
}

/* ---------------------------------------------------------------- sparse attention
 * Sparse generation over the assembled context [A, 推論パイプライン "スパース生成"];
 * [C, 三阶段推理流程 "稀疏生成"], with global RoPE on the active context: the query's start
 * index is shifted by k, the number of retrieved blocks [A, グローバル RoPE]; [B, MSAの提案手法].
 *
 * Q [B, T, h_q, d]; K_loc, V_loc [B, L, h_kv, d] (K_loc before RoPE); memory rows are bank
 * rows Kbar/Vbar [*, h_kv, d] selected by gather_idx [B, max_ctx] (first ctx_len[b] used).
 * Query head h reads KV head floor(h / (h_q / h_kv)). Output O [B, T, h_q, d] (double).
 * scale <= 0 means 1 / sqrt(d). Returns 0 or -1. */
int orc_attend(int dtype, const void* Q, int B, int T, int h_q, const void* K_loc,
               const void* V_loc, int L, const void* Kbar, const void* Vbar,
               const int32_t* gather_idx, const int32_t* ctx_len, int max_ctx, int h_kv, int d,
               int pos0, double rope_base, double scale, double* O) {
    if (T <= 0 || L < T || h_q <= 0 || h_kv <= 0 || h_q % h_kv || d <= 0 || (d & 1)) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int grp = h_q / h_kv;
    for (int b = 0; b < B; ++b) {
        int n_ctx = ctx_len[b];
        if (n_ctx < 0 || n_ctx > max_ctx) return -1;
        /* local keys rotated at pos0 + j, once per (row, kv head) */
        double* kl = (double*)malloc(sizeof(double) * (size_t)L * h_kv * d);
        for (int64_t j = 0; j < L; ++j)
            for (int g = 0; g < h_kv; ++g) {
                double* r = kl + (j * h_kv + g) * d;
                for (int e = 0; e < d; ++e)
                    r[e] = orc_at(K_loc, dtype, (((int64_t)b * L + j) * h_kv + g) * d + e);
                orc_rope(r, d, (double)pos0 + (double)j, rope_base);
            }
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < h_q; ++h) {
                int g = h / grp;
                int64_t qi = (int64_t)L - T + t; /* local index of this query token */
                double* q = (double*)malloc(sizeof(double) * (size_t)d);
                double* lg = (double*)malloc(sizeof(double) * (size_t)(n_ctx + L));
                for (int e = 0; e < d; ++e)
                    q[e] = orc_at(Q, dtype, (((int64_t)b * T + t) * h_q + h) * d + e);
                orc_rope(q, d, (double)pos0 + (double)qi, rope_base);
                int n = 0;
                double mx = -INFINITY;
                for (int j = 0; j < n_ctx; ++j) { /* memory rows: all visible */
                    int64_t c = gather_idx[(int64_t)b * max_ctx + j];
                    double s = 0.0;
                    for (int e = 0; e < d; ++e)
                        s += q[e] * orc_at(Kbar, dtype, (c * h_kv + g) * (int64_t)d + e);
                    lg[n] = s * scale;
                    if (lg[n] > mx) mx = lg[n];
                    ++n;
                }
                for (int64_t j = 0; j <= qi; ++j) { /* local rows: causal */
                    const double* r = kl + (j * h_kv + g) * d;
                    double s = 0.0;
                    for (int e = 0; e < d; ++e) s += q[e] * r[e];
                    lg[n] = s * scale;
                    if (lg[n] > mx) mx = lg[n];
                    ++n;
                }
                double den = 0.0;
                for (int j = 0; j < n; ++j) { lg[j] = exp(lg[j] - mx); den += lg[j]; }
                double* o = O + (((int64_t)b * T + t) * h_q + h) * d;
                for (int e = 0; e < d; ++e) o[e] = 0.0;
                n = 0;
                for (int j = 0; j < n_ctx; ++j, ++n) {
                    int64_t c = gather_idx[(int64_t)b * max_ctx + j];
                    for (int e = 0; e < d; ++e)
                        o[e] += lg[n] * orc_at(Vbar, dtype, (c * h_kv + g) * (int64_t)d + e);
                }
                for (int64_t j = 0; j <= qi; ++j, ++n)
                    for (int e = 0; e < d; ++e)
                        o[e] += lg[n] *
                                orc_at(V_loc, dtype, (((int64_t)b * L + j) * h_kv + g) * d + e);
                for (int e = 0; e < d; ++e) o[e] /= den;
                free(q);
                free(lg);
            }
        free(kl);
    }
    return 0;
}

/* ---------------------------------------------------------------- its gradients
 * Reverse mode of orc_attend, for training the routed layer: continued pre-training uses the
 * standard generation loss through the sparse attention plus an auxiliary routing loss
 * [C, 训练策略 "连续预训练阶段"].
 * Given dO [B, T, h_q, d] (double), writes (double, zeroed here):
 *   dQ [B, T, h_q, d]; dK_loc, dV_loc [B, L, h_kv, d] (w.r.t. the pre-RoPE local keys);
 *   dK_ctx, dV_ctx [B, max_ctx, h_kv, d] w.r.t. the gathered memory rows as used (row j of
 *   query b is bank row gather_idx[b, j]; rows j >= ctx_len[b] get zero).
 * Per query row: P = softmax(scale q k^T) over the visible rows, dV_j += P_j dO,
 * dP_j = dO . v_j, dS_j = P_j (dP_j - sum_i P_i dP_i), dq_rot = scale sum_j dS_j k_j,
 * dk_j += scale dS_j q_rot; rotated vectors go back through the inverse rotation (RoPE is
 * orthogonal: the rotation by -pos). Sequential over query rows (small cases). Returns 0 or -1. */
int orc_attend_backward(int dtype, const void* Q, int B, int T, int h_q, const void* K_loc,
                        const void* V_loc, int L, const void* Kbar, const void* Vbar,
                        const int32_t* gather_idx, const int32_t* ctx_len, int max_ctx, int h_kv,
                        int d, int pos0, double rope_base, double scale, const double* dO,
                        double* dQ, double* dK_loc, double* dV_loc, double* dK_ctx,
                        double* dV_ctx) {
    if (T <= 0 || L < T || h_q <= 0 || h_kv <= 0 || h_q % h_kv || d <= 0 || (d & 1)) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    int grp = h_q / h_kv;
    memset(dQ, 0, sizeof(double) * (size_t)B * T * h_q * d);
    memset(dK_loc, 0, sizeof(double) * (size_t)B * L * h_kv * d);
    memset(dV_loc, 0, sizeof(double) * (size_t)B * L * h_kv * d);
    memset(dK_ctx, 0, sizeof(double) * (size_t)B * max_ctx * h_kv * d);
    memset(dV_ctx, 0, sizeof(double) * (size_t)B * max_ctx * h_kv * d);
    double* q = (double*)malloc(sizeof(double) * (size_t)d);
    double* dq = (double*)malloc(sizeof(double) * (size_t)d);
    for (int b = 0; b < B; ++b) {
        int n_ctx = ctx_len[b];
        if (n_ctx < 0 || n_ctx > max_ctx) { free(q); free(dq); return -1; }
        int n_max = n_ctx + L;
        /* rotated local keys and their (rotated) gradients */
        double* kl = (double*)malloc(sizeof(double) * (size_t)L * h_kv * d);
        double* dkl = (double*)calloc((size_t)L * h_kv * d, sizeof(double));
        double* p = (double*)malloc(sizeof(double) * (size_t)n_max);
        double* dp = (double*)malloc(sizeof(double) * (size_t)n_max);
        for (int64_t j = 0; j < L; ++j)
            for (int g = 0; g < h_kv; ++g) {
                double* r = kl + (j * h_kv + g) * d;
                for (int e = 0; e < d; ++e)
                    r[e] = orc_at(K_loc, dtype, (((int64_t)b * L + j) * h_kv + g) * d + e);
                orc_rope(r, d, (double)pos0 + (double)j, rope_base);
            }
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < h_q; ++h) {
                int g = h / grp;
                int64_t qi = (int64_t)L - T + t;
                const double pos = (double)pos0 + (double)qi;
                for (int e = 0; e < d; ++e)
                    q[e] = orc_at(Q, dtype, (((int64_t)b * T + t) * h_q + h) * d + e);
                orc_rope(q, d, pos, rope_base);
                const double* go = dO + (((int64_t)b * T + t) * h_q + h) * d;
                /* forward again: logits, softmax */
                int n = 0;
                double mx = -INFINITY;
                for (int j = 0; j < n_ctx; ++j, ++n) {
                    int64_t c = gather_idx[(int64_t)b * max_ctx + j];
                    double sdot = 0.0;
                    for (int e = 0; e < d; ++e)
                        sdot += q[e] * orc_at(Kbar, dtype, (c * h_kv + g) * (int64_t)d + e);
                    p[n] = sdot * scale;
                    if (p[n] > mx) mx = p[n];
                }
                for (int64_t j = 0; j <= qi; ++j, ++n) {
                    const double* r = kl + (j * h_kv + g) * d;
                    double sdot = 0.0;
                    for (int e = 0; e < d; ++e) sdot += q[e] * r[e];
                    p[n] = sdot * scale;
                    if (p[n] > mx) mx = p[n];
                }
                double den = 0.0;
                for (int j = 0; j < n; ++j) { p[j] = exp(p[j] - mx); den += p[j]; }
                for (int j = 0; j < n; ++j) p[j] /= den;
                /* dV, dP and their weighted sum */
                double dsum = 0.0;
                n = 0;
                for (int j = 0; j < n_ctx; ++j, ++n) {
                    int64_t c = gather_idx[(int64_t)b * max_ctx + j];
                    double* gv = dV_ctx + (((int64_t)b * max_ctx + j) * h_kv + g) * d;
                    double acc = 0.0;
                    for (int e = 0; e < d; ++e) {
                        gv[e] += p[n] * go[e];
                        acc += go[e] * orc_at(Vbar, dtype, (c * h_kv + g) * (int64_t)d + e);
                    }
                    dp[n] = acc;
                    dsum += p[n] * acc;
                }
                for (int64_t j = 0; j <= qi; ++j, ++n) {
                    double* gv = dV_loc + (((int64_t)b * L + j) * h_kv + g) * d;
                    double acc = 0.0;
                    for (int e = 0; e < d; ++e) {
                        gv[e] += p[n] * go[e];
                        acc += go[e] *
                               orc_at(V_loc, dtype, (((int64_t)b * L + j) * h_kv + g) * d + e);
                    }
                    dp[n] = acc;
                    dsum += p[n] * acc;
                }
                /* dS, then the query and key gradients (rotated frame) */
                for (int e = 0; e < d; ++e) dq[e] = 0.0;
                n = 0;
                for (int j = 0; j < n_ctx; ++j, ++n) {
                    int64_t c = gather_idx[(int64_t)b * max_ctx + j];
                    const double ds = p[n] * (dp[n] - dsum) * scale;
                    double* gk = dK_ctx + (((int64_t)b * max_ctx + j) * h_kv + g) * d;
                    for (int e = 0; e < d; ++e) {
                        dq[e] += ds * orc_at(Kbar, dtype, (c * h_kv + g) * (int64_t)d + e);
                        gk[e] += ds * q[e];
                    }
                }
                for (int64_t j = 0; j <= qi; ++j, ++n) {
                    const double ds = p[n] * (dp[n] - dsum) * scale;
                    const double* r = kl + (j * h_kv + g) * d;
                    double* gk = dkl + (j * h_kv + g) * d;
                    for (int e = 0; e < d; ++e) {
                        dq[e] += ds * r[e];
                        gk[e] += ds * q[e];
                    }
                }
                orc_rope(dq, d, -pos, rope_base); /* back through R(pos theta) */
                double* gq = dQ + (((int64_t)b * T + t) * h_q + h) * d;
                for (int e = 0; e < d; ++e) gq[e] = dq[e];
            }
        for (int64_t j = 0; j < L; ++j)
            for (int g = 0; g < h_kv; ++g) {
                double* r = dkl + (j * h_kv + g) * d;
                orc_rope(r, d, -((double)pos0 + (double)j), rope_base);
                double* gk = dK_loc + (((int64_t)b * L + j) * h_kv + g) * d;
                for (int e = 0; e < d; ++e) gk[e] = r[e];
            }
        free(kl);
        free(dkl);
        free(p);
        free(dp);
    }
    free(q);
    free(dq);
    return 0;
}
