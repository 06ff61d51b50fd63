// kernels.cuh - parameter blocks and launchers of the libmsa kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <string>

namespace msa {

// api.cu: thread-local message of msa_last_error
void set_last_error(const std::string& msg);
// api.cu: the device wait limit set by msa_set_device_wait_limit (0: default)
long long device_wait_limit();

// ---- encode_pool.cu
struct EncodeParams {
  const void* K;
  const void* V;
  const void* Kr;
  const int64_t* tok_off;    // [n_docs+1]
  const int64_t* chunk_off;  // [n_docs+1] (written by the chunk-offset kernel)
  int64_t n_docs, n_chunks;
  int chunk, h_kv;
  int rope;                  // 0: no rotation
  unsigned long long rope_turns[128];  // theta_i / (2 pi) mod 1, 64-bit fractions (i < d/2)
  void* Kb;
  void* Vb;
  void* Rb;
  float* inv_norm;           // nullable
};
cudaError_t launch_encode_pool(const EncodeParams& p, int dtype, int d, int sms, cudaStream_t st);
// encode_pool.cu: the pooling encode's status word (an expired bounded wait), read on `st`
cudaError_t read_encode_status(int* code, cudaStream_t st);
cudaError_t launch_inv_norm(const void* R, int64_t n_chunks, int h_kv, int d, int dtype, float* out,
                            int sms, cudaStream_t st);

// ---- route.cu
struct RouteParams {
  const void* qr;            // [B, T, h_qr, d] of this pass
  const void* kr;            // [n_chunks, h_kv, d]
  const float* invk;         // [n_chunks, h_kv]
  const int64_t* coff;       // [n_docs + 1]
  const uint32_t* excl;      // nullable [B, words] of this pass
  int64_t n_docs, n_chunks, words;
  int B, T, h_qr, h_kv, d, k;
  int32_t* top_ids;          // [B, k] of this pass
  float* top_scores;         // [B, k]
  float* doc_scores;         // nullable [B, n_docs]
  unsigned long long* cand;  // [grid, B, k]
  unsigned int* counter;
  int* err;
  int inv_bulk;              // inverse norms copied with each tile (h_kv % 4 == 0, aligned)
};
struct RouteChoice { int R, E; };
RouteChoice route_choose(int dtype, int rows, int W);
int route_grid(int dtype, RouteChoice c, int W, int h_kv, int h_qr, int sms, int64_t n_chunks);
cudaError_t route_launch(int dtype, RouteChoice c, const RouteParams& p, int grid, cudaStream_t st);

// ---- route_tc.cu (tensor-core scan for long queries)
struct TcPlan {
  bool ok;
  int NQ, N, grid, topk_grid, stages;
  int64_t n_qtiles, n_ctiles;
  size_t q_bytes, m_bytes, cand_bytes, smem;
};
struct RouteTcArgs {
  const void* Q_r;
  const void* Kr_hat;        // [n_chunks, h_kv * d] bf16 per-head unit rows
  const int64_t* coff;
  const uint32_t* excl;
  int64_t n_docs, n_chunks;
  int B, T, h_qr, h_kv, d, k, dtype;
  int32_t* top_ids;
  float* top_scores;
  float* doc_scores;
  __nv_bfloat16* q_hat;      // workspace [B*T, h_kv * d]
  float* mscore;             // unused (scores stay on chip)
  unsigned long long* cand;  // workspace
  unsigned int* counter;
  int* err;
  long long wait_limit;      // consumer-side device waits, SM clocks (0: default)
};
TcPlan tc_plan(int B, int T, int h_kv, int d, int64_t n_docs, int64_t n_chunks, int k, int sms);
cudaError_t launch_route_tc(const RouteTcArgs& a, const TcPlan& pl, cudaStream_t st);
cudaError_t launch_kr_normalize(const void* R, int64_t n_chunks, int h_kv, int d, int dtype,
                                void* out, int sms, cudaStream_t st);

// ---- gather.cu
struct GatherParams {
  const int32_t* ids;      // [B, k]
  const int64_t* coff;     // [n_docs + 1]
  int64_t n_docs;
  int B, k, max_ctx;
  int64_t row_bytes;       // h_kv * d * sizeof(T), a multiple of 16
  const void* Kb;          // nullable: index-only mode
  const void* Vb;
  int32_t* gidx;           // [B, max_ctx]
  int32_t* ctx_len;        // [B]
  void* ctxK;
  void* ctxV;
  int* err;
};
cudaError_t launch_gather(const GatherParams& p, cudaStream_t st);

// ---- attend.cu
struct AttendParams {
  const void* Q;        // [B, T, h_q, d]
  const void* Kl;       // [B, L, h_kv, d]
  const void* Vl;
  const void* cK;       // [B, max_ctx, h_kv, d]
  const void* cV;
  const int32_t* ctx_len;
  int B, T, h_q, h_kv, d, L, max_ctx;
  int rope;             // 0: no rotation
  const float2* cs;     // [L][d/2] cos/sin at positions pos0 + j
  float scale_log2;     // softmax scale * log2(e)
  int S, KPS, RB, NRB;  // splits, keys per split, rows per CTA, row blocks
  float* part_o;        // [B*T*h_q, S, d]
  float* part_ml;       // [B*T*h_q, S, 2]
  unsigned int* counters;  // [B*h_kv, NRB] split tickets
  void* O;              // [B, T, h_q, d]
};
struct AttendPlan {
  int RB, NRB, KPS, S;
  size_t cs_bytes, part_o_bytes, part_ml_bytes, ctr_bytes;
};
AttendPlan attend_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L, int sms);
cudaError_t launch_attend(AttendParams p, int dtype, double rope_base, int pos0, cudaStream_t st);

// api.cu: theta_i / (2 pi) mod 1 as 64-bit binary fractions, theta_i = base^(-2i/d), for
// i < d/2 (all zero when base <= 0)
void rope_turns(double base, int d, unsigned long long* out);

// tmap.cu: bf16 tensor map of a rank-dimensional array (dims innermost first, strides[rank-1]
// in bytes, box in elements; zero fill out of bounds), no swizzle or the 128-byte swizzle
bool encode_bf16_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, bool swizzle128);

// ---- attend_dec.cu: decode-shaped attention (bf16, d = 128, <= 8 query rows per KV head,
// h_kv in {1, 2, 4, 8})
struct DecParams {
  const __nv_bfloat16* Q;   // [B, T, h_q, 128]
  const __nv_bfloat16* Kl;  // [B, Ls, h_kv, 128], the first L rows of each query used
  const __nv_bfloat16* Vl;
  const __nv_bfloat16* cK;  // [B, max_ctx, h_kv, 128]
  const __nv_bfloat16* cV;
  const int32_t* ctx_len;
  int B, T, h_q, h_kv, L, max_ctx;
  int Ls;                   // local rows stored per query (row stride of Kl / Vl), >= L
  const int32_t* L_dev;     // nullable: the local length is read from here at run time
  int skip_on_err;          // write nothing if the status word already holds an error
  int start_status;         // the first CTA starts the status word (the call's first kernel;
                            // another CTA records an error only after a bounded wait has run
                            // out, long after every CTA started)
  int keys_rotated;         // local keys are stored rotated at their positions pos0 + j
  int rope, pos0;
  unsigned long long rope_turns[64];  // theta_i / (2 pi) mod 1 as 64-bit binary fractions,
                                      // theta_i = base^(-2i/128); all zero without RoPE
  float scale_log2;
  int CT, max_seg;          // tiles of 64/h_kv memory rows per query (the local tiles follow;
                            // the kernels count them from the live length); partial slots
                            // per query
  int grid;                 // CTAs of the attention kernel (tile ranges)
  float* part_o;            // [B, max_seg, h_kv, RB, 128]
  float* part_ml;           // [B, max_seg, h_kv, RB, 2]
  int* err;                 // workspace status word
  __nv_bfloat16* O;         // [B, T, h_q, 128]
  // decode step with the append fused in (16-warp kernel, L_dev set, keys_rotated): the T new
  // tokens' K/V [B, T, h_kv, 128] become local rows L_dev..L_dev+T-1, K rotated at pos0 + row;
  // the attention kernel writes them into Kl/Vl (and into the tiles it attends), starts the
  // status word and leaves the new length (-1 on overflow) in L_out; the merge kernel then
  // stores that length into L_dev
  const __nv_bfloat16* K_new;  // nullable: no fused append
  const __nv_bfloat16* V_new;
  int* L_out;
};
struct DecPlan {
  bool ok;
  int RB, TPP, CT, grid, max_seg;
  int NS;                   // stages of the 8-warp kernel's copy ring (4, or 6 when h_kv = 8)
  int64_t n_pairs, total;   // n_pairs: queries that own tiles (B)
  size_t ctr_bytes, part_ml_bytes, part_o_bytes, smem;
};
DecPlan attend_dec_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L, int sms);
DecPlan attend_dec_plan_cap(int B, int T, int h_q, int h_kv, int d, int max_ctx, int cap, int sms);
cudaError_t launch_attend_dec(const DecParams& p, const DecPlan& pl, cudaStream_t st);
// attend_dec_plain.cu: the same attention when every key is used as stored (rotated cache or
// no RoPE), 16 compute warps
size_t attend_dec_plain_smem(int RB);
cudaError_t launch_attend_dec_plain(const DecParams& p, const DecPlan& pl, const CUtensorMap& mkc,
                                    const CUtensorMap& mvc, const CUtensorMap& mkl,
                                    const CUtensorMap& mvl, cudaStream_t st);

// ---- encode_hidden.cu: projections of hidden states fused with doc-wise RoPE + pooling
struct EhParams {
  int64_t n_chunks, n_units;   // units = ceil(n_chunks / 2) x 3 projections x n_tiles
  int n_tiles;                 // head pairs: h_kv / 2
  int D, h_kv;                 // hidden size (multiple of 64), KV heads (even); d = 128
  const int32_t* ctab;         // [n_chunks][3]: first token row, valid rows, position of the
                               // first row within its document
  int rope;
  unsigned long long rope_turns[64];  // theta_i / (2 pi) mod 1, 64-bit fixed point
  __nv_bfloat16* Kbar;         // [n_chunks, h_kv, 128]
  __nv_bfloat16* Vbar;
  __nv_bfloat16* Kbar_r;
  int* err;                    // workspace status word
};
size_t encode_hidden_smem();
cudaError_t launch_encode_hidden(const EhParams& p, const void* H, int64_t n_tok,
                                 const void* Wk, const void* Wv, const void* Wr, int sms,
                                 cudaStream_t st);

// ---- assemble.cu: local context of a Memory Interleaving round
struct AssembleParams {
  int B, n_seg, T;
  int64_t L;                  // local rows per query: sum of the segment lengths + T
  int64_t row_bytes;          // h_kv * d * element size (multiple of 16)
  const void* const* seg_k;   // [B * n_seg] device pointers, each [seg_len, h_kv, d]
  const void* const* seg_v;
  const int32_t* seg_len;     // [B * n_seg]
  const void* K_q;            // [B, T, h_kv, d]
  const void* V_q;
  void* K_out;                // [B, L, h_kv, d]
  void* V_out;
  int* err;                   // workspace status word
};
// Sparse generation: rows [len, len + T_new) of every query's local cache <- the new tokens'
// K/V, then len += T_new (len read on the device)
struct AppendParams {
  int B, T_new, cap;
  int64_t row_bytes;          // h_kv * d * element size, a multiple of 16
  void* K_cache;              // [B, cap, h_kv, d]
  void* V_cache;
  const void* K_new;          // [B, T_new, h_kv, d]
  const void* V_new;
  int32_t* len;               // device, the rows the cache holds (shared by the batch)
  int* err;                   // workspace status word
  unsigned int* ticket;       // zero on entry; the last CTA advances len and resets it
  int single;                 // one CTA: sets the status word itself, needs no ticket
  int rope, pos0;             // keys stored rotated at position pos0 + row (rope != 0)
  unsigned long long rope_turns[64];  // theta_i / (2 pi) mod 1, 64-bit fixed point
  int d;                      // head dim (RoPE pairs i, i + d/2)
  int esize;                  // bytes per element (2: bf16, 4: fp32)
};
cudaError_t launch_kv_append(const AppendParams& p, int sms, cudaStream_t st);

cudaError_t launch_assemble_local(const AssembleParams& p, cudaStream_t st);

// ---- attend_tc.cu: long-query attention on tensor cores (bf16, d = 128, (h_q/h_kv) * T >= 64,
// h_q/h_kv dividing 128)
struct AtcParams {
  const __nv_bfloat16* Q;   // [B, T, h_q, 128]
  const __nv_bfloat16* Kl;  // [B, L, h_kv, 128] (before RoPE)
  const __nv_bfloat16* Vl;
  const __nv_bfloat16* cK;  // [B, max_ctx, h_kv, 128]
  const __nv_bfloat16* cV;
  const int32_t* ctx_len;
  int B, T, h_q, h_kv, L, max_ctx;
  int rope, pos0;
  unsigned long long rope_turns[64];  // theta_i / (2 pi) mod 1 as 64-bit binary fractions
  float scale_log2;
  int* err;                 // workspace status word
  __nv_bfloat16* O;         // [B, T, h_q, 128]
  float* O32;               // nullable: O in fp32 instead of bf16 (the backward's D)
  float* lse;               // nullable: per query row, log2 of the softmax denominator in the
                            // units of scale_log2 * score ([B, h_kv, lse_stride], row
                            // t * (h_q / h_kv) + head within the KV group)
  int lse_stride;
};
struct AtcPlan {
  bool ok;
  int n_qtiles;             // query tiles per (query, KV head)
  // scratch: rotated Q, rotated K (V is read as stored: vl_bytes = vc_bytes = 0)
  size_t q_bytes, k_bytes, vl_bytes, vc_bytes, smem;
};
// any_rows: accept fewer than 64 query rows per KV head (the backward's recompute)
AtcPlan attend_tc_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L,
                       bool any_rows = false);
cudaError_t launch_attend_tc(const AtcParams& p, const AtcPlan& pl, unsigned char* scratch,
                             int sms, cudaStream_t st);

// ---- attend_bwd.cu: backward of the sparse attention on tensor cores (bf16, d = 128,
// h_q / h_kv dividing 64)
struct BwdParams {
  const __nv_bfloat16* Q;   // [B, T, h_q, 128] (before RoPE)
  const __nv_bfloat16* Kl;  // [B, L, h_kv, 128] (before RoPE)
  const __nv_bfloat16* Vl;
  const __nv_bfloat16* cK;  // [B, max_ctx, h_kv, 128]
  const __nv_bfloat16* cV;
  const int32_t* ctx_len;
  const __nv_bfloat16* dO;  // [B, T, h_q, 128]
  int B, T, h_q, h_kv, L, max_ctx;
  int rope, pos0;
  unsigned long long rope_turns[64];
  float scale, scale_log2;
  float* dQ;                // [B, T, h_q, 128] fp32 outputs
  float* dKl;               // [B, L, h_kv, 128]
  float* dVl;
  float* dKc;               // [B, max_ctx, h_kv, 128]
  float* dVc;
  int* err;
};
struct BwdPlan {
  bool ok;
  AtcPlan fwd;              // the forward recompute (rotated Q and K, O, log-sum-exp)
  int Gq, NQT, Rpad, CT, LT;
  size_t fwd_bytes, o_bytes, lse_bytes, dq_bytes, smem;
};
BwdPlan attend_bwd_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L);
cudaError_t launch_attend_bwd(const BwdParams& p, const BwdPlan& pl, unsigned char* scratch,
                              int sms, cudaStream_t st);
cudaError_t launch_scatter_bank_grad(const int32_t* gidx, const int32_t* ctx_len, int B,
                                     int max_ctx, int64_t row_elems, const float* dKc,
                                     const float* dVc, float* dKbar, float* dVbar, int64_t n_chunks,
                                     int* err, int sms, cudaStream_t st);

// ---- aux_loss.cu: auxiliary routing loss over the chunk scores and its gradients
size_t aux_loss_scratch_bytes(int B, int64_t n_chunks);
cudaError_t launch_aux_routing_loss(const void* Q_r, int B, int T, int h_qr, const void* Kbar_r,
                                    int64_t n_chunks, int h_kv, int d, int dtype,
                                    const uint32_t* pos, float tau, float* loss, float* dQ_r,
                                    float* dKbar_r, unsigned char* scratch, int sms,
                                    cudaStream_t st);

}  // namespace msa
