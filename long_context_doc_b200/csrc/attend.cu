// attend.cu - sparse attention of MSA over [gathered memory ; causal local context] with
// global RoPE on the active context.
//
// Method: after routing, the compressed K/V of the selected documents are concatenated with
// the query's local K/V and used for autoregressive decoding
//   [news.neo-ai.one article, "全体設計 / アーキテクチャ" and "推論パイプライン"]; the active
// context uses "global RoPE": the query's start index is shifted by k, the number of Top-k
// retrieved blocks, so the causal order is background -> query -> generation
//   [news.neo-ai.one, "グローバル RoPE（アクティブコンテキスト）"; ai-papers.net summary,
//    "MSAの提案手法"].
//
// Kernel: split-K flash attention on CUDA cores (fp32 accumulation, online softmax).
// CTA = (key split, row block, batch x KV head); the rows of a CTA are RB of the G x T query
// rows that share one KV head (GQA), ordered token-major. Per 64-key tile, every load is in
// flight at once (key and value rows by cp.async, the RoPE pairs of the local keys by
// coalesced loads); the local keys are rotated once per CTA into an fp32 tile; logits,
// the online softmax and P·V then run from shared memory (two lanes per key for the logits,
// one thread per output dim for P·V). The last CTA of each (query, KV head, row block) to
// finish merges the splits.
#include "common.cuh"
#include "kernels.cuh"

#include <algorithm>

namespace msa {

constexpr int kAttThreads = 128;
constexpr int kAttWarps = 4;

// cos/sin table for positions pos0 .. pos0 + L - 1 (double-precision angles and sincos).
__global__ void rope_table_kernel(float2* cs, int L, int d, int pos0, double base) {
  const int half = d / 2;
  const int64_t n = (int64_t)L * half;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(idx / half), i = (int)(idx % half);
    const double theta = pow(base, -2.0 * (double)i / (double)d);
    double s, c;
    sincos((double)(pos0 + j) * theta, &s, &c);
    cs[idx] = make_float2((float)c, (float)s);
  }
}

// cp.async (16 bytes, L2 only) global -> shared
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

constexpr int kAttKT = 64;  // keys per tile

template <typename T, int D, int RB>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(AttendParams p) {
  constexpr int HALF = D / 2;
  constexpr int KP = D + 4;                          // padded fp32 key row
  constexpr int VEC = 16 / (int)sizeof(T);           // elements per 16-byte copy
  constexpr int PAIRS = kAttKT * HALF / kAttThreads;  // RoPE pairs per thread per tile
  constexpr int KPB = kAttThreads / D;               // key phases of the P.V step (1 or 2)
  extern __shared__ __align__(16) unsigned char att_smem[];
  T* kraw = reinterpret_cast<T*>(att_smem);                               // [KT][D]
  T* vraw = kraw + kAttKT * D;                                            // [KT][D]
  float* krot = reinterpret_cast<float*>(vraw + kAttKT * D);              // [KT][KP]
  float* qs = krot + kAttKT * KP;                                         // [RB][D]
  float* ps = qs + RB * D;                                                // [RB][KT]
  float* rowm = ps + RB * kAttKT;                                         // [RB] running max
  float* rowl = rowm + RB;                                                // [RB] running sum
  float* rowa = rowl + RB;                                                // [RB] rescale
  __shared__ int is_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x;
  const int rb = blockIdx.y;
  const int b = blockIdx.z / p.h_kv, g = blockIdx.z % p.h_kv;
  const int G = p.h_q / p.h_kv;
  const int rows_total = G * p.T;
  const int r0 = rb * RB;
  const int nr = min(RB, rows_total - r0);
  const int n_ctx = min(max(p.ctx_len[b], 0), p.max_ctx);
  const int n_keys = n_ctx + p.L;
  const int ks = split * p.KPS;
  const int t_hi = (r0 + nr - 1) / G;  // last local row any row of this block can see
  const int ke = min(min(ks + p.KPS, n_keys), n_ctx + p.L - p.T + t_hi + 1);
  const int64_t W = (int64_t)p.h_kv * D;

  // rotated, pre-scaled query rows; running softmax state
  for (int idx = tid; idx < RB * HALF; idx += kAttThreads) {
    const int rr = idx / HALF, i = idx % HALF;
    float x1 = 0.f, x2 = 0.f;
    if (rr < nr) {
      const int r = r0 + rr;
      const int t = r / G, h = g * G + r % G;
      const T* q = static_cast<const T*>(p.Q) + (((int64_t)b * p.T + t) * p.h_q + h) * D;
      x1 = Elem<T>::to_f(q[i]);
      x2 = Elem<T>::to_f(q[i + HALF]);
      if (p.rope) {
        const float2 c = p.cs[(int64_t)(p.L - p.T + t) * HALF + i];
        const float y1 = x1 * c.x - x2 * c.y, y2 = x2 * c.x + x1 * c.y;
        x1 = y1;
        x2 = y2;
      }
    }
    qs[rr * D + i] = x1 * p.scale_log2;
    qs[rr * D + i + HALF] = x2 * p.scale_log2;
  }
  if (tid < RB) { rowm[tid] = -INFINITY; rowl[tid] = 0.f; }

  const int e_own = tid % D;       // output dim of this thread in the P.V step
  const int kph = tid / D;         // key phase of this thread in the P.V step
  float acc[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) acc[r] = 0.f;

  for (int kt = ks; kt < ke; kt += kAttKT) {
    const int nk = min(kAttKT, ke - kt);
    // 1. all loads of the tile in flight at once: K and V rows (cp.async) and RoPE pairs
    for (int idx = tid; idx < nk * (D / VEC); idx += kAttThreads) {
      const int j = idx / (D / VEC), sg = idx % (D / VEC);
      const int key = kt + j;
      const T* ks_src = key < n_ctx
          ? static_cast<const T*>(p.cK) + ((int64_t)b * p.max_ctx + key) * W + (int64_t)g * D
          : static_cast<const T*>(p.Kl) + ((int64_t)b * p.L + (key - n_ctx)) * W + (int64_t)g * D;
      const T* vs_src = key < n_ctx
          ? static_cast<const T*>(p.cV) + ((int64_t)b * p.max_ctx + key) * W + (int64_t)g * D
          : static_cast<const T*>(p.Vl) + ((int64_t)b * p.L + (key - n_ctx)) * W + (int64_t)g * D;
      cp_async16(kraw + j * D + sg * VEC, ks_src + sg * VEC);
      cp_async16(vraw + j * D + sg * VEC, vs_src + sg * VEC);
    }
    float2 cs[PAIRS];
#pragma unroll
    for (int q = 0; q < PAIRS; ++q) {
      const int idx = q * kAttThreads + tid;
      const int j = idx / HALF, i = idx % HALF;
      const int key = kt + j;
      cs[q] = make_float2(1.f, 0.f);
      if (p.rope && j < nk && key >= n_ctx) cs[q] = __ldg(p.cs + (int64_t)(key - n_ctx) * HALF + i);
    }
    cp_async_wait_all();
    __syncthreads();
    // 2. rotate the local keys once (memory rows pass through), fp32
#pragma unroll
    for (int q = 0; q < PAIRS; ++q) {
      const int idx = q * kAttThreads + tid;
      const int j = idx / HALF, i = idx % HALF;
      float y1 = 0.f, y2 = 0.f;
      if (j < nk) {
        const float a = Elem<T>::to_f(kraw[j * D + i]), c = Elem<T>::to_f(kraw[j * D + i + HALF]);
        y1 = a * cs[q].x - c * cs[q].y;
        y2 = c * cs[q].x + a * cs[q].y;
      }
      krot[j * KP + i] = y1;
      krot[j * KP + i + HALF] = y2;
    }
    __syncthreads();
    // 3. logits: two lanes per key (half the dims each), 16 keys per warp
    {
      const int j = warp * 16 + (lane & 15);
      const int hh = lane >> 4;
      float s[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) s[r] = 0.f;
      const float4* kr4 = reinterpret_cast<const float4*>(krot + j * KP + hh * HALF);
#pragma unroll 4
      for (int v = 0; v < HALF / 4; ++v) {
        const float4 kv = kr4[v];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const float4 qv = reinterpret_cast<const float4*>(qs + r * D + hh * HALF)[v];
          s[r] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, s[r]))));
        }
      }
      const int key = kt + j;
      const bool kin = j < nk;
      const bool is_ctx = key < n_ctx;
      const int jl = key - n_ctx;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        s[r] += __shfl_xor_sync(0xffffffffu, s[r], 16);
        const int t = (r0 + r) / G;
        const bool vis = kin && r < nr && (is_ctx || jl <= p.L - p.T + t);
        if (hh == 0) ps[r * kAttKT + j] = vis ? s[r] : -INFINITY;
      }
    }
    __syncthreads();
    // 4. online softmax: warp w owns rows w, w + 4, ...
    for (int r = warp; r < RB; r += kAttWarps) {
      const float a0 = ps[r * kAttKT + lane], a1 = ps[r * kAttKT + lane + 32];
      float mx = fmaxf(a0, a1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mo = rowm[r];
      const float mn = fmaxf(mo, mx);
      float p0 = 0.f, p1 = 0.f, alpha = 1.f;
      if (mn != -INFINITY) {
        p0 = a0 == -INFINITY ? 0.f : exp2f(a0 - mn);
        p1 = a1 == -INFINITY ? 0.f : exp2f(a1 - mn);
        alpha = mo == -INFINITY ? 0.f : exp2f(mo - mn);
      }
      float sum = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      ps[r * kAttKT + lane] = p0;
      ps[r * kAttKT + lane + 32] = p1;
      if (lane == 0) {
        rowl[r] = rowl[r] * alpha + sum;
        rowm[r] = mn;
        rowa[r] = alpha;
      }
    }
    __syncthreads();
    // 5. P.V: thread owns one output dim (and a key phase when D < 128)
#pragma unroll
    for (int r = 0; r < RB; ++r) acc[r] *= rowa[r];
    for (int j = kph; j < nk; j += KPB) {
      const float v = Elem<T>::to_f(vraw[j * D + e_own]);
#pragma unroll
      for (int r = 0; r < RB; ++r) acc[r] = fmaf(ps[r * kAttKT + j], v, acc[r]);
    }
    __syncthreads();  // the tiles are rewritten by the next iteration
  }

  // combine the key phases (D < 128), then write this split's partial or the output
  float* part = krot;  // free after the loop: [KPB][RB][D]
#pragma unroll
  for (int r = 0; r < RB; ++r) part[(kph * RB + r) * D + e_own] = acc[r];
  __syncthreads();
  for (int idx = tid; idx < nr * D; idx += kAttThreads) {
    const int r = idx / D, e = idx % D;
    float oo = 0.f;
    for (int k2 = 0; k2 < KPB; ++k2) oo += part[(k2 * RB + r) * D + e];
    const float mm = rowm[r], ll = rowl[r];
    const int rr = r0 + r;
    const int t = rr / G, h = g * G + rr % G;
    const int64_t row = ((int64_t)b * p.T + t) * p.h_q + h;
    if (p.S == 1) {
      static_cast<T*>(p.O)[row * D + e] = Elem<T>::from_f(ll > 0.f ? oo / ll : 0.f);
    } else {
      p.part_o[(row * p.S + split) * D + e] = oo;
      if (e == 0) {
        p.part_ml[(row * p.S + split) * 2 + 0] = mm;
        p.part_ml[(row * p.S + split) * 2 + 1] = ll;
      }
    }
  }
  if (p.S == 1) return;
  // the last split CTA of this (query, KV head, row block) merges the splits
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    unsigned int* ctr = p.counters + ((int64_t)blockIdx.z * p.NRB + rb);
    is_last = (atomicInc(ctr, (unsigned)(p.S - 1)) == (unsigned)(p.S - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int idx = tid; idx < nr * D; idx += kAttThreads) {
    const int r = idx / D, e = idx % D;
    const int rr = r0 + r;
    const int t = rr / G, h = g * G + rr % G;
    const int64_t row = ((int64_t)b * p.T + t) * p.h_q + h;
    float mm = -INFINITY;
#pragma unroll 8
    for (int sp = 0; sp < p.S; ++sp) mm = fmaxf(mm, __ldcg(p.part_ml + (row * p.S + sp) * 2));
    float ll = 0.f, oo = 0.f;
    if (mm != -INFINITY) {
#pragma unroll 8
      for (int sp = 0; sp < p.S; ++sp) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (row * p.S + sp) * 2));
        const float a = ml.x == -INFINITY ? 0.f : exp2f(ml.x - mm);
        ll += ml.y * a;
        oo += __ldcg(p.part_o + (row * p.S + sp) * D + e) * a;
      }
    }
    static_cast<T*>(p.O)[row * D + e] = Elem<T>::from_f(ll > 0.f ? oo / ll : 0.f);
  }
}

// ------------------------------------------------------------------------------ planning

AttendPlan attend_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L, int sms) {
  AttendPlan pl{};
  const int G = h_q / h_kv;
  const int rows = G * T;
  pl.RB = rows >= 8 ? 8 : rows >= 4 ? 4 : rows >= 2 ? 2 : 1;
  pl.NRB = (rows + pl.RB - 1) / pl.RB;
  pl.KPS = 64;
  const int keys = max_ctx + L;
  const int max_s = (keys + pl.KPS - 1) / pl.KPS;
  const int64_t base = (int64_t)B * h_kv * pl.NRB;
  int64_t want = base > 0 ? ((int64_t)sms * 12 + base - 1) / base : 1;
  if (want > max_s) want = max_s;
  if (want < 1) want = 1;
  pl.S = (int)want;
  pl.KPS = ((keys + pl.S - 1) / pl.S + 63) / 64 * 64;
  if (pl.KPS < 64) pl.KPS = 64;
  pl.S = (keys + pl.KPS - 1) / pl.KPS;
  if (pl.S < 1) pl.S = 1;
  pl.cs_bytes = ((size_t)L * (d / 2) * sizeof(float2) + 255) & ~(size_t)255;
  const size_t nrow = (size_t)B * T * h_q;
  pl.part_o_bytes = pl.S > 1 ? ((nrow * pl.S * d * sizeof(float) + 255) & ~(size_t)255) : 0;
  pl.part_ml_bytes = pl.S > 1 ? ((nrow * pl.S * 2 * sizeof(float) + 255) & ~(size_t)255) : 0;
  pl.ctr_bytes = pl.S > 1 ? (((size_t)B * h_kv * pl.NRB * sizeof(unsigned int) + 255) & ~(size_t)255) : 0;
  return pl;
}

cudaError_t launch_attend(AttendParams p, int dtype, double rope_base, int pos0,
                          cudaStream_t st) {
  if (p.rope) {
    const int64_t n = (int64_t)p.L * (p.d / 2);
    int grid = (int)((n + 255) / 256);
    if (grid > 4096) grid = 4096;
    if (grid < 1) grid = 1;
    rope_table_kernel<<<grid, 256, 0, st>>>(const_cast<float2*>(p.cs), p.L, p.d, pos0, rope_base);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.S > 1) {  // split-merge tickets of the last-CTA combine
    cudaError_t e = cudaMemsetAsync(p.counters, 0, sizeof(unsigned int) * (size_t)p.B * p.h_kv * p.NRB, st);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.S, p.NRB, p.B * p.h_kv);
  cudaError_t e = cudaSuccess;
#define MSA_ATT(TT, DD, RR)                                                                    \
  {                                                                                            \
    const size_t sm = sizeof(TT) * 2 * kAttKT * DD + sizeof(float) * kAttKT * (DD + 4) +         \
                      sizeof(float) * (RR * DD + RR * kAttKT + 3 * RR);                         \
    auto kf = attend_kernel<TT, DD, RR>;                                                       \
    e = cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);        \
    if (e == cudaSuccess) kf<<<grid, kAttThreads, sm, st>>>(p);                               \
  }
#define MSA_ATT_RB(TT, DD)                                                                     \
  switch (p.RB) {                                                                              \
    case 1: MSA_ATT(TT, DD, 1) break;                                                          \
    case 2: MSA_ATT(TT, DD, 2) break;                                                          \
    case 4: MSA_ATT(TT, DD, 4) break;                                                          \
    default: MSA_ATT(TT, DD, 8) break;                                                         \
  }
  if (dtype == 1) {
    if (p.d == 128) { MSA_ATT_RB(__nv_bfloat16, 128) } else { MSA_ATT_RB(__nv_bfloat16, 64) }
  } else {
    if (p.d == 128) { MSA_ATT_RB(float, 128) } else { MSA_ATT_RB(float, 64) }
  }
#undef MSA_ATT_RB
#undef MSA_ATT
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace msa
