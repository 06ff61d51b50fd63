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
// rows that share one KV head (GQA), ordered token-major. Each warp owns 32-key tiles: the
// tile's key and value rows are staged with coalesced 16-byte loads into padded shared
// memory (all loads in flight at once); then lane = key reads its key row (memory rows as
// stored, local rows rotated in registers with the cos/sin table), dots it with the CTA's
// rotated, pre-scaled query rows (broadcast reads), and the warp updates its running
// max/sum; P·V is accumulated with lane = output dims. Warps are merged in shared memory;
// the last CTA of each (query, KV head, row block) to finish merges the splits.
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

// One warp's 32 key rows (or value rows) of KV head g, staged with coalesced 16-byte loads
// into a shared-memory tile with padded rows (row stride D + 16 / sizeof(T) elements), so
// that one-row-per-lane reads are free of bank conflicts.
template <typename T, int D>
__device__ __forceinline__ void stage_rows(T* tile, const AttendParams& p, const void* ctx_base,
                                           const void* loc_base, int b, int g, int kt, int nk,
                                           int n_ctx, int lane) {
  constexpr int SEG = D * (int)sizeof(T) / 16;       // 16-byte segments per row
  constexpr int RPI = 32 / SEG;                      // rows per warp instruction
  constexpr int PAD = D + 16 / (int)sizeof(T);
  const int64_t W = (int64_t)p.h_kv * D;
#pragma unroll
  for (int it = 0; it < SEG; ++it) {
    const int r = it * RPI + lane / SEG, sg = lane % SEG;
    const int key = kt + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < nk) {
      const T* src = key < n_ctx
          ? static_cast<const T*>(ctx_base) + ((int64_t)b * p.max_ctx + key) * W + (int64_t)g * D
          : static_cast<const T*>(loc_base) + ((int64_t)b * p.L + (key - n_ctx)) * W + (int64_t)g * D;
      v = reinterpret_cast<const uint4*>(src)[sg];
    }
    *reinterpret_cast<uint4*>(tile + r * PAD + sg * (16 / (int)sizeof(T))) = v;
  }
}

template <typename T, int D, int RB>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(AttendParams p) {
  constexpr int HALF = D / 2;
  constexpr int DPL = D / 32;  // output dims per lane
  constexpr int PAD = D + 16 / (int)sizeof(T);
  constexpr int E = 16 / (int)sizeof(T);
  constexpr int kMaxRB = RB;
  using VecT = Vec<T, E>;
  // dynamic shared memory: query rows, then per-warp key/value tiles; after the key loop the
  // tiles are reused for the warp merge
  extern __shared__ __align__(16) unsigned char att_smem[];
  float (*qs)[D] = reinterpret_cast<float (*)[D]>(att_smem);
  T* tiles = reinterpret_cast<T*>(att_smem + sizeof(float) * RB * D);
  float (*wo)[RB][D] = reinterpret_cast<float (*)[RB][D]>(tiles);
  __shared__ float wm[kAttWarps][RB], wl[kAttWarps][RB];
  __shared__ int is_last;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int split = blockIdx.x;
  const int rb = blockIdx.y;
  const int b = blockIdx.z / p.h_kv, g = blockIdx.z % p.h_kv;
  const int G = p.h_q / p.h_kv;
  const int rows_total = G * p.T;
  const int r0 = rb * p.RB;
  const int nr = min(p.RB, rows_total - r0);
  const int n_ctx = min(max(p.ctx_len[b], 0), p.max_ctx);
  const int n_keys = n_ctx + p.L;
  const int ks = split * p.KPS;
  const int t_hi = (r0 + nr - 1) / G;  // last local row any row of this block can see
  const int ke = min(min(ks + p.KPS, n_keys), n_ctx + p.L - p.T + t_hi + 1);

  // rotated, pre-scaled query rows
  for (int idx = threadIdx.x; idx < nr * HALF; idx += blockDim.x) {
    const int rr = idx / HALF, i = idx % HALF;
    const int r = r0 + rr;
    const int t = r / G, h = g * G + r % G;
    const T* q = static_cast<const T*>(p.Q) + (((int64_t)b * p.T + t) * p.h_q + h) * D;
    float x1 = Elem<T>::to_f(q[i]), x2 = Elem<T>::to_f(q[i + HALF]);
    if (p.rope) {
      const float2 c = p.cs[(int64_t)(p.L - p.T + t) * HALF + i];
      const float y1 = x1 * c.x - x2 * c.y, y2 = x2 * c.x + x1 * c.y;
      x1 = y1;
      x2 = y2;
    }
    qs[rr][i] = x1 * p.scale_log2;
    qs[rr][i + HALF] = x2 * p.scale_log2;
  }
  __syncthreads();

  float m[kMaxRB], l[kMaxRB], acc[kMaxRB][DPL];
#pragma unroll
  for (int r = 0; r < kMaxRB; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[r][e] = 0.f;
  }

  T* kt_s = tiles + (size_t)(2 * warp) * 32 * PAD;
  T* vt_s = tiles + (size_t)(2 * warp + 1) * 32 * PAD;
  for (int kt = ks + warp * 32; kt < ke; kt += kAttWarps * 32) {
    const int nk = min(32, ke - kt);
    // both tiles' loads are issued before either is used
    stage_rows<T, D>(kt_s, p, p.cK, p.Kl, b, g, kt, nk, n_ctx, lane);
    stage_rows<T, D>(vt_s, p, p.cV, p.Vl, b, g, kt, nk, n_ctx, lane);
    __syncwarp();
    const int key = kt + lane;
    const bool kin = lane < nk;
    const bool is_ctx = key < n_ctx;
    const int j = key - n_ctx;  // local row (if not memory)
    float s[kMaxRB];
#pragma unroll
    for (int r = 0; r < kMaxRB; ++r) s[r] = 0.f;
    if (kin) {
      const bool rot = !is_ctx && p.rope;
      const float4* csr = reinterpret_cast<const float4*>(p.cs + (int64_t)(rot ? j : 0) * HALF);
      const T* krow = kt_s + lane * PAD;
#pragma unroll 2
      for (int v = 0; v < HALF / E; ++v) {
        float a[E], c[E];
        VecT::unpack(reinterpret_cast<const typename VecT::raw*>(krow)[v], a);
        VecT::unpack(reinterpret_cast<const typename VecT::raw*>(krow + HALF)[v], c);
        if (rot) {
#pragma unroll
          for (int e2 = 0; e2 < E / 2; ++e2) {
            const float4 t2 = __ldg(csr + (v * E) / 2 + e2);  // (cos, sin) of two pairs
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = 2 * e2 + h2;
              const float co = h2 ? t2.z : t2.x, si = h2 ? t2.w : t2.y;
              const float y1 = a[e] * co - c[e] * si, y2 = c[e] * co + a[e] * si;
              a[e] = y1;
              c[e] = y2;
            }
          }
        }
#pragma unroll
        for (int r = 0; r < kMaxRB; ++r) {
          if (r < nr) {
            float acc_r = s[r];
#pragma unroll
            for (int e = 0; e < E; ++e) {
              acc_r = fmaf(qs[r][v * E + e], a[e], acc_r);
              acc_r = fmaf(qs[r][HALF + v * E + e], c[e], acc_r);
            }
            s[r] = acc_r;
          }
        }
      }
    }
    // mask + online softmax per row (base-2 exponent; q was pre-scaled by log2 e)
#pragma unroll
    for (int r = 0; r < kMaxRB; ++r) {
      if (r >= nr) continue;
      const int t = (r0 + r) / G;
      const bool vis = kin && (is_ctx || j <= p.L - p.T + t);
      const float sv = vis ? s[r] : -INFINITY;
      float mx = sv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mn = fmaxf(m[r], mx);
      if (mn == -INFINITY) { s[r] = 0.f; continue; }
      const float pr = vis ? exp2f(sv - mn) : 0.f;
      const float alpha = exp2f(m[r] - mn);
      float ps = pr;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l[r] = l[r] * alpha + ps;
      m[r] = mn;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[r][e] *= alpha;
      s[r] = pr;
    }
    // P V: lane owns DPL consecutive dims; value rows from the staged tile
    using VecV = Vec<T, DPL>;
    for (int kk = 0; kk < nk; ++kk) {
      float vv[DPL];
      VecV::unpack(reinterpret_cast<const typename VecV::raw*>(vt_s + kk * PAD)[lane], vv);
#pragma unroll
      for (int r = 0; r < kMaxRB; ++r) {
        if (r >= nr) continue;
        const float pr = __shfl_sync(0xffffffffu, s[r], kk);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[r][e] = fmaf(pr, vv[e], acc[r][e]);
      }
    }
    __syncwarp();  // the tiles are rewritten by the next iteration
  }

  // merge the warps (the tiles are free once every warp has left the key loop)
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMaxRB; ++r) {
    if (r >= nr) continue;
    if (lane == 0) { wm[warp][r] = m[r]; wl[warp][r] = l[r]; }
#pragma unroll
    for (int e = 0; e < DPL; ++e) wo[warp][r][lane * DPL + e] = acc[r][e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) {
    const int r = idx / D, e = idx % D;
    float mm = -INFINITY;
    for (int w = 0; w < kAttWarps; ++w) mm = fmaxf(mm, wm[w][r]);
    float ll = 0.f, oo = 0.f;
    if (mm != -INFINITY) {
      for (int w = 0; w < kAttWarps; ++w) {
        const float a = exp2f(wm[w][r] - mm);
        ll += wl[w][r] * a;
        oo += wo[w][r][e] * a;
      }
    }
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
  if (threadIdx.x == 0) {
    unsigned int* ctr = p.counters + ((int64_t)blockIdx.z * p.NRB + rb);
    is_last = (atomicInc(ctr, (unsigned)(p.S - 1)) == (unsigned)(p.S - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) {
    const int r = idx / D, e = idx % D;
    const int rr = r0 + r;
    const int t = rr / G, h = g * G + rr % G;
    const int64_t row = ((int64_t)b * p.T + t) * p.h_q + h;
    float mm = -INFINITY;
    for (int sp = 0; sp < p.S; ++sp) mm = fmaxf(mm, __ldcg(p.part_ml + (row * p.S + sp) * 2));
    float ll = 0.f, oo = 0.f;
    if (mm != -INFINITY) {
      for (int sp = 0; sp < p.S; ++sp) {
        const float ms = __ldcg(p.part_ml + (row * p.S + sp) * 2);
        const float a = ms == -INFINITY ? 0.f : exp2f(ms - mm);
        ll += __ldcg(p.part_ml + (row * p.S + sp) * 2 + 1) * a;
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
  pl.KPS = 128;
  const int keys = max_ctx + L;
  const int max_s = (keys + pl.KPS - 1) / pl.KPS;
  const int64_t base = (int64_t)B * h_kv * pl.NRB;
  int64_t want = base > 0 ? ((int64_t)sms * 8 + base - 1) / base : 1;
  if (want > max_s) want = max_s;
  if (want < 1) want = 1;
  pl.S = (int)want;
  pl.KPS = ((keys + pl.S - 1) / pl.S + 127) / 128 * 128;
  if (pl.KPS < 128) pl.KPS = 128;
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
    const size_t sm = sizeof(float) * RR * DD +                                                 \
                      std::max(sizeof(TT) * 2 * kAttWarps * 32 * (DD + 16 / sizeof(TT)),       \
                               sizeof(float) * kAttWarps * RR * DD);                           \
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
