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
// rows that share one KV head (GQA), ordered token-major. Each warp owns 32-key tiles
// (lane = key): the lane reads its key row straight from global memory (16-byte vectors,
// memory rows as stored, local rows rotated in registers with the cos/sin table), dots it
// with the CTA's rotated, pre-scaled query rows (shared memory, broadcast reads), and the
// warp updates its running max/sum; P·V is accumulated with lane = 4 output dims, V rows
// read coalesced. Warps are merged in shared memory; splits are merged by a second kernel
// (or normalised in place when there is a single split).
#include "common.cuh"
#include "kernels.cuh"

namespace msa {

constexpr int kAttThreads = 128;
constexpr int kAttWarps = 4;
constexpr int kMaxRB = 8;

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

template <typename T, int D>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(AttendParams p) {
  constexpr int HALF = D / 2;
  constexpr int DPL = D / 32;  // output dims per lane
  __shared__ __align__(16) float qs[kMaxRB][D];
  __shared__ float wm[kAttWarps][kMaxRB], wl[kAttWarps][kMaxRB];
  __shared__ __align__(16) float wo[kAttWarps][kMaxRB][D];

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
  // last local row any row of this block can see
  const int t_hi = (r0 + nr - 1) / G;
  const int ke = min(min(ks + p.KPS, n_keys), n_ctx + p.L - p.T + t_hi + 1);
  const int64_t W = (int64_t)p.h_kv * D;

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

  for (int kt = ks + warp * 32; kt < ke; kt += kAttWarps * 32) {
    const int key = kt + lane;
    const bool kin = key < ke;
    const bool is_ctx = key < n_ctx;
    const int j = key - n_ctx;  // local row (if not memory)
    const T* krow = nullptr;
    if (kin) {
      krow = is_ctx ? static_cast<const T*>(p.cK) + ((int64_t)b * p.max_ctx + key) * W + (int64_t)g * D
                    : static_cast<const T*>(p.Kl) + ((int64_t)b * p.L + j) * W + (int64_t)g * D;
    }
    // logits for this lane's key against every row
    float s[kMaxRB];
#pragma unroll
    for (int r = 0; r < kMaxRB; ++r) s[r] = 0.f;
    if (kin) {
      constexpr int E = 16 / sizeof(T);
      using VecT = Vec<T, E>;
      const bool rot = !is_ctx && p.rope;
      const float2* csr = p.cs + (int64_t)(rot ? j : 0) * HALF;
#pragma unroll 2
      for (int v = 0; v < HALF / E; ++v) {
        float a[E], c[E];
        VecT::unpack(reinterpret_cast<const typename VecT::raw*>(krow)[v], a);
        VecT::unpack(reinterpret_cast<const typename VecT::raw*>(krow + HALF)[v], c);
        if (rot) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float2 t = csr[v * E + e];
            const float y1 = a[e] * t.x - c[e] * t.y, y2 = c[e] * t.x + a[e] * t.y;
            a[e] = y1;
            c[e] = y2;
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
    // P V: lane owns DPL consecutive dims
    const int nk = min(32, ke - kt);
    for (int kk = 0; kk < nk; ++kk) {
      const int key2 = kt + kk;
      const T* vrow = key2 < n_ctx
          ? static_cast<const T*>(p.cV) + ((int64_t)b * p.max_ctx + key2) * W + (int64_t)g * D
          : static_cast<const T*>(p.Vl) + ((int64_t)b * p.L + (key2 - n_ctx)) * W + (int64_t)g * D;
      float vv[DPL];
      using VecV = Vec<T, DPL>;
      VecV::unpack(reinterpret_cast<const typename VecV::raw*>(vrow)[lane], vv);
#pragma unroll
      for (int r = 0; r < kMaxRB; ++r) {
        if (r >= nr) continue;
        const float pr = __shfl_sync(0xffffffffu, s[r], kk);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[r][e] = fmaf(pr, vv[e], acc[r][e]);
      }
    }
  }

  // merge the warps
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
}

template <typename T>
__global__ void attend_combine_kernel(AttendParams p) {
  const int64_t row = blockIdx.x;
  const int D = p.d;
  float mm = -INFINITY;
  for (int s = 0; s < p.S; ++s) mm = fmaxf(mm, p.part_ml[(row * p.S + s) * 2]);
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float ll = 0.f, oo = 0.f;
    if (mm != -INFINITY) {
      for (int s = 0; s < p.S; ++s) {
        const float ms = p.part_ml[(row * p.S + s) * 2];
        const float a = ms == -INFINITY ? 0.f : exp2f(ms - mm);
        ll += p.part_ml[(row * p.S + s) * 2 + 1] * a;
        oo += p.part_o[(row * p.S + s) * D + e] * a;
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
  pl.RB = rows < kMaxRB ? rows : kMaxRB;
  if (pl.RB < 1) pl.RB = 1;
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
  dim3 grid(p.S, p.NRB, p.B * p.h_kv);
  if (dtype == 1) {
    if (p.d == 128) attend_kernel<__nv_bfloat16, 128><<<grid, kAttThreads, 0, st>>>(p);
    else attend_kernel<__nv_bfloat16, 64><<<grid, kAttThreads, 0, st>>>(p);
  } else {
    if (p.d == 128) attend_kernel<float, 128><<<grid, kAttThreads, 0, st>>>(p);
    else attend_kernel<float, 64><<<grid, kAttThreads, 0, st>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.S == 1) return e;
  const int64_t rows = (int64_t)p.B * p.T * p.h_q;
  if (dtype == 1) attend_combine_kernel<__nv_bfloat16><<<(unsigned)rows, 128, 0, st>>>(p);
  else attend_combine_kernel<float><<<(unsigned)rows, 128, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace msa
