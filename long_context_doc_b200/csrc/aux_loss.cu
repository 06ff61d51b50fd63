// aux_loss.cu - the auxiliary routing loss of MSA training and its gradients with respect to
// the router queries and the router-key bank.
//
// MSA trains its router with an auxiliary loss next to the generation loss, described as a
// supervised contrastive loss that separates the chunks of relevant documents from those of
// irrelevant ones [ruixiangma.github.io blog, "训练策略"]. The pages give no formula; the reading
// implemented here (the same as the oracle's) works on the routing scan's chunk scores before
// the document maximum,
//   s[b, c] = max_t (1/h_qr) sum_h cos(Q_r[b, t, h], Kbar_r[c, g(h)]),  g(h) = h / (h_qr/h_kv),
// with the positives P_b = the chunks marked relevant for query b:
//   loss_b = -(1/|P_b|) sum_{c in P_b} log softmax_c(s[b, :] / tau),
//   loss   = mean of loss_b over the queries with at least one positive.
// The maximum over tokens passes its gradient to the first maximising token t*(b, c); the
// cosine's gradients are d cos / d q = (k^ - cos q^) / |q| and symmetrically for k (zero vectors
// have cosine 0 and no gradient).
//
// Kernels (CUDA cores; the scores are cosines of short row sets, gathered per warp):
//  * scores: warp per (chunk, query): for every token and router head the cosine by warp dot
//    products, head mean, max over tokens and its first argmax;
//  * loss: one block; per query the log-sum-exp over the chunks and the positives' mean,
//    the loss, and dL/ds[b, c] = (softmax - [c in P_b] / |P_b|) / (tau * n_rows);
//  * dKbar_r: warp per (chunk, KV head); dQ_r: warp per (query, token, router head), gathering
//    the chunks whose maximum sits at that token (deterministic, no atomics).
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace aux {

constexpr int kD = 128;  // largest head dim; lanes hold d / 32 elements

template <typename T>
__device__ __forceinline__ void load_row(const T* src, int d, int lane, float* x) {
#pragma unroll
  for (int j = 0; j < kD / 32; ++j) {
    const int e = lane + 32 * j;
    x[j] = e < d ? Elem<T>::to_f(src[e]) : 0.f;
  }
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct Args {
  const void* Q;      // [B, T, h_qr, d]
  const void* K;      // [n_chunks, h_kv, d]
  const uint32_t* pos;  // [B, words]
  int64_t n_chunks, words;
  int B, T, h_qr, h_kv, d;
  float tau;
  float* s;           // [B, n_chunks]
  int32_t* tstar;     // [B, n_chunks]
  float* ds;          // [B, n_chunks]
  float* loss;        // [1]
  float* dQ;          // nullable [B, T, h_qr, d]
  float* dK;          // nullable [n_chunks, h_kv, d]
};

template <typename T>
__global__ void __launch_bounds__(256) scores_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const T* Q = static_cast<const T*>(a.Q);
  const T* K = static_cast<const T*>(a.K);
  const int m = a.h_qr / a.h_kv;
  for (int64_t i = w; i < a.n_chunks * a.B; i += nw) {
    const int64_t c = i / a.B;
    const int b = (int)(i % a.B);
    float best = -INFINITY;
    int bt = 0;
    for (int t = 0; t < a.T; ++t) {
      float acc = 0.f;
      for (int h = 0; h < a.h_qr; ++h) {
        float q[kD / 32], k[kD / 32];
        load_row(Q + (((int64_t)b * a.T + t) * a.h_qr + h) * a.d, a.d, lane, q);
        load_row(K + (c * a.h_kv + h / m) * a.d, a.d, lane, k);
        float qq = 0.f, kk = 0.f, qk = 0.f;
#pragma unroll
        for (int j = 0; j < kD / 32; ++j) {
          qq += q[j] * q[j];
          kk += k[j] * k[j];
          qk += q[j] * k[j];
        }
        qq = warp_sum(qq);
        kk = warp_sum(kk);
        qk = warp_sum(qk);
        acc += (qq > 0.f && kk > 0.f) ? qk / (sqrtf(qq) * sqrtf(kk)) : 0.f;
      }
      const float st = acc / (float)a.h_qr;
      if (st > best) {  // the first maximising token keeps the gradient
        best = st;
        bt = t;
      }
    }
    if (lane == 0) {
      a.s[(int64_t)b * a.n_chunks + c] = best;
      a.tstar[(int64_t)b * a.n_chunks + c] = bt;
    }
  }
}

// One block: per query the log-sum-exp over the chunks (two passes), the positives, the loss
// and dL/ds. Block-wide reductions through shared memory.
__global__ void __launch_bounds__(1024) loss_kernel(Args a) {
  __shared__ float red[32];
  __shared__ float bc[4];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  auto block_reduce = [&](float v, bool is_max) -> float {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float x = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, x) : v + x;
    }
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
      v = lane < nwarps ? red[lane] : (is_max ? -INFINITY : 0.f);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float x = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmaxf(v, x) : v + x;
      }
      if (lane == 0) bc[0] = v;
    }
    __syncthreads();
    const float r = bc[0];
    __syncthreads();
    return r;
  };
  const float inv_tau = 1.0f / a.tau;
  // rows with positives
  int n_rows = 0;
  for (int b = 0; b < a.B; ++b) {
    float cnt = 0.f;
    for (int64_t j = tid; j < a.words; j += blockDim.x) cnt += (float)__popc(a.pos[b * a.words + j]);
    n_rows += block_reduce(cnt, false) > 0.f ? 1 : 0;
  }
  float total = 0.f;
  for (int b = 0; b < a.B; ++b) {
    const float* s = a.s + (int64_t)b * a.n_chunks;
    const uint32_t* P = a.pos + (int64_t)b * a.words;
    float mx = -INFINITY;
    for (int64_t c = tid; c < a.n_chunks; c += blockDim.x) mx = fmaxf(mx, s[c] * inv_tau);
    mx = block_reduce(mx, true);
    float se = 0.f, ps = 0.f, pc = 0.f;
    for (int64_t c = tid; c < a.n_chunks; c += blockDim.x) {
      const float z = s[c] * inv_tau;
      se += expf(z - mx);
      if ((P[c >> 5] >> (c & 31)) & 1u) {
        ps += z;
        pc += 1.f;
      }
    }
    se = block_reduce(se, false);
    ps = block_reduce(ps, false);
    pc = block_reduce(pc, false);
    const float lse = mx + logf(se);
    if (pc > 0.f) total += lse - ps / pc;
    for (int64_t c = tid; c < a.n_chunks; c += blockDim.x) {
      float g = 0.f;
      if (pc > 0.f) {
        const float p = expf(s[c] * inv_tau - lse);
        const float y = ((P[c >> 5] >> (c & 31)) & 1u) ? 1.f / pc : 0.f;
        g = (p - y) * inv_tau / (float)n_rows;
      }
      a.ds[(int64_t)b * a.n_chunks + c] = g;
    }
  }
  if (tid == 0) *a.loss = n_rows > 0 ? total / (float)n_rows : 0.f;
}

// dKbar_r[c, g] = sum_b (ds[b, c] / h_qr) sum_{h in g} (q^ - cos k^) / |k|, q = Q_r[b, t*(b, c), h]
template <typename T>
__global__ void __launch_bounds__(256) grad_k_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const T* Q = static_cast<const T*>(a.Q);
  const T* K = static_cast<const T*>(a.K);
  const int m = a.h_qr / a.h_kv;
  for (int64_t i = w; i < a.n_chunks * a.h_kv; i += nw) {
    const int64_t c = i / a.h_kv;
    const int g = (int)(i % a.h_kv);
    float k[kD / 32], acc[kD / 32] = {};
    load_row(K + (c * a.h_kv + g) * a.d, a.d, lane, k);
    float kk = 0.f;
#pragma unroll
    for (int j = 0; j < kD / 32; ++j) kk += k[j] * k[j];
    kk = warp_sum(kk);
    if (kk > 0.f) {
      const float kn = sqrtf(kk), ik = 1.f / kn;
      for (int b = 0; b < a.B; ++b) {
        const float gs = a.ds[(int64_t)b * a.n_chunks + c] / (float)a.h_qr;
        if (gs == 0.f) continue;
        const int t = a.tstar[(int64_t)b * a.n_chunks + c];
        for (int hm = 0; hm < m; ++hm) {
          float q[kD / 32];
          load_row(Q + (((int64_t)b * a.T + t) * a.h_qr + g * m + hm) * a.d, a.d, lane, q);
          float qq = 0.f, qk = 0.f;
#pragma unroll
          for (int j = 0; j < kD / 32; ++j) {
            qq += q[j] * q[j];
            qk += q[j] * k[j];
          }
          qq = warp_sum(qq);
          qk = warp_sum(qk);
          if (qq <= 0.f) continue;
          const float iq = 1.f / sqrtf(qq);
          const float cs = qk * iq * ik;
#pragma unroll
          for (int j = 0; j < kD / 32; ++j) acc[j] += gs * (q[j] * iq - cs * k[j] * ik) * ik;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kD / 32; ++j) {
      const int e = lane + 32 * j;
      if (e < a.d) a.dK[(c * a.h_kv + g) * a.d + e] = acc[j];
    }
  }
}

// dQ_r[b, t, h] = sum_{c: t*(b, c) = t} (ds[b, c] / h_qr) (k^ - cos q^) / |q|, k = Kbar_r[c, g(h)]
template <typename T>
__global__ void __launch_bounds__(256) grad_q_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const T* Q = static_cast<const T*>(a.Q);
  const T* K = static_cast<const T*>(a.K);
  const int m = a.h_qr / a.h_kv;
  const int64_t rows = (int64_t)a.B * a.T * a.h_qr;
  for (int64_t i = w; i < rows; i += nw) {
    const int h = (int)(i % a.h_qr);
    const int t = (int)((i / a.h_qr) % a.T);
    const int b = (int)(i / ((int64_t)a.h_qr * a.T));
    float q[kD / 32], acc[kD / 32] = {};
    load_row(Q + i * a.d, a.d, lane, q);
    float qq = 0.f;
#pragma unroll
    for (int j = 0; j < kD / 32; ++j) qq += q[j] * q[j];
    qq = warp_sum(qq);
    if (qq > 0.f) {
      const float iq = 1.f / sqrtf(qq);
      for (int64_t c = 0; c < a.n_chunks; ++c) {
        const int64_t at = (int64_t)b * a.n_chunks + c;
        if (a.tstar[at] != t) continue;
        const float gs = a.ds[at] / (float)a.h_qr;
        if (gs == 0.f) continue;
        float k[kD / 32];
        load_row(K + (c * a.h_kv + h / m) * a.d, a.d, lane, k);
        float kk = 0.f, qk = 0.f;
#pragma unroll
        for (int j = 0; j < kD / 32; ++j) {
          kk += k[j] * k[j];
          qk += q[j] * k[j];
        }
        kk = warp_sum(kk);
        qk = warp_sum(qk);
        if (kk <= 0.f) continue;
        const float ik = 1.f / sqrtf(kk);
        const float cs = qk * iq * ik;
#pragma unroll
        for (int j = 0; j < kD / 32; ++j) acc[j] += gs * (k[j] * ik - cs * q[j] * iq) * iq;
      }
    }
#pragma unroll
    for (int j = 0; j < kD / 32; ++j) {
      const int e = lane + 32 * j;
      if (e < a.d) a.dQ[i * a.d + e] = acc[j];
    }
  }
}

template <typename T>
cudaError_t launch_t(const Args& a, int sms, cudaStream_t st) {
  auto grid_for = [&](int64_t warps) {
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>((warps * 32 + 255) / 256,
                                                              (int64_t)sms * 16));
  };
  scores_kernel<T><<<grid_for(a.n_chunks * a.B), 256, 0, st>>>(a);
  loss_kernel<<<1, 1024, 0, st>>>(a);
  if (a.dK) grad_k_kernel<T><<<grid_for(a.n_chunks * a.h_kv), 256, 0, st>>>(a);
  if (a.dQ) grad_q_kernel<T><<<grid_for((int64_t)a.B * a.T * a.h_qr), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aux

size_t aux_loss_scratch_bytes(int B, int64_t n_chunks) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return 3 * al((size_t)B * n_chunks * 4);
}

cudaError_t launch_aux_routing_loss(const void* Q_r, int B, int T, int h_qr, const void* Kbar_r,
                                    int64_t n_chunks, int h_kv, int d, int dtype,
                                    const uint32_t* pos, float tau, float* loss, float* dQ_r,
                                    float* dKbar_r, unsigned char* scratch, int sms,
                                    cudaStream_t st) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t part = al((size_t)B * n_chunks * 4);
  aux::Args a{};
  a.Q = Q_r;
  a.K = Kbar_r;
  a.pos = pos;
  a.n_chunks = n_chunks;
  a.words = (n_chunks + 31) / 32;
  a.B = B;
  a.T = T;
  a.h_qr = h_qr;
  a.h_kv = h_kv;
  a.d = d;
  a.tau = tau;
  a.s = reinterpret_cast<float*>(scratch);
  a.tstar = reinterpret_cast<int32_t*>(scratch + part);
  a.ds = reinterpret_cast<float*>(scratch + 2 * part);
  a.loss = loss;
  a.dQ = dQ_r;
  a.dK = dKbar_r;
  return dtype == 1 ? aux::launch_t<__nv_bfloat16>(a, sms, st) : aux::launch_t<float>(a, sms, st);
}

}  // namespace msa
