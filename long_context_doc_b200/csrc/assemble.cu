// assemble.cu - the local context of the attention call.
//  * Memory Interleaving round: per query, the raw per-token K/V of the documents appended so
//    far (in the order appended) followed by the query's own token rows, written contiguously.
//  * Sparse generation: each generated token's K/V joins the end of a preallocated local cache
//    whose length lives in device memory, so a captured decode step replays unchanged while
//    the cache grows.
//
// Method: each round's retrieved documents have their original text appended to the query's
// context for the next round [ai-papers.net summary, "MSAの提案手法"; ruixiangma.github.io blog,
// "Memory Interleaving"]; the tokens of that text precede the query tokens.
//
// CTA = (16 output rows, query). The query's segment offsets are a prefix sum over seg_len in
// shared memory; each output row is found by a binary search over them and copied with 16-byte
// vector loads and stores (rows of h_kv * d elements).
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {

constexpr int kAsmRows = 16;
constexpr int kAppendTab = 8;  // appends of at most this many rows per query use a RoPE table
constexpr int kAsmMaxSeg = 1024;

__global__ void __launch_bounds__(256) assemble_local_kernel(AssembleParams p) {
  __shared__ int64_t off[kAsmMaxSeg + 1];
  __shared__ int ok;
  const int b = blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * kAsmRows;
  if (threadIdx.x == 0) {
    int64_t s = 0;
    off[0] = 0;
    for (int q = 0; q < p.n_seg; ++q) {
      s += max(p.seg_len[(int64_t)b * p.n_seg + q], 0);
      off[q + 1] = s;
    }
    ok = (s + p.T == p.L);
    if (!ok && blockIdx.x == 0) set_err(p.err, kErrBadIndex);
  }
  __syncthreads();
  if (!ok) return;
  const int64_t S = off[p.n_seg];
  const int vecs = (int)(p.row_bytes / 16);  // 16-byte vectors per row
  for (int idx = threadIdx.x; idx < kAsmRows * vecs; idx += blockDim.x) {
    const int64_t j = j0 + idx / vecs;
    const int v = idx % vecs;
    if (j >= p.L) break;
    const uint4 *ks, *vs;
    if (j < S) {  // segment holding row j: last q with off[q] <= j
      int lo = 0, hi = p.n_seg - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= j) lo = mid;
        else hi = mid - 1;
      }
      const int64_t r = j - off[lo];
      const int64_t si = (int64_t)b * p.n_seg + lo;
      ks = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(p.seg_k[si]) + r * p.row_bytes);
      vs = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(p.seg_v[si]) + r * p.row_bytes);
    } else {  // the query's own rows
      const int64_t r = ((int64_t)b * p.T + (j - S)) * p.row_bytes;
      ks = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(p.K_q) + r);
      vs = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(p.V_q) + r);
    }
    const int64_t o = ((int64_t)b * p.L + j) * p.row_bytes;
    reinterpret_cast<uint4*>(static_cast<unsigned char*>(p.K_out) + o)[v] = ks[v];
    reinterpret_cast<uint4*>(static_cast<unsigned char*>(p.V_out) + o)[v] = vs[v];
  }
}

// Sparse generation: once the context is assembled, generation runs autoregressively over it
// with the routed memory fixed [news.neo-ai.one article, "推論パイプライン"; ruixiangma.github.io
// blog, "三阶段推理流程"]; each new token's K/V joins the end of the local context. Every CTA reads the length first; the last CTA to take a ticket
// (after all reads) advances it, so one launch both writes rows [len, len + T_new) and
// publishes len + T_new to the launches after it. A write past the capacity records
// kErrCtxOverflow and leaves cache and length unchanged.
__global__ void __launch_bounds__(256) kv_append_kernel(AppendParams p) {
  __shared__ int len_s;
  __shared__ unsigned long long turns[64];
  __shared__ float2 rtab[kAppendTab * 64];  // (cos, sin) per (new row t, pair i) for short appends
  if (threadIdx.x == 0) len_s = *reinterpret_cast<volatile int32_t*>(p.len);
  if (threadIdx.x < p.d / 2) turns[threadIdx.x] = p.rope_turns[threadIdx.x];
  __syncthreads();
  const int len = len_s;
  const bool ok = len >= 0 && (int64_t)len + p.T_new <= p.cap;
  const bool tab = p.rope && ok && p.T_new <= kAppendTab;  // a decode step's few rows
  if (tab) {
    const int half = p.d / 2;
    for (int e = threadIdx.x; e < p.T_new * half; e += blockDim.x)
      rtab[e] = rot_turns((int64_t)p.pos0 + len + e / half, turns[e % half]);
    __syncthreads();
  }
  // a one-CTA launch (a decode step) starts the call's status word itself
  if (p.single && threadIdx.x == 0) *p.err = ok ? 0 : kErrCtxOverflow;
  if (ok) {
    const int64_t vecs = p.row_bytes / 16;
    const int64_t n = (int64_t)p.B * p.T_new * vecs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
      const int64_t row = i / vecs, v = i % vecs;  // row = b * T_new + t
      const int64_t b = row / p.T_new, t = row % p.T_new;
      const int64_t dst = ((b * p.cap + len + t) * p.row_bytes) / 16 + v;
      if (!p.rope)
        reinterpret_cast<uint4*>(p.K_cache)[dst] = reinterpret_cast<const uint4*>(p.K_new)[i];
      reinterpret_cast<uint4*>(p.V_cache)[dst] = reinterpret_cast<const uint4*>(p.V_new)[i];
    }
    if (p.rope) {  // keys rotated at their global positions pos0 + len + t (pairs i, i + d/2)
      // one 16-byte vector of the first half of a (row, head) and its partner vector at + d/2
      const int half = p.d / 2, E = 16 / p.esize, cpr = half / E;  // vectors per half row
      const int64_t heads = p.row_bytes / ((int64_t)p.esize * p.d);
      const int64_t n_vec = (int64_t)p.B * p.T_new * heads * cpr;
      for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n_vec; w += stride) {
        const int c = (int)(w % cpr);
        const int64_t rh = w / cpr;  // (b * T_new + t) * heads + head
        const int64_t row = rh / heads, b = row / p.T_new, t = row % p.T_new;
        const int64_t src = (rh * p.d + (int64_t)c * E) * p.esize / 16;  // in 16-byte vectors
        const int64_t dst =
            ((((b * p.cap + len + t) * heads + rh % heads) * p.d + (int64_t)c * E) * p.esize) / 16;
        const uint4 lo = reinterpret_cast<const uint4*>(p.K_new)[src];
        const uint4 hi = reinterpret_cast<const uint4*>(p.K_new)[src + half * p.esize / 16];
        float x[8], y[8];
        if (p.esize == 2) {
          Vec<__nv_bfloat16, 8>::unpack(lo, x);
          Vec<__nv_bfloat16, 8>::unpack(hi, y);
        } else {
          Vec<float, 4>::unpack(*reinterpret_cast<const float4*>(&lo), x);
          Vec<float, 4>::unpack(*reinterpret_cast<const float4*>(&hi), y);
        }
        float xr[8], yr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (e >= E) break;
          const int i = c * E + e;
          const float2 cs = tab ? rtab[t * half + i] : rot_turns((int64_t)p.pos0 + len + t, turns[i]);
          xr[e] = x[e] * cs.x - y[e] * cs.y;
          yr[e] = y[e] * cs.x + x[e] * cs.y;
        }
        uint4 olo, ohi;
        if (p.esize == 2) {
          __nv_bfloat162* a2 = reinterpret_cast<__nv_bfloat162*>(&olo);
          __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            a2[e] = __floats2bfloat162_rn(xr[2 * e], xr[2 * e + 1]);
            b2[e] = __floats2bfloat162_rn(yr[2 * e], yr[2 * e + 1]);
          }
        } else {
          olo = make_uint4(__float_as_uint(xr[0]), __float_as_uint(xr[1]), __float_as_uint(xr[2]),
                           __float_as_uint(xr[3]));
          ohi = make_uint4(__float_as_uint(yr[0]), __float_as_uint(yr[1]), __float_as_uint(yr[2]),
                           __float_as_uint(yr[3]));
        }
        reinterpret_cast<uint4*>(p.K_cache)[dst] = olo;
        reinterpret_cast<uint4*>(p.K_cache)[dst + half * p.esize / 16] = ohi;
      }
    }
  } else if (!p.single && blockIdx.x == 0 && threadIdx.x == 0) {
    set_err(p.err, kErrCtxOverflow);
  }
  __syncthreads();
  if (p.single) {  // every thread's rows are written: publish the new length
    if (threadIdx.x == 0 && ok) *reinterpret_cast<volatile int32_t*>(p.len) = len + p.T_new;
    return;
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.ticket, 1u) == gridDim.x - 1) {
      if (ok) *reinterpret_cast<volatile int32_t*>(p.len) = len + p.T_new;
      *p.ticket = 0u;
      __threadfence();
    }
  }
}

cudaError_t launch_kv_append(const AppendParams& p, int sms, cudaStream_t st) {
  const int64_t n = (int64_t)p.B * p.T_new * (p.row_bytes / 16);
  const int64_t blocks =
      p.single ? 1 : std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 4LL * sms));
  kv_append_kernel<<<(unsigned)blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_assemble_local(const AssembleParams& p, cudaStream_t st) {
  if (p.B == 0 || p.L == 0) return cudaSuccess;
  dim3 grid((unsigned)((p.L + kAsmRows - 1) / kAsmRows), (unsigned)p.B);
  assemble_local_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace msa
