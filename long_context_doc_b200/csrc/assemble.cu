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
  if (threadIdx.x == 0) len_s = *reinterpret_cast<volatile int32_t*>(p.len);
  __syncthreads();
  const int len = len_s;
  const bool ok = len >= 0 && (int64_t)len + p.T_new <= p.cap;
  if (ok) {
    const int64_t vecs = p.row_bytes / 16;
    const int64_t n = (int64_t)p.B * p.T_new * vecs;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
      const int64_t row = i / vecs, v = i % vecs;  // row = b * T_new + t
      const int64_t b = row / p.T_new, t = row % p.T_new;
      const int64_t dst = ((b * p.cap + len + t) * p.row_bytes) / 16 + v;
      reinterpret_cast<uint4*>(p.K_cache)[dst] = reinterpret_cast<const uint4*>(p.K_new)[i];
      reinterpret_cast<uint4*>(p.V_cache)[dst] = reinterpret_cast<const uint4*>(p.V_new)[i];
    }
  } else if (blockIdx.x == 0 && threadIdx.x == 0) {
    set_err(p.err, kErrCtxOverflow);
  }
  __syncthreads();
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
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 4LL * sms));
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
