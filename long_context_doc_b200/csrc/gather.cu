// gather.cu - context assembly of MSA: only the selected documents' pooled K̄/V̄ are loaded
// and laid out as the memory part of each query's context, in ascending doc id, each doc's
// chunks in order [news.neo-ai.one article, "推論パイプライン": the selected K̄/V̄ are loaded
// and concatenated with the local context].
//
// One CTA per (selected slot j, query b). Its first warp ranks the doc among the query's valid
// ids (lane q holds id q, k <= 32; sums by shuffles), which gives its row offset in the context;
// the CTA writes the gather indices of its chunks and copies its chunks' rows with 16-byte
// vector loads/stores, four of each tensor in flight per thread (the source may be HBM or
// pinned host memory mapped into the device address space). Slot 0 also writes ctx_len and pads
// gather_idx with -1.
#include "common.cuh"
#include "kernels.cuh"

namespace msa {


__global__ void __launch_bounds__(256) gather_kernel(GatherParams p) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int32_t* ids = p.ids + (int64_t)b * p.k;
  __shared__ int64_t s_off, s_n, s_src, s_total;
  if (threadIdx.x < 32) {
    const int q = threadIdx.x;
    const int32_t o = q < p.k ? ids[q] : -1;
    const bool ok = o >= 0 && o < p.n_docs;
    const int64_t c0 = ok ? p.coff[o] : 0;
    const int64_t n = ok ? p.coff[o + 1] - c0 : 0;
    const int32_t me = __shfl_sync(0xffffffffu, o, j);
    const bool ok_me = me >= 0 && me < p.n_docs;
    // rows of the valid docs before this one: smaller id, or the same id at an earlier slot
    int64_t before = ok && ok_me && (o < me || (o == me && q < j)) ? n : 0;
    int64_t total = n;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, s);
      total += __shfl_xor_sync(0xffffffffu, total, s);
    }
    const int64_t n_me = __shfl_sync(0xffffffffu, n, j);
    const int64_t src_me = __shfl_sync(0xffffffffu, c0, j);
    if (q == 0) {
      if (me >= p.n_docs) set_err(p.err, kErrBadIndex);
      s_off = before;
      s_n = ok_me ? n_me : 0;
      s_src = ok_me ? src_me : 0;
      s_total = total;
      if (total > p.max_ctx && j == 0) set_err(p.err, kErrCtxOverflow);
    }
  }
  __syncthreads();
  const int64_t off = s_off, src = s_src, total = s_total;
  int64_t n = s_n;
  if (off >= p.max_ctx) n = 0;
  else if (off + n > p.max_ctx) n = p.max_ctx - off;
  int32_t* gi = p.gidx + (int64_t)b * p.max_ctx;
  for (int64_t x = threadIdx.x; x < n; x += blockDim.x) gi[off + x] = (int32_t)(src + x);
  if (j == 0) {
    const int64_t len = total < p.max_ctx ? total : p.max_ctx;
    for (int64_t x = len + threadIdx.x; x < p.max_ctx; x += blockDim.x) gi[x] = -1;
    if (threadIdx.x == 0) p.ctx_len[b] = (int32_t)len;
  }
  if (p.Kb == nullptr || n == 0) return;
  const int64_t vecs = n * p.row_bytes / 16;
  const int64_t dst0 = (((int64_t)b * p.max_ctx + off) * p.row_bytes) / 16;
  const int64_t src0 = (src * p.row_bytes) / 16;
  const uint4* sk = static_cast<const uint4*>(p.Kb) + src0;
  const uint4* sv = static_cast<const uint4*>(p.Vb) + src0;
  uint4* dk = static_cast<uint4*>(p.ctxK) + dst0;
  uint4* dv = static_cast<uint4*>(p.ctxV) + dst0;
  constexpr int U = 4;  // vectors of each tensor in flight per thread
  const int64_t nt = blockDim.x;
  for (int64_t x0 = threadIdx.x; x0 < vecs; x0 += U * nt) {
    uint4 a[U], c[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (x0 + u * nt < vecs) {
        a[u] = sk[x0 + u * nt];
        c[u] = sv[x0 + u * nt];
      }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (x0 + u * nt < vecs) {
        dk[x0 + u * nt] = a[u];
        dv[x0 + u * nt] = c[u];
      }
  }
}

cudaError_t launch_gather(const GatherParams& p, cudaStream_t st) {
  if (p.B == 0 || p.k == 0) return cudaSuccess;
  dim3 grid(p.k, p.B);
  gather_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace msa
