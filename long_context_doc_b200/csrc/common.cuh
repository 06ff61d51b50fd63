// common.cuh - device helpers shared by the libmsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace msa {

// ---------------------------------------------------------------- element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Unpack E elements held in a 16/8/4-byte vector into floats.
template <typename T, int E> struct Vec;
template <> struct Vec<__nv_bfloat16, 8> {
  using raw = uint4;
  static __device__ __forceinline__ void unpack(const raw& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <> struct Vec<__nv_bfloat16, 4> {
  using raw = uint2;
  static __device__ __forceinline__ void unpack(const raw& v, float* f) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xFFFF0000u);
  }
};
template <> struct Vec<__nv_bfloat16, 2> {
  using raw = uint32_t;
  static __device__ __forceinline__ void unpack(const raw& v, float* f) {
    f[0] = __uint_as_float(v << 16);
    f[1] = __uint_as_float(v & 0xFFFF0000u);
  }
};
template <> struct Vec<float, 4> {
  using raw = float4;
  static __device__ __forceinline__ void unpack(const raw& v, float* f) {
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
};
template <> struct Vec<float, 2> {
  using raw = float2;
  static __device__ __forceinline__ void unpack(const raw& v, float* f) { f[0] = v.x; f[1] = v.y; }
};
template <> struct Vec<float, 8> {
  using raw = float4;  // unused (fp32 uses at most 4 per 16 bytes)
  static __device__ __forceinline__ void unpack(const raw&, float*) {}
};

// ---------------------------------------------------------------- status word
// Workspaces start with a 256-byte header: [0] device status (0 = ok), [1] a counter.
constexpr int kErrWaitTimeout = 1;
constexpr int kErrCtxOverflow = 2;
constexpr int kErrBadIndex = 3;

__device__ __forceinline__ void set_err(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- mbarrier + bulk copy
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The dynamic shared memory array advanced to the next 1024-byte boundary of the shared window
// (the 128-byte swizzle atoms of TMA boxes and tensor-core operands). The pad is added to the
// array itself, so every pointer derived from the result stays in the shared state space and
// compiles to shared loads and stores with 32-bit addresses (a detour through an integer
// address makes them generic 64-bit accesses).
__device__ __forceinline__ unsigned char* smem_align1024(unsigned char* raw) {
  return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One-dimensional bulk copy global -> shared, completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after ~2^31 SM clocks (about a second) and records the failure.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << 31)) {
      set_err(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

constexpr long long kDefaultWaitLimit = 1ll << 31;  // SM clocks, about a second

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait by polling (non-blocking test, short sleeps between tests): for waits whose
// phase usually completes within a microsecond or two, where a blocking try_wait can keep the
// thread suspended well past the completion. Same limit and error as mbar_wait_bounded.
__device__ __forceinline__ bool mbar_wait_poll_bounded(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_test_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test_wait(bar, parity)) {
    __nanosleep(32);
    if (clock64() - t0 > (1ll << 31)) {
      set_err(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// Bounded wait with a caller-chosen limit in SM clocks: the default limit takes the blocking
// form above; a shorter one polls with the non-blocking test so that the limit, not the
// hardware's suspend time, decides when the wait gives up.
__device__ __forceinline__ bool mbar_wait_limited(uint64_t* bar, uint32_t parity, int* err,
                                                  long long limit) {
  if (limit <= 0 || limit >= kDefaultWaitLimit) return mbar_wait_bounded(bar, parity, err);
  const long long t0 = clock64();
  while (!mbar_test_wait(bar, parity)) {
    if (clock64() - t0 > limit) {
      set_err(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- RoPE angles
// (cos, sin) of n * theta_i for an integer position n. F = theta_i / (2 pi) mod 1 as a 64-bit
// binary fraction (host-computed), so n * F mod 2^64 is the exact turn count of the angle mod 1
// (two's complement for negative n); its top 32 bits, as a signed fraction of a half turn, go
// to the single-precision sincospi. Angle error < 2^-24 half turns at any position.
__device__ __forceinline__ float2 rot_turns(int64_t n, unsigned long long F) {
  const unsigned long long t = (unsigned long long)n * F;
  const float x = (float)(int)(t >> 32) * 0x1p-31f;  // angle / pi in [-1, 1)
  float s, c;
  sincospif(x, &s, &c);
  return make_float2(c, s);
}

// ---------------------------------------------------------------- order-preserving keys
// 64-bit key: larger key = larger score, then lower doc id. 0 is "empty".
__device__ __forceinline__ unsigned long long score_key(float s, uint32_t id) {
  if (s == 0.0f) s = 0.0f;  // -0.0 ranks as +0.0
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned long long)(~id);
}
__device__ __forceinline__ float key_score(unsigned long long key) {
  uint32_t u = (uint32_t)(key >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}
__device__ __forceinline__ int32_t key_id(unsigned long long key) {
  return (int32_t)(~(uint32_t)(key & 0xFFFFFFFFull));
}

// Binary search: first index j in [0, n] with off[j] >= x (off non-decreasing, length n+1).
__device__ __forceinline__ int64_t lower_bound_i64(const int64_t* off, int64_t n, int64_t x) {
  int64_t lo = 0, hi = n;
  while (lo < hi) {
    int64_t mid = (lo + hi) >> 1;
    if (off[mid] < x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// The same search by one warp with 32-way splits: ceil(log32(n)) + 1 dependent loads instead
// of log2(n). Needs x <= off[n]. Every lane returns j; *val = off[j].
__device__ __forceinline__ int64_t warp_lower_bound(const int64_t* off, int64_t n, int64_t x,
                                                    int lane, int64_t* val) {
  int64_t lo = 0, hi = n;  // off[lo - 1] < x <= off[hi]
  while (hi - lo >= 32) {
    const int64_t pos = lo + ((hi - lo) * (lane + 1)) / 32;  // lane 31 probes hi
    const unsigned m = __ballot_sync(0xffffffffu, __ldg(off + pos) >= x);
    const int f = __ffs(m) - 1;
    const int64_t prev = __shfl_sync(0xffffffffu, pos, f > 0 ? f - 1 : 0);
    hi = __shfl_sync(0xffffffffu, pos, f);
    lo = f > 0 ? prev + 1 : lo;
  }
  const int64_t pos = lo + lane;
  const int64_t v = pos <= hi ? __ldg(off + pos) : INT64_MAX;
  const int f = __ffs(__ballot_sync(0xffffffffu, v >= x)) - 1;
  *val = __shfl_sync(0xffffffffu, v, f);
  return lo + f;
}

// Document-aligned chunk range of CTA i of G: documents [D0, D1) whose chunks [cb, ce) start
// in the CTA's equal share of the n_chunks rows (the last CTA takes every remaining document).
// Run by warps 0 and 1 of the block (whole warps); writes {D0, D1, cb, ce} to out, which the
// block reads after its next barrier.
__device__ __forceinline__ void cta_doc_range(const int64_t* coff, int64_t n_docs,
                                              int64_t n_chunks, int64_t i, int64_t G,
                                              int64_t* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp > 1) return;
  int64_t D, cv;
  if (warp == 1 && i == G - 1) {
    D = n_docs;
    cv = __ldg(coff + n_docs);
  } else {
    D = warp_lower_bound(coff, n_docs, ((i + warp) * n_chunks) / G, lane, &cv);
  }
  if (lane == 0) {
    out[warp] = D;
    out[2 + warp] = cv;
  }
}

// ---------------------------------------------------------------- warp reductions
// Transposing warp reduction of N values per lane: at each of the five butterfly steps a lane
// keeps one half of its values, sends the other half to its XOR partner and adds what it
// receives, so the values per lane halve while every kept value gathers more lanes. After the call,
// if N >= 32 lane l holds flat indices [l*N/32, (l+1)*N/32) in v[0..N/32); otherwise v[0]
// holds index l / (32/N), summed over all 32 lanes.
template <int N, int O>
__device__ __forceinline__ void tr_reduce(float* v, int lane) {
  if constexpr (O >= 1) {
    if constexpr (N >= 2) {
      constexpr int H = N / 2;
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < H; ++i) {
        const float send = up ? v[i] : v[i + H];
        const float keep = up ? v[i + H] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      tr_reduce<H, O / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      tr_reduce<1, O / 2>(v, lane);
    }
  }
}

// ---------------------------------------------------------------- warp top-k lists
// Insert the lanes' candidate keys into the warp-held sorted list (lane i < k holds the
// i-th largest key; 0 = empty).
__device__ __forceinline__ void list_insert(unsigned long long& li, unsigned long long key,
                                            int lane, int k) {
  const unsigned long long thr = __shfl_sync(0xffffffffu, li, k - 1);
  unsigned m = __ballot_sync(0xffffffffu, key > thr);
  while (m) {
    const int src = __ffs(m) - 1;
    m &= m - 1;
    const unsigned long long x = __shfl_sync(0xffffffffu, key, src);
    const unsigned gt = __ballot_sync(0xffffffffu, lane < k && li > x);
    const int pos = __popc(gt);
    const unsigned long long up = __shfl_up_sync(0xffffffffu, li, 1);
    if (pos < k) {
      if (lane > pos && lane < k) li = up;
      if (lane == pos) li = x;
    }
  }
}

__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}

// Merge of one query's per-CTA lists by insertion: every key >= tau enters the warp-held
// top-k list (cand rows of CTA c for query b start at (c * B + b) * k).
__device__ __forceinline__ unsigned long long merge_by_insertion(const unsigned long long* src,
                                                                 bool in_smem, int G, int B, int b,
                                                                 int k, unsigned long long tau,
                                                                 int lane) {
  unsigned long long lst = 0ull;
  for (int c0 = 0; c0 < G; c0 += 32) {
    const int c = c0 + lane;
    const int row = (c * B + b) * k;
    for (int j = 0; j < k; ++j) {
      unsigned long long key = 0ull;
      if (c < G) key = in_smem ? src[row + j] : __ldcg(src + row + j);
      key = key >= tau ? key : 0ull;
      if (__ballot_sync(0xffffffffu, key != 0ull) == 0u) break;  // lists are sorted
      list_insert(lst, key, lane, k);
    }
  }
  return lst;
}

constexpr int kMergeCap = 256;  // survivors ranked directly, per warp

// Final merge of the per-CTA candidate lists cand[G][B][k] (run by the last CTA, every thread
// of the block). Each list is sorted (descending keys, 0 = empty) and the keys of different
// lists are distinct. The lists are first copied into shared memory with every copy in
// flight; warp w then takes queries w, w + nwarps, ...:
//   tau = max(largest k-th key of a list, largest per-lane maximum of the list heads that at
//         least k per-lane maxima reach): either way at least k distinct keys are >= tau,
//         so the global top-k lies in the keys >= tau;
//   the keys >= tau (a prefix of every list) are compacted into a per-warp buffer and each
//         one's rank is the number of larger survivors: rank r < k goes to output slot r.
// A query with more than kMergeCap survivors (or a block without the shared memory) falls
// back to inserting the keys >= tau into a warp-held sorted list.
__device__ __forceinline__ void merge_candidates(const unsigned long long* cand, int G, int B,
                                                 int k, unsigned char* smem, size_t smem_bytes,
                                                 int32_t* top_ids, float* top_scores) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const int n = G * B * k;
  const bool staged = (size_t)(n + nwarps * kMergeCap) * 8 <= smem_bytes;
  const unsigned long long* src = cand;
  unsigned long long* surv = nullptr;
  if (staged) {
    fence_proxy_async_smem();  // the region last held bulk-copied operand tiles
    unsigned long long* dst = reinterpret_cast<unsigned long long*>(smem);
    for (int i = 2 * tid; i + 1 < n; i += 2 * nthreads) cp_async16_cg(dst + i, cand + i);
    if ((n & 1) && tid == 0) dst[n - 1] = __ldcg(cand + n - 1);
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    src = dst;
    surv = dst + n + warp * kMergeCap;
  }
  for (int b = warp; b < B; b += nwarps) {
    // largest k-th key of a list
    unsigned long long tau = 0ull;
    for (int c = lane; c < G; c += 32) {
      const int at = (c * B + b) * k + (k - 1);
      const unsigned long long kth = staged ? src[at] : __ldcg(src + at);
      tau = kth > tau ? kth : tau;
    }
    // lane maxima of the list heads: heads of different lists are distinct documents, so the
    // largest lane maximum that k of the 32 lane maxima reach is a lower bound as well
    {
      unsigned long long hm = 0ull;
      for (int c = lane; c < G; c += 32) {
        const int at = (c * B + b) * k;
        const unsigned long long h = staged ? src[at] : __ldcg(src + at);
        hm = h > hm ? h : hm;
      }
      int ge = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) ge += __shfl_sync(0xffffffffu, hm, j) >= hm ? 1 : 0;
      if (hm != 0ull && ge >= k) tau = hm > tau ? hm : tau;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, tau, o);
      tau = other > tau ? other : tau;
    }
    // compact the survivors
    int total = 0;
    if (staged) {
      for (int c0 = 0; c0 < G; c0 += 32) {
        const int c = c0 + lane;
        const int row = (c * B + b) * k;
        int m = 0;
        if (c < G)
          while (m < k && src[row + m] != 0ull && src[row + m] >= tau) ++m;
        int incl = m;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int at = total + incl - m;
        if (at + m <= kMergeCap)
          for (int j = 0; j < m; ++j) surv[at + j] = src[row + j];
        total += __shfl_sync(0xffffffffu, incl, 31);
      }
      __syncwarp();
    }
    if (staged && total <= kMergeCap) {
      for (int i = lane; i < total; i += 32) {
        const unsigned long long x = surv[i];
        int r = 0;
        for (int j = 0; j < total; ++j) r += surv[j] > x ? 1 : 0;
        if (r < k) {
          top_ids[b * k + r] = key_id(x);
          top_scores[b * k + r] = key_score(x);
        }
      }
      if (lane < k && lane >= total) {
        top_ids[b * k + lane] = -1;
        top_scores[b * k + lane] = -INFINITY;
      }
      __syncwarp();  // the buffer is refilled for the warp's next query
    } else {
      const unsigned long long lst = merge_by_insertion(src, staged, G, B, b, k, tau, lane);
      if (lane < k) {
        top_ids[b * k + lane] = lst ? key_id(lst) : -1;
        top_scores[b * k + lane] = lst ? key_score(lst) : -INFINITY;
      }
    }
  }
}

}  // namespace msa
