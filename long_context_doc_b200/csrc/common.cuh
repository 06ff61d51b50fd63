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

}  // namespace msa
