// synth_dev.cu - device twin of synth.c: the same counter-based generator, run on the
// GPU so that multi-gigabyte synthetic banks (a 100M-token router-key bank is ~59 GB)
// can be created in place. It implements exactly the integer definitions written at the
// top of synth.c (SplitMix64 words, sum-of-twelve-uniforms normal, bf16 round-to-nearest-
// even); the only floating-point operations are an exact int->float conversion, an exact
// division by 2^17 and the caller's scale. Tests compare it with the host side bit for bit.
//
// This is workload construction, not part of the MSA path: nothing here computes any
// step of the method.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kG = 0x9E3779B97F4A7C15ULL;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t e) {
  int64_t s = 0;
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    uint64_t r = mix64(key + (3ULL * e + (uint64_t)w + 1ULL) * kG);
    s += (int64_t)(r & 0xFFFF) + (int64_t)((r >> 16) & 0xFFFF) +
         (int64_t)((r >> 32) & 0xFFFF) + (int64_t)(r >> 48);
  }
  return __int2float_rn((int)(2 * s - 12 * 65535)) * (1.0f / 131072.0f);
}

__device__ __forceinline__ uint16_t bf16_rne_bits(float x) {
  uint32_t b = __float_as_uint(x);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

__global__ void fill_normal_kernel(void* out, int64_t n, int dtype, uint64_t key,
                                   uint64_t first, float scale) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    float x = normal_at(key, first + (uint64_t)i) * scale;
    if (dtype == 0) static_cast<float*>(out)[i] = x;
    else static_cast<uint16_t*>(out)[i] = bf16_rne_bits(x);
  }
}

}  // namespace

extern "C" {

// Fill the device buffer out[0..n) with normal(key(seed, tag), first + i) * scale.
// dtype 0 = fp32, 1 = bf16. Returns a cudaError_t value (0 = success).
int synth_dev_fill_normal(void* out, int64_t n, int dtype, uint64_t seed, uint64_t tag,
                          uint64_t first, float scale, void* stream) {
  if (n <= 0) return 0;
  if (out == nullptr || (dtype != 0 && dtype != 1)) return (int)cudaErrorInvalidValue;
  uint64_t key = mix64((seed * kG) ^ mix64(tag));
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (n + 255) / 256;
  int64_t cap = (int64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  fill_normal_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(out, n, dtype, key,
                                                                        first, scale);
  return (int)cudaGetLastError();
}

}  // extern "C"
