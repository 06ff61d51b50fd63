// noalloc.cu - msa_route_topk for callers that cannot allocate device memory.
//
// Some callers cannot hand libmsa a workspace: code that runs under another framework's
// memory planner, which owns every device allocation and offers no scratch hook; paths that
// must not synchronise the device (cudaMalloc and cudaFree may synchronise); and serving loops
// that forbid allocator calls between steps. msa_route_topk_noalloc serves them with the same
// routing as msa_route_topk, using a fixed scratch array compiled into the library instead
// of a caller workspace.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes (2 MiB) that every
// GPU loading the library holds until the process exits. Host code cannot pass the array's
// name to a kernel (on the host it is only a stand-in, not a device address), so the first
// call on each device, with that device current, looks up the array's device address with
// cudaGetSymbolAddress and caches it; that first call should therefore come before any
// stream capture. All calls share the array and it keeps the previous call's contents:
// msa_route_topk clears the parts that must start at zero on every call, and calls that
// overlap on the GPU (different streams, or host threads) race on the array, so they must be
// serialised by the caller. Its first word is the status word that the kernels set when a
// bounded wait runs out or an index is bad; msa_route_topk_noalloc_status reads it.
//
// The cached address belongs to the device's primary context (the one the CUDA runtime uses);
// it goes stale after cudaDeviceReset, and a caller that switches to another driver-API
// context on the same device cannot use it.
#include <atomic>
#include <string>

#include "../../include/msa.h"
#include "kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

std::atomic<void*> g_scratch_addr[kMaxDevices];

}  // namespace

namespace {

// Device address of the scratch array on the current device (looked up once per device).
msa_status scratch_address(const char* who, void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    msa::set_last_error(std::string(who) + ": cudaGetDevice: " + cudaGetErrorString(e));
    return MSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    msa::set_last_error(std::string(who) + ": device ordinal " + std::to_string(dev) +
                        " beyond the " + std::to_string(kMaxDevices) + " supported");
    return MSA_ERR_UNSUPPORTED;
  }
  void* scratch = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (scratch == nullptr) {
    // set-up, once per device: the device address of the static scratch array
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_route_scratch);
    if (e != cudaSuccess || addr == nullptr) {
      msa::set_last_error(std::string(who) + ": cudaGetSymbolAddress: " +
                          cudaGetErrorString(e));
      return MSA_ERR_CUDA;
    }
    g_scratch_addr[dev].store(addr, std::memory_order_release);
    scratch = addr;
  }
  *out = scratch;
  return MSA_OK;
}

}  // namespace

extern "C" msa_status msa_route_topk_noalloc_status(int32_t* code, void* stream) {
  if (code == nullptr) {
    msa::set_last_error("msa_route_topk_noalloc_status: null code pointer");
    return MSA_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  const msa_status s = scratch_address("msa_route_topk_noalloc_status", &scratch);
  if (s != MSA_OK) return s;
  // the scratch starts with the same status word as a caller workspace
  return msa_workspace_status(scratch, code, stream);
}

extern "C" msa_status msa_route_topk_noalloc(
    const void* Q_r, int32_t B, int32_t T, int32_t h_qr, const void* Kbar_r,
    const float* kr_inv_norm, const void* Kbar_r_hat, const int64_t* doc_chunk_off,
    int64_t n_docs, int64_t n_chunks, int32_t h_kv, int32_t d, int32_t dtype, int32_t k,
    const uint32_t* exclude_bits, int32_t* top_ids, float* top_scores, float* doc_scores,
    void* stream) {
  void* scratch = nullptr;
  const msa_status s = scratch_address("msa_route_topk_noalloc", &scratch);
  if (s != MSA_OK) return s;
  const size_t need = msa_route_topk_workspace(B, T, h_qr, h_kv, d, dtype, n_docs, n_chunks, k);
  if (need > kNoAllocScratchBytes) {
    msa::set_last_error("msa_route_topk_noalloc: this call needs " + std::to_string(need) +
                        " bytes of scratch, more than the built-in " +
                        std::to_string(kNoAllocScratchBytes) +
                        "; use msa_route_topk with a workspace");
    return MSA_ERR_UNSUPPORTED;
  }
  return msa_route_topk(Q_r, B, T, h_qr, Kbar_r, kr_inv_norm, Kbar_r_hat, doc_chunk_off, n_docs,
                        n_chunks, h_kv, d, dtype, k, exclude_bits, top_ids, top_scores,
                        doc_scores, scratch, kNoAllocScratchBytes, stream);
}
