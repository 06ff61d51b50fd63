// encode_hidden.cu - the offline memory encoding from hidden states in one kernel: the key,
// value and router-key projections of every token on the 5th-generation tensor cores, with
// document-wise RoPE and chunk mean pooling applied to the fp32 accumulators, so the per-token
// K, V and K_r never reach memory.
//
// Method: the router K projector makes each document's routing keys and the attention layer
// its keys and values, all from the document's hidden states (ruixiangma.github.io blog,
// "稀疏注意力机制"); keys and router keys are rotated at the token's position within its
// document and every fixed-length chunk is mean-pooled (news.neo-ai.one article,
// "アーキテクチャ" and "並列（ドキュメント単位）RoPE").
//
// Kernel (one CTA per SM; work unit = two chunks x one projection x two KV heads):
//   warp 0     : TMA producer: per 64-wide slice of the hidden dimension, the two chunks'
//                hidden rows (two boxes of 64 rows, stacked into the 128-row A tile) and 256
//                weight rows (the two heads' outputs, B tile), 128-byte swizzle, no multicast,
//                into a 4-stage ring;
//   warp 1     : one thread issues tcgen05.mma kind::f16 (bf16 -> fp32, M = 128, N = 256,
//                K = 16) into one of two TMEM accumulators;
//   warps 2-5  : epilogue; a thread owns one token row (its TMEM lane): 32 columns and their
//                RoPE partners 64 columns on are read with tcgen05.ld, rotated at the token's
//                position (keys and router keys), masked to the chunk's valid rows, summed over
//                the warp's 32 rows by a transposing shuffle reduction and added into a
//                shared-memory row per chunk; the means are stored in bf16.
// Units are ordered chunk pair by chunk pair and dealt to the CTAs in turn, so the twelve
// units of a pair run at about the same time and the pair's hidden rows are read from HBM once
// and from L2 by its other units. Every wait is bounded; on expiry the CTA records an
// error in the status word, stops issuing work, drains what it issued and frees its TMEM.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace eh {

constexpr int kStages = 4;
constexpr int kBM = 128;        // token rows of a unit (two chunks of up to 64)
constexpr int kBN = 256;        // output columns of a unit (two KV heads of d = 128)
constexpr int kBK = 64;         // slice of the hidden dimension (128 bytes of bf16)
constexpr int kThreads = 192;   // 6 warps
constexpr uint32_t kABytes = kBM * kBK * 2;      // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;      // 32 KB
constexpr uint32_t kStage = kABytes + kBBytes;   // 48 KB

__device__ __forceinline__ void tma2(uint32_t dst, const CUtensorMap* map, int x, int y,
                                     uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// K-major tile [rows][64 bf16], 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}
__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                    uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t par, int* err,
                                             volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_wait_bounded(bar, par, err)) return true;
  *abort_flag = 1;
  return false;
}
__device__ __forceinline__ void epi_sync() {  // the 128 epilogue threads
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// The same barrier, returning on every epilogue thread whether all 128 passed true (one
// decision for the four warps, so none leaves the loop while another waits on a barrier).
__device__ __forceinline__ bool epi_sync_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
// Sum over the 32 lanes of v[j] for every j: afterwards v[0] of lane l holds the sum of the
// lanes' v[l] (a transposing butterfly: 31 shuffles for 32 sums).
__device__ __forceinline__ void lane_sums(float* v, int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
encode_hidden_kernel(const __grid_constant__ CUtensorMap map_h,
                     const __grid_constant__ CUtensorMap map_wk,
                     const __grid_constant__ CUtensorMap map_wv,
                     const __grid_constant__ CUtensorMap map_wr, EhParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = smem_align1024(smem_raw);
  float* pool = reinterpret_cast<float*>(base + kStages * kStage);   // [2 chunks][256]
  uint64_t* full = reinterpret_cast<uint64_t*>(pool + 2 * kBN);      // [kStages]
  uint64_t* empty = full + kStages;                                  // [kStages]
  uint64_t* tfull = empty + kStages;                                 // [2]
  uint64_t* tempty = tfull + 2;                                      // [2]
  uint64_t* done = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  unsigned long long* turns = reinterpret_cast<unsigned long long*>(tmem_holder + 4);  // [64]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x, ci = blockIdx.x;
  // units u = ci, ci + G, ...: at any time the CTAs work on about G consecutive units, the
  // twelve units of a chunk pair among them, so a pair's hidden rows come from HBM once and
  // from L2 for the other units (a contiguous range per CTA re-read them from HBM per unit)
  const int n_k = p.D / kBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 64) turns[threadIdx.x] = p.rope_turns[threadIdx.x];
  for (int j = threadIdx.x; j < 2 * kBN; j += kThreads) pool[j] = 0.f;
  if (warp == 0) {  // two fp32 accumulators of 256 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_holder;
  const int per_pair = 3 * p.n_tiles;  // units of one chunk pair: K, V, K_r x head pairs

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t u = ci; u < p.n_units; u += G) {
        const int64_t pr = u / per_pair;
        const int rest = (int)(u % per_pair), j = rest / p.n_tiles, t = rest % p.n_tiles;
        const int64_t ca = 2 * pr, cb = min(2 * pr + 1, p.n_chunks - 1);
        const int ya = __ldg(p.ctab + 3 * ca), yb = __ldg(p.ctab + 3 * cb);
        const CUtensorMap* mw = j == 0 ? &map_wk : (j == 1 ? &map_wv : &map_wr);
        for (int kk = 0; kk < n_k; ++kk) {
          if (issued >= kStages && !wait_or_fail(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
          const uint32_t st = smem_u32(base + (size_t)s * kStage);
          mbar_arrive_expect_tx(&full[s], kStage);
          tma2(st, &map_h, kk * kBK, ya, &full[s]);                     // rows 0..63
          tma2(st + kABytes / 2, &map_h, kk * kBK, yb, &full[s]);       // rows 64..127
          tma2(st + kABytes, mw, kk * kBK, t * kBN, &full[s]);          // 256 weight rows
          ++issued;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (*abort_flag) break;
      }
      for (int64_t q = (issued > kStages ? issued - kStages : 0); q < issued; ++q)
        mbar_wait_bounded(&full[q % kStages], (uint32_t)((q / kStages) & 1), p.err);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                             ((uint32_t)(kBM >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      for (int64_t u = ci, i = 0; u < p.n_units; u += G, ++i) {
        const int a = (int)(i & 1);
        const uint32_t aph = (uint32_t)((i >> 1) & 1);
        if (i >= 2 && !wait_or_fail(&tempty[a], aph ^ 1u, p.err, abort_flag)) break;
        fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * kBN);
        bool ok = true;
        for (int kk = 0; kk < n_k; ++kk) {
          if (!wait_or_fail(&full[s], ph, p.err, abort_flag)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t st = smem_u32(base + (size_t)s * kStage);
          const uint64_t ad = desc_sw128(st), bd = desc_sw128(st + kABytes);
#pragma unroll
          for (int k16 = 0; k16 < kBK / 16; ++k16)  // K = 16 per instruction: +32 bytes
            mma(d_tmem, ad + 2 * k16, bd + 2 * k16, idesc, (kk | k16) ? 1u : 0u);
          commit(&empty[s]);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        commit(&tfull[a]);
      }
      commit(done);
      mbar_wait_bounded(done, 0, p.err);
    }
  } else {
    // ---------------- epilogue (warps 2..5 -> TMEM lane groups 2, 3, 0, 1)
    const int lg = warp & 3;
    const int row = lg * 32 + lane;   // token row of the unit (TMEM lane)
    const int slot = row >> 6;        // chunk 0 or 1 of the pair
    const int ri = row & 63;          // row within the chunk
    const int HALF = kBN / 4;         // 64: RoPE partner offset within a head of d = 128
    for (int64_t u = ci, i = 0; u < p.n_units; u += G, ++i) {
      const int a = (int)(i & 1);
      const uint32_t aph = (uint32_t)((i >> 1) & 1);
      const int64_t pr = u / per_pair;
      const int rest = (int)(u % per_pair), j = rest / p.n_tiles, t = rest % p.n_tiles;
      const int64_t c = 2 * pr + slot;
      const bool chunk_ok = c < p.n_chunks;
      const int len = chunk_ok ? __ldg(p.ctab + 3 * c + 1) : 0;
      const int pos = chunk_ok ? __ldg(p.ctab + 3 * c + 2) + ri : 0;
      const bool valid = ri < len;
      const bool rotate = p.rope && j != 1;  // keys and router keys; values are not rotated
      if (!epi_sync_and(wait_or_fail(&tfull[a], aph, p.err, abort_flag))) break;
      fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(a * kBN);
      for (int cb = 0; cb < HALF; cb += 32) {  // pairs cb .. cb + 31 of each head
        float2 cs[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          cs[e] = rotate ? rot_turns(pos, turns[cb + e]) : make_float2(1.f, 0.f);
        for (int hh = 0; hh < 2; ++hh) {
          float lo[32], hi[32];
          ld32(tbase + (uint32_t)(hh * 128 + cb), lo);
          ld32(tbase + (uint32_t)(hh * 128 + cb + HALF), hi);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float x = lo[e], y = hi[e];
            lo[e] = valid ? x * cs[e].x - y * cs[e].y : 0.f;
            hi[e] = valid ? y * cs[e].x + x * cs[e].y : 0.f;
          }
          lane_sums(lo, lane);
          lane_sums(hi, lane);
          atomicAdd(&pool[slot * kBN + hh * 128 + cb + lane], lo[0]);
          atomicAdd(&pool[slot * kBN + hh * 128 + cb + HALF + lane], hi[0]);
        }
      }
      fence_before();
      mbar_arrive(&tempty[a]);  // the accumulator may be overwritten
      epi_sync();
      // means of the two chunks: warps of chunk slot s2 (lane groups 2 s2, 2 s2 + 1) split its
      // 256 columns; column col of the unit is element col % 128 of KV head 2 t + col / 128
      {
        const int s2 = slot, half_w = lg & 1;
        const int64_t c2 = 2 * pr + s2;
        const int n = c2 < p.n_chunks ? __ldg(p.ctab + 3 * c2 + 1) : 0;
        __nv_bfloat16* out = j == 0 ? p.Kbar : (j == 1 ? p.Vbar : p.Kbar_r);
        for (int col = half_w * 128 + lane; col < half_w * 128 + 128; col += 32) {
          const float m = n > 0 ? pool[s2 * kBN + col] / (float)n : 0.f;
          if (n > 0 && !*abort_flag) {
            const int head = 2 * t + col / 128;
            out[(c2 * p.h_kv + head) * 128 + (col & 127)] = __float2bfloat16_rn(m);
          }
          pool[s2 * kBN + col] = 0.f;
        }
      }
      epi_sync();  // the pool rows are zero again before the next unit's sums
    }
  }

  // ---------------- teardown: every MMA completed (the issuer waited on `done`)
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
}

}  // namespace eh

size_t encode_hidden_smem() {
  return 1024 + (size_t)eh::kStages * eh::kStage + 2 * eh::kBN * 4 + (2 * eh::kStages + 5) * 8 +
         16 + 64 * 8;
}

cudaError_t launch_encode_hidden(const EhParams& p, const void* H, int64_t n_tok,
                                 const void* Wk, const void* Wv, const void* Wr, int sms,
                                 cudaStream_t st) {
  if (p.n_units == 0) return cudaSuccess;
  CUtensorMap mh, mk, mv, mr;
  const uint64_t row = (uint64_t)p.D * 2;
  {
    const uint64_t dims[2] = {(uint64_t)p.D, (uint64_t)n_tok};
    const uint64_t str[1] = {row};
    const uint32_t box[2] = {(uint32_t)eh::kBK, 64};
    if (!encode_bf16_map(&mh, H, 2, dims, str, box, true)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)p.D, (uint64_t)p.h_kv * 128};
    const uint64_t str[1] = {row};
    const uint32_t box[2] = {(uint32_t)eh::kBK, (uint32_t)eh::kBN};
    if (!encode_bf16_map(&mk, Wk, 2, dims, str, box, true) ||
        !encode_bf16_map(&mv, Wv, 2, dims, str, box, true) ||
        !encode_bf16_map(&mr, Wr, 2, dims, str, box, true))
      return cudaErrorInvalidValue;
  }
  const size_t smem = encode_hidden_smem();
  cudaError_t e = cudaFuncSetAttribute(eh::encode_hidden_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<int64_t>(sms, p.n_units);
  eh::encode_hidden_kernel<<<grid, eh::kThreads, smem, st>>>(mh, mk, mv, mr, p);
  return cudaGetLastError();
}

}  // namespace msa
