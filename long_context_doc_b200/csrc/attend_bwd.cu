// attend_bwd.cu - backward pass of MSA's sparse attention on the 5th-generation tensor cores:
// the gradients of the loss with respect to the queries, the local keys and values and the
// gathered memory rows, which then flow into the bank rows the documents were gathered from.
//
// MSA is trained end to end: continued pre-training on the generation loss with an auxiliary
// routing loss, the top-k selection fused with the sparse attention so that the attention over
// [routed memory ; local context] is differentiable [ruixiangma.github.io blog, "训练策略";
// news.neo-ai.one article, "プロジェクト概要", Fig. 1]. The forward operation is that of
// attend_tc.cu: O = softmax(scale * q k^T over [memory ; causal local]) V with Q and the local K
// rotated at positions pos0 + row. With P the probabilities, dP = dO V^T, D = rowsum(dO * O)
// and dS = P * (dP - D) * scale:
//   dV = P^T dO,  dK = dS^T q_rot (local keys rotated back by -(pos0 + j)),  dQ = R^-1 (dS K).
//
// Kernels:
//  * the forward of attend_tc.cu again, writing the rotated Q and local K, the output O (fp32,
//    so that D carries no storage rounding) and the per-row log-sum-exp (log2 units) into the
//    workspace;
//  * a row pass: D = rowsum(dO * O) in the query-tile row order, the fp32 dQ accumulator zeroed;
//  * the main kernel, one CTA per (128-key tile, KV head, query): the tile's K and V stay in
//    shared memory while the query tiles that can see it (64 rows each: 64 / (h_q / h_kv)
//    tokens x the KV head's query heads) stream through a 2-stage ring (TMA, 128-byte swizzle).
//    One thread issues tcgen05.mma (bf16 x bf16 -> fp32 in TMEM):
//      S^T = K Q^T and dP^T = V dO^T              (M = 128 keys, N = 64 rows, K = 128 dims)
//      dV += P^T dO, dK += dS^T Q                 (M = 128 keys, N = 128 dims, K = 64 rows)
//      dQ^T = K^T dS^T                            (M = 128 dims, N = 64 rows, K = 128 keys)
//    The last three read dO, Q and K as MN-major operands straight from the tiles loaded for
//    the first two, and P^T / dS^T from the shared memory the softmax warps wrote them to, so
//    nothing is transposed in global memory. Eight warps (two per TMEM lane quarter: thread =
//    key row x half of the tile's rows) form
//    P^T = 2^(S^T * scale_log2 - lse) and dS^T under the visibility mask, then stage the tile's
//    dQ^T (thread = head dimension) as [row][dim] rows in shared memory that the bulk-copy
//    engine adds into the fp32 dQ accumulator (cp.reduce.async.bulk .add.f32, 512 bytes per
//    row); at the end they write dK (rotated back for local keys) and dV;
//  * a last row pass rotates dQ back by -(pos0 + L - T + t).
// Every wait is bounded; on expiry the CTA records kErrWaitTimeout in the status word, stops
// issuing, lets its copies and MMAs land, frees its TMEM and returns.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace abw {

constexpr int kKeys = 128;      // keys per CTA (TMEM lanes of S^T, dK, dV)
constexpr int kRows = 64;       // query rows per streamed tile
constexpr int kD = 128;
constexpr int kThreads = 320;   // warp 0 copies, warp 1 MMA, warps 2-9 softmax / epilogues
constexpr int kSoftmax = 256;   // softmax / epilogue threads
constexpr uint32_t kKSlice = kKeys * 128;     // [128 keys][64 dims] bf16: 16 KB
constexpr uint32_t kRSlice = kRows * 128;     // [64 rows][64 dims] bf16: 8 KB
constexpr uint32_t kStageBytes = 4 * kRSlice + 1024;  // Q, dO (2 slices each), lse + D
constexpr uint32_t kQStage = kRows * kD * 4;          // dQ of a tile, fp32 [64 rows][128]
constexpr uint32_t kSmem = 1024 + 4 * kKSlice + 2 * kStageBytes + 2 * kKSlice + kQStage + 256;

__device__ __forceinline__ void tma3(void* dst, const CUtensorMap* map, int x, int y, int z,
                                     uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// K-major operand slice [rows][64 bf16] with the 128-byte swizzle: 8-row groups 1024 bytes
// apart; a K step of 16 elements is +32 bytes.
__device__ __forceinline__ uint64_t desc_k(const void* slice) {
  const uint64_t a = (uint64_t)(smem_u32(slice) & 0x3FFFFu) >> 4;
  return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// MN-major operand over the same [rows][64 bf16] swizzled slices read the other way: the 64
// elements of a 128-byte row run along M (or N), the rows along K. 8-row K groups are 1024
// bytes apart, the next 64 elements along M/N start `lbo` bytes on (the next slice); a K step
// of 16 rows is +2048 bytes.
__device__ __forceinline__ uint64_t desc_mn(const void* slice, uint32_t lbo) {
  const uint64_t a = (uint64_t)(smem_u32(slice) & 0x3FFFFu) >> 4;
  return a | ((uint64_t)(lbo >> 4) << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                    uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t* r) {
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
}
// The same load without the wait: several loads in flight, then one tmem_wait_ld().
__device__ __forceinline__ void ld32_nowait(uint32_t taddr, uint32_t* r) {
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
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void red_add(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}
// global[0 .. bytes) += shared[0 .. bytes) (fp32, element-wise) by the bulk-copy engine;
// addresses 16-byte aligned, bytes a multiple of 16
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                   dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {  // sources of committed groups read
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {  // committed groups complete
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void softmax_sync() {  // the 256 softmax / epilogue threads
  asm volatile("bar.sync 1, 256;" ::: "memory");
}
// The same barrier, returning on every thread whether all 256 threads passed true: the
// softmax warps leave their loop together (a named barrier waits for all of them).
__device__ __forceinline__ bool softmax_sync_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 256, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t par, int* err,
                                              volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_wait_bounded(bar, par, err)) return true;
  *abort_flag = 1;
  return false;
}
struct Geo {
  int B, T, h_q, h_kv, L, max_ctx, Gq, R, Rpad, NQT, CT, LT;
};

// ------------------------------------------------------------------------------ row passes
// D[b, g, r] = sum_e dO[row] * O[row] for the query-tile row order r = t * Gq + head in group
// (rows past T*Gq up to Rpad: 0); one warp per row.
__global__ void __launch_bounds__(256) rows_d_kernel(const __nv_bfloat16* __restrict__ dO,
                                                     const float* __restrict__ O,
                                                     float* __restrict__ Dr, Geo g) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = (int64_t)g.B * g.h_kv * g.Rpad;
  for (int64_t i = w; i < total; i += nw) {
    const int r = (int)(i % g.Rpad);
    const int64_t bg = i / g.Rpad;
    const int gg = (int)(bg % g.h_kv), b = (int)(bg / g.h_kv);
    float s = 0.f;
    if (r < g.R) {
      const int t = r / g.Gq, hq = gg * g.Gq + r % g.Gq;
      const int64_t off = (((int64_t)b * g.T + t) * g.h_q + hq) * kD + lane * 4;
      const uint2 a = *reinterpret_cast<const uint2*>(dO + off);
      const float4 c = *reinterpret_cast<const float4*>(O + off);
      float x[4];
      Vec<__nv_bfloat16, 4>::unpack(a, x);
      s = x[0] * c.x + x[1] * c.y + x[2] * c.z + x[3] * c.w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    }
    if (lane == 0) Dr[i] = s;
  }
}

struct Turns {
  unsigned long long v[64];  // theta_i / (2 pi) mod 1 as 64-bit binary fractions
};

// dQ[row] = R(-(pos0 + L - T + t)) dQacc[row], in place (fp32). Thread per (row, pair i).
__global__ void __launch_bounds__(256) dq_rotate_back_kernel(float* __restrict__ dQ, Geo g,
                                                             int rope, int pos0, Turns turns) {
  const int64_t n = (int64_t)g.B * g.T * g.h_q * (kD / 2);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(i % (kD / 2));
    const int64_t row = i / (kD / 2);
    const int t = (int)((row / g.h_q) % g.T);
    float* r = dQ + row * kD;
    const float2 cs = rope ? rot_turns((int64_t)pos0 + g.L - g.T + t, turns.v[e])
                           : make_float2(1.f, 0.f);
    const float a = r[e], c = r[e + kD / 2];
    r[e] = a * cs.x + c * cs.y;
    r[e + kD / 2] = c * cs.x - a * cs.y;
  }
}

// ------------------------------------------------------------------------------ main kernel
struct MainArgs {
  Geo g;
  const int32_t* ctx_len;
  const float* lse;   // [B, h_kv, Rpad] log2 units
  const float* Dr;    // [B, h_kv, Rpad]
  float* dQacc;       // [B, T, h_q, 128]
  float* dKl;
  float* dVl;
  float* dKc;
  float* dVc;
  int rope, pos0;
  unsigned long long rope_turns[64];
  float scale, scale_log2;
  int* err;
};

__global__ void __launch_bounds__(kThreads, 1)
attend_bwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                  const __grid_constant__ CUtensorMap map_kc, const __grid_constant__ CUtensorMap map_kl,
                  const __grid_constant__ CUtensorMap map_vc, const __grid_constant__ CUtensorMap map_vl,
                  MainArgs p) {
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* base = smem_align1024(sm_raw);
  unsigned char* k_s = base;                          // [2 slices][128 keys][64 dims]
  unsigned char* v_s = base + 2 * kKSlice;            // [2 slices][128 keys][64 dims]
  unsigned char* stg = base + 4 * kKSlice;            // [2 stages][Q 2 slices | dO 2 | lse | D]
  unsigned char* pt_s = stg + 2 * kStageBytes;        // P^T  [128 keys][64 rows]
  unsigned char* dst_s = pt_s + kKSlice;              // dS^T [128 keys][64 rows]
  float* qst = reinterpret_cast<float*>(dst_s + kKSlice);  // dQ of a tile [64 rows][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(dst_s + kKSlice + kQStage);
  uint64_t* kvfull = bars;          // K and V tiles landed
  uint64_t* qfull = bars + 1;       // [2] stage landed
  uint64_t* qempty = bars + 3;      // [2] stage consumed by every MMA of its tile
  uint64_t* sfull = bars + 5;       // [2] S^T and dP^T of a TMEM buffer computed
  uint64_t* pfull = bars + 7;       // P^T, dS^T written (256 threads)
  uint64_t* pempty = bars + 8;      // the MMAs reading P^T, dS^T completed
  uint64_t* dqfull = bars + 9;      // [2] dQ^T of a TMEM buffer computed
  uint64_t* tfree = bars + 11;      // [2] dQ^T of a buffer drained (256 threads)
  uint64_t* done = bars + 13;       // every issued MMA completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const Geo& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, gk = blockIdx.y, b = blockIdx.z;
  const bool is_ctx = kt < g.CT;
  const int k0 = is_ctx ? kt * kKeys : (kt - g.CT) * kKeys;
  const int n_ctx = min(max(p.ctx_len[b], 0), g.max_ctx);
  const int kvalid = is_ctx ? min(kKeys, max(n_ctx - k0, 0)) : min(kKeys, g.L - k0);
  // query tiles that can see a key of this tile: every tile for memory keys; for local keys
  // the tokens t with L - T + t >= k0
  int qt0 = 0;
  if (!is_ctx) qt0 = (max(0, k0 - (g.L - g.T)) * g.Gq) / kRows;
  const int n_tiles = kvalid > 0 ? g.NQT - qt0 : 0;

  if (threadIdx.x == 0) {
    mbar_init(kvfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&dqfull[s], 1);
      mbar_init(&tfree[s], kSoftmax);
    }
    mbar_init(pfull, kSoftmax);
    mbar_init(pempty, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {  // buffers a = 0, 1: S^T / dQ^T at 128a, dP^T at 128a + 64; dK 256; dV 384
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

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0 && n_tiles > 0) {
      const CUtensorMap* mk = is_ctx ? &map_kc : &map_kl;
      const CUtensorMap* mv = is_ctx ? &map_vc : &map_vl;
      const int krow = is_ctx ? b * g.max_ctx + k0 : b * g.L + k0;
      mbar_arrive_expect_tx(kvfull, 4 * kKSlice);
      tma3(k_s, mk, 0, gk, krow, kvfull);
      tma3(k_s + kKSlice, mk, 64, gk, krow, kvfull);
      tma3(v_s, mv, 0, gk, krow, kvfull);
      tma3(v_s + kKSlice, mv, 64, gk, krow, kvfull);
      const int TQ = kRows / g.Gq;
      const int64_t rbase = ((int64_t)b * g.h_kv + gk) * g.Rpad;
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i & 1, qt = qt0 + i;
        if (i >= 2 && !wait_or_abort(&qempty[s], (uint32_t)(((i >> 1) - 1) & 1), p.err, abort_flag))
          break;
        unsigned char* st = stg + s * kStageBytes;
        mbar_arrive_expect_tx(&qfull[s], 4 * kRSlice + 512);
        const int z = b * g.T + qt * TQ;
        tma3(st, &map_q, 0, gk * g.Gq, z, &qfull[s]);
        tma3(st + kRSlice, &map_q, 64, gk * g.Gq, z, &qfull[s]);
        tma3(st + 2 * kRSlice, &map_do, 0, gk * g.Gq, z, &qfull[s]);
        tma3(st + 3 * kRSlice, &map_do, 64, gk * g.Gq, z, &qfull[s]);
        bulk_g2s(st + 4 * kRSlice, p.lse + rbase + (int64_t)qt * kRows, 256, &qfull[s]);
        bulk_g2s(st + 4 * kRSlice + 256, p.Dr + rbase + (int64_t)qt * kRows, 256, &qfull[s]);
        ++issued;
      }
      // the copies issued land before the CTA can exit
      mbar_wait_bounded(kvfull, 0, p.err);
      for (int j = max(0, issued - 2); j < issued; ++j)
        mbar_wait_bounded(&qfull[j & 1], (uint32_t)((j >> 1) & 1), p.err);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t kF32 = 1u << 4, kBf16A = 1u << 7, kBf16B = 1u << 10;
      constexpr uint32_t kMnA = 1u << 15, kMnB = 1u << 16;
      const uint32_t id_s = kF32 | kBf16A | kBf16B | ((uint32_t)(kRows >> 3) << 17) |
                            ((uint32_t)(kKeys >> 4) << 24);
      const uint32_t id_kv = kF32 | kBf16A | kBf16B | kMnB | ((uint32_t)(kD >> 3) << 17) |
                             ((uint32_t)(kKeys >> 4) << 24);
      const uint32_t id_q = kF32 | kBf16A | kBf16B | kMnA | kMnB |
                            ((uint32_t)(kRows >> 3) << 17) | ((uint32_t)(kD >> 4) << 24);
      auto issue_s = [&](int i) -> bool {  // S^T, dP^T of tile i into buffer i & 1
        const int s = i & 1;
        if (!wait_or_abort(&qfull[s], (uint32_t)((i >> 1) & 1), p.err, abort_flag)) return false;
        if (i >= 2 && !wait_or_abort(&tfree[s], (uint32_t)(((i >> 1) - 1) & 1), p.err, abort_flag))
          return false;
        fence_after();
        const unsigned char* st = stg + s * kStageBytes;
        const uint32_t d_s = tmem + (uint32_t)(s * 128), d_p = d_s + 64u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // over the 128 head dims, 16 per instruction
          const int sl = kk >> 2, o = 2 * (kk & 3);
          mma(d_s, desc_k(k_s + sl * kKSlice) + o, desc_k(st + sl * kRSlice) + o, id_s, kk ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int sl = kk >> 2, o = 2 * (kk & 3);
          mma(d_p, desc_k(v_s + sl * kKSlice) + o, desc_k(st + (2 + sl) * kRSlice) + o, id_s,
              kk ? 1u : 0u);
        }
        commit(&sfull[s]);
        return true;
      };
      bool ok = wait_or_abort(kvfull, 0, p.err, abort_flag) && issue_s(0);
      for (int i = 0; ok && i < n_tiles; ++i) {
        if (i + 1 < n_tiles && !issue_s(i + 1)) break;
        if (!wait_or_abort(pfull, (uint32_t)(i & 1), p.err, abort_flag)) break;
        fence_after();
        const int s = i & 1;
        const unsigned char* st = stg + s * kStageBytes;
        // dV += P^T dO and dK += dS^T Q over the tile's 64 rows (16 per instruction)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (i | kk) ? 1u : 0u;
          mma(tmem + 384u, desc_k(pt_s) + 2 * kk, desc_mn(st + 2 * kRSlice + kk * 2048, kRSlice),
              id_kv, acc);
          mma(tmem + 256u, desc_k(dst_s) + 2 * kk, desc_mn(st + kk * 2048, kRSlice), id_kv, acc);
        }
        // dQ^T = K^T dS^T over the tile's 128 keys, into the buffer S^T occupied
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma(tmem + (uint32_t)(s * 128), desc_mn(k_s + kk * 2048, kKSlice),
              desc_mn(dst_s + kk * 2048, 1024u), id_q, kk ? 1u : 0u);  // one 64-row chunk
        commit(&qempty[s]);
        commit(pempty);
        commit(&dqfull[s]);
      }
      commit(done);
      mbar_wait_bounded(done, 0, p.err);
    }
  } else {
    // ---------------- softmax + epilogues: warps 2-9, two per TMEM lane quarter (warp w reads
    // lanes 32 (w % 4) ..); thread = (lane = key row, half of the tile's 64 rows / of the dims)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int kr = quarter * 32 + lane;           // key row (and head dim for dQ^T)
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int key = k0 + kr;
    const bool key_ok = kr < kvalid;
    const float c = p.scale_log2;
    // a local key is visible to the tile rows r with token r / Gq >= key - (L - T): rows
    // r >= rmin (memory keys: every valid row)
    const int rmin = is_ctx ? 0 : max(0, key - (g.L - g.T)) * g.Gq;
    bool bad = false;
    int i = 0;
    for (; i < n_tiles && !bad; ++i) {
      const int s = i & 1, qt = qt0 + i;
      // the stage and S^T / dP^T have landed, and the MMAs of the previous tile no longer read
      // P^T / dS^T; leaving is decided by all 256 threads together
      bool ok = __all_sync(0xffffffffu, wait_or_abort(&qfull[s], (uint32_t)((i >> 1) & 1), p.err,
                                                      abort_flag) &&
                                            wait_or_abort(&sfull[s], (uint32_t)((i >> 1) & 1),
                                                          p.err, abort_flag));
      if (ok && i > 0)
        ok = __all_sync(0xffffffffu,
                        wait_or_abort(pempty, (uint32_t)((i - 1) & 1), p.err, abort_flag));
      if (!softmax_sync_and(ok)) {
        bad = true;
        break;
      }
      if (i == 0 && !key_ok) {
        // rows past the valid keys (memory rows past ctx_len hold whatever the buffer held):
        // zero them in K so that dQ^T = K^T dS^T reads no stale values (their dS^T is 0); each
        // half clears one of the two 64-dim slices
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(k_s + half * kKSlice + kr * 128 + ch * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      fence_after();
      const unsigned char* st = stg + s * kStageBytes;
      const float* lse_s = reinterpret_cast<const float*>(st + 4 * kRSlice) + half * 32;
      const float* d_s = lse_s + 64;
      const int r0 = qt * kRows + half * 32;       // tile row of this thread's first column
      const int lo_vis = max(rmin - r0, 0);        // columns [lo_vis, hi_vis) visible
      const int hi_vis = key_ok ? min(32, g.R - r0) : 0;
      uint32_t sr[32], dr[32];
      ld32_nowait(lane_base + (uint32_t)(s * 128 + half * 32), sr);  // S^T and dP^T together
      ld32_nowait(lane_base + (uint32_t)(s * 128 + 64 + half * 32), dr);
      tmem_wait_ld();
      uint32_t pk[16], dk[16];
      const float sc = p.scale;
#pragma unroll
      for (int q = 0; q < 32; q += 2) {
        float pv[2], dv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = q + u;
          const bool vis = col >= lo_vis && col < hi_vis;
          const float pp = vis ? ex2(fmaf(__uint_as_float(sr[col]), c, -lse_s[col])) : 0.f;
          pv[u] = pp;
          dv[u] = vis ? pp * (__uint_as_float(dr[col]) - d_s[col]) * sc : 0.f;
        }
        const __nv_bfloat162 h0 = __floats2bfloat162_rn(pv[0], pv[1]);
        const __nv_bfloat162 h1 = __floats2bfloat162_rn(dv[0], dv[1]);
        pk[q >> 1] = *reinterpret_cast<const uint32_t*>(&h0);
        dk[q >> 1] = *reinterpret_cast<const uint32_t*>(&h1);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {  // 16-byte chunk index XOR row % 8 (128-byte swizzle)
        const int chunk = half * 4 + q4;
        const int off = kr * 128 + ((chunk ^ (kr & 7)) << 4);
        *reinterpret_cast<uint4*>(pt_s + off) =
            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        *reinterpret_cast<uint4*>(dst_s + off) =
            make_uint4(dk[4 * q4], dk[4 * q4 + 1], dk[4 * q4 + 2], dk[4 * q4 + 3]);
      }
      fence_before();
      fence_proxy_async_smem();  // P^T, dS^T and the zeroed K rows are read by the tensor core
      mbar_arrive(pfull);
      // dQ^T of this tile: thread = head dim kr, this half's 32 of the tile's rows
      if (!softmax_sync_and(__all_sync(0xffffffffu, wait_or_abort(&dqfull[s],
                                                                  (uint32_t)((i >> 1) & 1), p.err,
                                                                  abort_flag)))) {
        bad = true;
        break;
      }
      fence_after();
      uint32_t qr[32];
      ld32(lane_base + (uint32_t)(s * 128 + half * 32), qr);
      fence_before();
      mbar_arrive(&tfree[s]);  // the TMEM buffer is drained into registers
      // the previous tile's reductions have read the staging rows; then every thread writes its
      // head dim of its 32 rows ([row][dim] fp32) and one thread per warp adds 8 whole rows
      // (512 bytes each) into the dQ accumulator with the bulk-copy engine
      if (lane == 0) bulk_wait_read_all();
      softmax_sync();
#pragma unroll
      for (int q = 0; q < 32; ++q) qst[(half * 32 + q) * kD + kr] = __uint_as_float(qr[q]);
      fence_proxy_async_smem();
      softmax_sync();
      if (lane == 0) {
        const int wq = warp - 2;  // rows [8 wq, 8 wq + 8) of the tile
        for (int q = 8 * wq; q < 8 * wq + 8; ++q) {
          const int r = qt * kRows + q;
          if (r >= g.R) break;
          const int t = r / g.Gq, hq = gk * g.Gq + r % g.Gq;
          bulk_reduce_add_f32(p.dQacc + (((int64_t)b * g.T + t) * g.h_q + hq) * kD, qst + q * kD,
                              kD * 4);
        }
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();  // the dQ reductions complete before the CTA exits
    // epilogue: dK (rotated back for local keys) and dV of the tile's valid rows, this half's
    // RoPE pairs (dims [32 half, 32 half + 32) and their partners 64 on). The TMEM loads are
    // warp-collective: every lane loads (a warp-uniform decision), valid rows store.
    const bool fin = n_tiles > 0 && !bad &&
                     __all_sync(0xffffffffu, wait_or_abort(done, 0, p.err, abort_flag));
    const bool store = key_ok && !*abort_flag;
    float* dk = is_ctx ? p.dKc + (((int64_t)b * g.max_ctx + key) * g.h_kv + gk) * kD
                       : p.dKl + (((int64_t)b * g.L + key) * g.h_kv + gk) * kD;
    float* dv = is_ctx ? p.dVc + (((int64_t)b * g.max_ctx + key) * g.h_kv + gk) * kD
                       : p.dVl + (((int64_t)b * g.L + key) * g.h_kv + gk) * kD;
    const int e0 = half * 32;
    if (n_tiles == 0 && store) {  // no query row sees the key
      for (int e = 0; e < 32; e += 4) {
        *reinterpret_cast<float4*>(dk + e0 + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(dk + 64 + e0 + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(dv + e0 + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(dv + 64 + e0 + e) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (fin) {  // warp-uniform
      fence_after();
      const bool rot = !is_ctx && p.rope;
      uint32_t lo[32], hi[32];
      ld32_nowait(lane_base + 256u + e0, lo);
      ld32_nowait(lane_base + 256u + 64 + e0, hi);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32 && store; q += 4) {
        float a4[4], h4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float x = __uint_as_float(lo[q + u]), y = __uint_as_float(hi[q + u]);
          if (rot) {
            const float2 cs = rot_turns((int64_t)p.pos0 + key, p.rope_turns[e0 + q + u]);
            a4[u] = x * cs.x + y * cs.y;
            h4[u] = y * cs.x - x * cs.y;
          } else {
            a4[u] = x;
            h4[u] = y;
          }
        }
        *reinterpret_cast<float4*>(dk + e0 + q) = make_float4(a4[0], a4[1], a4[2], a4[3]);
        *reinterpret_cast<float4*>(dk + 64 + e0 + q) = make_float4(h4[0], h4[1], h4[2], h4[3]);
      }
      ld32_nowait(lane_base + 384u + e0, lo);
      ld32_nowait(lane_base + 384u + 64 + e0, hi);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32 && store; q += 4) {
        *reinterpret_cast<float4*>(dv + e0 + q) =
            make_float4(__uint_as_float(lo[q]), __uint_as_float(lo[q + 1]),
                        __uint_as_float(lo[q + 2]), __uint_as_float(lo[q + 3]));
        *reinterpret_cast<float4*>(dv + 64 + e0 + q) =
            make_float4(__uint_as_float(hi[q]), __uint_as_float(hi[q + 1]),
                        __uint_as_float(hi[q + 2]), __uint_as_float(hi[q + 3]));
      }
    }
    // memory rows of the tile past ctx_len: zero gradients (each half its 64 dims)
    if (is_ctx && !key_ok && key < g.max_ctx && !*abort_flag) {
      for (int e = 64 * half; e < 64 * half + 64; e += 4) {
        *reinterpret_cast<float4*>(dk + e) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(dv + e) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
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

// ------------------------------------------------------------------------------ bank scatter
// dKbar[gidx[b, j]] += dKc[b, j] (and V) for j < ctx_len[b]: thread per 4 elements.
__global__ void __launch_bounds__(256) scatter_bank_grad_kernel(
    const int32_t* __restrict__ gidx, const int32_t* __restrict__ ctx_len, int B, int max_ctx,
    int64_t row_elems, const float* __restrict__ dKc, const float* __restrict__ dVc,
    float* __restrict__ dKbar, float* __restrict__ dVbar, int64_t n_chunks, int* err) {
  const int64_t per_row = row_elems / 4;
  const int64_t n = (int64_t)B * max_ctx * per_row;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / per_row, e = (i % per_row) * 4;
    const int b = (int)(row / max_ctx), j = (int)(row % max_ctx);
    if (j >= min(max(ctx_len[b], 0), max_ctx)) continue;
    const int64_t c = gidx[row];
    if (c < 0 || c >= n_chunks) {
      set_err(err, kErrBadIndex);
      continue;
    }
    const float4 k = *reinterpret_cast<const float4*>(dKc + row * row_elems + e);
    const float4 v = *reinterpret_cast<const float4*>(dVc + row * row_elems + e);
    float* dk = dKbar + c * row_elems + e;
    float* dv = dVbar + c * row_elems + e;
    red_add(dk, k.x); red_add(dk + 1, k.y); red_add(dk + 2, k.z); red_add(dk + 3, k.w);
    red_add(dv, v.x); red_add(dv + 1, v.y); red_add(dv + 2, v.z); red_add(dv + 3, v.w);
  }
}

}  // namespace abw

// ------------------------------------------------------------------------------ host side
BwdPlan attend_bwd_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L) {
  BwdPlan pl{};
  const int Gq = h_kv > 0 ? h_q / h_kv : 0;
  pl.fwd = attend_tc_plan(B, T, h_q, h_kv, d, max_ctx, L, true);
  pl.ok = pl.fwd.ok && Gq >= 1 && abw::kRows % Gq == 0;
  if (!pl.ok) return pl;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  pl.Gq = Gq;
  const int R = T * Gq;
  pl.NQT = (R + abw::kRows - 1) / abw::kRows;
  pl.Rpad = pl.NQT * abw::kRows;
  pl.CT = (max_ctx + abw::kKeys - 1) / abw::kKeys;
  pl.LT = (L + abw::kKeys - 1) / abw::kKeys;
  pl.fwd_bytes = pl.fwd.q_bytes + pl.fwd.k_bytes + pl.fwd.vl_bytes + pl.fwd.vc_bytes;
  pl.o_bytes = al((size_t)B * T * h_q * abw::kD * 4);
  pl.lse_bytes = al((size_t)B * h_kv * pl.Rpad * 4);
  pl.dq_bytes = al((size_t)B * T * h_q * abw::kD * 4);
  pl.smem = abw::kSmem;
  return pl;
}

cudaError_t launch_attend_bwd(const BwdParams& p, const BwdPlan& pl, unsigned char* scratch,
                              int sms, cudaStream_t st) {
  using namespace abw;
  unsigned char* fwd_ws = scratch;
  float* O = reinterpret_cast<float*>(scratch + pl.fwd_bytes);  // fp32 O of the recompute
  float* lse = reinterpret_cast<float*>(scratch + pl.fwd_bytes + pl.o_bytes);
  float* Dr = reinterpret_cast<float*>(scratch + pl.fwd_bytes + pl.o_bytes + pl.lse_bytes);
  const __nv_bfloat16* q_rot = reinterpret_cast<const __nv_bfloat16*>(fwd_ws);
  const __nv_bfloat16* k_rot = reinterpret_cast<const __nv_bfloat16*>(fwd_ws + pl.fwd.q_bytes);
  // 1. the forward again: rotated Q and K, O, log-sum-exp per row
  cudaError_t e = cudaMemsetAsync(lse, 0, pl.lse_bytes, st);
  if (e != cudaSuccess) return e;
  AtcParams a{};
  a.Q = p.Q;
  a.Kl = p.Kl;
  a.Vl = p.Vl;
  a.cK = p.cK;
  a.cV = p.cV;
  a.ctx_len = p.ctx_len;
  a.B = p.B;
  a.T = p.T;
  a.h_q = p.h_q;
  a.h_kv = p.h_kv;
  a.L = p.L;
  a.max_ctx = p.max_ctx;
  a.rope = p.rope;
  a.pos0 = p.pos0;
  for (int i = 0; i < 64; ++i) a.rope_turns[i] = p.rope_turns[i];
  a.scale_log2 = p.scale_log2;
  a.err = p.err;
  a.O = nullptr;
  a.O32 = O;
  a.lse = lse;
  a.lse_stride = pl.Rpad;
  e = launch_attend_tc(a, pl.fwd, fwd_ws, sms, st);
  if (e != cudaSuccess) return e;
  // 2. D per row; dQ accumulator zeroed (it is the dQ output, rotated back at the end)
  Geo g{p.B, p.T, p.h_q, p.h_kv, p.L, p.max_ctx, pl.Gq, p.T * pl.Gq, pl.Rpad, pl.NQT, pl.CT,
        pl.LT};
  {
    const int64_t rows = (int64_t)p.B * p.h_kv * pl.Rpad;
    const int64_t grid = std::min<int64_t>((rows * 32 + 255) / 256, (int64_t)sms * 16);
    rows_d_kernel<<<(unsigned)std::max<int64_t>(grid, 1), 256, 0, st>>>(p.dO, O, Dr, g);
    e = cudaMemsetAsync(p.dQ, 0, (size_t)p.B * p.T * p.h_q * kD * 4, st);
    if (e != cudaSuccess) return e;
  }
  // 3. tensor maps (bf16, 128-byte swizzle, zero fill out of bounds)
  CUtensorMap mq, mdo, mkc, mkl, mvc, mvl;
  const uint64_t row = kD * 2;
  {
    const uint64_t dims[3] = {kD, (uint64_t)p.h_q, (uint64_t)p.B * p.T};
    const uint64_t str[2] = {row, row * p.h_q};
    const uint32_t box[3] = {64, (uint32_t)pl.Gq, (uint32_t)(kRows / pl.Gq)};
    if (!encode_bf16_map(&mq, q_rot, 3, dims, str, box, true)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&mdo, p.dO, 3, dims, str, box, true)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {kD, (uint64_t)p.h_kv, (uint64_t)p.B * p.L};
    const uint64_t str[2] = {row, row * p.h_kv};
    const uint32_t box[3] = {64, 1, kKeys};
    if (!encode_bf16_map(&mkl, k_rot, 3, dims, str, box, true)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&mvl, p.Vl, 3, dims, str, box, true)) return cudaErrorInvalidValue;
  }
  if (p.max_ctx > 0) {
    const uint64_t dims[3] = {kD, (uint64_t)p.h_kv, (uint64_t)p.B * p.max_ctx};
    const uint64_t str[2] = {row, row * p.h_kv};
    const uint32_t box[3] = {64, 1, kKeys};
    if (!encode_bf16_map(&mkc, p.cK, 3, dims, str, box, true)) return cudaErrorInvalidValue;
    if (!encode_bf16_map(&mvc, p.cV, 3, dims, str, box, true)) return cudaErrorInvalidValue;
  } else {  // no memory tiles: never read
    mkc = mkl;
    mvc = mvl;
  }
  MainArgs m{};
  m.g = g;
  m.ctx_len = p.ctx_len;
  m.lse = lse;
  m.Dr = Dr;
  m.dQacc = p.dQ;
  m.dKl = p.dKl;
  m.dVl = p.dVl;
  m.dKc = p.dKc;
  m.dVc = p.dVc;
  m.rope = p.rope;
  m.pos0 = p.pos0;
  for (int i = 0; i < 64; ++i) m.rope_turns[i] = p.rope_turns[i];
  m.scale = p.scale;
  m.scale_log2 = p.scale_log2;
  m.err = p.err;
  e = cudaFuncSetAttribute(attend_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)pl.smem);
  if (e != cudaSuccess) return e;
  attend_bwd_kernel<<<dim3((unsigned)(pl.CT + pl.LT), (unsigned)p.h_kv, (unsigned)p.B), kThreads,
                      pl.smem, st>>>(mq, mdo, mkc, mkl, mvc, mvl, m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 4. dQ rotated back to the frame of the unrotated queries
  if (p.rope) {
    const int64_t n = (int64_t)p.B * p.T * p.h_q * (kD / 2);
    const int64_t grid = std::min<int64_t>((n + 255) / 256, (int64_t)sms * 16);
    Turns t{};
    for (int i = 0; i < 64; ++i) t.v[i] = p.rope_turns[i];
    dq_rotate_back_kernel<<<(unsigned)std::max<int64_t>(grid, 1), 256, 0, st>>>(p.dQ, g, p.rope,
                                                                                p.pos0, t);
  }
  return cudaGetLastError();
}

cudaError_t launch_scatter_bank_grad(const int32_t* gidx, const int32_t* ctx_len, int B,
                                     int max_ctx, int64_t row_elems, const float* dKc,
                                     const float* dVc, float* dKbar, float* dVbar, int64_t n_chunks,
                                     int* err, int sms, cudaStream_t st) {
  const int64_t n = (int64_t)B * max_ctx * (row_elems / 4);
  if (n == 0) return cudaSuccess;
  const int64_t grid = std::min<int64_t>((n + 255) / 256, (int64_t)sms * 16);
  abw::scatter_bank_grad_kernel<<<(unsigned)grid, 256, 0, st>>>(gidx, ctx_len, B, max_ctx,
                                                               row_elems, dKc, dVc, dKbar, dVbar,
                                                               n_chunks, err);
  return cudaGetLastError();
}

}  // namespace msa
