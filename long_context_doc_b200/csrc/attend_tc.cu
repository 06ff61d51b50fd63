// attend_tc.cu - sparse attention of MSA for long queries (prefill and Memory Interleaving
// rounds: at least 64 query rows per KV head) on the 5th-generation tensor cores.
//
// Method (the same operation as attend.cu): each query token attends over the compressed K/V
// of the routed documents (memory rows, used as stored, always visible) followed by the local
// context (causal: query token t sits at local row L - T + t), one softmax with scale 1/sqrt(d);
// Q and the local K are rotated at positions pos0 + row, pos0 = k
//   [news.neo-ai.one article, "グローバル RoPE（アクティブコンテキスト）" and "推論パイプライン";
//    ruixiangma.github.io blog, "三阶段推理流程" and "Memory Interleaving"].
//
// Two kernels:
//  * A pre-pass rotates Q and the local K once (bf16 out; angles as exact fixed-point turn
//    counts through sincospi).
//  * The attention kernel, one CTA per (128 query rows of one KV head, KV head, query): the rows
//    are 128 / (h_q / h_kv) tokens x the KV head's query heads. Warp 0 loads Q once and the
//    key tiles (128 rows of K and of V as stored, two 128-byte-swizzled TMA boxes of 64 dims
//    each, no multicast) into a 2-stage ring; one thread of warp 1 issues tcgen05.mma (bf16 x
//    bf16 -> fp32 in TMEM): S_j = Q K_j^T into one of two S buffers, issued one tile ahead, and
//    O += P_j V_j into a TMEM accumulator, V_j read as an MN-major operand straight from its
//    [key][dim] tile (nothing is transposed in memory); warps 2-9 (two per TMEM lane quarter:
//    thread = one query row x one half
//    of the keys and of the output dims) read S_j, mask, keep the online softmax (the halves
//    exchange the tile's row maximum through shared memory; the running maximum is raised only
//    when a tile's maximum exceeds it by more than 8 in log2 units, and only then is O rescaled
//    in TMEM), write P_j in bf16 to shared memory in the operand layout (and clear the V rows
//    of a memory tile past ctx_len, whose contents are not defined: 0 * NaN would reach O),
//    and finally normalise O and store it.
// Every wait is bounded; on expiry the CTA records kErrWaitTimeout in the workspace status word,
// stops, lets its copies and MMAs land, frees its TMEM and writes nothing.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace atc {

constexpr int kM = 128;         // query rows per tile (TMEM lanes)
constexpr int kN = 128;         // key rows per tile
constexpr int kD = 128;         // head dim
constexpr int kThreads = 320;   // warp 0 copies, warp 1 MMA, warps 2-9 softmax
constexpr uint32_t kSlice = 128 * 128;           // one 128-row x 64-element bf16 slice: 16 KB
constexpr uint32_t kQBytes = 2 * kSlice;         // Q tile (two 64-wide K slices)
constexpr uint32_t kKBytes = 2 * kSlice;         // K tile
constexpr uint32_t kVBytes = 2 * kSlice;         // V tile (two 64-dim slices)
constexpr uint32_t kStage = kKBytes + kVBytes;   // 64 KB
constexpr int kStages = 2;
constexpr float kRaise = 8.f;  // log2 headroom before the running maximum is raised

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
// K-major operand slice [rows][64 bf16], 128-byte swizzle: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc128(const void* slice) {
  const uint64_t a = (uint64_t)(smem_u32(slice) & 0x3FFFFu) >> 4;
  return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// MN-major operand over [rows][64 bf16] swizzled slices read the other way: the 64 elements of
// a 128-byte row run along N, the rows along K; 8-row K groups are 1024 bytes apart, the next
// 64 elements along N start `lbo` bytes on (the next slice); a K step of 16 rows is +2048 bytes.
__device__ __forceinline__ uint64_t desc_mn(const void* slice, uint32_t lbo) {
  const uint64_t a = (uint64_t)(smem_u32(slice) & 0x3FFFFu) >> 4;
  return a | ((uint64_t)(lbo >> 4) << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
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
__device__ __forceinline__ void st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Barrier of the 256 softmax threads (id 2), returning whether every one of them passed true.
__device__ __forceinline__ bool named_sync_softmax_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 2, 256, p;\n"
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

// 2^x by the hardware approximation (max relative error 2^-22; the probabilities are stored
// in bf16)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------------------ pre-pass
// Rotated bf16 copies of Q and the local K.
// RoPE of the rows of one position at a time (Q: the h_q heads of a token; local K: the h_kv
// heads of a row): warp per position, lane l on the pairs 2l, 2l + 1 (dims 2l, 2l+1 and their
// partners + 64), so each cos/sin is computed once per position and reused for every head, and
// a head row is two coalesced 128-byte reads and writes. Position of position-row r:
// base + r % mod.
__global__ void __launch_bounds__(256) rope_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                        __nv_bfloat16* __restrict__ dst,
                                                        int64_t n_pos, int heads, int64_t mod,
                                                        int64_t base, AtcParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const unsigned long long F0 = p.rope_turns[2 * lane], F1 = p.rope_turns[2 * lane + 1];
  for (int64_t r = w0; r < n_pos; r += nw) {
    const int64_t pos = base + r % mod;
    const float2 c0 = p.rope ? rot_turns(pos, F0) : make_float2(1.f, 0.f);
    const float2 c1 = p.rope ? rot_turns(pos, F1) : make_float2(1.f, 0.f);
    const uint32_t* s32 = reinterpret_cast<const uint32_t*>(src + r * heads * kD);
    uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + r * heads * kD);
#pragma unroll 8
    for (int h = 0; h < heads; ++h) {
      const uint32_t lo = __ldg(s32 + h * (kD / 2) + lane);
      const uint32_t hi = __ldg(s32 + h * (kD / 2) + 32 + lane);
      const float a0 = __uint_as_float(lo << 16), a1 = __uint_as_float(lo & 0xFFFF0000u);
      const float b0 = __uint_as_float(hi << 16), b1 = __uint_as_float(hi & 0xFFFF0000u);
      const __nv_bfloat162 ol =
          __floats2bfloat162_rn(a0 * c0.x - b0 * c0.y, a1 * c1.x - b1 * c1.y);
      const __nv_bfloat162 oh =
          __floats2bfloat162_rn(b0 * c0.x + a0 * c0.y, b1 * c1.x + a1 * c1.y);
      d32[h * (kD / 2) + lane] = *reinterpret_cast<const uint32_t*>(&ol);
      d32[h * (kD / 2) + 32 + lane] = *reinterpret_cast<const uint32_t*>(&oh);
    }
  }
}


// ------------------------------------------------------------------------------ attention
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kc,
                 const __grid_constant__ CUtensorMap map_kl, const __grid_constant__ CUtensorMap map_vc,
                 const __grid_constant__ CUtensorMap map_vl, AtcParams p) {
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* base = smem_align1024(sm_raw);
  unsigned char* q_s = base;                                  // [2][128][64]
  unsigned char* stages = base + kQBytes;                     // [S][K 2 slices | V 2 slices]
  unsigned char* p_s = stages + kStages * kStage;             // [2][128][64] probabilities
  float* xmax = reinterpret_cast<float*>(p_s + 2 * kSlice);  // [2 tiles][2 halves][128 rows]
  float* xsum = xmax + 512;                                  // [2 halves][128 rows]
  uint64_t* bars = reinterpret_cast<uint64_t*>(xsum + 256);
  uint64_t* qfull = bars;                    // Q landed
  uint64_t* kfull = bars + 1;                // [2] K half of the stage landed
  uint64_t* kempty = bars + 3;               // [2] K half consumed (S = Q K^T done)
  uint64_t* sfull = bars + 5;                // [2] S buffer written
  uint64_t* sfree = bars + 7;                // [2] S buffer read (256 threads)
  uint64_t* pfull = bars + 9;                // P written (256 threads)
  uint64_t* ofull = bars + 10;               // P.V of the tile completed
  uint64_t* done = bars + 11;                // every issued MMA completed
  uint64_t* vfull = bars + 12;               // [2] V half of the stage landed
  uint64_t* vempty = bars + 14;              // [2] V half consumed (P.V done)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int Gq = p.h_q / p.h_kv;
  const int TQ = kM / Gq;                         // tokens per query tile
  const int t0 = qt * TQ;
  const int t_last = min(t0 + TQ - 1, p.T - 1);
  const int n_ctx = min(max(p.ctx_len[b], 0), p.max_ctx);
  const int CT = (n_ctx + kN - 1) / kN;           // memory tiles
  const int jmax = p.L - p.T + t_last;            // last local row the tile's rows can see
  const int LT = jmax / kN + 1;                   // local tiles
  const int n_tiles = CT + LT;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&sfree[s], 256);
    }
    mbar_init(pfull, 256);
    mbar_init(ofull, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {  // S0 at column 0, S1 at 128, O at 256
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
    if (lane == 0) {
      int issued = 0;
      mbar_arrive_expect_tx(qfull, kQBytes);
      tma3(q_s, &map_q, 0, g * Gq, b * p.T + t0, qfull);
      tma3(q_s + kSlice, &map_q, 64, g * Gq, b * p.T + t0, qfull);
      // K of tile j may load once S_{j-2} is done, V once P_{j-2} V_{j-2} is done
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        const uint32_t par = (uint32_t)(((j >> 1) - 1) & 1);
        unsigned char* st = stages + s * kStage;
        const bool ctx = j < CT;
        const int r0 = ctx ? j * kN : (j - CT) * kN;
        const CUtensorMap* mk = ctx ? &map_kc : &map_kl;
        const CUtensorMap* mv = ctx ? &map_vc : &map_vl;
        const int krow = ctx ? b * p.max_ctx + r0 : b * p.L + r0;
        if (j >= 2 && !wait_or_abort(&kempty[s], par, p.err, abort_flag)) break;
        mbar_arrive_expect_tx(&kfull[s], kKBytes);
        tma3(st, mk, 0, g, krow, &kfull[s]);
        tma3(st + kSlice, mk, 64, g, krow, &kfull[s]);
        if (j >= 2 && !wait_or_abort(&vempty[s], par, p.err, abort_flag)) {
          ++issued;  // the K half is in flight
          break;
        }
        mbar_arrive_expect_tx(&vfull[s], kVBytes);
        tma3(st + kKBytes, mv, 0, g, krow, &vfull[s]);
        tma3(st + kKBytes + kSlice, mv, 64, g, krow, &vfull[s]);
        ++issued;
      }
      // the copies issued land before the CTA can exit
      mbar_wait_bounded(qfull, 0, p.err);
      for (int j = max(0, issued - 2); j < issued; ++j) {
        mbar_wait_bounded(&kfull[j & 1], (uint32_t)((j >> 1) & 1), p.err);
        mbar_wait_bounded(&vfull[j & 1], (uint32_t)((j >> 1) & 1), p.err);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                             ((uint32_t)(kM >> 4) << 24);
      const uint32_t idesc_pv = idesc | (1u << 16);  // B (V) MN-major
      const uint64_t qd0 = desc128(q_s), qd1 = desc128(q_s + kSlice);
      const uint64_t pd0 = desc128(p_s), pd1 = desc128(p_s + kSlice);
      auto issue_s = [&](int j) -> bool {  // S_j = Q K_j^T into buffer j & 1
        const int s = j & 1;
        if (!wait_or_abort(&kfull[s], (uint32_t)((j >> 1) & 1), p.err, abort_flag)) return false;
        if (j >= 2 && !wait_or_abort(&sfree[s], (uint32_t)(((j >> 1) - 1) & 1), p.err, abort_flag))
          return false;
        fence_after();
        const unsigned char* st = stages + s * kStage;
        const uint64_t kd0 = desc128(st), kd1 = desc128(st + kSlice);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 16 per instruction: +32 bytes within a slice
          const uint64_t a = (kk < 4 ? qd0 : qd1) + 2 * (kk & 3);
          const uint64_t bb = (kk < 4 ? kd0 : kd1) + 2 * (kk & 3);
          mma(tmem + (uint32_t)(s * kN), a, bb, idesc, kk ? 1u : 0u);
        }
        commit(&sfull[s]);
        commit(&kempty[s]);
        return true;
      };
      bool ok = wait_or_abort(qfull, 0, p.err, abort_flag) && (n_tiles == 0 || issue_s(0));
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_s(j + 1)) break;
        if (!wait_or_abort(pfull, (uint32_t)(j & 1), p.err, abort_flag)) break;
        if (!wait_or_abort(&vfull[j & 1], (uint32_t)((j >> 1) & 1), p.err, abort_flag)) break;
        fence_after();
        const unsigned char* st = stages + (j & 1) * kStage;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // O += P_j V_j over the tile's 128 keys, 16 per step
          const uint64_t a = (kk < 4 ? pd0 : pd1) + 2 * (kk & 3);
          const uint64_t bb = desc_mn(st + kKBytes + kk * 2048, kSlice);
          mma(tmem + 2u * kN, a, bb, idesc_pv, (j | kk) ? 1u : 0u);
        }
        commit(ofull);
        commit(&vempty[j & 1]);
      }
      commit(done);
      mbar_wait_bounded(done, 0, p.err);
    }
  } else {
    // ---------------- softmax: warps 2-9, two per TMEM lane quarter; thread = (query row, half
    // of the keys and of the output dims). The halves exchange only the row maximum per tile.
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const int tok = t0 + row / Gq;              // query token of this row
    const int hq = g * Gq + row % Gq;           // query head
    const bool row_ok = tok < p.T;
    const int vis = p.L - p.T + min(tok, p.T - 1);  // last visible local row
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t col0 = (uint32_t)(half * 64);
    const float c = p.scale_log2;
    float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
    bool bad = false;              // a wait gave up: no more tensor-memory work
    int j = 0;
    // tcgen05.ld/st are warp-collective: decisions around them are warp-uniform; leaving the
    // loop is a vote of all 256 softmax threads at the per-tile barrier
    for (; j < n_tiles; ++j) {
      const int sb = j & 1;
      bool ok = !bad && __all_sync(0xffffffffu, wait_or_abort(&sfull[sb], (uint32_t)((j >> 1) & 1),
                                                               p.err, abort_flag));
      const bool is_ctx = j < CT;
      const int k0 = (is_ctx ? j * kN : (j - CT) * kN) + half * 64;
      const int lim = is_ctx ? n_ctx - 1 - k0 : vis - k0;  // this half's keys [0, lim] visible
      const uint32_t sa = lane_base + (uint32_t)(sb * kN) + col0;
      const bool all_vis = lim >= 63;  // every key of this half visible to the row
      float mx = -INFINITY;
      uint32_t sr[64];  // this half's 64 scores of the row, loaded once for both passes
      if (ok) {
        fence_after();
        ld32_nowait(sa, sr);
        ld32_nowait(sa + 32, sr + 32);
        tmem_wait_ld();
        if (all_vis) {
#pragma unroll
          for (int q = 0; q < 64; ++q) mx = fmaxf(mx, __uint_as_float(sr[q]));
        } else {
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if (q <= lim) mx = fmaxf(mx, __uint_as_float(sr[q]));
        }
        mx *= c;  // the scale is positive: max of the scaled scores
      }
      xmax[(j & 1) * 256 + half * 128 + row] = mx;
      if (!named_sync_softmax_and(ok)) break;  // every softmax thread leaves together
      mx = fmaxf(mx, xmax[(j & 1) * 256 + (half ^ 1) * 128 + row]);
      // the running maximum moves only by more than kRaise (then O is rescaled)
      const bool raise = mx > m + kRaise || m == -INFINITY;
      const float m_new = raise ? mx : m;
      float alpha = 1.f;
      if (raise && m != -INFINITY) alpha = exp2f(m - m_new);
      // P_{j-1} . V_{j-1} must be done before P is rewritten and before O is rescaled
      if (j > 0) {
        ok = __all_sync(0xffffffffu, wait_or_abort(ofull, (uint32_t)((j - 1) & 1), p.err, abort_flag));
        if (!ok) {
          bad = true;
          continue;  // the next barrier vote ends the loop for everyone
        }
        fence_after();
        if (__any_sync(0xffffffffu, raise && m != -INFINITY)) {  // lanes not raising scale by 1
#pragma unroll 1
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t r[32];
            ld32(lane_base + 2u * kN + col0 + ch * 32, r);
#pragma unroll
            for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(__uint_as_float(r[q]) * alpha);
            st32(lane_base + 2u * kN + col0 + ch * 32, r);
          }
        }
      }
      m = (m_new == -INFINITY) ? m : m_new;
      l *= alpha;
      // pass 2: this half's probabilities in bf16 into P slice `half` (row-major 64 keys,
      // 16-byte chunk index XOR row % 8)
      float sum0 = 0.f, sum1 = 0.f;
      unsigned char* slice = p_s + half * kSlice + row * 128;
      const float negm = -m;
      const bool none = m == -INFINITY;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {  // the scores loaded in pass 1
        const uint32_t* r = sr + ch * 32;
        uint32_t pk[16];
        if (all_vis && !none) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float p0 = ex2(fmaf(__uint_as_float(r[2 * q]), c, negm));
            const float p1 = ex2(fmaf(__uint_as_float(r[2 * q + 1]), c, negm));
            sum0 += p0;
            sum1 += p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[q] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int k = ch * 32 + 2 * q;
            const float p0 = (k <= lim && !none) ? ex2(fmaf(__uint_as_float(r[2 * q]), c, negm)) : 0.f;
            const float p1 = (k + 1 <= lim && !none) ? ex2(fmaf(__uint_as_float(r[2 * q + 1]), c, negm)) : 0.f;
            sum0 += p0;
            sum1 += p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[q] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // 4 chunks of 16 bytes (8 keys) of this 32-key group
          const int chunk = ch * 4 + q4;
          *reinterpret_cast<uint4*>(slice + ((chunk ^ (row & 7)) << 4)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      l += sum0 + sum1;
      // a memory tile reaching past ctx_len: its V rows there are cleared once the tile has
      // landed, before P_j V_j (thread: key row `row` of the tile, its half of the dims)
      if (is_ctx && (j + 1) * kN > n_ctx) {
        bad = bad || !__all_sync(0xffffffffu, wait_or_abort(&vfull[sb], (uint32_t)((j >> 1) & 1),
                                                            p.err, abort_flag));
        if (!bad && j * kN + row >= n_ctx) {
          uint4* vr = reinterpret_cast<uint4*>(stages + sb * kStage + kKBytes + half * kSlice +
                                               row * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q) vr[q] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_before();
      fence_proxy_async_smem();  // P (and the cleared V rows) are read by the tensor core
      mbar_arrive(&sfree[sb]);
      mbar_arrive(pfull);
    }
    // epilogue: O / l of the last tile's accumulator (the halves add their shares of l)
    const bool fin = j == n_tiles && n_tiles > 0 && !bad &&
                     __all_sync(0xffffffffu, wait_or_abort(ofull, (uint32_t)((n_tiles - 1) & 1),
                                                           p.err, abort_flag));
    xsum[half * 128 + row] = l;
    const bool all_fin = named_sync_softmax_and(fin);
    if (all_fin) {
      fence_after();
      const float lt = l + xsum[(half ^ 1) * 128 + row];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if (p.lse != nullptr && half == 0 && row_ok && !*abort_flag)  // for the backward
        p.lse[((int64_t)b * p.h_kv + g) * p.lse_stride + qt * kM + row] = m + log2f(lt);
      __nv_bfloat16* out = p.O + (((int64_t)b * p.T + tok) * p.h_q + hq) * kD + half * 64;
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t r[32];
        ld32(lane_base + 2u * kN + col0 + ch * 32, r);
        if (row_ok && !*abort_flag && p.O32 != nullptr) {
          float* o32 = p.O32 + (((int64_t)b * p.T + tok) * p.h_q + hq) * kD + half * 64 + ch * 32;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<float4*>(o32 + 4 * q4) =
                make_float4(__uint_as_float(r[4 * q4]) * inv, __uint_as_float(r[4 * q4 + 1]) * inv,
                            __uint_as_float(r[4 * q4 + 2]) * inv,
                            __uint_as_float(r[4 * q4 + 3]) * inv);
        } else if (row_ok && !*abort_flag) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(
                  __uint_as_float(r[8 * q8 + 2 * q]) * inv, __uint_as_float(r[8 * q8 + 2 * q + 1]) * inv);
              w[q] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(out + ch * 32 + q8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
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

}  // namespace atc

// ------------------------------------------------------------------------------ host side

AtcPlan attend_tc_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L,
                       bool any_rows) {
  AtcPlan pl{};
  const int Gq = h_kv > 0 ? h_q / h_kv : 0;
  pl.ok = d == atc::kD && B >= 1 && T >= 1 && L >= T && Gq >= 1 && atc::kM % Gq == 0 &&
          (any_rows || Gq * T >= 64);
  if (!pl.ok) return pl;
  pl.n_qtiles = (Gq * T + atc::kM - 1) / atc::kM;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  pl.q_bytes = al((size_t)B * T * h_q * atc::kD * 2);
  pl.k_bytes = al((size_t)B * L * h_kv * atc::kD * 2);
  pl.vl_bytes = 0;  // V is read as stored (no transposed copy)
  pl.vc_bytes = 0;
  pl.smem = 1024 + atc::kQBytes + atc::kStages * atc::kStage + 2 * atc::kSlice + 768 * 4 +
            20 * 8 + 16;
  return pl;
}

cudaError_t launch_attend_tc(const AtcParams& p0, const AtcPlan& pl, unsigned char* scratch,
                             int sms, cudaStream_t st) {
  AtcParams p = p0;
  __nv_bfloat16* q_rot = reinterpret_cast<__nv_bfloat16*>(scratch);
  __nv_bfloat16* k_rot = reinterpret_cast<__nv_bfloat16*>(scratch + pl.q_bytes);
  const int Gq = p.h_q / p.h_kv;
  // pre-pass: rotated Q and local K
  {
    const int64_t qpos = (int64_t)p.B * p.T, kpos = (int64_t)p.B * p.L;  // warp per position
    const int64_t grid_q = std::min<int64_t>((qpos + 7) / 8, (int64_t)sms * 8);
    const int64_t grid_k = std::min<int64_t>((kpos + 7) / 8, (int64_t)sms * 8);
    atc::rope_rows_kernel<<<(unsigned)std::max<int64_t>(grid_q, 1), 256, 0, st>>>(
        p.Q, q_rot, qpos, p.h_q, p.T, (int64_t)p.pos0 + p.L - p.T, p);
    atc::rope_rows_kernel<<<(unsigned)std::max<int64_t>(grid_k, 1), 256, 0, st>>>(
        p.Kl, k_rot, kpos, p.h_kv, p.L, (int64_t)p.pos0, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // tensor maps (bf16, 128-byte swizzle, zero fill out of bounds)
  CUtensorMap mq, mkc, mkl, mvc, mvl;
  const uint64_t row = atc::kD * 2;
  {
    const uint64_t dims[3] = {atc::kD, (uint64_t)p.h_q, (uint64_t)p.B * p.T};
    const uint64_t str[2] = {row, row * p.h_q};
    const uint32_t box[3] = {64, (uint32_t)Gq, (uint32_t)(atc::kM / Gq)};
    if (!encode_bf16_map(&mq, q_rot, 3, dims, str, box, true)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {atc::kD, (uint64_t)p.h_kv, (uint64_t)p.B * p.L};
    const uint64_t str[2] = {row, row * p.h_kv};
    const uint32_t box[3] = {64, 1, atc::kN};
    if (!encode_bf16_map(&mkl, k_rot, 3, dims, str, box, true) ||
        !encode_bf16_map(&mvl, p.Vl, 3, dims, str, box, true))
      return cudaErrorInvalidValue;
  }
  if (p.max_ctx > 0) {
    const uint64_t dims[3] = {atc::kD, (uint64_t)p.h_kv, (uint64_t)p.B * p.max_ctx};
    const uint64_t str[2] = {row, row * p.h_kv};
    const uint32_t box[3] = {64, 1, atc::kN};
    if (!encode_bf16_map(&mkc, p.cK, 3, dims, str, box, true) ||
        !encode_bf16_map(&mvc, p.cV, 3, dims, str, box, true))
      return cudaErrorInvalidValue;
  } else {  // no memory tiles: never read
    mkc = mkl;
    mvc = mvl;
  }
  cudaError_t e = cudaFuncSetAttribute(atc::attend_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
  if (e != cudaSuccess) return e;
  atc::attend_tc_kernel<<<dim3((unsigned)pl.n_qtiles, (unsigned)p.h_kv, (unsigned)p.B),
                          atc::kThreads, pl.smem, st>>>(mq, mkc, mkl, mvc, mvl, p);
  return cudaGetLastError();
}

}  // namespace msa
