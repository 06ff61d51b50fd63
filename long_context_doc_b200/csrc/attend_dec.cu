// attend_dec.cu - sparse attention of MSA for decode-shaped queries (at most 8 query rows per
// KV head, bf16, d = 128, 1/2/4/8 KV heads): a bandwidth-bound stream over
// [gathered memory ; local context].
//
// Method (the same operation as attend.cu): the query attends over the compressed K/V of the
// routed documents followed by its own local K/V, one softmax, global RoPE on the active
// context: local row j sits at position pos0 + j with pos0 = k, the number of retrieved
// documents, memory rows are used as stored
//   [news.neo-ai.one article, "グローバル RoPE（アクティブコンテキスト）" and "推論パイプライン"].
//
// Kernel design (one CTA of eight warps per SM):
//  * A tile is KT = 64 / h_kv consecutive key rows of one query with all their KV heads (16 KB
//    of K and 16 KB of V, contiguous in the [row][KV head][d] storage order). One thread
//    moves it with four TMA boxes of [KV head][key row][64 dims] (each half of d of K and of V)
//    whose 128-byte swizzle makes every later shared-memory read conflict-free. Per query the
//    memory rows come first, then the local rows (a tile holds one kind). The flattened tile
//    list of all queries is cut into one contiguous range per CTA; a 4-stage ring keeps
//    128 KB of loads in flight per SM (an mbarrier per stage signals its copies' arrival;
//    the last warp to release a stage, counted in shared memory, issues its next copies).
//  * Warp w owns KV head w % h_kv and eight key rows of every tile, with its own online
//    softmax state; the warps meet only at the end of a query's segment (no block barrier per
//    tile). The logits and P.V run on the tensor cores as warp-level bf16 MMAs (fp32
//    accumulation): the query rows of the head (<= 8) are the rows of a 16-row A operand,
//    ldmatrix hands each lane its key and value fragments (8 MMAs of k = 16 over d for the
//    logits, 16 MMAs of k = 8 for P.V), and the probabilities of the logits' accumulator
//    fragment are the A fragment of P.V without leaving registers. This is a bandwidth-bound
//    stream, not a GEMM: the MMAs replace ~100 fp32 instructions per (key, KV head) row with
//    ~4, which is what lets eight warps keep up with HBM.
//  * RoPE by angle addition: key c of a local tile whose rows start at position P is rotated
//    by c*theta (per-CTA table, applied to the key fragments in registers before they are
//    rounded back to bf16), and the rotation by P*theta moves to the query
//    (<R((P+c)th) k, q> = <R(c th) k, R(-P th) q>); from one local tile to the next the query
//    turns by a fixed -KT*theta. Angles are exact integer turn counts (64-bit fixed point) fed
//    to a single-precision sincospi. The rotated query and keys and the probabilities are
//    rounded to bf16 for the MMAs (fp32 accumulation, softmax in fp32).
//  * A query split over several CTAs leaves one fp32 partial (m, l, o) per CTA in the workspace;
//    a second, short kernel merges them with one CTA per output row spread over all SMs.
// Every wait is bounded; on expiry the CTA records kErrWaitTimeout in the workspace status
// word, skips the remaining waits (all warps still pass every barrier), lets the copies it
// issued land and writes nothing.
#include <cmath>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {

constexpr int kDecCW = 8;                        // compute warps
constexpr int kDecThreads = kDecCW * 32;
constexpr int kDecRowsPerTile = 64;              // key rows x KV heads per tile
constexpr int kDecStages = 4;
constexpr int kDecD = 128;
constexpr uint32_t kDecRow = kDecD * 2;                   // bytes of one (key, KV head) row
constexpr uint32_t kDecHalf = kDecRowsPerTile * kDecRow;  // K (or V) of a tile: 16 KB
constexpr uint32_t kDecStage = 2 * kDecHalf;

// First CTA whose tile range contains flattened tile x.
__device__ __forceinline__ int64_t dec_cta_of(int64_t x, int64_t G, int64_t total) {
  return ((x + 1) * G + total - 1) / total - 1;
}

__device__ __forceinline__ void named_sync_compute() {  // the 256 compute threads
  asm volatile("bar.sync 1, 256;" ::: "memory");
}
// The same barrier, returning on every thread whether any of the 256 threads passed true.
__device__ __forceinline__ bool named_sync_compute_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 256, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// ---- register-level helpers of the tensor-core (mma.sync) logits and P.V
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// D = A B + C for a 16 x 8 x 16 bf16 product whose A rows 8..15 are zero: only the row-g
// accumulators (c0, c1) are kept.
__device__ __forceinline__ void mma_k16(float& c0, float& c1, uint32_t a0, uint32_t a2,
                                        uint32_t b0, uint32_t b1) {
  float d2, d3;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %10, %11};"
      : "+f"(c0), "+f"(c1), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(0.f), "f"(0.f));
}
// The same for a 16 x 8 x 8 product.
__device__ __forceinline__ void mma_k8(float& c0, float& c1, uint32_t a0, uint32_t b0) {
  float d2, d3;
  asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %7, %8};"
      : "+f"(c0), "+f"(c1), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(0u), "r"(b0), "f"(0.f), "f"(0.f));
}
__device__ __forceinline__ float2 bf2_unpack(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t bf2_pack(float2 v) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ void tma3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                      uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(0), "r"(smem_u32(bar))
      : "memory");
}

// Shared memory of the 8-warp kernel with an NS-stage ring: the stages, then the rotation
// tables (R(c theta) for the KT = 64 / h_kv in-tile key offsets and 11 rows of 32 entries),
// the RoPE turn counts, the combine buffer of the warps of a KV head (none when each warp owns
// a KV head, h_kv = 8), the per-warp scratch and the ring's barriers and counters.
__host__ __device__ constexpr size_t dec_comb_floats(int h_kv) {
  return h_kv == 8 ? 0 : (size_t)kDecCW * 8 * kDecD;
}
__host__ __device__ constexpr size_t dec_smem(int NS, int h_kv) {
  return 1024 + (size_t)NS * kDecStage + (size_t)(64 / h_kv) * 32 * 16 + 11 * 32 * 16 +
         (kDecD / 2) * 8 + sizeof(float) * (dec_comb_floats(h_kv) + (size_t)kDecCW * 88) +
         (size_t)NS * 12 + 16;
}

template <int NS>
__global__ void __launch_bounds__(kDecThreads, 1)
attend_dec_kernel(const __grid_constant__ CUtensorMap map_kc, const __grid_constant__ CUtensorMap map_vc,
                  const __grid_constant__ CUtensorMap map_kl, const __grid_constant__ CUtensorMap map_vl,
                  DecParams p) {
  constexpr int D = kDecD, HALF = D / 2;
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* sm = smem_align1024(sm_raw);
  unsigned char* stages = sm;                                                 // [NS][K|V]
  float4* rstep = reinterpret_cast<float4*>(sm + NS * kDecStage);             // [KT][32]
  float4* kturn = rstep + (64 / p.h_kv) * 32;                                 // [32]
  float4* qrot = kturn + 32;   // [T][32]: R(pos theta) at each query token's position
  float4* turn0 = qrot + 8 * 32;  // [32]: R(-pos0 theta), a query's first local tile
  float4* turn1 = turn0 + 32;     // [32]: R(-P theta), P = the CTA's first local tile start
  unsigned long long* turns = reinterpret_cast<unsigned long long*>(turn1 + 32);  // [HALF]
  const int RB = (p.h_q / p.h_kv) * p.T <= 4 ? 4 : 8;  // combine-buffer rows per KV head
  constexpr int WS = 11 * 8;                            // per-warp scratch floats
  float* comb = reinterpret_cast<float*>(turns + HALF);  // [8][RB][D] (h_kv < 8 only)
  float* wscr = comb + dec_comb_floats(p.h_kv);          // [8][WS]: max at 9 RB, sum at 10 RB
  uint64_t* full = reinterpret_cast<uint64_t*>(wscr + kDecCW * WS);  // [NS]
  unsigned int* released = reinterpret_cast<unsigned int*>(full + NS);  // [NS] warp releases
  volatile int* abort_flag = reinterpret_cast<volatile int*>(released + NS);
  volatile int* issued = abort_flag + 1;  // tiles whose copies were issued
  __shared__ int skip_call;
  __shared__ int ctx_first[32];  // context rows of the CTA's first 32 queries

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HKV = p.h_kv;
  const int KT = kDecRowsPerTile / HKV;  // key rows per tile
  const int Gq = p.h_q / HKV;
  const int nr = Gq * p.T;  // query rows per KV head (<= 8)
  // local rows per query: fixed, or read from the device (a cache that grows between launches)
  if (p.start_status && blockIdx.x == 0 && tid == 0) *p.err = 0;
  const int L = p.L_dev != nullptr ? *p.L_dev : p.L;
  if (L < p.T || L > p.Ls) {  // uniform over the grid: nothing is read or written
    if (blockIdx.x == 0 && tid == 0) set_err(p.err, kErrBadIndex);
    return;
  }
  const int TPP = p.CT + (L + KT - 1) / KT;  // tiles per query
  const int64_t total = (int64_t)p.B * TPP;
  // tile ranges: one per CTA, at most one per tile (a grid planned for a longer context
  // leaves its surplus CTAs idle, so every range a query spans is non-empty)
  const int64_t G = min((int64_t)gridDim.x, total), ci = blockIdx.x;
  if (ci >= G) return;
  const int64_t x0 = ci * total / G, x1 = (ci + 1) * total / G;
  const int n_tiles = (int)(x1 - x0);
  const int b_first = (int)(x0 / TPP), tt_first = (int)(x0 % TPP);

  // Copies of tile v of this CTA's range into stage v % NS: four TMA boxes of
  // [KV head][key row][64 dims] (128-byte swizzle), the K and V halves of d. Issued by one
  // thread: the first NS tiles here, each later one by the warp that releases the stage last.
  auto issue = [&](int v, bool check_ctx) {
    const int64_t x = x0 + v;
    const int bb = (int)(x / TPP), tv = (int)(x % TPP);
    const bool ctx = tv < p.CT;
    const int kt = ctx ? tv * KT : (tv - p.CT) * KT;
    // memory tiles past the query's context are not read (local tiles hold >= 1 row)
    // (the first tiles go out before ctx_len is read: rows past it are masked like a partial
    // tile's)
    const bool any = !ctx || !check_ctx || kt < min(max(__ldg(p.ctx_len + bb), 0), p.max_ctx);
    const int s = v % NS;
    const uint32_t st = smem_u32(stages + (size_t)s * kDecStage);
    fence_proxy_async_smem();  // the stage's earlier reads come before the new writes
    mbar_arrive_expect_tx(&full[s], any ? kDecStage : 0u);
    if (any) {
      const CUtensorMap* mk = ctx ? &map_kc : &map_kl;
      const CUtensorMap* mv = ctx ? &map_vc : &map_vl;
      const int y = ctx ? bb * p.max_ctx + kt : bb * p.Ls + kt;
      tma3d(st, mk, 0, y, &full[s]);
      tma3d(st + kDecHalf / 2, mk, HALF, y, &full[s]);
      tma3d(st + kDecHalf, mv, 0, y, &full[s]);
      tma3d(st + kDecHalf + kDecHalf / 2, mv, HALF, y, &full[s]);
    }
    *issued = v + 1;
  };
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      released[s] = 0u;
    }
    *abort_flag = 0;
    *issued = 0;
    // an error an earlier kernel of the same call recorded (a failed append) skips the call
    skip_call = (p.skip_on_err && *reinterpret_cast<volatile int*>(p.err) != 0) ? 1 : 0;
    fence_mbar_init();
    // the first copies go out before the tables are built, so the prologue overlaps them
    // (none when the call is skipped: a CTA never exits with a copy in flight)
    if (!skip_call)
      for (int v = 0; v < min(NS, n_tiles); ++v) issue(v, false);
  }
  if (tid < HALF) turns[tid] = p.rope_turns[tid];
  if (tid < 32)
    ctx_first[tid] = b_first + tid < p.B ? min(max(__ldg(p.ctx_len + b_first + tid), 0), p.max_ctx) : 0;
  __syncthreads();
  if (skip_call) return;
  auto ctx_rows = [&](int bb) {
    return bb - b_first < 32 ? ctx_first[bb - b_first]
                             : min(max(__ldg(p.ctx_len + bb), 0), p.max_ctx);
  };  // written once before the barrier: one value for the whole CTA


  // ---------------- compute warps
  const int g = warp % HKV;    // KV head of this warp
  const int sl = warp / HKV;   // its eight key rows of a tile: [8 sl, 8 sl + 8)
  const int gr = lane >> 2;    // fragment row: query row gr (logits) / key 8 sl + gr (keys)
  const int t4 = lane & 3;     // fragment column pair
  // per-CTA rotation tables, (cos, cos, sin, sin) of the pairs 2pp, 2pp + 1 (32 per row):
  // qrot[t] R(pos theta) at each query token's position; for caches whose keys are rotated
  // here also rstep[c] R(c theta) of the in-tile key offsets, kturn R(-KT theta) (the query's
  // turn from one local tile to the next), turn0 R(-pos0 theta) and turn1 R(-P theta) with P
  // the start of the CTA's first local tile
  {
    const bool rot_keys = p.rope && !p.keys_rotated;
    const int n_rows = p.T + (rot_keys ? KT + 3 : 0);
    const int64_t kt_first = (int64_t)max(tt_first - p.CT, 0) * KT;
    for (int idx = tid; idx < n_rows * 32; idx += kDecCW * 32) {
      const int r = idx >> 5, pp = idx & 31;
      int64_t n;
      float4* dst;
      if (r < p.T) {
        n = (int64_t)p.pos0 + L - p.T + r;
        dst = qrot + idx;
      } else if (r < p.T + KT) {
        n = r - p.T;
        dst = rstep + (r - p.T) * 32 + pp;
      } else if (r == p.T + KT) {
        n = -KT;
        dst = kturn + pp;
      } else if (r == p.T + KT + 1) {
        n = -(int64_t)p.pos0;
        dst = turn0 + pp;
      } else {
        n = -((int64_t)p.pos0 + kt_first);
        dst = turn1 + pp;
      }
      const float2 r0 = rot_turns(n, turns[2 * pp]), r1 = rot_turns(n, turns[2 * pp + 1]);
      *dst = make_float4(r0.x, r1.x, r0.y, r1.y);
    }
  }
  named_sync_compute();  // tables complete

  // ldmatrix row addresses of this lane: key row 8 sl + (lane & 7) of KV head g, dim chunk
  // 4 (m & 1) + (lane >> 3) of the half m >> 1 (128-byte swizzle: chunk ^ (line & 7))
  const int line = g * KT + 8 * sl + (lane & 7);
  uint32_t lofs[4];
#pragma unroll
  for (int m = 0; m < 4; ++m)
    lofs[m] = (uint32_t)((m >> 1) * (kDecHalf / 2) + line * 128 +
                         ((((m & 1) * 4 + (lane >> 3)) ^ (line & 7)) << 4));

  // the query rows of KV head g in fragment order: element (m, q) holds dims 32m + 8q + 2 t4
  // and +1 of row gr (zero for gr >= nr); ql rotated at the query position and pre-scaled,
  // qa turned back by the current local tile's start position
  float2 ql[4][4], qa[4][4];
  float2 o[16];  // P.V accumulators of row gr: dims 8 nt + 2 t4, +1
  float mrow = -INFINITY, lsum = 0.f;
  int b = b_first, tt = tt_first, cur = -1, n_ctx = 0;
  const int WPH = kDecCW / HKV;  // warps per KV head

  // combine the warps of each KV head over the open segment of query fb; write O (a query
  // within one CTA) or this CTA's partial
  auto finish_segment = [&](int fb) {
    float l = lsum;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    // the warps of head g other than its leader (warp g) leave (m, l, o) of their rows in shared
    // memory, o in fragment order ([warp][nt][lane], conflict-free); the leader folds them into
    // its registers and writes the rows
    const bool leader = warp == g;
    if (!leader && gr < RB) {
      float2* cw = reinterpret_cast<float2*>(comb) + warp * 16 * (RB * 4);
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) cw[nt * (RB * 4) + lane] = o[nt];
      if (t4 == 0) {
        wscr[warp * WS + 9 * RB + gr] = mrow;
        wscr[warp * WS + 10 * RB + gr] = l;
      }
    }
    const bool write = !named_sync_compute_or(*abort_flag != 0);  // one decision for all warps
    if (leader && write && gr < nr) {
      float M = mrow;
      for (int k2 = 1; k2 < WPH; ++k2) M = fmaxf(M, wscr[(g + k2 * HKV) * WS + 9 * RB + gr]);
      const float a0 = mrow == -INFINITY ? 0.f : exp2f(mrow - M);
      float2* ov = o;  // the segment's accumulators are folded in place
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) ov[nt] = __fmul2_rn(o[nt], make_float2(a0, a0));
      float lv = l * a0;
      for (int k2 = 1; k2 < WPH; ++k2) {
        const int w = g + k2 * HKV;
        const float m = wscr[w * WS + 9 * RB + gr];
        const float a = m == -INFINITY ? 0.f : exp2f(m - M);
        const float2* cw = reinterpret_cast<const float2*>(comb) + w * 16 * (RB * 4);
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
          ov[nt] = __ffma2_rn(cw[nt * (RB * 4) + lane], make_float2(a, a), ov[nt]);
        lv = fmaf(wscr[w * WS + 10 * RB + gr], a, lv);
      }
      const int64_t first = dec_cta_of((int64_t)fb * TPP, G, total);
      const int64_t last = dec_cta_of((int64_t)fb * TPP + TPP - 1, G, total);
      const int t = gr / Gq, h = g * Gq + gr % Gq;
      if (first == last) {  // the whole query in this CTA: O itself
        const float inv = lv > 0.f ? 1.f / lv : 0.f;
        __nv_bfloat16* out = p.O + (((int64_t)fb * p.T + t) * p.h_q + h) * D + 2 * t4;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
          *reinterpret_cast<uint32_t*>(out + 8 * nt) =
              bf2_pack(make_float2(ov[nt].x * inv, ov[nt].y * inv));
      } else {  // this CTA's partial of a split query
        const int64_t slot = (((int64_t)fb * p.max_seg + (ci - first)) * HKV + g) * RB + gr;
        float* out = p.part_o + slot * D + 2 * t4;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) *reinterpret_cast<float2*>(out + 8 * nt) = ov[nt];
        if (t4 == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = lv;
        }
      }
    }
    if (WPH > 1) named_sync_compute();  // the shared fragments are refilled by the next segment
  };

  bool qa_ok = false;  // qa matches the current local tile
  for (int u = 0; u < n_tiles; ++u) {
    const bool is_ctx = tt < p.CT;
    const int kt = is_ctx ? tt * KT : (tt - p.CT) * KT;  // first memory row / first local row
    if (b != cur) {
      if (cur >= 0) finish_segment(cur);
      cur = b;
      n_ctx = ctx_rows(b);
      const int tq = min(gr / Gq, p.T - 1), h = g * Gq + gr % Gq;
      const __nv_bfloat16* q = p.Q + (((int64_t)b * p.T + tq) * p.h_q + h) * D;
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int i = 32 * m + 8 * qq + 2 * t4;  // RoPE pairs i, i + 1 (partners + 64)
          float2 lo = make_float2(0.f, 0.f), hi = lo;
          if (gr < nr) {
            const float2 a = bf2_unpack(*reinterpret_cast<const uint32_t*>(q + i));
            const float2 c = bf2_unpack(*reinterpret_cast<const uint32_t*>(q + i + HALF));
            const float4 cs = qrot[tq * 32 + i / 2];
            const float2 c2 = make_float2(cs.x, cs.y), s2 = make_float2(cs.z, cs.w);
            lo = __fmul2_rn(__ffma2_rn(a, c2, __fmul2_rn(c, make_float2(-s2.x, -s2.y))), sc2);
            hi = __fmul2_rn(__ffma2_rn(c, c2, __fmul2_rn(a, s2)), sc2);
          }
          ql[m][qq] = lo;
          ql[m + 2][qq] = hi;
        }
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) o[nt] = make_float2(0.f, 0.f);
      mrow = -INFINITY;
      lsum = 0.f;
      qa_ok = false;
    }
    const int nk = is_ctx ? min(max(n_ctx - kt, 0), KT) : min(L - kt, KT);
    // keys used as stored: memory rows, and local rows of a cache that holds rotated keys
    const bool plain = is_ctx || p.keys_rotated || !p.rope;
    if (!plain && !qa_ok) {  // the query turned back by the tile's start position P
      // P = pos0 (a query's first local tile) or, for the CTA's first tile only, pos0 + kt
      const float4* A = kt == 0 ? turn0 : turn1;
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const float4 cs = A[16 * m + 4 * qq + t4];
          const float2 c2 = make_float2(cs.x, cs.y), s2 = make_float2(cs.z, cs.w);
          const float2 lo = ql[m][qq], hi = ql[m + 2][qq];
          qa[m][qq] = __ffma2_rn(lo, c2, __fmul2_rn(hi, make_float2(-s2.x, -s2.y)));
          qa[m + 2][qq] = __ffma2_rn(hi, c2, __fmul2_rn(lo, s2));
        }
      qa_ok = true;
    }
    const int s = u % NS;
    if (!*abort_flag && !mbar_wait_bounded(&full[s], (uint32_t)((u / NS) & 1), p.err))
      *abort_flag = 1;
    const uint32_t kb = smem_u32(stages + (size_t)s * kDecStage), vb = kb + kDecHalf;

    // ---- logits S[row gr][keys 8 sl + 2 t4, +1]: 8 MMAs over d, keys rotated in registers
    uint32_t kr[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) ldsm_x4(kb + lofs[m], kr[m]);
    if (!plain) {  // local keys: R(c theta), c = 8 sl + gr within the tile
      const float4* R = rstep + (8 * sl + gr) * 32 + t4;
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const float4 cs = R[16 * m + 4 * qq];
          const float2 c2 = make_float2(cs.x, cs.y), s2 = make_float2(cs.z, cs.w);
          const float2 x = bf2_unpack(kr[m][qq]), y = bf2_unpack(kr[m + 2][qq]);
          kr[m][qq] = bf2_pack(__ffma2_rn(x, c2, __fmul2_rn(y, make_float2(-s2.x, -s2.y))));
          kr[m + 2][qq] = bf2_pack(__ffma2_rn(y, c2, __fmul2_rn(x, s2)));
        }
    }
    // four independent accumulator pairs (one per quarter of d) shorten the MMA chain
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    if (plain) {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          mma_k16(sa[m], sb[m], bf2_pack(ql[m][2 * hh]), bf2_pack(ql[m][2 * hh + 1]),
                  kr[m][2 * hh], kr[m][2 * hh + 1]);
    } else {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          mma_k16(sa[m], sb[m], bf2_pack(qa[m][2 * hh]), bf2_pack(qa[m][2 * hh + 1]),
                  kr[m][2 * hh], kr[m][2 * hh + 1]);
    }
    const float s0 = (sa[0] + sa[1]) + (sa[2] + sa[3]), s1 = (sb[0] + sb[1]) + (sb[2] + sb[3]);

    // ---- online softmax of row gr over this warp's 8 keys (a lane holds keys 2 t4, 2 t4 + 1)
    const int jj = 8 * sl + 2 * t4;          // tile key of s0 (s1: jj + 1)
    const bool k0 = jj < nk, k1 = jj + 1 < nk;
    bool v0 = k0, v1 = k1;
    if (!is_ctx) {
      const int lim = L - p.T + gr / Gq - kt;  // causal: local row kt + j visible if <= lim
      v0 = v0 && jj <= lim;
      v1 = v1 && jj + 1 <= lim;
    }
    const float xa = v0 ? s0 : -INFINITY, xb = v1 ? s1 : -INFINITY;
    float mx = fmaxf(xa, xb);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mn = fmaxf(mrow, mx);
    const float alpha = mn == -INFINITY ? 1.f : exp2f(mrow - mn);
    const float p0 = v0 ? exp2f(xa - mn) : 0.f, p1 = v1 ? exp2f(xb - mn) : 0.f;
    lsum = fmaf(lsum, alpha, p0 + p1);
    mrow = mn;
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) o[nt] = __fmul2_rn(o[nt], make_float2(alpha, alpha));
    }
    const uint32_t pa = bf2_pack(make_float2(p0, p1));

    // ---- P.V: O[row gr][dims] += P[row gr][8 keys] V[8 keys][dims], 16 MMAs; V rows of keys
    // past the tile's valid rows are cleared (their probabilities are zero, their contents
    // are not defined)
    const uint32_t vmask = (k0 ? 0x0000FFFFu : 0u) | (k1 ? 0xFFFF0000u : 0u);
    const bool partial = __any_sync(0xffffffffu, vmask != 0xFFFFFFFFu);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      uint32_t vr[4];
      ldsm_x4_trans(vb + lofs[m], vr);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        const uint32_t bv = partial ? (vr[qq] & vmask) : vr[qq];
        mma_k8(o[4 * m + qq].x, o[4 * m + qq].y, pa, bv);
      }
    }
    __syncwarp();
    // release the stage; the last of the eight warps refills it with tile u + NS
    if (lane == 0 && atomicAdd(&released[s], 1u) % kDecCW == kDecCW - 1 && u + NS < n_tiles &&
        !*abort_flag)
      issue(u + NS, true);
    // next local tile: advance the position by KT (turn the query back by KT theta)
    if (!plain) {
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const float4 cs = kturn[16 * m + 4 * qq + t4];
          const float2 c2 = make_float2(cs.x, cs.y), s2 = make_float2(cs.z, cs.w);
          const float2 lo = qa[m][qq], hi = qa[m + 2][qq];
          qa[m][qq] = __ffma2_rn(lo, c2, __fmul2_rn(hi, make_float2(-s2.x, -s2.y)));
          qa[m + 2][qq] = __ffma2_rn(hi, c2, __fmul2_rn(lo, s2));
        }
    }
    if (++tt == TPP) {
      tt = 0;
      ++b;
    }
  }
  if (cur >= 0) finish_segment(cur);
  // every copy issued lands before the CTA exits (after an expired wait some were not
  // consumed; bounded)
  named_sync_compute();
  if (tid == 0)
    for (int j = max(0, *issued - NS); j < *issued; ++j)
      mbar_wait_bounded(&full[j % NS], (uint32_t)((j / NS) & 1), p.err);
}

// Merge of the partials of the queries split over several CTAs: CTA = one output row (query b,
// query head h, token t); warp w folds segments w, w + 8, ... with lane l on dims 4l .. 4l+3,
// each with its own running maximum, then the eight warps combine in shared memory.
constexpr int kMergeWarps = 8;
__global__ void __launch_bounds__(kMergeWarps * 32) attend_dec_merge_kernel(DecParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int HKV = p.h_kv, Gq = p.h_q / HKV;
  const int row = blockIdx.x;  // ((b * T + t) * h_q + h)
  const int h = row % p.h_q, t = (row / p.h_q) % p.T, b = row / (p.h_q * p.T);
  const int gh = h / Gq, r = t * Gq + h % Gq;
  const int RB = (Gq * p.T) <= 4 ? 4 : 8;
  // the length and the status word, loaded together
  const int L = p.K_new != nullptr ? __ldcg(p.L_out)  // fused append: the length it used
                                   : (p.L_dev != nullptr ? __ldcg(p.L_dev) : p.L);
  const int err = p.skip_on_err ? __ldcg(p.err) : 0;
  if (p.K_new != nullptr) {
    if (L < 0) return;  // overflow: the cache length stays
    // the cache length advances here, after every attention CTA has read it
    if (blockIdx.x == 0 && threadIdx.x == 0) *const_cast<int32_t*>(p.L_dev) = L;
  }
  if (L < p.T || L > p.Ls) return;  // reported by the attention kernel
  if (err != 0) return;
  const int KT = kDecRowsPerTile / HKV;
  const int TPP = p.CT + (L + KT - 1) / KT;
  const int64_t total = (int64_t)p.B * TPP, G = min((int64_t)p.grid, total);
  const int64_t first = dec_cta_of((int64_t)b * TPP, G, total);
  const int64_t last = dec_cta_of((int64_t)b * TPP + TPP - 1, G, total);
  const int n_seg = (int)(last - first + 1);
  if (n_seg == 1) return;  // written directly by the attention kernel
  __shared__ float sm_m[kMergeWarps], sm_l[kMergeWarps];
  __shared__ float4 sm_o[kMergeWarps][32];
  auto slot_of = [&](int sg) { return (((int64_t)b * p.max_seg + sg) * HKV + gh) * RB + r; };
  // warp w folds segments w, w + 8, ... four at a time (their loads in flight together) with
  // its own running maximum; the eight warps are then combined in shared memory
  float M = -INFINITY, l = 0.f;
  float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sg0 = warp; sg0 < n_seg; sg0 += 4 * kMergeWarps) {
    float2 ml[4];
    float4 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int sg = sg0 + i * kMergeWarps;
      ml[i] = make_float2(-INFINITY, 0.f);
      x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (sg < n_seg) {
        const int64_t sl = slot_of(sg);
        ml[i] = __ldcg(reinterpret_cast<const float2*>(p.part_ml + sl * 2));
        x[i] = __ldcg(reinterpret_cast<const float4*>(p.part_o + sl * kDecD) + lane);
      }
    }
    float mb = M;
#pragma unroll
    for (int i = 0; i < 4; ++i) mb = fmaxf(mb, ml[i].x);
    if (mb == -INFINITY) continue;
    const float a = M == -INFINITY ? 0.f : exp2f(M - mb);
    l *= a;
    o4 = make_float4(o4.x * a, o4.y * a, o4.z * a, o4.w * a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float w = ml[i].x == -INFINITY ? 0.f : exp2f(ml[i].x - mb);
      l = fmaf(ml[i].y, w, l);
      o4.x = fmaf(x[i].x, w, o4.x);
      o4.y = fmaf(x[i].y, w, o4.y);
      o4.z = fmaf(x[i].z, w, o4.z);
      o4.w = fmaf(x[i].w, w, o4.w);
    }
    M = mb;
  }
  sm_o[warp][lane] = o4;
  if (lane == 0) {
    sm_m[warp] = M;
    sm_l[warp] = l;
  }
  __syncthreads();
  if (warp == 0) {
    float Mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) Mt = fmaxf(Mt, sm_m[w]);
    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
    float ls = 0.f;
    if (Mt != -INFINITY)
#pragma unroll
      for (int w = 0; w < kMergeWarps; ++w) {
        const float a = sm_m[w] == -INFINITY ? 0.f : exp2f(sm_m[w] - Mt);
        const float4 y = sm_o[w][lane];
        s4.x = fmaf(y.x, a, s4.x);
        s4.y = fmaf(y.y, a, s4.y);
        s4.z = fmaf(y.z, a, s4.z);
        s4.w = fmaf(y.w, a, s4.w);
        ls = fmaf(sm_l[w], a, ls);
      }
    __nv_bfloat162* out = reinterpret_cast<__nv_bfloat162*>(p.O + (int64_t)row * kDecD + 4 * lane);
    out[0] = __floats2bfloat162_rn(ls > 0.f ? s4.x / ls : 0.f, ls > 0.f ? s4.y / ls : 0.f);
    out[1] = __floats2bfloat162_rn(ls > 0.f ? s4.z / ls : 0.f, ls > 0.f ? s4.w / ls : 0.f);
  }
}

// ------------------------------------------------------------------------------ planning
DecPlan attend_dec_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L, int sms) {
  DecPlan pl{};
  const int rows = (h_kv > 0 ? h_q / h_kv : 0) * T;
  pl.ok = d == kDecD && rows >= 1 && rows <= 8 && B >= 1 &&
          (h_kv == 1 || h_kv == 2 || h_kv == 4 || h_kv == 8);
  if (!pl.ok) return pl;
  const int KT = kDecRowsPerTile / h_kv;
  pl.RB = rows <= 4 ? 4 : 8;
  pl.n_pairs = B;  // work owners: queries
  pl.CT = (max_ctx + KT - 1) / KT;
  pl.TPP = pl.CT + (L + KT - 1) / KT;
  pl.total = (int64_t)B * pl.TPP;
  pl.grid = (int)std::min<int64_t>(sms, pl.total);
  const int64_t G = pl.grid;
  auto cta_of = [&](int64_t x) { return ((x + 1) * G + pl.total - 1) / pl.total - 1; };
  int max_seg = 1;
  for (int64_t q = 0; q < B; ++q) {
    const int64_t n = cta_of(q * pl.TPP + pl.TPP - 1) - cta_of(q * pl.TPP) + 1;
    if (n > max_seg) max_seg = (int)n;
  }
  pl.max_seg = max_seg;
  const size_t slots = (size_t)B * max_seg * h_kv * pl.RB;
  pl.ctr_bytes = ((size_t)B * sizeof(unsigned int) + 255) & ~(size_t)255;
  pl.part_ml_bytes = max_seg > 1 ? ((slots * 2 * sizeof(float) + 255) & ~(size_t)255) : 0;
  pl.part_o_bytes = max_seg > 1 ? ((slots * kDecD * sizeof(float) + 255) & ~(size_t)255) : 0;
  // a deeper ring where the shared memory allows it (no combine buffer at h_kv = 8)
  pl.NS = dec_smem(6, h_kv) <= 227 * 1024 ? 6 : kDecStages;
  pl.smem = dec_smem(pl.NS, h_kv);
  return pl;
}

// Plan for a local length known only on the device (1 <= T <= L <= cap): the grid is fixed
// and the kernel cuts the tile list for the live length. A query's TPP tiles out of B * TPP
// meet fewer than G / B + 2 of the G tile ranges, so ceil(G / B) + 1 partial slots suffice.
DecPlan attend_dec_plan_cap(int B, int T, int h_q, int h_kv, int d, int max_ctx, int cap,
                            int sms) {
  DecPlan pl = attend_dec_plan(B, T, h_q, h_kv, d, max_ctx, cap, sms);
  if (!pl.ok) return pl;
  pl.grid = sms;
  const int max_seg = std::min<int64_t>(sms, (sms + B - 1) / B + 1);
  pl.max_seg = max_seg;
  const size_t slots = (size_t)B * max_seg * h_kv * pl.RB;
  pl.part_ml_bytes = (slots * 2 * sizeof(float) + 255) & ~(size_t)255;
  pl.part_o_bytes = (slots * kDecD * sizeof(float) + 255) & ~(size_t)255;
  return pl;
}

cudaError_t launch_attend_dec(const DecParams& p, const DecPlan& pl, cudaStream_t st) {
  // tensor maps of [rows][KV head][d] (bf16, 128-byte swizzle, zero fill out of bounds) read
  // as boxes of [KV head][KT rows][64 dims]: dims (d, rows of all queries, KV head)
  const uint64_t row = (uint64_t)p.h_kv * kDecRow;
  const uint32_t box[3] = {64, (uint32_t)(kDecRowsPerTile / p.h_kv), (uint32_t)p.h_kv};
  const uint64_t str[2] = {row, kDecRow};
  CUtensorMap mkl, mvl, mkc, mvc;
  {
    const uint64_t dims[3] = {kDecD, (uint64_t)p.B * p.Ls, (uint64_t)p.h_kv};
    if (!encode_bf16_map(&mkl, p.Kl, 3, dims, str, box, true) ||
        !encode_bf16_map(&mvl, p.Vl, 3, dims, str, box, true))
      return cudaErrorInvalidValue;
  }
  if (p.max_ctx > 0) {
    const uint64_t dims[3] = {kDecD, (uint64_t)p.B * p.max_ctx, (uint64_t)p.h_kv};
    if (!encode_bf16_map(&mkc, p.cK, 3, dims, str, box, true) ||
        !encode_bf16_map(&mvc, p.cV, 3, dims, str, box, true))
      return cudaErrorInvalidValue;
  } else {  // no memory tiles: never read
    mkc = mkl;
    mvc = mvl;
  }
  cudaError_t e;
  if (p.keys_rotated || !p.rope) {  // keys used as stored: the 16-warp kernel
    e = launch_attend_dec_plain(p, pl, mkc, mvc, mkl, mvl, st);
  } else {
    auto kfn = pl.NS == 6 ? attend_dec_kernel<6> : attend_dec_kernel<kDecStages>;
    e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
    if (e == cudaSuccess) kfn<<<pl.grid, kDecThreads, pl.smem, st>>>(mkc, mvc, mkl, mvl, p);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  // (a fused append needs the merge kernel for the length update even with no split query)
  if (e != cudaSuccess || (pl.max_seg == 1 && p.K_new == nullptr)) return e;
  // split queries: merge their partials (one CTA per output row; y carries the grid size)
  attend_dec_merge_kernel<<<(unsigned)(p.B * p.T * p.h_q), kMergeWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace msa
