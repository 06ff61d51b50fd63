// attend_dec_plain.cu - decode-shaped sparse attention over keys used as stored: the memory rows
// of the routed documents and a local context whose keys are already rotated at their global
// positions (the cache of sparse generation, which rotates each key once when it is appended,
// or any call without RoPE). The operation is that of attend_dec.cu
//   [news.neo-ai.one article, "グローバル RoPE（アクティブコンテキスト）" and "推論パイプライン";
//    ruixiangma.github.io blog, "三阶段推理流程"]:
// the query, rotated at its global position, attends over [gathered memory ; local context].
//
// Why a second kernel: with no key to rotate, a warp needs no fp32 copy of the query for the
// per-tile turn nor the key-rotation tables, so its live state (the packed bf16 query
// fragments, the P.V accumulators) fits 128 registers and a CTA runs 16 compute warps instead
// of 8. The stream is latency-bound at 8 warps per SM (fixed-latency dependencies between the
// warp-level MMAs, the softmax shuffles and the shared-memory fragment loads), so twice the
// warps hide twice the latency. Design otherwise as attend_dec.cu: one CTA per SM over a
// contiguous range of the flattened (query, tile) list, tiles of 64 / h_kv key rows x all KV
// heads (16 KB of K and 16 KB of V by four 128-byte-swizzled TMA boxes) in a 4-stage ring;
// the warps form two groups of eight that take alternate tiles (stages u % 4 with u even belong
// to group 0, odd to group 1; the last warp of a group to release a stage refills it); warp w
// of a group owns KV head w % h_kv and eight key rows of the tile, with its own online softmax;
// at the end of each query's segment the 16 warps combine (two per head and key slot) and
// write O, or this CTA's partial, which attend_dec_merge_kernel folds.
// Every wait is bounded; on expiry the CTA records kErrWaitTimeout in the workspace status
// word, skips the remaining waits, lets the copies it issued land and writes nothing.
#include "common.cuh"
#include "kernels.cuh"

namespace msa {
namespace adp {

constexpr int kGroups = 2;
constexpr int kGroupWarps = 8;
constexpr int kCW = kGroups * kGroupWarps;   // compute warps
constexpr int kThreads = kCW * 32;
constexpr int kRowsPerTile = 64;             // key rows x KV heads per tile
constexpr int kStages = 4;
constexpr int kD = 128;
constexpr uint32_t kRow = kD * 2;
constexpr uint32_t kHalf = kRowsPerTile * kRow;  // K (or V) of a tile: 16 KB
constexpr uint32_t kStage = 2 * kHalf;
constexpr int kWS = 11 * 8;                      // per-warp scratch floats

__device__ __forceinline__ int64_t cta_of(int64_t x, int64_t G, int64_t total) {
  return ((x + 1) * G + total - 1) / total - 1;
}
__device__ __forceinline__ void sync_compute() {
  asm volatile("bar.sync 1, 512;" ::: "memory");
}
__device__ __forceinline__ bool sync_compute_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 512, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
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

__global__ void __launch_bounds__(kThreads, 1)
attend_dec_plain_kernel(const __grid_constant__ CUtensorMap map_kc,
                        const __grid_constant__ CUtensorMap map_vc,
                        const __grid_constant__ CUtensorMap map_kl,
                        const __grid_constant__ CUtensorMap map_vl, DecParams p) {
  constexpr int D = kD, HALF = D / 2, NS = kStages;
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* sm = smem_align1024(sm_raw);
  unsigned char* stages = sm;                                              // [NS][K | V]
  float4* qrot = reinterpret_cast<float4*>(sm + NS * kStage);              // [T][32]
  const int RB = (p.h_q / p.h_kv) * p.T <= 4 ? 4 : 8;  // combine-buffer rows per KV head
  float* comb = reinterpret_cast<float*>(qrot + 8 * 32);                   // [16][RB][D]
  float* wscr = comb + kCW * RB * D;                   // [16][WS]: max at 9 RB, sum at 10 RB
  uint64_t* full = reinterpret_cast<uint64_t*>(wscr + kCW * kWS);          // [NS]
  unsigned int* released = reinterpret_cast<unsigned int*>(full + NS);     // [NS]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(released + NS);
  // copies issued into each stage (its latest copy is the only one that can be in flight)
  unsigned int* issued = reinterpret_cast<unsigned int*>(const_cast<int*>(abort_flag) + 1);
  __shared__ int skip_call;
  __shared__ int ctx_first[32];  // context rows of the CTA's first 32 queries

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = warp / kGroupWarps, lw = warp % kGroupWarps;
  const int HKV = p.h_kv;
  const int KT = kRowsPerTile / HKV;  // key rows per tile
  const int Gq = p.h_q / HKV;
  const int nr = Gq * p.T;            // query rows per KV head (<= 8)
  // local rows per query: fixed, read from the device, or (fused append) the device length
  // plus the T tokens this call appends
  const bool fused = p.K_new != nullptr;
  if (p.start_status && !fused && blockIdx.x == 0 && tid == 0) *p.err = 0;
  const int L = fused ? *reinterpret_cast<const volatile int32_t*>(p.L_dev) + p.T
                      : (p.L_dev != nullptr ? *p.L_dev : p.L);
  const bool bad = L < p.T || L > p.Ls;  // uniform over the grid: nothing is read or written
  if (fused && blockIdx.x == 0 && tid == 0) {
    // the first CTA starts the call's status word (another CTA records an error only after a
    // bounded wait has run out, long after every CTA started) and hands the new length to the
    // merge kernel
    *p.err = bad ? kErrCtxOverflow : 0;
    *p.L_out = bad ? -1 : L;
  }
  if (bad) {
    if (!fused && blockIdx.x == 0 && tid == 0) set_err(p.err, kErrBadIndex);
    return;
  }
  const int TPP = p.CT + (L + KT - 1) / KT;  // tiles per query
  const int64_t total = (int64_t)p.B * TPP;
  const int64_t G = min((int64_t)gridDim.x, total), ci = blockIdx.x;
  if (ci >= G) return;
  const int64_t x0 = ci * total / G, x1 = (ci + 1) * total / G;
  const int n_tiles = (int)(x1 - x0);
  const int b_first = (int)(x0 / TPP);

  // Copies of tile v of this CTA's range into stage v % NS: four TMA boxes of
  // [KV head][key row][64 dims] (128-byte swizzle), the K and V halves of d.
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
    const uint32_t st = smem_u32(stages + (size_t)s * kStage);
    fence_proxy_async_smem();  // the stage's earlier reads come before the new writes
    mbar_arrive_expect_tx(&full[s], any ? kStage : 0u);
    if (any) {
      const CUtensorMap* mk = ctx ? &map_kc : &map_kl;
      const CUtensorMap* mv = ctx ? &map_vc : &map_vl;
      const int y = ctx ? bb * p.max_ctx + kt : bb * p.Ls + kt;
      tma3d(st, mk, 0, y, &full[s]);
      tma3d(st + kHalf / 2, mk, HALF, y, &full[s]);
      tma3d(st + kHalf, mv, 0, y, &full[s]);
      tma3d(st + kHalf + kHalf / 2, mv, HALF, y, &full[s]);
    }
    atomicAdd(&issued[s], 1u);
  };
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      released[s] = 0u;
      issued[s] = 0u;
    }
    *abort_flag = 0;
    skip_call = (!fused && p.skip_on_err && *reinterpret_cast<volatile int*>(p.err) != 0) ? 1 : 0;
    fence_mbar_init();
    // the first copies go out before the tables are built, so the prologue overlaps them
    // (none when the call is skipped: a CTA never exits with a copy in flight)
    if (!skip_call)
      for (int v = 0; v < min(NS, n_tiles); ++v) issue(v, false);
  }
  if (tid < 32)
    ctx_first[tid] =
        b_first + tid < p.B ? min(max(__ldg(p.ctx_len + b_first + tid), 0), p.max_ctx) : 0;
  // R(pos theta) at each query token's position, (cos, cos, sin, sin) of the pairs 2pp, 2pp+1
  for (int idx = tid; idx < p.T * 32; idx += kThreads) {
    const int r = idx >> 5, pp = idx & 31;
    const int64_t n = (int64_t)p.pos0 + L - p.T + r;
    const float2 r0 = p.rope ? rot_turns(n, p.rope_turns[2 * pp]) : make_float2(1.f, 0.f);
    const float2 r1 = p.rope ? rot_turns(n, p.rope_turns[2 * pp + 1]) : make_float2(1.f, 0.f);
    qrot[idx] = make_float4(r0.x, r1.x, r0.y, r1.y);
  }
  __syncthreads();
  if (skip_call) return;
  auto ctx_rows = [&](int bb) {
    return bb - b_first < 32 ? ctx_first[bb - b_first]
                             : min(max(__ldg(p.ctx_len + bb), 0), p.max_ctx);
  };


  // ---------------- compute warps
  const int g = lw % HKV;      // KV head of this warp
  const int sl = lw / HKV;     // its eight key rows of a tile: [8 sl, 8 sl + 8)
  const int gr = lane >> 2;    // fragment row: query row gr (logits) / key 8 sl + gr (keys)
  const int t4 = lane & 3;     // fragment column pair
  // ldmatrix row address of this lane for fragment m: key row 8 sl + (lane & 7) of KV head g,
  // dim chunk 4 (m & 1) + (lane >> 3) of the half m >> 1 (128-byte swizzle: chunk ^ (line & 7))
  const int line = g * KT + 8 * sl + (lane & 7);
  const uint32_t lbase = (uint32_t)(line * 128);
  const uint32_t lx0 = (uint32_t)(((lane >> 3) ^ (line & 7)) << 4);
  const uint32_t lx1 = (uint32_t)(((4 + (lane >> 3)) ^ (line & 7)) << 4);
  auto lofs = [&](int m) -> uint32_t {
    return (uint32_t)((m >> 1) * (kHalf / 2)) + lbase + ((m & 1) ? lx1 : lx0);
  };
  const int WPH = kCW / HKV;  // warps per KV head
  // Fused append of new local row j (token t = j - (L - T)) of query bb, KV head g, line
  // g * KT + r of the tile: K rotated at its position pos0 + j (the query's table entry t; the
  // formula of kv_append), V as given; written into the tile in shared memory (128-byte
  // swizzle: 16-byte chunk c of a line at c ^ (line & 7)) and into the cache. Lane l: RoPE
  // pairs 2l, 2l+1 (dims 2l, 2l+1 and their partners + 64) of K, dims 4l..4l+3 of V.
  auto append_row = [&](int bb, int j, int r, uint32_t kb, uint32_t vb) {
    const int t = j - (L - p.T);
    const int line = g * KT + r;
    const int64_t src = (((int64_t)bb * p.T + t) * HKV + g) * D;
    const int64_t dst = (((int64_t)bb * p.Ls + j) * HKV + g) * D;
    const float2 x = bf2_unpack(__ldg(reinterpret_cast<const unsigned int*>(p.K_new + src) + lane));
    const float2 y =
        bf2_unpack(__ldg(reinterpret_cast<const unsigned int*>(p.K_new + src + HALF) + lane));
    const float4 cs = qrot[t * 32 + lane];  // (cos, cos, sin, sin) of pairs 2l, 2l+1
    const uint32_t xr = bf2_pack(make_float2(x.x * cs.x - y.x * cs.z, x.y * cs.y - y.y * cs.w));
    const uint32_t yr = bf2_pack(make_float2(y.x * cs.x + x.x * cs.z, y.y * cs.y + x.y * cs.w));
    const uint32_t ko = (uint32_t)(line * 128 + ((((lane >> 2) ^ (line & 7))) << 4) + (lane & 3) * 4);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(kb + ko), "r"(xr) : "memory");
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(kb + kHalf / 2 + ko), "r"(yr) : "memory");
    unsigned int* kc = reinterpret_cast<unsigned int*>(const_cast<__nv_bfloat16*>(p.Kl) + dst);
    kc[lane] = xr;
    kc[HALF / 2 + lane] = yr;
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.V_new + src) + lane);
    const int hv = lane >> 4, cv = (lane & 15) >> 1;  // half of d, 16-byte chunk in the half
    const uint32_t vo = (uint32_t)(hv * (kHalf / 2) + line * 128 + ((cv ^ (line & 7)) << 4) +
                                   (lane & 1) * 8);
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(vb + vo), "r"(v.x), "r"(v.y)
                 : "memory");
    reinterpret_cast<uint2*>(const_cast<__nv_bfloat16*>(p.Vl) + dst)[lane] = v;
    __syncwarp();  // the row is in the tile before the warp's fragment loads
  };

  uint32_t qa[4][4];  // the query rows of head g in fragment order, rotated, scaled, bf16
  float2 o[16];       // P.V accumulators of row gr: dims 8 nt + 2 t4, +1
  float mrow = -INFINITY, lsum = 0.f;

  // combine the 16 warps over the segment of query fb; write O (a query within one CTA) or
  // this CTA's partial
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
        wscr[warp * kWS + 9 * RB + gr] = mrow;
        wscr[warp * kWS + 10 * RB + gr] = l;
      }
    }
    const bool write = !sync_compute_or(*abort_flag != 0);  // one decision for all warps
    if (leader && write && gr < nr) {
      float M = mrow;
      for (int k2 = 1; k2 < WPH; ++k2) M = fmaxf(M, wscr[(g + k2 * HKV) * kWS + 9 * RB + gr]);
      const float a0 = mrow == -INFINITY ? 0.f : exp2f(mrow - M);
      float2* ov = o;  // the segment's accumulators are folded in place
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) ov[nt] = __fmul2_rn(o[nt], make_float2(a0, a0));
      float lv = l * a0;
      for (int k2 = 1; k2 < WPH; ++k2) {
        const int w = g + k2 * HKV;
        const float m = wscr[w * kWS + 9 * RB + gr];
        const float a = m == -INFINITY ? 0.f : exp2f(m - M);
        const float2* cw = reinterpret_cast<const float2*>(comb) + w * 16 * (RB * 4);
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
          ov[nt] = __ffma2_rn(cw[nt * (RB * 4) + lane], make_float2(a, a), ov[nt]);
        lv = fmaf(wscr[w * kWS + 10 * RB + gr], a, lv);
      }
      const int64_t first = cta_of((int64_t)fb * TPP, G, total);
      const int64_t last = cta_of((int64_t)fb * TPP + TPP - 1, G, total);
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
    if (WPH > 1) sync_compute();  // the shared fragments are refilled by the next segment
  };

  int64_t x = x0;
  while (x < x1) {  // one query's segment of the CTA's range at a time, all 16 warps
    const int b = (int)(x / TPP);
    const int64_t xe = min(x1, (int64_t)(b + 1) * TPP);
    const int n_ctx = ctx_rows(b);
    {  // the query rows of KV head g, rotated at their positions and pre-scaled, in bf16
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
          qa[m][qq] = bf2_pack(lo);
          qa[m + 2][qq] = bf2_pack(hi);
        }
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt] = make_float2(0.f, 0.f);
    mrow = -INFINITY;
    lsum = 0.f;
    for (int64_t xx = x; xx < xe; ++xx) {
      const int u = (int)(xx - x0);
      if ((u & 1) != grp) continue;  // the other group's tile
      const int tt = (int)(xx % TPP);
      const bool is_ctx = tt < p.CT;
      const int kt = is_ctx ? tt * KT : (tt - p.CT) * KT;
      const int nk = is_ctx ? min(max(n_ctx - kt, 0), KT) : min(L - kt, KT);
      const int s = u % NS;
      if (!*abort_flag && !mbar_wait_bounded(&full[s], (uint32_t)((u / NS) & 1), p.err))
        *abort_flag = 1;
      const uint32_t kb = smem_u32(stages + (size_t)s * kStage), vb = kb + kHalf;
      if (fused && !is_ctx) {  // this warp's rows of the tile that the call appends
        const int r0 = kt + 8 * sl;
        const int j1 = min(r0 + 8, L);
        for (int j = max(r0, L - p.T); j < j1; ++j) append_row(b, j, j - kt, kb, vb);
      }

      // ---- logits S[row gr][keys 8 sl + 2 t4, +1]: 8 MMAs over d in four chains
      uint32_t kr[4][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) ldsm_x4(kb + lofs(m), kr[m]);
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          mma_k16(sa[m], sb[m], qa[m][2 * hh], qa[m][2 * hh + 1], kr[m][2 * hh],
                  kr[m][2 * hh + 1]);
      const float s0 = (sa[0] + sa[1]) + (sa[2] + sa[3]), s1 = (sb[0] + sb[1]) + (sb[2] + sb[3]);

      // ---- online softmax of row gr over this warp's 8 keys (a lane holds keys 2 t4, +1)
      const int jj = 8 * sl + 2 * t4;
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

      // ---- P.V: 16 MMAs; V rows of keys past the tile's valid rows are cleared
      const uint32_t vmask = (k0 ? 0x0000FFFFu : 0u) | (k1 ? 0xFFFF0000u : 0u);
      const bool partial = __any_sync(0xffffffffu, vmask != 0xFFFFFFFFu);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t vr[4];
        ldsm_x4_trans(vb + lofs(m), vr);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const uint32_t bv = partial ? (vr[qq] & vmask) : vr[qq];
          mma_k8(o[4 * m + qq].x, o[4 * m + qq].y, pa, bv);
        }
      }
      __syncwarp();
      // release the stage; the last of the group's eight warps refills it with tile u + NS
      // (the same parity: the same group's)
      if (lane == 0 &&
          atomicAdd(&released[s], 1u) % kGroupWarps == kGroupWarps - 1 && u + NS < n_tiles &&
          !*abort_flag)
        issue(u + NS, true);
    }
    finish_segment(b);
    x = xe;
  }
  // every copy issued lands before the CTA exits (bounded)
  sync_compute();
  if (tid == 0)
    for (int s = 0; s < NS; ++s) {
      const unsigned int n = *reinterpret_cast<volatile unsigned int*>(&issued[s]);
      if (n > 0u) mbar_wait_bounded(&full[s], (n - 1u) & 1u, p.err);
    }
}

}  // namespace adp

size_t attend_dec_plain_smem(int RB) {
  return 1024 + (size_t)adp::kStages * adp::kStage + (size_t)8 * 32 * 16 +
         sizeof(float) * ((size_t)adp::kCW * RB * adp::kD + (size_t)adp::kCW * adp::kWS) +
         adp::kStages * 16 + 16;
}

cudaError_t launch_attend_dec_plain(const DecParams& p, const DecPlan& pl, const CUtensorMap& mkc,
                                    const CUtensorMap& mvc, const CUtensorMap& mkl,
                                    const CUtensorMap& mvl, cudaStream_t st) {
  const size_t smem = attend_dec_plain_smem(pl.RB);
  cudaError_t e = cudaFuncSetAttribute(adp::attend_dec_plain_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  adp::attend_dec_plain_kernel<<<pl.grid, adp::kThreads, smem, st>>>(mkc, mvc, mkl, mvl, p);
  return cudaGetLastError();
}

}  // namespace msa
