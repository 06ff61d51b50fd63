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
// Kernel design (one CTA per SM: eight compute warps and one copy warp):
//  * A tile is KT = 64 / h_kv consecutive key rows of one query with all their KV heads: one
//    contiguous 16 KB block of K and one of V ([row][KV head][d] is the storage order), so the
//    copy warp moves a tile with two one-dimensional bulk copies and DRAM sees long sequential
//    reads. Per query the memory rows come first, then the local rows (a tile holds one kind).
//    The flattened tile list of all queries is cut into one contiguous range per CTA; a 4-stage
//    ring (full/empty mbarriers) keeps ~128 KB of loads in flight per SM.
//  * Compute warp w owns KV head w % h_kv and eight key rows of every tile, with its own online
//    softmax state (running max, sum, P.V accumulators of its head's query rows); the warps
//    meet only at the end of a query's segment (no block barrier per tile).
//  * RoPE by angle addition: key c of a local tile whose rows start at position P is rotated by
//    c*theta from a per-CTA table, and the rotation by P*theta moves to the query
//    (<R((P+c)th) k, q> = <R(c th) k, R(-P th) q>); from one local tile to the next the query
//    turns by a fixed -KT*theta, so no position table is read or built. Angles are exact
//    integer turn counts (64-bit fixed point) fed to a single-precision sincospi.
//  * Logits: the lanes split each key's RoPE pairs (16 lanes per key for 4 query rows, 32 for
//    8) and a transposing reduction hands each lane finished logits; P.V: lane l owns output
//    dims 4l .. 4l+3; packed fp32 FMA throughout.
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
constexpr int kDecThreads = (kDecCW + 1) * 32;   // + the copy warp
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

template <int RB>
__global__ void __launch_bounds__(kDecThreads, 1) attend_dec_kernel(DecParams p) {
  constexpr int D = kDecD, HALF = D / 2, NS = kDecStages;
  constexpr int LPK = RB == 4 ? 16 : 32;  // lanes sharing one key's dims in the logits
  constexpr int NG = 32 / LPK;            // key groups per warp
  constexpr int KG = 8 / NG;              // keys per group
  constexpr int PPL = HALF / LPK;         // RoPE pairs per lane (4 or 2)
  constexpr int PH = PPL / 2;             // packed float2 of pairs per lane
  constexpr int NV = KG * RB;             // logits per lane before the group reduction
  constexpr int PER = NV / LPK;           // logits per lane after it (RB / 4)
  constexpr int WS = 8 * RB + 3 * RB;     // per-warp scratch: probabilities, alpha, max, sum
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* stages = sm;                                                 // [NS][K|V]
  float4* rstep = reinterpret_cast<float4*>(sm + NS * kDecStage);             // [KT][32]
  unsigned long long* turns = reinterpret_cast<unsigned long long*>(rstep + 64 * 32);  // [HALF]
  float* comb = reinterpret_cast<float*>(turns + HALF);                       // [8][RB][D]
  float* wscr = comb + kDecCW * RB * D;                                       // [8][WS]
  uint64_t* full = reinterpret_cast<uint64_t*>(wscr + kDecCW * WS);           // [NS]
  uint64_t* empty = full + NS;                                                // [NS]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
  __shared__ int skip_call;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HKV = p.h_kv;
  const int KT = kDecRowsPerTile / HKV;  // key rows per tile
  const int Gq = p.h_q / HKV;
  const int nr = Gq * p.T;  // query rows per KV head (<= RB)
  // local rows per query: fixed, or read from the device (a cache that grows between launches)
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

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecCW);
    }
    *abort_flag = 0;
    // an error an earlier kernel of the same call recorded (a failed append) skips the call
    skip_call = (p.skip_on_err && *reinterpret_cast<volatile int*>(p.err) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  if (tid < HALF) turns[tid] = p.rope_turns[tid];
  __syncthreads();
  if (skip_call) return;  // written once before the barrier: one value for the whole CTA

  if (warp == kDecCW) {
    // ---------------- copy warp (lane 0): tile u -> stage u % NS
    if (lane == 0) {
      int b = b_first, tt = tt_first, cb = -1, n_ctx = 0;
      const int64_t row_elems = (int64_t)HKV * D;  // one key row, all KV heads
      int u = 0;
      for (; u < n_tiles; ++u) {
        const int s = u % NS;
        if (u >= NS) {  // the compute warps released this stage
          const bool ok = !*abort_flag &&
                          mbar_wait_bounded(&empty[s], (uint32_t)(((u / NS) - 1) & 1), p.err);
          if (!ok) {
            *abort_flag = 1;
            break;
          }
        }
        if (b != cb) {
          cb = b;
          n_ctx = min(max(__ldg(p.ctx_len + b), 0), p.max_ctx);
        }
        int nk;
        const __nv_bfloat16 *ks, *vs;
        if (tt < p.CT) {  // memory rows [KT tt, KT tt + KT)
          const int kt = tt * KT;
          nk = min(max(n_ctx - kt, 0), KT);
          const int64_t off = ((int64_t)b * p.max_ctx + kt) * row_elems;
          ks = p.cK + off;
          vs = p.cV + off;
        } else {  // local rows [KT i, KT i + KT)
          const int j0 = (tt - p.CT) * KT;
          nk = min(L - j0, KT);
          const int64_t off = ((int64_t)b * p.Ls + j0) * row_elems;
          ks = p.Kl + off;
          vs = p.Vl + off;
        }
        const uint32_t bytes = (uint32_t)nk * (uint32_t)HKV * kDecRow;
        unsigned char* st = stages + (size_t)s * kDecStage;
        mbar_arrive_expect_tx(&full[s], 2u * bytes);
        if (bytes) {
          bulk_g2s(st, ks, bytes, &full[s]);
          bulk_g2s(st + kDecHalf, vs, bytes, &full[s]);
        }
        if (++tt == TPP) {
          tt = 0;
          ++b;
        }
      }
      // every copy issued lands before the CTA can exit (bounded; the last NS stages)
      for (int j = max(0, u - NS); j < u; ++j)
        mbar_wait_bounded(&full[j % NS], (uint32_t)((j / NS) & 1), p.err);
    }
    return;
  }

  // ---------------- compute warps
  const int g = warp % HKV;    // KV head of this warp
  const int sl = warp / HKV;   // its eight key rows of a tile: [8 sl, 8 sl + 8)
  const int grp = lane / LPK, dl = lane % LPK;
  const int i0 = PPL * dl;     // first RoPE pair of this lane in the logits
  // in-tile rotations: rstep[c][pp] = (cos, cos, sin, sin) of c*theta for the pairs 2pp, 2pp+1
  for (int idx = tid; idx < KT * 32; idx += kDecCW * 32) {
    const int c = idx >> 5, pp = idx & 31;
    const float2 r0 = rot_turns(c, turns[2 * pp]), r1 = rot_turns(c, turns[2 * pp + 1]);
    rstep[idx] = make_float4(r0.x, r1.x, r0.y, r1.y);
  }
  // the query's turn from one local tile to the next: R(-KT theta) on the lane's pairs
  float2 stc[PH], sts[PH];  // (cos, cos), (sin, sin) of the packed pairs
#pragma unroll
  for (int h = 0; h < PH; ++h) {
    const float2 r0 = rot_turns(-KT, turns[i0 + 2 * h]), r1 = rot_turns(-KT, turns[i0 + 2 * h + 1]);
    stc[h] = make_float2(r0.x, r1.x);
    sts[h] = make_float2(r0.y, r1.y);
  }
  named_sync_compute();  // rstep complete

  float* wp = wscr + warp * WS;  // [8 keys][RB] probabilities
  float* wa = wp + 8 * RB;       // [RB] rescale of this tile
  float* wm = wa + RB;           // [RB] running max
  float* wl = wm + RB;           // [RB] running sum
  // rotated, pre-scaled query on this lane's pairs, packed by two: lo = dims i0 + 2h, +1,
  // hi = the same + 64; ql as rotated, qa turned back by the local tile's start position
  float2 ql_lo[RB][PH], ql_hi[RB][PH], qa_lo[RB][PH], qa_hi[RB][PH];
  float2 acc[RB][2];             // P.V: dims 4l .. 4l+3
  int b = b_first, tt = tt_first, cur = -1, n_ctx = 0;
  const int WPH = kDecCW / HKV;  // warps per KV head

  // combine the warps of each KV head over the open segment of query fb; write O (a query
  // within one CTA) or this CTA's partial
  auto finish_segment = [&](int fb) {
#pragma unroll
    for (int r = 0; r < RB; ++r)
      *reinterpret_cast<float4*>(comb + (warp * RB + r) * D + 4 * lane) =
          make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
    const bool write = !named_sync_compute_or(*abort_flag != 0);  // one decision for all warps
    const int64_t first = dec_cta_of((int64_t)fb * TPP, G, total);
    const int64_t last = dec_cta_of((int64_t)fb * TPP + TPP - 1, G, total);
    const int n_seg = (int)(last - first + 1);
    const int seg = (int)(ci - first);
    const int n_out = HKV * nr * D;
    for (int idx = tid; idx < n_out; idx += kDecCW * 32) {
      const int gh = idx / (nr * D), r = (idx / D) % nr, e = idx % D;
      float M = -INFINITY;
      for (int k2 = 0; k2 < WPH; ++k2) M = fmaxf(M, wscr[(gh + k2 * HKV) * WS + 9 * RB + r]);
      float o = 0.f, l = 0.f;
      if (M != -INFINITY)
        for (int k2 = 0; k2 < WPH; ++k2) {
          const int w = gh + k2 * HKV;
          const float m = wscr[w * WS + 9 * RB + r];
          const float a = m == -INFINITY ? 0.f : exp2f(m - M);
          o = fmaf(comb[(w * RB + r) * D + e], a, o);
          l = fmaf(wscr[w * WS + 10 * RB + r], a, l);
        }
      if (!write) continue;
      const int t = r / Gq, h = gh * Gq + r % Gq;
      if (n_seg == 1) {
        p.O[(((int64_t)fb * p.T + t) * p.h_q + h) * D + e] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
      } else {
        const int64_t slot = (((int64_t)fb * p.max_seg + seg) * HKV + gh) * RB + r;
        p.part_o[slot * D + e] = o;
        if (e == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = l;
        }
      }
    }
    named_sync_compute();  // comb and the warps' scratch are reused by the next segment
  };

  bool qa_ok = false;  // qa matches the current local tile
  for (int u = 0; u < n_tiles; ++u) {
    const bool is_ctx = tt < p.CT;
    const int kt = is_ctx ? tt * KT : (tt - p.CT) * KT;  // first memory row / first local row
    if (b != cur) {
      if (cur >= 0) finish_segment(cur);
      cur = b;
      n_ctx = min(max(__ldg(p.ctx_len + b), 0), p.max_ctx);
      // rotated, pre-scaled query rows of this warp's KV head
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        float xl[PPL], xh[PPL];
#pragma unroll
        for (int m = 0; m < PPL; ++m) xl[m] = xh[m] = 0.f;
        if (r < nr) {
          const int t = r / Gq, h = g * Gq + r % Gq;
          const __nv_bfloat16* q = p.Q + (((int64_t)b * p.T + t) * p.h_q + h) * D;
          const int64_t pos = (int64_t)p.pos0 + L - p.T + t;
#pragma unroll
          for (int m = 0; m < PPL; ++m) {
            const float a = __bfloat162float(q[i0 + m]), c = __bfloat162float(q[i0 + m + HALF]);
            const float2 cs = rot_turns(pos, turns[i0 + m]);
            xl[m] = (a * cs.x - c * cs.y) * p.scale_log2;
            xh[m] = (c * cs.x + a * cs.y) * p.scale_log2;
          }
        }
#pragma unroll
        for (int hh = 0; hh < PH; ++hh) {
          ql_lo[r][hh] = make_float2(xl[2 * hh], xl[2 * hh + 1]);
          ql_hi[r][hh] = make_float2(xh[2 * hh], xh[2 * hh + 1]);
        }
        acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
      }
      qa_ok = false;
      if (lane < RB) {
        wm[lane] = -INFINITY;
        wl[lane] = 0.f;
      }
      __syncwarp();
    }
    const int nk = is_ctx ? min(max(n_ctx - kt, 0), KT) : min(L - kt, KT);
    if (!is_ctx && !qa_ok) {  // the query turned back by the tile's start position P
      const int64_t P = (int64_t)p.pos0 + kt;
#pragma unroll
      for (int hh = 0; hh < PH; ++hh) {
        const float2 r0 = rot_turns(-P, turns[i0 + 2 * hh]);
        const float2 r1 = rot_turns(-P, turns[i0 + 2 * hh + 1]);
        const float2 c2 = make_float2(r0.x, r1.x), s2 = make_float2(r0.y, r1.y);
        const float2 ns2 = make_float2(-s2.x, -s2.y);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          qa_lo[r][hh] = __ffma2_rn(ql_lo[r][hh], c2, __fmul2_rn(ql_hi[r][hh], ns2));
          qa_hi[r][hh] = __ffma2_rn(ql_hi[r][hh], c2, __fmul2_rn(ql_lo[r][hh], s2));
        }
      }
      qa_ok = true;
    }
    const int s = u % NS;
    if (!*abort_flag && !mbar_wait_bounded(&full[s], (uint32_t)((u / NS) & 1), p.err))
      *abort_flag = 1;
    const unsigned char* stg = stages + (size_t)s * kDecStage;

    // ---- logits of this warp's eight keys x RB rows: lane group grp takes keys
    // [KG grp, KG grp + KG) of them, lane dl of the group the RoPE pairs [PPL dl, PPL dl + PPL)
    float v[NV];
#pragma unroll
    for (int kk = 0; kk < KG; ++kk) {
      const int j = 8 * sl + grp * KG + kk;  // key row within the tile
      const unsigned char* row = stg + (j * HKV + g) * kDecRow;
      float2 x2[PH], y2[PH];
      if constexpr (PPL == 4) {
        const uint2 lo = *reinterpret_cast<const uint2*>(row + 2 * i0);
        const uint2 hi = *reinterpret_cast<const uint2*>(row + 2 * HALF + 2 * i0);
        x2[0] = make_float2(__uint_as_float(lo.x << 16), __uint_as_float(lo.x & 0xFFFF0000u));
        x2[1] = make_float2(__uint_as_float(lo.y << 16), __uint_as_float(lo.y & 0xFFFF0000u));
        y2[0] = make_float2(__uint_as_float(hi.x << 16), __uint_as_float(hi.x & 0xFFFF0000u));
        y2[1] = make_float2(__uint_as_float(hi.y << 16), __uint_as_float(hi.y & 0xFFFF0000u));
      } else {
        const uint32_t lo = *reinterpret_cast<const uint32_t*>(row + 2 * i0);
        const uint32_t hi = *reinterpret_cast<const uint32_t*>(row + 2 * HALF + 2 * i0);
        x2[0] = make_float2(__uint_as_float(lo << 16), __uint_as_float(lo & 0xFFFF0000u));
        y2[0] = make_float2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xFFFF0000u));
      }
      if (!is_ctx) {  // local row: rotate by c * theta within the tile, dot with qa
#pragma unroll
        for (int hh = 0; hh < PH; ++hh) {
          const float4 R = rstep[j * 32 + i0 / 2 + hh];
          const float2 c2 = make_float2(R.x, R.y), s2 = make_float2(R.z, R.w);
          const float2 a2 = __ffma2_rn(x2[hh], c2, __fmul2_rn(y2[hh], make_float2(-s2.x, -s2.y)));
          const float2 b2 = __ffma2_rn(y2[hh], c2, __fmul2_rn(x2[hh], s2));
          x2[hh] = a2;
          y2[hh] = b2;
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          float2 t2 = __fmul2_rn(qa_lo[r][0], x2[0]);
          t2 = __ffma2_rn(qa_hi[r][0], y2[0], t2);
#pragma unroll
          for (int hh = 1; hh < PH; ++hh) {
            t2 = __ffma2_rn(qa_lo[r][hh], x2[hh], t2);
            t2 = __ffma2_rn(qa_hi[r][hh], y2[hh], t2);
          }
          v[kk * RB + r] = t2.x + t2.y;
        }
      } else {  // memory row: as stored, against the unshifted query
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          float2 t2 = __fmul2_rn(ql_lo[r][0], x2[0]);
          t2 = __ffma2_rn(ql_hi[r][0], y2[0], t2);
#pragma unroll
          for (int hh = 1; hh < PH; ++hh) {
            t2 = __ffma2_rn(ql_lo[r][hh], x2[hh], t2);
            t2 = __ffma2_rn(ql_hi[r][hh], y2[hh], t2);
          }
          v[kk * RB + r] = t2.x + t2.y;
        }
      }
    }
    tr_reduce<NV, LPK / 2>(v, lane);

    // ---- online softmax over the warp's 8 keys: lane holds the logits of the warp's key
    // grp * KG + (dl * PER + e) / RB and row (dl * PER + e) % RB
    {
      const int kk = grp * KG + (dl * PER) / RB;
      const int jrow = kt + 8 * sl + kk;  // memory row or local row
      float pe[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int r = (dl * PER + e) % RB;
        const int t = r / Gq;
        const bool vis = 8 * sl + kk < nk && r < nr && (is_ctx || jrow <= L - p.T + t);
        float x = vis ? v[e] : -INFINITY;
        float mx = x;
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mo = wm[r];
        const float mn = fmaxf(mo, mx);
        const float pr = (x == -INFINITY) ? 0.f : exp2f(x - mn);
        float sum = pr;
        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
        sum += __shfl_xor_sync(0xffffffffu, sum, 8);
        sum += __shfl_xor_sync(0xffffffffu, sum, 16);
        pe[e] = pr;
        v[e] = mn;         // reuse: new max of row r
        v[PER + e] = sum;  // and the tile's sum (NV >= 2 * PER)
      }
      __syncwarp();  // every lane read the old maxima
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int r = (dl * PER + e) % RB;
        wp[kk * RB + r] = pe[e];
        if (kk == 0) {
          const float mo = wm[r], mn = v[e];
          const float alpha = mn == -INFINITY ? 1.f : (mo == -INFINITY ? 0.f : exp2f(mo - mn));
          wa[r] = alpha;
          wm[r] = mn;
          wl[r] = fmaf(wl[r], alpha, v[PER + e]);
        }
      }
      __syncwarp();
    }
    // ---- P.V over the warp's 8 keys: dims 4l .. 4l+3
    {
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const float a = wa[r];
        acc[r][0].x *= a; acc[r][0].y *= a; acc[r][1].x *= a; acc[r][1].y *= a;
      }
      const unsigned char* vt = stg + kDecHalf;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int j = 8 * sl + kk;
        if (j >= nk) break;
        const uint2 w = *reinterpret_cast<const uint2*>(vt + (j * HKV + g) * kDecRow + 8 * lane);
        const float2 v01 = make_float2(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u));
        const float2 v23 = make_float2(__uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
#pragma unroll
        for (int r4 = 0; r4 < RB; r4 += 4) {
          const float4 pr = *reinterpret_cast<const float4*>(wp + kk * RB + r4);
          const float pv[4] = {pr.x, pr.y, pr.z, pr.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 pp = make_float2(pv[i], pv[i]);
            acc[r4 + i][0] = __ffma2_rn(pp, v01, acc[r4 + i][0]);
            acc[r4 + i][1] = __ffma2_rn(pp, v23, acc[r4 + i][1]);
          }
        }
      }
      __syncwarp();  // probabilities and rescale are rewritten by the next tile
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // next local tile: advance the position by KT (turn the query back by KT theta)
    if (!is_ctx) {
#pragma unroll
      for (int hh = 0; hh < PH; ++hh) {
        const float2 ns2 = make_float2(-sts[hh].x, -sts[hh].y);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const float2 lo = __ffma2_rn(qa_lo[r][hh], stc[hh], __fmul2_rn(qa_hi[r][hh], ns2));
          const float2 hi = __ffma2_rn(qa_hi[r][hh], stc[hh], __fmul2_rn(qa_lo[r][hh], sts[hh]));
          qa_lo[r][hh] = lo;
          qa_hi[r][hh] = hi;
        }
      }
    }
    if (++tt == TPP) {
      tt = 0;
      ++b;
    }
  }
  if (cur >= 0) finish_segment(cur);
}

// Merge of the partials of the queries split over several CTAs: CTA = one output row (query b,
// query head h, token t); warp w folds segments w, w + 8, ... with lane l on dims 4l .. 4l+3,
// then the eight warps combine in shared memory.
constexpr int kMergeWarps = 8;
__global__ void __launch_bounds__(kMergeWarps * 32) attend_dec_merge_kernel(DecParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int HKV = p.h_kv, Gq = p.h_q / HKV;
  const int row = blockIdx.x;  // ((b * T + t) * h_q + h)
  const int h = row % p.h_q, t = (row / p.h_q) % p.T, b = row / (p.h_q * p.T);
  const int gh = h / Gq, r = t * Gq + h % Gq;
  const int RB = (Gq * p.T) <= 4 ? 4 : 8;
  const int L = p.L_dev != nullptr ? *p.L_dev : p.L;
  if (L < p.T || L > p.Ls) return;  // reported by the attention kernel
  if (p.skip_on_err && *reinterpret_cast<volatile int*>(p.err) != 0) return;
  const int KT = kDecRowsPerTile / HKV;
  const int TPP = p.CT + (L + KT - 1) / KT;
  const int64_t total = (int64_t)p.B * TPP, G = min((int64_t)p.grid, total);
  const int64_t first = dec_cta_of((int64_t)b * TPP, G, total);
  const int64_t last = dec_cta_of((int64_t)b * TPP + TPP - 1, G, total);
  const int n_seg = (int)(last - first + 1);
  if (n_seg == 1) return;  // written directly by the attention kernel
  __shared__ float sm_l[kMergeWarps];
  __shared__ float4 sm_o[kMergeWarps][32];
  auto slot_of = [&](int sg) { return (((int64_t)b * p.max_seg + sg) * HKV + gh) * RB + r; };
  // the row's maximum over all segments
  float M = -INFINITY;
  for (int sg = lane; sg < n_seg; sg += 32) M = fmaxf(M, __ldcg(p.part_ml + slot_of(sg) * 2));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float l = 0.f;
  float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
#pragma unroll 2
    for (int sg = warp; sg < n_seg; sg += kMergeWarps) {
      const int64_t sl = slot_of(sg);
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + sl * 2));
      const float4 x = __ldcg(reinterpret_cast<const float4*>(p.part_o + sl * kDecD) + lane);
      const float a = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
      l = fmaf(ml.y, a, l);
      o4.x = fmaf(x.x, a, o4.x);
      o4.y = fmaf(x.y, a, o4.y);
      o4.z = fmaf(x.z, a, o4.z);
      o4.w = fmaf(x.w, a, o4.w);
    }
  }
  sm_o[warp][lane] = o4;
  if (lane == 0) sm_l[warp] = l;
  __syncthreads();
  if (warp == 0) {
    float4 s4 = sm_o[0][lane];
    float ls = sm_l[0];
#pragma unroll
    for (int w = 1; w < kMergeWarps; ++w) {
      const float4 y = sm_o[w][lane];
      s4.x += y.x; s4.y += y.y; s4.z += y.z; s4.w += y.w;
      ls += sm_l[w];
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
  pl.smem = 1024 + (size_t)kDecStages * kDecStage + (size_t)64 * 32 * 16 + (kDecD / 2) * 8 +
            sizeof(float) * ((size_t)kDecCW * pl.RB * kDecD + (size_t)kDecCW * 11 * pl.RB) +
            2 * kDecStages * 8 + 16;
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
  cudaError_t e = cudaSuccess;
  if (pl.RB == 4) {
    e = cudaFuncSetAttribute(attend_dec_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)pl.smem);
    if (e == cudaSuccess) attend_dec_kernel<4><<<pl.grid, kDecThreads, pl.smem, st>>>(p);
  } else {
    e = cudaFuncSetAttribute(attend_dec_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)pl.smem);
    if (e == cudaSuccess) attend_dec_kernel<8><<<pl.grid, kDecThreads, pl.smem, st>>>(p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || pl.max_seg == 1) return e;
  // split queries: merge their partials (one CTA per output row; y carries the grid size)
  attend_dec_merge_kernel<<<(unsigned)(p.B * p.T * p.h_q), kMergeWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace msa
