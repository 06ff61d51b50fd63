// attend_dec.cu - sparse attention of MSA for decode-shaped queries (at most 8 query rows per
// KV head, bf16, d = 128): a bandwidth-bound stream over [gathered memory ; local context].
//
// Method (the same operation as attend.cu): the query attends over the compressed K/V of the
// routed documents followed by its own local K/V, one softmax, global RoPE on the active
// context: local row j sits at position pos0 + j with pos0 = k, the number of retrieved
// documents, memory rows are used as stored
//   [news.neo-ai.one article, "グローバル RoPE（アクティブコンテキスト）" and "推論パイプライン"].
//
// Kernel design (one CTA per SM: eight compute warps and one copy warp):
//  * The work is the flattened list of 64-key tiles of every (query, KV head) pair: first the
//    tiles of its memory rows, then those of its local rows (each tile holds one kind only);
//    CTA i streams the contiguous tiles [i*total/G, (i+1)*total/G), which may span two pairs.
//    The copy warp moves a tile's K and V as two 16 KB TMA boxes (64 rows of one KV head of a
//    4-D tensor map, rows past the end zero-filled) into a 4-stage ring (full/empty mbarriers),
//    so every SM keeps ~128 KB of loads in flight.
//  * Compute warp w owns keys [8w, 8w + 8) of every tile and keeps its own online-softmax state
//    (running max, sum and P.V accumulators of the RB query rows); the warps meet only at the end
//    of a pair's segment, where their states are combined. No block barrier per tile.
//  * RoPE by angle addition: key c of a local tile whose rows start at position P = pos0 + 64i
//    is rotated by c*theta from a per-CTA table, and the rotation by P*theta moves to the query
//    (<R((P+c)th) k, q> = <R(c th) k, R(-P th) q>); from one local tile to the next the query
//    turns by a fixed -64*theta, so no position table is read or built.
//  * Logits: lane l owns the RoPE pairs 2l and 2l+1 of its warp's eight keys x RB rows and a
//    transposing warp reduction hands each lane finished logits; P.V: lane l owns output dims
//    4l .. 4l+3 (packed fp32 FMA).
//  * A pair split over several CTAs is merged by the last of them to finish (a ticket per
//    pair), from fp32 partial (m, l, o) in the workspace.
// Every wait is bounded; on expiry the CTA records kErrWaitTimeout in the workspace status
// word, skips the remaining waits (all warps still pass every barrier), lets the copies it
// issued land and writes nothing.
#include <cmath>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {

constexpr int kDecCW = 8;                        // compute warps
constexpr int kDecThreads = (kDecCW + 1) * 32;   // + the copy warp
constexpr int kDecKT = 64;      // keys per tile (8 per compute warp)
constexpr int kDecStages = 4;
constexpr int kDecD = 128;
constexpr uint32_t kDecRow = kDecD * 2;              // bytes of one key row of one KV head
constexpr uint32_t kDecHalf = kDecKT * kDecRow;      // K (or V) of a tile: 16 KB
constexpr uint32_t kDecStage = 2 * kDecHalf;

// cos/sin of an angle given in double precision: reduced modulo 2*pi in double, then the
// single-precision sincos of the remainder.
__device__ __forceinline__ float2 rot_of(double a) {
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  const double r = fma(-two_pi, rint(a * inv_two_pi), a);
  float s, c;
  sincosf((float)r, &s, &c);
  return make_float2(c, s);
}

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

// TMA load of a box of a 4-D tensor map into shared memory (no multicast); coordinate 0 (the
// innermost) is always 0 here, so every copy starts on a row boundary.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

template <int RB>
__global__ void __launch_bounds__(kDecThreads, 1)
attend_dec_kernel(const __grid_constant__ CUtensorMap map_kl, const __grid_constant__ CUtensorMap map_vl,
                  const __grid_constant__ CUtensorMap map_kc, const __grid_constant__ CUtensorMap map_vc,
                  DecParams p) {
  constexpr int D = kDecD, HALF = D / 2, KT = kDecKT, NS = kDecStages;
  constexpr int NV = 8 * RB;     // logits per lane before the warp reduction
  constexpr int PER = NV / 32;   // logits per lane after it
  constexpr int WS = 8 * RB + 3 * RB;  // per-warp scratch: probabilities, alpha, max, sum
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* stages = sm;                                                 // [NS][K|V]
  float4* rstep = reinterpret_cast<float4*>(sm + NS * kDecStage);             // [KT][32]
  double* theta = reinterpret_cast<double*>(rstep + KT * 32);                 // [HALF]
  float* comb = reinterpret_cast<float*>(theta + HALF);                       // [8][RB][D]
  float* wscr = comb + kDecCW * RB * D;                                       // [8][WS]
  uint64_t* full = reinterpret_cast<uint64_t*>(wscr + kDecCW * WS);           // [NS]
  uint64_t* empty = full + NS;                                                // [NS]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + NS);
  int* last_flag = const_cast<int*>(abort_flag) + 1;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Gq = p.h_q / p.h_kv;
  const int nr = Gq * p.T;  // query rows per pair (<= RB)
  const int64_t G = gridDim.x, ci = blockIdx.x;
  const int64_t x0 = ci * p.total / G, x1 = (ci + 1) * p.total / G;
  const int n_tiles = (int)(x1 - x0);
  const int pair0 = (int)(x0 / p.TPP), tt0 = (int)(x0 % p.TPP);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < HALF) theta[tid] = p.rope ? pow(p.rope_base, -2.0 * (double)tid / (double)D) : 0.0;
  __syncthreads();

  if (warp == kDecCW) {
    // ---------------- copy warp
    int pair = pair0, tt = tt0, cp = -1, n_ctx = 0;
    int u = 0;
    for (; u < n_tiles; ++u) {
      const int s = u % NS;
      if (u >= NS) {  // the compute warps released this stage
        const bool ok = !*abort_flag && mbar_wait_bounded(&empty[s], (uint32_t)(((u / NS) - 1) & 1), p.err);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
      if (pair != cp) {
        cp = pair;
        n_ctx = min(max(__ldg(p.ctx_len + pair / p.h_kv), 0), p.max_ctx);
      }
      const int b = pair / p.h_kv, g = pair % p.h_kv;
      unsigned char* st = stages + (size_t)s * kDecStage;
      if (tt < p.CT) {  // memory rows [64 tt, 64 tt + 64) (skipped when none is gathered)
        const bool any = tt * KT < n_ctx;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], any ? kDecStage : 0u);
          if (any) {
            tma_load_4d(st, &map_kc, 0, g, tt * KT, b, &full[s]);
            tma_load_4d(st + kDecHalf, &map_vc, 0, g, tt * KT, b, &full[s]);
          }
        }
      } else if (lane == 0) {  // local rows [64 i, 64 i + 64)
        const int j0 = (tt - p.CT) * KT;
        mbar_arrive_expect_tx(&full[s], kDecStage);
        tma_load_4d(st, &map_kl, 0, g, j0, b, &full[s]);
        tma_load_4d(st + kDecHalf, &map_vl, 0, g, j0, b, &full[s]);
      }
      if (++tt == p.TPP) {
        tt = 0;
        ++pair;
      }
    }
    // every copy issued lands before the CTA can exit (bounded; the last NS stages)
    if (lane == 0)
      for (int j = max(0, u - NS); j < u; ++j)
        mbar_wait_bounded(&full[j % NS], (uint32_t)((j / NS) & 1), p.err);
    return;
  }

  // ---------------- compute warps
  // in-tile rotations: rstep[c][l] = (cos, sin) of c*theta for the pairs 2l and 2l+1
  for (int idx = tid; idx < KT * 32; idx += kDecCW * 32) {
    const int c = idx >> 5, l = idx & 31;
    float4 v = make_float4(1.f, 0.f, 1.f, 0.f);
    if (p.rope) {
      const float2 r0 = rot_of((double)c * theta[2 * l]);
      const float2 r1 = rot_of((double)c * theta[2 * l + 1]);
      v = make_float4(r0.x, r0.y, r1.x, r1.y);
    }
    rstep[idx] = v;
  }
  // the query's turn from one tile to the next: R(-64 theta) on the pairs 2 lane, 2 lane + 1
  float2 st0 = make_float2(1.f, 0.f), st1 = make_float2(1.f, 0.f);
  if (p.rope) {
    st0 = rot_of(-(double)KT * theta[2 * lane]);
    st1 = rot_of(-(double)KT * theta[2 * lane + 1]);
  }
  named_sync_compute();  // rstep complete

  float* wp = wscr + warp * WS;  // [8 keys][RB] probabilities
  float* wa = wp + 8 * RB;       // [RB] rescale of this tile
  float* wm = wa + RB;           // [RB] running max
  float* wl = wm + RB;           // [RB] running sum
  float ql[RB][4];               // rotated, pre-scaled query: dims 2l, 2l+1, 2l+64, 2l+65
  float qa[RB][4];               // ql turned back by the tile's start position
  float2 acc[RB][2];             // P.V: dims 4l .. 4l+3
  int pair = pair0, tt = tt0, cur = -1, n_ctx = 0;

  // combine the warps' states of the open segment; write O or a partial; the last segment of
  // a pair merges the partials
  auto finish_segment = [&](int fp) {
#pragma unroll
    for (int r = 0; r < RB; ++r)
      *reinterpret_cast<float4*>(comb + (warp * RB + r) * D + 4 * lane) =
          make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
    const bool write = !named_sync_compute_or(*abort_flag != 0);  // one decision for all warps
    const int b = fp / p.h_kv, g = fp % p.h_kv;
    const int64_t first = dec_cta_of((int64_t)fp * p.TPP, G, p.total);
    const int64_t last = dec_cta_of((int64_t)fp * p.TPP + p.TPP - 1, G, p.total);
    const int n_seg = (int)(last - first + 1);
    const int seg = (int)(ci - first);
    for (int idx = tid; idx < nr * D; idx += kDecCW * 32) {
      const int r = idx / D, e = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecCW; ++w) M = fmaxf(M, wscr[w * WS + 9 * RB + r]);
      float o = 0.f, l = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kDecCW; ++w) {
          const float m = wscr[w * WS + 9 * RB + r];
          const float a = m == -INFINITY ? 0.f : exp2f(m - M);
          o = fmaf(comb[(w * RB + r) * D + e], a, o);
          l = fmaf(wscr[w * WS + 10 * RB + r], a, l);
        }
      }
      const int t = r / Gq, h = g * Gq + r % Gq;
      if (!write) continue;
      if (n_seg == 1) {
        p.O[(((int64_t)b * p.T + t) * p.h_q + h) * D + e] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
      } else {
        const int64_t slot = ((int64_t)fp * p.max_seg + seg) * RB + r;
        p.part_o[slot * D + e] = o;
        if (e == 0) {
          p.part_ml[slot * 2] = M;
          p.part_ml[slot * 2 + 1] = l;
        }
      }
    }
    if (n_seg > 1 && write) {
      __threadfence();
      named_sync_compute();
      if (tid == 0) *last_flag = atomicAdd(p.counters + fp, 1u) == (unsigned)(n_seg - 1);
      named_sync_compute();
      if (*last_flag) {
        __threadfence();
        for (int idx = tid; idx < nr * D; idx += kDecCW * 32) {
          const int r = idx / D, e = idx % D;
          const int64_t s0 = (int64_t)fp * p.max_seg * RB + r;
          float M = -INFINITY;
          for (int sg = 0; sg < n_seg; ++sg)
            M = fmaxf(M, __ldcg(p.part_ml + (s0 + (int64_t)sg * RB) * 2));
          float l = 0.f, o = 0.f;
          if (M != -INFINITY)
            for (int sg = 0; sg < n_seg; ++sg) {
              const int64_t sl = s0 + (int64_t)sg * RB;
              const float m = __ldcg(p.part_ml + sl * 2);
              const float a = m == -INFINITY ? 0.f : exp2f(m - M);
              l = fmaf(__ldcg(p.part_ml + sl * 2 + 1), a, l);
              o = fmaf(__ldcg(p.part_o + sl * D + e), a, o);
            }
          const int t = r / Gq, h = g * Gq + r % Gq;
          p.O[(((int64_t)b * p.T + t) * p.h_q + h) * D + e] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
        }
      }
    }
    named_sync_compute();  // comb and the warps' scratch are reused by the next segment
  };

  bool qa_ok = false;  // qa matches the current local tile
  for (int u = 0; u < n_tiles; ++u) {
    const int b = pair / p.h_kv, g = pair % p.h_kv;
    const bool is_ctx = tt < p.CT;
    const int kt = is_ctx ? tt * KT : (tt - p.CT) * KT;  // first memory row / first local row
    if (pair != cur) {
      if (cur >= 0) finish_segment(cur);
      cur = pair;
      n_ctx = min(max(__ldg(p.ctx_len + b), 0), p.max_ctx);
      // rotated, pre-scaled query rows of this pair (each warp keeps its own copy)
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (r < nr) {
          const int t = r / Gq, h = g * Gq + r % Gq;
          const __nv_bfloat16* q = p.Q + (((int64_t)b * p.T + t) * p.h_q + h) * D;
          const uint32_t lo = __ldg(reinterpret_cast<const unsigned int*>(q + 2 * lane));
          const uint32_t hi = __ldg(reinterpret_cast<const unsigned int*>(q + HALF + 2 * lane));
          const float a0 = __uint_as_float(lo << 16), a1 = __uint_as_float(lo & 0xFFFF0000u);
          const float c0 = __uint_as_float(hi << 16), c1 = __uint_as_float(hi & 0xFFFF0000u);
          float2 r0 = make_float2(1.f, 0.f), r1 = make_float2(1.f, 0.f);
          if (p.rope) {
            const double pos = (double)(p.pos0 + p.L - p.T + t);
            r0 = rot_of(pos * theta[2 * lane]);
            r1 = rot_of(pos * theta[2 * lane + 1]);
          }
          x[0] = (a0 * r0.x - c0 * r0.y) * p.scale_log2;
          x[2] = (c0 * r0.x + a0 * r0.y) * p.scale_log2;
          x[1] = (a1 * r1.x - c1 * r1.y) * p.scale_log2;
          x[3] = (c1 * r1.x + a1 * r1.y) * p.scale_log2;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) ql[r][i] = x[i];
        acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
      }
      qa_ok = false;
      if (lane < RB) {
        wm[lane] = -INFINITY;
        wl[lane] = 0.f;
      }
      __syncwarp();
    }
    const int nk = is_ctx ? min(max(n_ctx - kt, 0), KT) : min(p.L - kt, KT);
    if (!is_ctx && !qa_ok) {  // the query turned back by the tile's start position P
      float2 t0 = make_float2(1.f, 0.f), t1 = make_float2(1.f, 0.f);
      if (p.rope) {
        const double P = (double)((int64_t)p.pos0 + kt);
        t0 = rot_of(-P * theta[2 * lane]);
        t1 = rot_of(-P * theta[2 * lane + 1]);
      }
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        qa[r][0] = ql[r][0] * t0.x - ql[r][2] * t0.y;
        qa[r][2] = ql[r][2] * t0.x + ql[r][0] * t0.y;
        qa[r][1] = ql[r][1] * t1.x - ql[r][3] * t1.y;
        qa[r][3] = ql[r][3] * t1.x + ql[r][1] * t1.y;
      }
      qa_ok = true;
    }
    const int s = u % NS;
    if (!*abort_flag && !mbar_wait_bounded(&full[s], (uint32_t)((u / NS) & 1), p.err))
      *abort_flag = 1;
    const unsigned char* stg = stages + (size_t)s * kDecStage;

    // ---- logits of this warp's keys x RB rows
    float v[NV];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int j = warp * 8 + kk;
      const uint32_t wlo = *reinterpret_cast<const uint32_t*>(stg + j * kDecRow + 4 * lane);
      const uint32_t whi = *reinterpret_cast<const uint32_t*>(stg + j * kDecRow + 2 * HALF + 4 * lane);
      const float x0 = __uint_as_float(wlo << 16), x1 = __uint_as_float(wlo & 0xFFFF0000u);
      const float y0 = __uint_as_float(whi << 16), y1 = __uint_as_float(whi & 0xFFFF0000u);
      if (!is_ctx) {  // local row: rotate by c * theta within the tile
        const float4 R = rstep[j * 32 + lane];
        const float a0 = x0 * R.x - y0 * R.y, b0 = y0 * R.x + x0 * R.y;
        const float a1 = x1 * R.z - y1 * R.w, b1 = y1 * R.z + x1 * R.w;
#pragma unroll
        for (int r = 0; r < RB; ++r)
          v[kk * RB + r] = fmaf(qa[r][0], a0, fmaf(qa[r][1], a1, fmaf(qa[r][2], b0, qa[r][3] * b1)));
      } else {  // memory row: as stored, against the unshifted query
#pragma unroll
        for (int r = 0; r < RB; ++r)
          v[kk * RB + r] = fmaf(ql[r][0], x0, fmaf(ql[r][1], x1, fmaf(ql[r][2], y0, ql[r][3] * y1)));
      }
    }
    tr_reduce<NV, 16>(v, lane);

    // ---- online softmax over the warp's 8 keys: lane holds (key lane / 4, row (lane*PER+e) % RB)
    {
      const int kk = lane >> 2;
      const int jrow = kt + warp * 8 + kk;  // memory row or local row
      float pe[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int r = (lane * PER + e) % RB;
        const int t = r / Gq;
        const bool vis = warp * 8 + kk < nk && r < nr && (is_ctx || jrow <= p.L - p.T + t);
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
        v[e] = mn;     // reuse: new max of row r
        v[PER + e] = sum;  // and the tile's sum (NV >= 2 * PER)
      }
      __syncwarp();  // every lane read the old maxima
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int r = (lane * PER + e) % RB;
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
        const int j = warp * 8 + kk;
        if (j >= nk) break;
        const uint2 w = *reinterpret_cast<const uint2*>(vt + j * kDecRow + 8 * lane);
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
    // next local tile: advance the position by 64 (turn the query back by 64 theta)
    if (!is_ctx)
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      const float a0 = qa[r][0] * st0.x - qa[r][2] * st0.y, b0 = qa[r][2] * st0.x + qa[r][0] * st0.y;
      const float a1 = qa[r][1] * st1.x - qa[r][3] * st1.y, b1 = qa[r][3] * st1.x + qa[r][1] * st1.y;
      qa[r][0] = a0; qa[r][2] = b0; qa[r][1] = a1; qa[r][3] = b1;
    }
    if (++tt == p.TPP) {
      tt = 0;
      ++pair;
    }
  }
  if (cur >= 0) finish_segment(cur);
}

// ------------------------------------------------------------------------------ planning
DecPlan attend_dec_plan(int B, int T, int h_q, int h_kv, int d, int max_ctx, int L, int sms) {
  DecPlan pl{};
  const int rows = (h_q / h_kv) * T;
  pl.ok = d == kDecD && rows >= 1 && rows <= 8 && B >= 1;
  if (!pl.ok) return pl;
  pl.RB = rows <= 4 ? 4 : 8;
  pl.n_pairs = (int64_t)B * h_kv;
  pl.CT = (max_ctx + kDecKT - 1) / kDecKT;
  pl.TPP = pl.CT + (L + kDecKT - 1) / kDecKT;
  pl.total = pl.n_pairs * pl.TPP;
  pl.grid = (int)std::min<int64_t>(sms, pl.total);
  const int64_t G = pl.grid;
  auto cta_of = [&](int64_t x) { return ((x + 1) * G + pl.total - 1) / pl.total - 1; };
  int max_seg = 1;
  for (int64_t pr = 0; pr < pl.n_pairs; ++pr) {
    const int64_t n = cta_of(pr * pl.TPP + pl.TPP - 1) - cta_of(pr * pl.TPP) + 1;
    if (n > max_seg) max_seg = (int)n;
  }
  pl.max_seg = max_seg;
  const size_t slots = (size_t)pl.n_pairs * max_seg * pl.RB;
  pl.ctr_bytes = ((size_t)pl.n_pairs * sizeof(unsigned int) + 255) & ~(size_t)255;
  pl.part_ml_bytes = max_seg > 1 ? ((slots * 2 * sizeof(float) + 255) & ~(size_t)255) : 0;
  pl.part_o_bytes = max_seg > 1 ? ((slots * kDecD * sizeof(float) + 255) & ~(size_t)255) : 0;
  pl.smem = 1024 + (size_t)kDecStages * kDecStage + (size_t)kDecKT * 32 * 16 + (kDecD / 2) * 8 +
            sizeof(float) * ((size_t)kDecCW * pl.RB * kDecD + (size_t)kDecCW * 11 * pl.RB) +
            2 * kDecStages * 8 + 16;
  return pl;
}

cudaError_t launch_attend_dec(const DecParams& p, const DecPlan& pl, cudaStream_t st) {
  // 4-D maps (d, KV head, row, query) with 64-row boxes of one KV head
  CUtensorMap mkl, mvl, mkc, mvc;
  const uint64_t row = (uint64_t)kDecD * 2;
  const uint32_t box[4] = {(uint32_t)kDecD, 1u, (uint32_t)kDecKT, 1u};
  const uint64_t dl[4] = {(uint64_t)kDecD, (uint64_t)p.h_kv, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sl[3] = {row, row * p.h_kv, row * p.h_kv * p.L};
  if (!encode_bf16_map(&mkl, p.Kl, 4, dl, sl, box) || !encode_bf16_map(&mvl, p.Vl, 4, dl, sl, box))
    return cudaErrorInvalidValue;
  if (p.max_ctx > 0) {
    const uint64_t dc[4] = {(uint64_t)kDecD, (uint64_t)p.h_kv, (uint64_t)p.max_ctx, (uint64_t)p.B};
    const uint64_t sc[3] = {row, row * p.h_kv, row * p.h_kv * p.max_ctx};
    if (!encode_bf16_map(&mkc, p.cK, 4, dc, sc, box) || !encode_bf16_map(&mvc, p.cV, 4, dc, sc, box))
      return cudaErrorInvalidValue;
  } else {  // no memory tiles: never read
    mkc = mkl;
    mvc = mvl;
  }
  cudaError_t e = cudaSuccess;
  if (pl.RB == 4) {
    e = cudaFuncSetAttribute(attend_dec_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)pl.smem);
    if (e == cudaSuccess)
      attend_dec_kernel<4><<<pl.grid, kDecThreads, pl.smem, st>>>(mkl, mvl, mkc, mvc, p);
  } else {
    e = cudaFuncSetAttribute(attend_dec_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)pl.smem);
    if (e == cudaSuccess)
      attend_dec_kernel<8><<<pl.grid, kDecThreads, pl.smem, st>>>(mkl, mvl, mkc, mvc, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace msa
