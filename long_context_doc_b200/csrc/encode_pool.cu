// encode_pool.cu - offline memory encoding of MSA: document-wise RoPE on K and K_r fused with
// fixed-length chunk mean pooling of K, V and K_r, plus the fp32 inverse norms of the pooled
// router keys. One streaming pass over the per-token tensors (HBM-bound).
//
// Method: chunk-wise mean pooling compresses each document's K/V/K_r
//   [news.neo-ai.one article, "全体設計 / アーキテクチャ"; ruixiangma.github.io blog
//    "Memory-Sparse-Attention", "稀疏注意力机制 / 分块压缩"], with document-wise ("parallel")
//   RoPE whose positions restart at 0 in every document
//   [news.neo-ai.one, "並列（ドキュメント単位）RoPE"; ruixiangma blog, "文档级RoPE"].
//
// Layout: each CTA pools a contiguous range of chunks (the owning document advances with the
// chunk, no search per chunk). A thread owns one "pair group": E consecutive
// elements of the first half of a head and the E elements they pair with in the second half
// (RoPE rotates element i with i + d/2), for TP-strided tokens of the chunk; TP lanes that
// share a pair group sit next to each other in the warp and are reduced with shuffles.
// RoPE is linear, so sum_t R((P + c_t) theta) x_t = R(P theta) sum_t R(c_t theta) x_t: for chunks
// of at most 64 tokens one shared table of R(c theta), c < 64, built once per CTA, serves every
// chunk, and the chunk's sums are turned by its start position P once (longer chunks rebuild the
// table per 64-token block). Every cos/sin comes from the exact angle mod 2 pi (integer
// position x 64-bit fixed-point theta / 2 pi) through a single-precision sincospi; the padded
// table rows give conflict-free 16-byte reads.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {


template <typename T, int E, int D, int TP, bool SINGLE>
__global__ void __launch_bounds__(256) encode_pool_kernel(EncodeParams p) {
  constexpr int HALF = D / 2;
  constexpr int SUBS = HALF / E;     // pair groups per head
  constexpr int TB = 64;             // positions per cos/sin table block
  constexpr int ROW = HALF + 2;      // padded table row (float2 units)
  using V = Vec<T, E>;
  using raw = typename V::raw;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float2* cs = reinterpret_cast<float2*>(smem_raw);                 // [TB][ROW]
  unsigned long long* turns = reinterpret_cast<unsigned long long*>(cs + TB * ROW);  // [HALF]
  float* ssp = reinterpret_cast<float*>(turns + HALF);              // [PG] partial sum sq

  const int PG = p.h_kv * SUBS;
  const int tid = threadIdx.x;
  const int tp = tid % TP;
  const int pg = tid / TP;
  const bool active = pg < PG;
  const int h = pg / SUBS;
  const int e1 = (pg % SUBS) * E;    // first-half element offset within the head
  const int W = p.h_kv * D;          // row length
  const bool rope = p.rope != 0;

  if (rope) {
    for (int i = tid; i < HALF; i += blockDim.x) turns[i] = p.rope_turns[i];
    if constexpr (SINGLE) {  // in-chunk offsets 0 .. 63, shared by every chunk
      __syncthreads();
      for (int idx = tid; idx < TB * HALF; idx += blockDim.x) {
        const int pl = idx / HALF, i = idx % HALF;
        cs[pl * ROW + i] = rot_turns(pl, turns[i]);
      }
    }
  }
  __syncthreads();

  const T* K = static_cast<const T*>(p.K);
  const T* Vt = static_cast<const T*>(p.V);
  const T* Kr = static_cast<const T*>(p.Kr);

  const int64_t c_begin = (int64_t)blockIdx.x * p.n_chunks / gridDim.x;
  const int64_t c_end = ((int64_t)blockIdx.x + 1) * p.n_chunks / gridDim.x;
  // document owning chunk c: off[doc] <= c < off[doc+1] (found once, then advanced)
  int64_t doc = c_begin < c_end ? lower_bound_i64(p.chunk_off, p.n_docs, c_begin + 1) - 1 : 0;
  for (int64_t c = c_begin; c < c_end; ++c) {
    while (p.chunk_off[doc + 1] <= c) ++doc;
    const int64_t j = c - p.chunk_off[doc];
    const int64_t tdoc = p.tok_off[doc];
    const int64_t t0 = tdoc + j * p.chunk;
    int64_t t1 = t0 + p.chunk;
    if (t1 > p.tok_off[doc + 1]) t1 = p.tok_off[doc + 1];
    const int n = (int)(t1 - t0);
    const int64_t pos0 = j * p.chunk;  // position of the chunk's first token in its doc

    float k1[E], k2[E], r1[E], r2[E], v1[E], v2[E];
#pragma unroll
    for (int e = 0; e < E; ++e) k1[e] = k2[e] = r1[e] = r2[e] = v1[e] = v2[e] = 0.f;

    for (int sb = 0; sb < n; sb += TB) {
      const int nb = min(TB, n - sb);
      if (!SINGLE && rope) {
        __syncthreads();  // the previous table block is no longer read
        for (int idx = tid; idx < nb * HALF; idx += blockDim.x) {
          const int pl = idx / HALF, i = idx % HALF;
          cs[pl * ROW + i] = rot_turns(pos0 + sb + pl, turns[i]);
        }
        __syncthreads();
      }
      if (active) {
#pragma unroll 2
        for (int tl = tp; tl < nb; tl += TP) {
          const int64_t base = (t0 + sb + tl) * (int64_t)W + (int64_t)h * D + e1;
          float a1[E], a2[E], b1[E], b2[E], c1[E], c2[E];
          V::unpack(*reinterpret_cast<const raw*>(K + base), a1);
          V::unpack(*reinterpret_cast<const raw*>(K + base + HALF), a2);
          V::unpack(*reinterpret_cast<const raw*>(Kr + base), b1);
          V::unpack(*reinterpret_cast<const raw*>(Kr + base + HALF), b2);
          V::unpack(*reinterpret_cast<const raw*>(Vt + base), c1);
          V::unpack(*reinterpret_cast<const raw*>(Vt + base + HALF), c2);
          if (rope) {
            const float2* row = cs + tl * ROW + e1;
#pragma unroll
            for (int e = 0; e < E; ++e) {
              const float2 t = row[e];
              k1[e] += a1[e] * t.x - a2[e] * t.y;
              k2[e] += a2[e] * t.x + a1[e] * t.y;
              r1[e] += b1[e] * t.x - b2[e] * t.y;
              r2[e] += b2[e] * t.x + b1[e] * t.y;
            }
          } else {
#pragma unroll
            for (int e = 0; e < E; ++e) {
              k1[e] += a1[e]; k2[e] += a2[e]; r1[e] += b1[e]; r2[e] += b2[e];
            }
          }
#pragma unroll
          for (int e = 0; e < E; ++e) { v1[e] += c1[e]; v2[e] += c2[e]; }
        }
      }
    }

    if (SINGLE && rope) {  // turn the sums by the chunk's start position
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float2 t = rot_turns(pos0, turns[e1 + e]);
        const float a = k1[e] * t.x - k2[e] * t.y, b = k2[e] * t.x + k1[e] * t.y;
        k1[e] = a;
        k2[e] = b;
        const float ar = r1[e] * t.x - r2[e] * t.y, br = r2[e] * t.x + r1[e] * t.y;
        r1[e] = ar;
        r2[e] = br;
      }
    }
    // reduce over the TP lanes sharing this pair group (adjacent lanes)
#pragma unroll
    for (int o = TP / 2; o > 0; o >>= 1) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        k1[e] += __shfl_xor_sync(0xffffffffu, k1[e], o);
        k2[e] += __shfl_xor_sync(0xffffffffu, k2[e], o);
        r1[e] += __shfl_xor_sync(0xffffffffu, r1[e], o);
        r2[e] += __shfl_xor_sync(0xffffffffu, r2[e], o);
        v1[e] += __shfl_xor_sync(0xffffffffu, v1[e], o);
        v2[e] += __shfl_xor_sync(0xffffffffu, v2[e], o);
      }
    }

    if (active) {
      const float fn = (float)n;
      const int64_t ob = c * (int64_t)W + (int64_t)h * D + e1;
      T* Kb = static_cast<T*>(p.Kb);
      T* Vb = static_cast<T*>(p.Vb);
      T* Rb = static_cast<T*>(p.Rb);
      float ss = 0.f;
      // every lane of the TP group holds the totals; lane tp stores vectors tp, tp+TP, ...
#pragma unroll
      for (int vct = 0; vct < 6; ++vct) {
        const bool mine = (vct % TP) == tp;
        const float* src = vct == 0 ? k1 : vct == 1 ? k2 : vct == 2 ? r1 : vct == 3 ? r2
                         : vct == 4 ? v1 : v2;
        T* dst = (vct < 2 ? Kb : vct < 4 ? Rb : Vb) + ob + ((vct & 1) ? HALF : 0);
        T out[E];
#pragma unroll
        for (int e = 0; e < E; ++e) out[e] = Elem<T>::from_f(src[e] / fn);
        if (mine) *reinterpret_cast<raw*>(dst) = *reinterpret_cast<const raw*>(out);
        if (vct == 2 || vct == 3) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float s = Elem<T>::to_f(out[e]);
            ss += s * s;
          }
        }
      }
      if (tp == 0) ssp[pg] = ss;
    }
    __syncthreads();
    if (p.inv_norm != nullptr) {
      for (int hh = tid; hh < p.h_kv; hh += blockDim.x) {
        float s = 0.f;
        for (int q = 0; q < SUBS; ++q) s += ssp[hh * SUBS + q];
        p.inv_norm[c * p.h_kv + hh] = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
      }
    }
    __syncthreads();
  }
}

// Status word of the pooling encode (bounded waits of encode_pool_tma_kernel), zeroed by
// each call's chunk-offset kernel, read by msa_encode_pool_status.
__device__ int g_encode_status;

// The same pooling for bf16, d = 128, chunks of at most 64 tokens and h_kv <= 8, fed by the
// bulk-copy engine: one CTA per SM over a contiguous chunk range; warp 0 copies each chunk's
// token rows (contiguous in [token][KV head][d]) of K, V and K_r in blocks of kEpTB tokens into
// a kEpNS-stage ring (one 1-D bulk copy per tensor and block, completion counted in bytes on
// the stage's mbarrier); consumer warp h owns KV head h, lane l its RoPE pairs 2l, 2l+1 (dims
// 2l, 2l+1 and their partners + 64), and reads a block's rows from shared memory (a warp reads
// 128 contiguous bytes per row half). Each thread sums its pairs over the chunk's tokens in
// order (keys rotated by c*theta from the per-CTA table, c the offset in the chunk), turns the
// sums by the chunk's start position, divides by the token count and stores the means; the
// warp reduces the squares of its head's bf16 K̄_r for the inverse norm. No shuffle
// reduction and no barrier between chunks: the copies of the next blocks are in flight while a
// chunk is finished.
constexpr int kEpTB = 8;   // tokens per copy block
constexpr int kEpNS = 4;   // ring stages
__global__ void __launch_bounds__(32 + 8 * 32, 1) encode_pool_tma_kernel(EncodeParams p) {
  constexpr int D = 128, HALF = 64;
  const int W = p.h_kv * D;                  // elements of a token row
  const uint32_t row_bytes = (uint32_t)W * 2;
  const uint32_t blk_bytes = kEpTB * row_bytes;  // one tensor's block in a stage
  extern __shared__ __align__(1024) unsigned char sm_raw[];
  unsigned char* stages = smem_align1024(sm_raw);                          // [NS][K|V|Kr]
  float2* cs = reinterpret_cast<float2*>(stages + kEpNS * 3 * blk_bytes);  // [64][64]
  unsigned long long* turns = reinterpret_cast<unsigned long long*>(cs + 64 * HALF);  // [64]
  uint64_t* full = reinterpret_cast<uint64_t*>(turns + HALF);             // [NS]
  uint64_t* empty = full + kEpNS;                                           // [NS]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kEpNS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool rope = p.rope != 0;
  const int64_t c_begin = (int64_t)blockIdx.x * p.n_chunks / gridDim.x;
  const int64_t c_end = ((int64_t)blockIdx.x + 1) * p.n_chunks / gridDim.x;
  if (tid == 0) {
    for (int s = 0; s < kEpNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], p.h_kv);  // one arrival per consumer warp
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (rope) {
    for (int i = tid; i < HALF; i += blockDim.x) turns[i] = p.rope_turns[i];
    __syncthreads();
    for (int idx = tid; idx < 64 * HALF; idx += blockDim.x)
      cs[idx] = rot_turns(idx / HALF, turns[idx % HALF]);  // R(c theta), c < 64
  }
  __syncthreads();
  int64_t doc = c_begin < c_end ? lower_bound_i64(p.chunk_off, p.n_docs, c_begin + 1) - 1 : 0;

  if (warp == 0) {
    // ---------------- copies
    if (lane == 0) {
      const unsigned char* src[3] = {static_cast<const unsigned char*>(p.K),
                                     static_cast<const unsigned char*>(p.V),
                                     static_cast<const unsigned char*>(p.Kr)};
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t c = c_begin; c < c_end && !*abort_flag; ++c) {
        while (p.chunk_off[doc + 1] <= c) ++doc;
        const int64_t t0 = p.tok_off[doc] + (c - p.chunk_off[doc]) * p.chunk;
        const int n = (int)(min(t0 + p.chunk, p.tok_off[doc + 1]) - t0);
        for (int tb = 0; tb < n; tb += kEpTB) {
          const uint32_t bytes = (uint32_t)min(kEpTB, n - tb) * row_bytes;
          if (issued >= kEpNS && !mbar_wait_bounded(&empty[s], ph ^ 1u, &g_encode_status)) {
            *abort_flag = 1;
            break;
          }
          unsigned char* st = stages + (size_t)s * 3 * blk_bytes;
          mbar_arrive_expect_tx(&full[s], 3 * bytes);
#pragma unroll
          for (int q = 0; q < 3; ++q)
            bulk_g2s(st + q * blk_bytes, src[q] + (t0 + tb) * (int64_t)row_bytes, bytes, &full[s]);
          ++issued;
          if (++s == kEpNS) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // every copy issued lands before the CTA exits (bounded)
      for (int64_t j = (issued > kEpNS ? issued - kEpNS : 0); j < issued; ++j)
        mbar_wait_bounded(&full[j % kEpNS], (uint32_t)((j / kEpNS) & 1), &g_encode_status);
    }
    return;
  }
  // ---------------- consumers: warp h = KV head h - 1 + 1 (warps 1..h_kv)
  const int h = warp - 1;
  if (h >= p.h_kv) return;
  const int e1 = 2 * lane;  // first-half dims e1, e1 + 1 of the head; partners + 64
  const uint32_t col = (uint32_t)(h * D + e1) * 2;  // byte offset of dims e1, e1+1 in a row
  int s = 0;
  uint32_t ph = 0;
  bool ok = true;
  for (int64_t c = c_begin; c < c_end; ++c) {
    while (p.chunk_off[doc + 1] <= c) ++doc;
    const int64_t j = c - p.chunk_off[doc];
    const int64_t t0 = p.tok_off[doc] + j * p.chunk;
    const int n = (int)(min(t0 + p.chunk, p.tok_off[doc + 1]) - t0);
    float k1[2] = {0.f, 0.f}, k2[2] = {0.f, 0.f}, r1[2] = {0.f, 0.f}, r2[2] = {0.f, 0.f};
    float v1[2] = {0.f, 0.f}, v2[2] = {0.f, 0.f};
    for (int tb = 0; tb < n; tb += kEpTB) {
      const int nt = min(kEpTB, n - tb);
      if (ok && !mbar_wait_bounded(&full[s], ph, &g_encode_status)) {
        ok = false;
        *abort_flag = 1;
      }
      if (ok) {
        const unsigned char* st = stages + (size_t)s * 3 * blk_bytes + col;
#pragma unroll 4
        for (int t = 0; t < nt; ++t) {
          const unsigned char* rk = st + t * row_bytes;
          const uint32_t ka = *reinterpret_cast<const uint32_t*>(rk);
          const uint32_t kb = *reinterpret_cast<const uint32_t*>(rk + HALF * 2);
          const uint32_t va = *reinterpret_cast<const uint32_t*>(rk + blk_bytes);
          const uint32_t vb = *reinterpret_cast<const uint32_t*>(rk + blk_bytes + HALF * 2);
          const uint32_t ra = *reinterpret_cast<const uint32_t*>(rk + 2 * blk_bytes);
          const uint32_t rb = *reinterpret_cast<const uint32_t*>(rk + 2 * blk_bytes + HALF * 2);
          const float a[2] = {__uint_as_float(ka << 16), __uint_as_float(ka & 0xFFFF0000u)};
          const float b[2] = {__uint_as_float(kb << 16), __uint_as_float(kb & 0xFFFF0000u)};
          const float x[2] = {__uint_as_float(ra << 16), __uint_as_float(ra & 0xFFFF0000u)};
          const float y[2] = {__uint_as_float(rb << 16), __uint_as_float(rb & 0xFFFF0000u)};
          v1[0] += __uint_as_float(va << 16);
          v1[1] += __uint_as_float(va & 0xFFFF0000u);
          v2[0] += __uint_as_float(vb << 16);
          v2[1] += __uint_as_float(vb & 0xFFFF0000u);
          if (rope) {
            const float4 t2 = *reinterpret_cast<const float4*>(cs + (tb + t) * HALF + e1);
            const float2 c0 = make_float2(t2.x, t2.y), c1 = make_float2(t2.z, t2.w);
            k1[0] += a[0] * c0.x - b[0] * c0.y;
            k2[0] += b[0] * c0.x + a[0] * c0.y;
            k1[1] += a[1] * c1.x - b[1] * c1.y;
            k2[1] += b[1] * c1.x + a[1] * c1.y;
            r1[0] += x[0] * c0.x - y[0] * c0.y;
            r2[0] += y[0] * c0.x + x[0] * c0.y;
            r1[1] += x[1] * c1.x - y[1] * c1.y;
            r2[1] += y[1] * c1.x + x[1] * c1.y;
          } else {
            k1[0] += a[0]; k1[1] += a[1]; k2[0] += b[0]; k2[1] += b[1];
            r1[0] += x[0]; r1[1] += x[1]; r2[0] += y[0]; r2[1] += y[1];
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // the stage's rows of this head are consumed
      if (++s == kEpNS) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (!ok) continue;  // an expired wait: nothing more is written
    if (rope) {  // turn the sums by the chunk's start position
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 t = rot_turns(j * p.chunk, turns[e1 + e]);
        const float a = k1[e] * t.x - k2[e] * t.y, b = k2[e] * t.x + k1[e] * t.y;
        k1[e] = a;
        k2[e] = b;
        const float ar = r1[e] * t.x - r2[e] * t.y, br = r2[e] * t.x + r1[e] * t.y;
        r1[e] = ar;
        r2[e] = br;
      }
    }
    const float fn = (float)n;
    const int64_t ob = c * (int64_t)W + h * D + e1;
    const __nv_bfloat162 ok1 = __floats2bfloat162_rn(k1[0] / fn, k1[1] / fn);
    const __nv_bfloat162 ok2 = __floats2bfloat162_rn(k2[0] / fn, k2[1] / fn);
    const __nv_bfloat162 or1 = __floats2bfloat162_rn(r1[0] / fn, r1[1] / fn);
    const __nv_bfloat162 or2 = __floats2bfloat162_rn(r2[0] / fn, r2[1] / fn);
    const __nv_bfloat162 ov1 = __floats2bfloat162_rn(v1[0] / fn, v1[1] / fn);
    const __nv_bfloat162 ov2 = __floats2bfloat162_rn(v2[0] / fn, v2[1] / fn);
    __nv_bfloat16* Kb = static_cast<__nv_bfloat16*>(p.Kb);
    __nv_bfloat16* Vb = static_cast<__nv_bfloat16*>(p.Vb);
    __nv_bfloat16* Rb = static_cast<__nv_bfloat16*>(p.Rb);
    *reinterpret_cast<__nv_bfloat162*>(Kb + ob) = ok1;
    *reinterpret_cast<__nv_bfloat162*>(Kb + ob + HALF) = ok2;
    *reinterpret_cast<__nv_bfloat162*>(Rb + ob) = or1;
    *reinterpret_cast<__nv_bfloat162*>(Rb + ob + HALF) = or2;
    *reinterpret_cast<__nv_bfloat162*>(Vb + ob) = ov1;
    *reinterpret_cast<__nv_bfloat162*>(Vb + ob + HALF) = ov2;
    if (p.inv_norm != nullptr) {  // of the stored bf16 K̄_r row of this head
      const float2 f1 = __bfloat1622float2(or1), f2 = __bfloat1622float2(or2);
      float ss = f1.x * f1.x + f1.y * f1.y + f2.x * f2.x + f2.y * f2.y;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) p.inv_norm[c * p.h_kv + h] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
    }
  }
}

size_t encode_pool_tma_smem(int h_kv) {
  const size_t blk = (size_t)kEpTB * h_kv * 128 * 2;
  return 1024 + kEpNS * 3 * blk + sizeof(float2) * 64 * 64 + 64 * 8 + 2 * kEpNS * 8 + 16;
}

// Inverse norms of a pre-pooled bank: one warp per (chunk, head) row.
template <typename T>
__global__ void __launch_bounds__(256) inv_norm_kernel(const T* __restrict__ R, int64_t rows,
                                                       int d, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += nw) {
    float s = 0.f;
    for (int e = lane; e < d; e += 32) {
      const float x = Elem<T>::to_f(R[r * d + e]);
      s += x * x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) out[r] = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
  }
}

// chunk offsets: doc_chunk_off[i+1] = sum_{j<=i} ceil(len_j / chunk). One CTA of 1024.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int64_t* __restrict__ tok_off,
                                                             int64_t n_docs, int chunk,
                                                             int64_t* __restrict__ out) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  if (tid == 0) g_encode_status = 0;  // the call's status word starts at zero
  const int64_t per = (n_docs + blockDim.x - 1) / blockDim.x;
  const int64_t a = min(n_docs, (int64_t)tid * per), b = min(n_docs, a + per);
  int64_t s = 0;
  for (int64_t i = a; i < b; ++i) s += (tok_off[i + 1] - tok_off[i] + chunk - 1) / chunk;
  part[tid] = s;
  __syncthreads();
  for (int o = 1; o < (int)blockDim.x; o <<= 1) {  // inclusive scan
    const int64_t v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int64_t run = tid ? part[tid - 1] : 0;
  if (tid == 0) out[0] = 0;
  for (int64_t i = a; i < b; ++i) {
    run += (tok_off[i + 1] - tok_off[i] + chunk - 1) / chunk;
    out[i + 1] = run;
  }
}

// ------------------------------------------------------------------------------- launch
template <typename T, int E, int D, int TP, bool SINGLE>
static cudaError_t launch_encode_s(const EncodeParams& p, int sms, cudaStream_t st) {
  constexpr int HALF = D / 2;
  const int PG = p.h_kv * (HALF / E);
  const size_t smem = sizeof(float2) * 64 * (HALF + 2) + sizeof(unsigned long long) * HALF +
                      sizeof(float) * PG;
  auto kfn = encode_pool_kernel<T, E, D, TP, SINGLE>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, PG * TP, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  int64_t grid = (int64_t)sms * per_sm;  // every CTA resident; contiguous chunk ranges
  if (grid > p.n_chunks) grid = p.n_chunks;
  if (grid < 1) grid = 1;
  kfn<<<(unsigned)grid, PG * TP, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int E, int D, int TP>
static cudaError_t launch_encode_t(const EncodeParams& p, int sms, cudaStream_t st) {
  return p.chunk <= 64 ? launch_encode_s<T, E, D, TP, true>(p, sms, st)
                       : launch_encode_s<T, E, D, TP, false>(p, sms, st);
}

template <typename T, int E, int D>
static cudaError_t launch_encode_e(const EncodeParams& p, int sms, cudaStream_t st) {
  const int PG = p.h_kv * (D / 2 / E);
  const int tp = 256 / PG;
  switch (tp >= 32 ? 32 : tp) {
    case 32: return launch_encode_t<T, E, D, 32>(p, sms, st);
    case 16: return launch_encode_t<T, E, D, 16>(p, sms, st);
    case 8: return launch_encode_t<T, E, D, 8>(p, sms, st);
    case 4: return launch_encode_t<T, E, D, 4>(p, sms, st);
    case 2: return launch_encode_t<T, E, D, 2>(p, sms, st);
    case 1: return launch_encode_t<T, E, D, 1>(p, sms, st);
    default: return cudaErrorInvalidConfiguration;
  }
}

// Host entry (validated by the caller): dtype 0 fp32, 1 bf16; d 64 or 128; h_kv a power of
// two with h_kv * (d/2) / E <= 256.
cudaError_t launch_encode_pool(const EncodeParams& p, int dtype, int d, int sms,
                               cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  if (p.n_docs > 0) {  // (also starts the status word)
    chunk_offsets_kernel<<<1, 1024, 0, st>>>(p.tok_off, p.n_docs, p.chunk,
                                             const_cast<int64_t*>(p.chunk_off));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    void* sw = nullptr;
    e = cudaGetSymbolAddress(&sw, g_encode_status);
    if (e == cudaSuccess) e = cudaMemsetAsync(sw, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
  }
  if (p.n_chunks == 0) return cudaSuccess;
  if (dtype == 1 && d == 128 && p.chunk <= 64 && p.h_kv >= 1 && p.h_kv <= 8) {
    const size_t smem = encode_pool_tma_smem(p.h_kv);
    e = cudaFuncSetAttribute(encode_pool_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(sms, p.n_chunks);
    encode_pool_tma_kernel<<<(unsigned)grid, 32 + 32 * p.h_kv, smem, st>>>(p);
    return cudaGetLastError();
  }
  if (dtype == 1) {
    return d == 128 ? launch_encode_e<__nv_bfloat16, 8, 128>(p, sms, st)
                    : launch_encode_e<__nv_bfloat16, 8, 64>(p, sms, st);
  }
  return d == 128 ? launch_encode_e<float, 4, 128>(p, sms, st)
                  : launch_encode_e<float, 4, 64>(p, sms, st);
}

cudaError_t read_encode_status(int* code, cudaStream_t st) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_encode_status, sizeof v, 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *code = v;
  return e;
}

cudaError_t launch_inv_norm(const void* R, int64_t n_chunks, int h_kv, int d, int dtype,
                            float* out, int sms, cudaStream_t st) {
  const int64_t rows = n_chunks * h_kv;
  if (rows == 0) return cudaSuccess;
  int64_t grid = (rows * 32 + 255) / 256;
  if (grid > (int64_t)sms * 32) grid = (int64_t)sms * 32;
  if (dtype == 1)
    inv_norm_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(R), rows, d, out);
  else
    inv_norm_kernel<float><<<(unsigned)grid, 256, 0, st>>>(static_cast<const float*>(R), rows,
                                                           d, out);
  return cudaGetLastError();
}

}  // namespace msa
