// route.cu - online routing of MSA: cosine scoring of every chunk of the router-key bank
// against the router queries, document scores, and an exact top-k, in ONE kernel launch.
//
// Method: the router query Q_r is compared with every chunk's pooled router key K̄_r by
// cosine similarity; the similarities are averaged over heads, the maximum is taken over
// query tokens, and the Top-k documents are selected
//   [news.neo-ai.one article, "全体設計 / アーキテクチャ"; github-eval-reports "MSA 项目评测报告",
//    "核心模块 / 路由投影器"; ruixiangma.github.io blog, "稀疏注意力机制 / Top-k检索"].
// A document's score is the maximum over its chunks.
//
// Design (the bank is streamed once per query batch; HBM-bound for short queries):
//  * Persistent grid, one contiguous document-aligned chunk range per CTA (docs never straddle
//    CTAs, so each CTA's candidate list is an exact superset of its share of the top-k).
//  * K̄_r tiles (8-32 chunks, 16 KB) are staged into shared memory by 1-D bulk async copies
//    (cp.async.bulk + mbarrier transaction counts), STAGES deep, issued by one thread.
//  * The query side is folded once per CTA into q̃[r, g, :] = sum over the router heads h of
//    KV head g of Q_r[r,h,:] / (||Q_r[r,h]|| * h_qr), kept in registers (E elements x R rows
//    per thread). A chunk's score for row r is sum_g inv_norm[c,g] * <q̃[r,g], K̄_r[c,g]>.
//  * Each thread owns E consecutive elements of a chunk row; partial dots of U chunks x R rows
//    are reduced across the warp by a transposing butterfly (each halving step sends half of
//    the values), then across the warps that share a chunk through shared memory.
//  * Per tile: max over query tokens -> per-document max (segmented, with a carry for a
//    document that continues into the next tile) -> warp-register top-k insertion per query
//    (lane i holds the i-th best 64-bit key (score, ~doc id)).
//  * The CTA writes its k candidates per query; the last CTA to finish (threadfence + atomic
//    ticket, no spinning) merges all candidates into the final top-k.
#include "common.cuh"
#include "kernels.cuh"

#include <type_traits>

namespace msa {


constexpr int kNT = 512;
constexpr int kWarps = kNT / 32;
// chunks per thread per sub-tile (one warp reduction each) and sub-tiles per tile; a tile is
// kSub * kU = 8 vectors per thread (64 KB with 16-byte vectors). Wider query batches take
// smaller sub-tiles to stay within 128 registers.
template <int R> __host__ __device__ constexpr int kUof() { return R >= 8 ? 2 : 4; }
template <int R> __host__ __device__ constexpr int kSubOf() { return 8 / kUof<R>(); }
constexpr int kStages = 3;  // bulk-copy pipeline depth
constexpr int kWin = 1024;  // document offsets cached in shared memory

template <typename T, int R, int E>
__global__ void __launch_bounds__(kNT, 1) route_scan_kernel(RouteParams p) {
  using VecT = Vec<T, E>;
  using raw = typename VecT::raw;
  constexpr int kU = kUof<R>();
  constexpr int kSub = kSubOf<R>();
  constexpr int V = kU * R;
  constexpr int VPL = V >= 32 ? V / 32 : 1;  // values per lane after the warp reduction
  constexpr int E2 = E / 2;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = p.h_kv * p.d;
  const int LPC = W / E;             // threads per chunk (multiple of 32, <= kNT)
  const int CPG = kNT / LPC;         // chunk groups per CTA
  const int NWG = LPC / 32;          // warps per chunk group
  const int TCS = kU * CPG;          // chunks per sub-tile
  const int TC = kSub * TCS;         // chunks per tile
  const uint32_t tile_bytes = (uint32_t)(TC * W * (int)sizeof(T));

  extern __shared__ __align__(128) unsigned char sm[];
  unsigned char* stage = sm;                                                   // [S][tile]
  float* invs = reinterpret_cast<float*>(sm + kStages * tile_bytes);          // [S][TC*h_kv]
  float* red = invs + kStages * TC * p.h_kv;                                   // [kSub][warps][V]
  float* msc = red + kSub * kWarps * V;                                        // [TC][R]
  float* qn = msc + TC * R;                                                    // [R][h_qr]
  int64_t* win = reinterpret_cast<int64_t*>(qn + ((R * p.h_qr + 1) & ~1));    // [kWin+1]
  unsigned long long* lists = reinterpret_cast<unsigned long long*>(win + kWin + 1);  // [R][32]
  float* carry = reinterpret_cast<float*>(lists + R * 32);                    // [R]
  uint64_t* mbar = reinterpret_cast<uint64_t*>(carry + ((R + 1) & ~1) + 2);   // [S]
  // [0..1] current doc, [2] window start, [3..6] this CTA's {D0, D1, cb, ce}
  int64_t* docs = reinterpret_cast<int64_t*>(mbar + kStages);
  int* flags = reinterpret_cast<int*>(docs + 7);                              // [0] last

  // ---- document-aligned chunk range of this CTA
  const int64_t G = gridDim.x;
  const int64_t i = blockIdx.x;
  cta_doc_range(p.coff, p.n_docs, p.n_chunks, i, G, docs + 3);
  const T* kr = static_cast<const T*>(p.kr);
  const size_t row_bytes = (size_t)W * sizeof(T);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&mbar[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int64_t D0 = docs[3], D1 = docs[4], cb = docs[5], ce = docs[6];
  const int64_t n_tiles = (ce - cb + TC - 1) / TC;
  auto issue = [&](int s, int64_t t) {
    const int64_t c0 = cb + t * TC;
    const int64_t n = min((int64_t)TC, ce - c0);
    const uint32_t kb = (uint32_t)(n * row_bytes);
    const uint32_t ib = p.inv_bulk ? (uint32_t)(n * p.h_kv * 4) : 0u;
    mbar_arrive_expect_tx(&mbar[s], kb + ib);
    bulk_g2s(stage + (size_t)s * tile_bytes, kr + c0 * W, kb, &mbar[s]);
    if (ib) bulk_g2s(invs + s * TC * p.h_kv, p.invk + c0 * p.h_kv, ib, &mbar[s]);
  };
  if (tid == 0) {
    docs[0] = D0;
    docs[2] = D0;
  }
  if (tid == 0)
    for (int s = 0; s < kStages && s < n_tiles; ++s) issue(s, s);

  // ---- doc-offset window; inverse norms of the router query heads
  for (int j = tid; j <= kWin; j += kNT) win[j] = (D0 + j <= D1) ? p.coff[D0 + j] : INT64_MAX;
  const T* q = static_cast<const T*>(p.qr);
  const int rows = p.B * p.T;
  for (int pair = warp; pair < R * p.h_qr; pair += kWarps) {
    const int r = pair / p.h_qr, h = pair % p.h_qr;
    float ss = 0.f;
    if (r < rows)
      for (int e = lane; e < p.d; e += 32) {
        const float x = Elem<T>::to_f(q[((int64_t)r * p.h_qr + h) * p.d + e]);
        ss += x * x;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) qn[pair] = ss > 0.f ? (1.0f / sqrtf(ss)) / (float)p.h_qr : 0.f;
  }
  for (int b = warp; b < R; b += kWarps) lists[b * 32 + lane] = 0ull;
  if (tid < R) carry[tid] = -INFINITY;
  __syncthreads();

  // ---- this thread's slice of q̃: E elements of KV head g for every row, in registers
  const int cg = tid / LPC;
  const int li = tid % LPC;
  const int e0 = li * E;
  const int g = e0 / p.d;
  const int ed = e0 % p.d;
  float2 qreg[R][E2];
  {
    const int m = p.h_qr / p.h_kv;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float acc[E];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
      if (r < rows)
        for (int hm = 0; hm < m; ++hm) {
          const int h = g * m + hm;
          const float sc = qn[r * p.h_qr + h];
          float x[E];
          VecT::unpack(*reinterpret_cast<const raw*>(q + ((int64_t)r * p.h_qr + h) * p.d + ed), x);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] += x[e] * sc;
        }
#pragma unroll
      for (int e = 0; e < E2; ++e) qreg[r][e] = make_float2(acc[2 * e], acc[2 * e + 1]);
    }
  }

  bool failed = false;
  int64_t it = 0;
  for (; it < n_tiles; ++it) {
    const int s = (int)(it % kStages);
    const uint32_t par = (uint32_t)((it / kStages) & 1);
    const int64_t c0 = cb + it * TC;
    const int n = (int)min((int64_t)TC, ce - c0);
    const bool ok = mbar_wait_bounded(&mbar[s], par, p.err);

    const unsigned char* tile = stage + (size_t)s * tile_bytes;
    const float* itile = invs + s * TC * p.h_kv;
#pragma unroll
    for (int sub = 0; sub < kSub; ++sub) {
      float v[V];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int ci = sub * TCS + u * CPG + cg;
        float2 x2[E2];
        float inv = 0.f;
        if (ci < n) {
          float x[E];
          VecT::unpack(*reinterpret_cast<const raw*>(tile + ((size_t)ci * W + e0) * sizeof(T)), x);
#pragma unroll
          for (int e = 0; e < E2; ++e) x2[e] = make_float2(x[2 * e], x[2 * e + 1]);
          inv = p.inv_bulk ? itile[ci * p.h_kv + g] : __ldg(p.invk + (c0 + ci) * p.h_kv + g);
        } else {
#pragma unroll
          for (int e = 0; e < E2; ++e) x2[e] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float2 a = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < E2; ++e) a = __ffma2_rn(qreg[r][e], x2[e], a);
          v[u * R + r] = (a.x + a.y) * inv;
        }
      }
      tr_reduce<V, 16>(v, lane);
      float* rb = red + (sub * kWarps + warp) * V;
      if constexpr (V >= 32) {
#pragma unroll
        for (int j = 0; j < VPL; ++j) rb[lane * VPL + j] = v[j];
      } else {
        if ((lane % (32 / V)) == 0) rb[lane / (32 / V)] = v[0];
      }
    }
    if (!__syncthreads_and(ok)) {  // stage s consumed; partial sums complete
      failed = true;
      break;
    }
    if (tid == 0 && it + kStages < n_tiles) {
      fence_proxy_async_smem();
      issue(s, it + kStages);
    }
    // chunk score per query: sum over the chunk group's warps, max over the query tokens
    for (int idx = tid; idx < TC * p.B; idx += kNT) {
      const int ci = idx / p.B, b = idx % p.B;
      const int sub = ci / TCS, cs = ci % TCS;
      const int gi = cs % CPG, u = cs / CPG;
      float mx = -INFINITY;
      if (ci < n) {
        for (int t = 0; t < p.T; ++t) {
          const int f = u * R + b * p.T + t;
          float sum = 0.f;
          for (int w = 0; w < NWG; ++w) sum += red[(sub * kWarps + gi * NWG + w) * V + f];
          mx = fmaxf(mx, sum);
        }
      }
      msc[ci * R + b] = mx;
    }
    __syncthreads();
    // slide the doc-offset window when this tile's docs may run past it
    const int64_t dcur = docs[it & 1];
    if (dcur + TC + 2 > docs[2] + kWin) {
      for (int j = tid; j <= kWin; j += kNT) win[j] = (dcur + j <= D1) ? p.coff[dcur + j] : INT64_MAX;
      __syncthreads();
      if (tid == 0) docs[2] = dcur;
      __syncthreads();
    }
    const int64_t w0 = docs[2];
    // per-document max + top-k insertion; warp w serves queries w, w + kWarps, ...
    const int64_t tend = c0 + n;
    for (int b = warp; b < p.B; b += kWarps) {
      unsigned long long lst = lane < p.k ? lists[b * 32 + lane] : 0ull;
      float cr = carry[b];
      int64_t dd = dcur;
      int64_t next = dcur;
      while (true) {
        const int64_t doc = dd + lane;
        bool valid = doc < D1;
        int64_t ds = 0, de = 0;
        if (valid) {
          ds = (doc - w0 < kWin) ? win[doc - w0] : __ldg(p.coff + doc);
          de = (doc + 1 - w0 <= kWin) ? win[doc + 1 - w0] : __ldg(p.coff + doc + 1);
        }
        valid = valid && ds < tend;
        bool fin = false;
        float sc = -INFINITY;
        if (valid) {
          const int lo = (int)(max(ds, c0) - c0), hi = (int)(min(de, tend) - c0);
          for (int c = lo; c < hi; ++c) sc = fmaxf(sc, msc[c * R + b]);
          if (ds < c0) sc = fmaxf(sc, cr);
          fin = de <= tend;
        }
        unsigned long long key = 0ull;
        if (fin) {
          if (p.doc_scores) p.doc_scores[(int64_t)b * p.n_docs + doc] = sc;
          const bool ex = p.excl && ((p.excl[(int64_t)b * p.words + (doc >> 5)] >> (doc & 31)) & 1u);
          if (!ex) key = score_key(sc, (uint32_t)doc);
        }
        list_insert(lst, key, lane, p.k);
        const unsigned cont = __ballot_sync(0xffffffffu, valid && !fin);
        const unsigned vm = __ballot_sync(0xffffffffu, valid);
        if (cont) {
          const int src = __ffs(cont) - 1;
          cr = __shfl_sync(0xffffffffu, sc, src);
          next = dd + src;
          break;
        }
        if (vm != 0xffffffffu) {
          next = dd + __popc(vm);
          break;
        }
        dd += 32;
      }
      if (lane < p.k) lists[b * 32 + lane] = lst;
      if (lane == 0) carry[b] = cr;
      if (b == 0 && lane == 0) docs[(it + 1) & 1] = next;
    }
  }
  __syncthreads();

  if (failed) {
    // drain the copies still in flight into this CTA's shared memory (bounded)
    for (int64_t t = it; t < n_tiles && t < it + kStages; ++t)
      mbar_wait_bounded(&mbar[t % kStages], (uint32_t)((t / kStages) & 1), p.err);
    __syncthreads();
  } else {
    // documents without chunks at the end of the range score -inf
    const int64_t dcur = docs[n_tiles & 1];
    for (int b = warp; b < p.B; b += kWarps) {
      unsigned long long lst = lane < p.k ? lists[b * 32 + lane] : 0ull;
      for (int64_t dd = dcur; dd < D1; dd += 32) {
        const int64_t doc = dd + lane;
        unsigned long long key = 0ull;
        if (doc < D1) {
          if (p.doc_scores) p.doc_scores[(int64_t)b * p.n_docs + doc] = -INFINITY;
          const bool ex = p.excl && ((p.excl[(int64_t)b * p.words + (doc >> 5)] >> (doc & 31)) & 1u);
          if (!ex) key = score_key(-INFINITY, (uint32_t)doc);
        }
        list_insert(lst, key, lane, p.k);
      }
      if (lane < p.k) lists[b * 32 + lane] = lst;
    }
    __syncthreads();
  }

  // ---- publish this CTA's candidates; the last CTA merges
  for (int b = warp; b < p.B; b += kWarps)
    if (lane < p.k) p.cand[(i * p.B + b) * p.k + lane] = lists[b * 32 + lane];
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicInc(p.counter, (unsigned)(G - 1));
    flags[0] = (t == (unsigned)(G - 1));
  }
  __syncthreads();
  if (!flags[0]) return;
  __threadfence();
  merge_candidates(p.cand, (int)G, p.B, p.k, stage, (size_t)kStages * tile_bytes, p.top_ids,
                   p.top_scores);
}

// ------------------------------------------------------------------------------- launch
template <typename T, int R, int E>
static size_t route_smem_bytes(int W, int h_kv, int h_qr) {
  constexpr int kU = kUof<R>(), kSub = kSubOf<R>();
  const int LPC = W / E, CPG = kNT / LPC, TC = kSub * kU * CPG;
  const size_t tile = (size_t)TC * W * sizeof(T);
  size_t s = kStages * tile + sizeof(float) * ((size_t)kStages * TC * h_kv +
                                               (size_t)kSub * kWarps * kU * R + (size_t)TC * R +
                                               (size_t)((R * h_qr + 1) & ~1));
  s = (s + 7) & ~(size_t)7;
  s += sizeof(int64_t) * (kWin + 1) + sizeof(unsigned long long) * R * 32;
  s += sizeof(float) * (((R + 1) & ~1) + 2);
  s += sizeof(uint64_t) * kStages + sizeof(int64_t) * 7 + sizeof(int) * 4;
  return (s + 127) & ~(size_t)127;
}

template <typename T, int R, int E>
static cudaError_t route_launch_t(const RouteParams& p, int grid, cudaStream_t st) {
  const size_t smem = route_smem_bytes<T, R, E>(p.h_kv * p.d, p.h_kv, p.h_qr);
  auto kfn = route_scan_kernel<T, R, E>;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kfn<<<grid, kNT, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int R, int E>
static int route_grid_t(int W, int h_kv, int h_qr, int sms, int64_t n_chunks) {
  const size_t smem = route_smem_bytes<T, R, E>(W, h_kv, h_qr);
  auto kfn = route_scan_kernel<T, R, E>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return -1;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, kNT, smem) != cudaSuccess || per_sm < 1)
    return -1;
  const int TC = kSubOf<R>() * kUof<R>() * (kNT / (W / E));
  int64_t want = (n_chunks + 2 * TC - 1) / (2 * TC);  // at least two tiles per CTA
  int64_t cap = (int64_t)per_sm * sms;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return (int)want;
}

// Dispatch on (dtype, rows per pass, vector width). Returns false if unsupported.

RouteChoice route_choose(int dtype, int rows, int W) {
  int R = 1;
  while (R < rows) R <<= 1;
  if (R > 16) return {0, 0};
  int E = dtype == 1 ? (R <= 8 ? 8 : 4) : 4;
  if (dtype == 1 && E == 8 && ((W / 8) % 32 != 0 || W / 8 > kNT)) E = 4;
  if (W % E != 0 || (W / E) % 32 != 0 || W / E > kNT) return {0, 0};
  return {R, E};
}

#define MSA_ROUTE_CASES(X)                                                              \
  X(float, 1, 4) X(float, 2, 4) X(float, 4, 4) X(float, 8, 4) X(float, 16, 4)           \
  X(__nv_bfloat16, 1, 8) X(__nv_bfloat16, 2, 8) X(__nv_bfloat16, 4, 8)                  \
  X(__nv_bfloat16, 8, 8) X(__nv_bfloat16, 1, 4) X(__nv_bfloat16, 2, 4)                  \
  X(__nv_bfloat16, 4, 4) X(__nv_bfloat16, 8, 4) X(__nv_bfloat16, 16, 4)

int route_grid(int dtype, RouteChoice c, int W, int h_kv, int h_qr, int sms, int64_t n_chunks) {
#define X(TT, RR, EE)                                                                     \
  if ((dtype == 1) == std::is_same<TT, __nv_bfloat16>::value && c.R == RR && c.E == EE)   \
    return route_grid_t<TT, RR, EE>(W, h_kv, h_qr, sms, n_chunks);
  MSA_ROUTE_CASES(X)
#undef X
  return -1;
}

cudaError_t route_launch(int dtype, RouteChoice c, const RouteParams& p, int grid, cudaStream_t st) {
#define X(TT, RR, EE)                                                                     \
  if ((dtype == 1) == std::is_same<TT, __nv_bfloat16>::value && c.R == RR && c.E == EE)   \
    return route_launch_t<TT, RR, EE>(p, grid, st);
  MSA_ROUTE_CASES(X)
#undef X
  return cudaErrorInvalidConfiguration;
}

}  // namespace msa
