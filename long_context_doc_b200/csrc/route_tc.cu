// route_tc.cu - routing for long queries (B*T rows beyond the CUDA-core scan) on the
// 5th-generation tensor cores: the chunk-vs-query cosine matrix is a dense contraction.
//
// Method (as in route.cu): cosine of Q_r against every chunk's K̄_r, mean over heads, max
// over query tokens, max over a document's chunks, top-k documents
//   [news.neo-ai.one article, "全体設計 / アーキテクチャ"; github-eval-reports, "核心模块"].
//
// Because the cosine normalises each head separately, the contraction runs on per-head unit
// vectors: K̂_r[c, g, :] = K̄_r[c, g, :] / ||K̄_r[c, g]|| (bank preparation, bf16, once per
// bank) and q̂[r, g, :] = sum_{h in g} Q_r[r, h, :] / (||Q_r[r, h]|| h_qr) (bf16, per call).
// Then s[c, r] = <K̂_r[c, :], q̂[r, :]> over the full h_kv * d row is exactly the head-mean
// cosine up to the bf16 rounding of the two unit operands.
//
// Kernel (one CTA per SM; work units = 128 chunks x one tile of query rows):
//   warp 0     : TMA producer (cp.async.bulk.tensor 2-D, 128-byte swizzle, no multicast)
//                of 64-wide K slices of K̂_r (128 rows) and q̂ (N rows) into a 4-stage ring;
//   warp 1     : one elected thread issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32,
//                M = 128, N <= 256, K = 16) into one of two TMEM accumulators and commits to
//                mbarriers (stage free / accumulator full);
//   warps 2-5  : epilogue; each thread owns one chunk row (its TMEM lane), reads the
//                accumulator with tcgen05.ld and takes the max over each query's T columns.
// Each CTA owns a document-aligned contiguous chunk range; once a chunk tile has been scored
// against every query tile, the epilogue warps fold chunk scores into document maxima (with a
// carry for documents that continue into the next tile) and keep an exact per-query top-k in
// warp registers; the last CTA to finish merges the per-CTA candidates (no spinning).
// Every wait is bounded; on expiry the CTA records an error in the workspace status word,
// stops issuing work, drains what it issued and frees its TMEM. The epilogue's waits for
// accumulators take the limit msa_set_device_wait_limit sets (the MMA issuer's and the
// producer's waits keep the default one: a limit check in the issue loop costs the scan ~1.5%,
// measured), so that no copy or MMA is in flight when the CTA frees its TMEM and exits.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace msa {

constexpr int kTcMaxStages = 12;
constexpr int kTcBM = 128;        // chunks per tile (TMEM lanes)
constexpr int kTcBK = 64;         // K slice (128 bytes of bf16: one swizzle row)
// 6 warps (copies, MMA issue, 4 epilogue warps), or 8 for decode batches of more than 6
// queries: the 2 more wait for the final merge, which then takes a query per warp in one round
// (measured: 3 us less at 8 decode queries; 13 us more per call at 4 queries over the 100M-token
// bank, where the 6-warp form keeps the scan at the copy peak)
constexpr int kTcWarpsMerge = 8;

// ------------------------------------------------------------------ PTX wrappers (sm_100a)
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand tile [rows][64 bf16] with the 128-byte swizzle: 8-row groups 1024 bytes
// apart (SBO), leading offset unused for swizzled K-major (1), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(const void* tile) {
  const uint64_t a = (uint64_t)(smem_u32(tile) & 0x3FFFFu) >> 4;
  return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
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

// ------------------------------------------------------------------ bank / query prep
// K̂_r rows: per (chunk, head) unit vectors in bf16 (zero rows stay zero). One warp per row.
template <typename T>
__global__ void __launch_bounds__(256) kr_normalize_kernel(const T* __restrict__ R, int64_t rows,
                                                           int d, __nv_bfloat16* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = warp; r < rows; r += nw) {
    float x[4];
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = lane + 32 * j;
      x[j] = e < d ? Elem<T>::to_f(R[r * d + e]) : 0.f;
      s += x[j] * x[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv = s > 0.f ? 1.0f / sqrtf(s) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = lane + 32 * j;
      if (e < d) out[r * d + e] = __float2bfloat16_rn(x[j] * inv);
    }
  }
}

// q̂ [rows, h_kv * d] bf16: one warp per (row, KV head).
template <typename T>
__global__ void __launch_bounds__(256) q_fold_kernel(const T* __restrict__ q, int rows, int h_qr,
                                                     int h_kv, int d,
                                                     __nv_bfloat16* __restrict__ out,
                                                     int* __restrict__ header) {
  const int lane = threadIdx.x & 31;
  // the call's workspace header (status word, merge ticket) starts at zero for the scan
  if (blockIdx.x == 0 && threadIdx.x < 64) header[threadIdx.x] = 0;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int m = h_qr / h_kv;
  const float inv_h = 1.0f / (float)h_qr;
  for (int64_t pr = warp; pr < (int64_t)rows * h_kv; pr += nw) {
    const int64_t r = pr / h_kv;
    const int g = (int)(pr % h_kv);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int hm = 0; hm < m; ++hm) {
      const T* qh = q + (r * h_qr + g * m + hm) * d;
      float x[4];
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = lane + 32 * j;
        x[j] = e < d ? Elem<T>::to_f(qh[e]) : 0.f;
        s += x[j] * x[j];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float sc = s > 0.f ? (1.0f / sqrtf(s)) * inv_h : 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] += x[j] * sc;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = lane + 32 * j;
      if (e < d) out[(r * h_kv + g) * d + e] = __float2bfloat16_rn(acc[j]);
    }
  }
}

// ------------------------------------------------------------------ tcgen05 scoring + top-k
struct TcParams {
  const int64_t* coff;   // [n_docs + 1]
  const uint32_t* excl;  // nullable [B, words]
  int64_t n_docs, n_chunks, words;
  int K;                 // h_kv * d (multiple of 64)
  int B, T, NQ, N;       // queries per row tile, row-tile width (multiple of 16, <= 256)
  int n_qtiles, stages, k;
  int32_t* top_ids;      // [B, k]
  float* top_scores;     // [B, k]
  float* doc_scores;     // nullable [B, n_docs]
  unsigned long long* cand;  // [grid, B, k]
  unsigned int* counter;
  int* err;
  long long wait_limit;  // the epilogue's waits for accumulators, SM clocks; 0: default
};

constexpr int kTcWin = 1024;  // document offsets cached in shared memory

__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, uint32_t par, int* err,
                                             volatile int* abort_flag,
                                             long long limit = kDefaultWaitLimit) {
  if (*abort_flag) return false;
  if (mbar_wait_limited(bar, par, err, limit)) return true;
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ void epi_sync() {  // the 128 epilogue threads only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Work of a CTA: the chunk tiles (128 rows from the CTA's first chunk) of its document-aligned
// chunk range, each against every row tile of queries; units are (chunk tile, query tile),
// query tiles innermost.
template <int NW>
__global__ void __launch_bounds__(NW * 32, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                TcParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // generic base on purpose: with shared-space pointers (smem_align1024) this kernel's scan
  // measured ~5% slower at the 100M-token bank
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t a_bytes = kTcBM * kTcBK * 2;
  const uint32_t b_bytes = (uint32_t)p.N * kTcBK * 2;
  const uint32_t stage_bytes = (a_bytes + b_bytes + 1023) & ~1023u;
  const int S = p.stages;
  float* msc = reinterpret_cast<float*>(base + S * stage_bytes);                // [128][B]
  int64_t* win = reinterpret_cast<int64_t*>(msc + kTcBM * p.B);                 // [kTcWin+1]
  unsigned long long* lists = reinterpret_cast<unsigned long long*>(win + kTcWin + 1);  // [B][32]
  float* carry = reinterpret_cast<float*>(lists + p.B * 32);                    // [B]
  uint64_t* full = reinterpret_cast<uint64_t*>(carry + ((p.B + 1) & ~1));       // [max]
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* tfull = empty + kTcMaxStages;  // [2]
  uint64_t* tempty = tfull + 2;            // [2]
  uint64_t* done = tempty + 2;             // MMA issuer: every issued MMA has completed
  // [0..1] current doc, [2] window start, [3..6] this CTA's {D0, D1, cb, ce}
  int64_t* docs = reinterpret_cast<int64_t*>(done + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(docs + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* last_flag = const_cast<int*>(abort_flag) + 1;
  // epilogue give-up flags, one per chunk-tile parity: written (only by epilogue threads whose
  // wait failed) before a chunk tile's barrier, read by all of them after it, so the four
  // epilogue warps leave together; a flag is written again two chunk tiles later, after the
  // next barrier, so no thread reads one that is being rewritten
  volatile int* epi_abort = const_cast<int*>(abort_flag) + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_k = p.K / kTcBK;

  const int64_t G = gridDim.x, ci = blockIdx.x;
  cta_doc_range(p.coff, p.n_docs, p.n_chunks, ci, G, docs + 3);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    epi_abort[0] = 0;
    epi_abort[1] = 0;
    fence_mbar_init();
  }
  for (int j = threadIdx.x; j < p.B * 32; j += NW * 32) lists[j] = 0ull;
  for (int j = threadIdx.x; j < p.B; j += NW * 32) carry[j] = -INFINITY;
  if (warp == 0) {  // two fp32 accumulators of up to 256 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int64_t D0 = docs[3], D1 = docs[4], cb = docs[5], ce = docs[6];
  const int64_t n_ct = (ce - cb + kTcBM - 1) / kTcBM;
  const int64_t n_units = n_ct * p.n_qtiles;
  // a range's partial last tile is loaded ending at the range's end: its first `shift` rows
  // repeat rows of the tile before (just read, in L2) and are dropped, so no row past the range
  // (the next CTA's) is read from memory; a range shorter than a tile reads past its end
  auto tile_shift = [&](int64_t ct) -> int64_t {
    return (ct == n_ct - 1 && ce - cb >= kTcBM) ? cb + (ct + 1) * kTcBM - ce : 0;
  };

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t u = 0; u < n_units; ++u) {
        const int64_t ct = u / p.n_qtiles, qt = u % p.n_qtiles;
        const int y_a = (int)(cb + ct * kTcBM - tile_shift(ct)), y_b = (int)(qt * p.NQ * p.T);
        for (int kk = 0; kk < n_k; ++kk) {
          if (issued >= S && !wait_or_fail(&empty[s], ph ^ 1u, p.err, abort_flag)) break;
          unsigned char* st = base + (size_t)s * stage_bytes;
          mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
          tma_load_2d(st, &map_k, kk * kTcBK, y_a, &full[s]);
          tma_load_2d(st + a_bytes, &map_q, kk * kTcBK, y_b, &full[s]);
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (*abort_flag) break;
      }
      for (int64_t j = (issued > S ? issued - S : 0); j < issued; ++j)
        mbar_wait_bounded(&full[j % S], (uint32_t)((j / S) & 1), p.err);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.N >> 3) << 17) |
                             ((uint32_t)(kTcBM >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      for (int64_t u = 0; u < n_units; ++u) {
        const int a = (int)(u & 1);
        const uint32_t aph = (uint32_t)((u >> 1) & 1);
        if (u >= 2 && !wait_or_fail(&tempty[a], aph ^ 1u, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * 256);
        bool ok = true;
        for (int kk = 0; kk < n_k; ++kk) {
          if (!wait_or_fail(&full[s], ph, p.err, abort_flag)) { ok = false; break; }
          tc_fence_after();
          unsigned char* st = base + (size_t)s * stage_bytes;
          const uint64_t ad = sw128_desc(st), bd = sw128_desc(st + a_bytes);
#pragma unroll
          for (int j = 0; j < kTcBK / 16; ++j)  // K = 16 per instruction: +32 bytes
            tc_mma(d_tmem, ad + 2 * j, bd + 2 * j, idesc, (kk | j) ? 1u : 0u);
          tc_commit(&empty[s]);
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&tfull[a]);
      }
      tc_commit(done);
      mbar_wait_bounded(done, 0, p.err);
    }
  } else if (warp < 6) {
    // ---------------- epilogue (warps 2..5 -> TMEM lane groups 2, 3, 0, 1)
    const int lg = warp & 3;
    const int ew = warp - 2;                 // epilogue warp 0..3
    const int row = lg * 32 + lane;          // chunk row of the tile (TMEM lane)
    const int ncols = p.NQ * p.T;
    bool aborted = false;
    // document-offset window (the producer is already streaming the first tiles)
    for (int j = ew * 32 + lane; j <= kTcWin; j += 128)
      win[j] = (D0 + j <= D1) ? __ldg(p.coff + D0 + j) : INT64_MAX;
    if (ew == 0 && lane == 0) {
      docs[0] = D0;
      docs[2] = D0;
    }
    epi_sync();
    for (int64_t u = 0; u < n_units; ++u) {
      const int a = (int)(u & 1);
      const uint32_t aph = (uint32_t)((u >> 1) & 1);
      const int64_t ct = u / p.n_qtiles, qt = u % p.n_qtiles;
      // a warp whose wait fails skips the tensor-memory loads (warp-collective: a warp-uniform
      // decision), flags the chunk tile and leaves with the others after its barrier
      const bool got = !aborted && __all_sync(0xffffffffu, wait_or_fail(&tfull[a], aph, p.err,
                                                                       abort_flag, p.wait_limit));
      if (!got) {
        aborted = true;
        epi_abort[ct & 1] = 1;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(lg * 32) << 16) + (uint32_t)(a * 256);
      const int mrow = row - (int)tile_shift(ct);  // the row's chunk offset in the tile
      int q = 0, t = 0;
      float cur = -INFINITY;
      for (int col = 0; got && col < ncols; col += 32) {
        float v[32];
        tmem_ld32(tbase + (uint32_t)col, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (col + j < ncols) {
            cur = fmaxf(cur, v[j]);
            if (++t == p.T) {  // max over the query's tokens done
              const int b = (int)qt * p.NQ + q;
              if (b < p.B && mrow >= 0) msc[mrow * p.B + b] = cur;
              cur = -INFINITY;
              t = 0;
              ++q;
            }
          }
        }
      }
      tc_fence_before();
      if (got) mbar_arrive(&tempty[a]);
      if (qt != p.n_qtiles - 1) continue;
      // ---- chunk tile complete for every query: per-document max + top-k insertion
      epi_sync();
      if (epi_abort[ct & 1]) {  // every epilogue thread leaves here
        aborted = true;
        break;
      }
      const int64_t c0 = cb + ct * kTcBM;
      const int64_t tend = min(c0 + kTcBM, ce);
      const int64_t dcur = docs[ct & 1];
      if (dcur + kTcBM + 2 > docs[2] + kTcWin) {  // slide the document-offset window
        for (int j = ew * 32 + lane; j <= kTcWin; j += 128)
          win[j] = (dcur + j <= D1) ? p.coff[dcur + j] : INT64_MAX;
        epi_sync();
        if (ew == 0 && lane == 0) docs[2] = dcur;
        epi_sync();
      }
      const int64_t w0 = docs[2];
      for (int b = ew; b < p.B; b += 4) {
        unsigned long long lst = lane < p.k ? lists[b * 32 + lane] : 0ull;
        float cr = carry[b];
        int64_t dd = dcur, next = dcur;
        while (true) {
          const int64_t doc = dd + lane;
          bool valid = doc < D1;
          int64_t ds = 0, de = 0;
          if (valid) {
            ds = (doc - w0 < kTcWin) ? win[doc - w0] : __ldg(p.coff + doc);
            de = (doc + 1 - w0 <= kTcWin) ? win[doc + 1 - w0] : __ldg(p.coff + doc + 1);
          }
          valid = valid && ds < tend;
          bool fin = false;
          float sc = -INFINITY;
          if (valid) {
            const int lo = (int)(max(ds, c0) - c0), hi = (int)(min(de, tend) - c0);
            for (int c = lo; c < hi; ++c) sc = fmaxf(sc, msc[c * p.B + b]);
            if (ds < c0) sc = fmaxf(sc, cr);
            fin = de <= tend;
          }
          unsigned long long key = 0ull;
          if (fin) {
            if (p.doc_scores) p.doc_scores[(int64_t)b * p.n_docs + doc] = sc;
            const bool ex =
                p.excl && ((p.excl[(int64_t)b * p.words + (doc >> 5)] >> (doc & 31)) & 1u);
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
        if (b == 0 && lane == 0) docs[(ct + 1) & 1] = next;
      }
      epi_sync();  // msc and the document cursor are reused by the next chunk tile
    }
    if (!aborted) {  // documents without chunks at the end of the range score -inf
      const int64_t dcur = docs[n_ct & 1];
      for (int b = ew; b < p.B; b += 4) {
        unsigned long long lst = lane < p.k ? lists[b * 32 + lane] : 0ull;
        for (int64_t dd = dcur; dd < D1; dd += 32) {
          const int64_t doc = dd + lane;
          unsigned long long key = 0ull;
          if (doc < D1) {
            if (p.doc_scores) p.doc_scores[(int64_t)b * p.n_docs + doc] = -INFINITY;
            const bool ex =
                p.excl && ((p.excl[(int64_t)b * p.words + (doc >> 5)] >> (doc & 31)) & 1u);
            if (!ex) key = score_key(-INFINITY, (uint32_t)doc);
          }
          list_insert(lst, key, lane, p.k);
        }
        if (lane < p.k) lists[b * 32 + lane] = lst;
      }
    }
  }

  // ---------------- teardown: every MMA completed (the issuer waited on `done`)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");

  // ---------------- publish this CTA's candidates; the last CTA merges
  for (int b = warp; b < p.B; b += NW)
    if (lane < p.k) p.cand[(ci * p.B + b) * p.k + lane] = lists[b * 32 + lane];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    *last_flag = (atomicInc(p.counter, (unsigned)(G - 1)) == (unsigned)(G - 1));
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  merge_candidates(p.cand, (int)G, p.B, p.k, base, (size_t)S * stage_bytes, p.top_ids,
                   p.top_scores);
}

// ------------------------------------------------------------------ host side
// 2-D bf16 tensor map over a [rows, cols] row-major matrix, box {64, box_rows}, 128B swizzle.
static bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)cols * 2};
  const uint32_t box[2] = {(uint32_t)kTcBK, (uint32_t)box_rows};
  return encode_bf16_map(m, ptr, 2, dims, strides, box, true);
}

TcPlan tc_plan(int B, int T, int h_kv, int d, int64_t n_docs, int64_t n_chunks, int k, int sms) {
  TcPlan pl{};
  pl.ok = (T >= 1 && T <= 256 && B >= 1 && B <= 64 && (h_kv * d) % kTcBK == 0);
  if (!pl.ok) return pl;
  pl.NQ = std::max(1, 256 / T);
  if (pl.NQ > B) pl.NQ = B;
  pl.N = ((pl.NQ * T + 15) / 16) * 16;
  if (pl.N < 16) pl.N = 16;
  pl.n_qtiles = (B + pl.NQ - 1) / pl.NQ;
  pl.n_ctiles = (n_chunks + kTcBM - 1) / kTcBM;
  pl.grid = (int)std::min<int64_t>(sms, std::max<int64_t>(1, pl.n_ctiles));
  pl.topk_grid = pl.grid;
  const size_t rows = (size_t)B * T;
  pl.q_bytes = ((rows * h_kv * d * 2) + 255) & ~(size_t)255;
  pl.m_bytes = 0;
  pl.cand_bytes = (((size_t)pl.grid * B * k * 8) + 255) & ~(size_t)255;
  const size_t stage = (((size_t)kTcBM * kTcBK * 2 + (size_t)pl.N * kTcBK * 2) + 1023) & ~(size_t)1023;
  const size_t fixed = (size_t)kTcBM * B * 4 + (kTcWin + 1) * 8 + (size_t)B * 32 * 8 +
                       ((B + 1) & ~1) * 4 + (2 * kTcMaxStages + 5) * 8 + 7 * 8 + 24;
  const size_t budget = 227 * 1024 - 1024 - fixed - 64;
  pl.stages = (int)std::min<size_t>(kTcMaxStages, budget / stage);
  if (pl.stages < 2) pl.ok = false;
  pl.smem = 1024 + pl.stages * stage + fixed + 64;
  (void)n_docs;
  return pl;
}

cudaError_t launch_kr_normalize(const void* R, int64_t n_chunks, int h_kv, int d, int dtype,
                                void* out, int sms, cudaStream_t st) {
  const int64_t rows = n_chunks * h_kv;
  if (rows == 0) return cudaSuccess;
  int64_t grid = (rows * 32 + 255) / 256;
  if (grid > (int64_t)sms * 32) grid = (int64_t)sms * 32;
  if (dtype == 1)
    kr_normalize_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(R), rows, d, static_cast<__nv_bfloat16*>(out));
  else
    kr_normalize_kernel<float><<<(unsigned)grid, 256, 0, st>>>(
        static_cast<const float*>(R), rows, d, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

cudaError_t launch_route_tc(const RouteTcArgs& a, const TcPlan& pl, cudaStream_t st) {
  // 1. fold the router queries into per-KV-head unit rows (bf16)
  const int rows = a.B * a.T;
  int64_t qgrid = ((int64_t)rows * a.h_kv * 32 + 255) / 256;
  if (qgrid > 4096) qgrid = 4096;
  if (a.dtype == 1)
    q_fold_kernel<__nv_bfloat16><<<(unsigned)qgrid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(a.Q_r), rows, a.h_qr, a.h_kv, a.d, a.q_hat, a.err);
  else
    q_fold_kernel<float><<<(unsigned)qgrid, 256, 0, st>>>(static_cast<const float*>(a.Q_r), rows,
                                                          a.h_qr, a.h_kv, a.d, a.q_hat, a.err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. tensor-core scores fused with the per-document max and the exact top-k
  CUtensorMap mk, mq;
  const int K = a.h_kv * a.d;
  if (!make_map(&mk, a.Kr_hat, a.n_chunks, K, kTcBM) || !make_map(&mq, a.q_hat, rows, K, pl.N))
    return cudaErrorInvalidValue;
  TcParams p{};
  p.coff = a.coff;
  p.excl = a.excl;
  p.n_docs = a.n_docs;
  p.n_chunks = a.n_chunks;
  p.words = (a.n_docs + 31) / 32;
  p.K = K;
  p.B = a.B;
  p.T = a.T;
  p.NQ = pl.NQ;
  p.N = pl.N;
  p.n_qtiles = (int)pl.n_qtiles;
  p.stages = pl.stages;
  p.k = a.k;
  p.top_ids = a.top_ids;
  p.top_scores = a.top_scores;
  p.doc_scores = a.doc_scores;
  p.cand = a.cand;
  p.counter = a.counter;
  p.err = a.err;
  p.wait_limit = a.wait_limit;
  // decode batches of more than 6 queries: 8 warps, one merge round
  const int nw = (pl.n_qtiles == 1 && a.B > 6 && a.B <= kTcWarpsMerge) ? kTcWarpsMerge : 6;
  auto kfn = nw == kTcWarpsMerge ? route_tc_kernel<kTcWarpsMerge> : route_tc_kernel<6>;
  e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem);
  if (e != cudaSuccess) return e;
  kfn<<<pl.grid, nw * 32, pl.smem, st>>>(mk, mq, p);
  return cudaGetLastError();
}

}  // namespace msa
