// api.cu - the extern "C" boundary of libmsa (declared in include/msa.h): argument
// validation, workspace sizing and kernel launches. No device memory is allocated here; the
// only allocation is the pinned staging area of an msa_fetch context, made at set-up time.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include "../../include/msa.h"
#include "common.cuh"
#include "kernels.cuh"

namespace {

thread_local std::string g_err;

msa_status fail(msa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
msa_status fail(msa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

msa_status ok() {
  g_err.clear();
  return MSA_OK;
}

msa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MSA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    return 148;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
size_t esize(int dtype) { return dtype == MSA_BF16 ? 2 : 4; }

constexpr size_t kHeader = 256;   // workspace header: [0] status word, [1..63] counters
constexpr int kMaxPasses = 63;

#define REQUIRE(cond, status, ...) \
  do {                             \
    if (!(cond)) return fail(status, __VA_ARGS__); \
  } while (0)

msa_status check_common(int32_t h_kv, int32_t d, int32_t dtype) {
  REQUIRE(dtype == MSA_FP32 || dtype == MSA_BF16, MSA_ERR_UNSUPPORTED, "dtype %d", dtype);
  REQUIRE(d == 64 || d == 128, MSA_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  REQUIRE(h_kv >= 1, MSA_ERR_INVALID_ARG, "h_kv %d", h_kv);
  return MSA_OK;
}

// route pass geometry: queries per pass and number of passes
void route_passes(int B, int T, int* bp, int* passes) {
  int per = std::max(1, 16 / std::max(T, 1));
  per = std::min(per, std::max(B, 1));
  int np = (B + per - 1) / per;
  per = (B + np - 1) / std::max(np, 1);
  *bp = std::max(per, 1);
  *passes = np;
}

}  // namespace

namespace msa {
void rope_turns(double base, int d, unsigned long long* out) {
  const long double pi2 = 6.283185307179586476925286766559005768L;
  for (int i = 0; i < d / 2; ++i) {
    unsigned long long F = 0;
    if (base > 0.0) {
      long double f = powl((long double)base, -2.0L * i / (long double)d) / pi2;
      f -= floorl(f);
      const long double scaled = ldexpl(f, 64);
      F = scaled >= 18446744073709551615.0L ? ~0ull : (unsigned long long)scaled;
    }
    out[i] = F;
  }
}
// Set the thread-local message returned by msa_last_error (for entry points defined in other
// translation units).
void set_last_error(const std::string& msg) { g_err = msg; }
static std::atomic<long long> g_wait_limit{0};
long long device_wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }
}  // namespace msa

extern "C" {

const char* msa_status_string(int s) {
  switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
    case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
    case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
    case MSA_ERR_DEVICE: return "MSA_ERR_DEVICE";
    default: return "MSA_ERR_UNKNOWN";
  }
}

const char* msa_last_error(void) { return g_err.c_str(); }

int msa_version(void) { return (1 << 16) | 0; }

int64_t msa_set_device_wait_limit(int64_t cycles) {
  return msa::g_wait_limit.exchange(cycles > 0 ? cycles : 0);
}

int64_t msa_count_chunks(const int64_t* off, int64_t n_docs, int32_t chunk) {
  if (off == nullptr || n_docs < 0 || chunk < 1) return -1;
  if (off[0] != 0) return -1;
  int64_t n = 0;
  for (int64_t i = 0; i < n_docs; ++i) {
    const int64_t len = off[i + 1] - off[i];
    if (len < 0) return -1;
    n += (len + chunk - 1) / chunk;
  }
  return n;
}

msa_status msa_encode_pool(const void* K, const void* V, const void* K_r, int64_t n_tok,
                           const int64_t* doc_tok_off_host, const int64_t* doc_tok_off,
                           int64_t n_docs, int32_t chunk, int32_t h_kv, int32_t d,
                           int32_t dtype, float rope_base, void* Kbar, void* Vbar,
                           void* Kbar_r, float* kr_inv_norm, int64_t* doc_chunk_off,
                           int64_t n_chunks, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(n_docs >= 0 && n_tok >= 0 && n_chunks >= 0, MSA_ERR_INVALID_ARG, "negative size");
  REQUIRE(chunk >= 1, MSA_ERR_INVALID_ARG, "chunk %d", chunk);
  REQUIRE(doc_tok_off_host && doc_tok_off && doc_chunk_off, MSA_ERR_INVALID_ARG,
          "null offset pointer");
  REQUIRE(doc_tok_off_host[n_docs] == n_tok, MSA_ERR_INVALID_ARG,
          "doc_tok_off[n_docs] = %lld != n_tok %lld", (long long)doc_tok_off_host[n_docs],
          (long long)n_tok);
  const int64_t nc = msa_count_chunks(doc_tok_off_host, n_docs, chunk);
  REQUIRE(nc >= 0, MSA_ERR_INVALID_ARG, "doc_tok_off must start at 0 and not decrease");
  REQUIRE(nc == n_chunks, MSA_ERR_INVALID_ARG, "n_chunks %lld != %lld implied by the offsets",
          (long long)n_chunks, (long long)nc);
  const int E = dtype == MSA_BF16 ? 8 : 4;
  REQUIRE(pow2(h_kv) && h_kv * (d / 2) / E <= 256, MSA_ERR_UNSUPPORTED,
          "encode needs h_kv a power of two with h_kv*d/2/%d <= 256 (h_kv=%d)", E, h_kv);
  if (n_chunks > 0) {
    REQUIRE(K && V && K_r && Kbar && Vbar && Kbar_r, MSA_ERR_INVALID_ARG, "null tensor");
    REQUIRE(aligned16(K) && aligned16(V) && aligned16(K_r) && aligned16(Kbar) &&
                aligned16(Vbar) && aligned16(Kbar_r),
            MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  }
  msa::EncodeParams p{};
  p.K = K;
  p.V = V;
  p.Kr = K_r;
  p.tok_off = doc_tok_off;
  p.chunk_off = doc_chunk_off;
  p.n_docs = n_docs;
  p.n_chunks = n_chunks;
  p.chunk = chunk;
  p.h_kv = h_kv;
  p.rope = rope_base > 0.f ? 1 : 0;
  msa::rope_turns(p.rope ? (double)rope_base : 0.0, d, p.rope_turns);
  p.Kb = Kbar;
  p.Vb = Vbar;
  p.Rb = Kbar_r;
  p.inv_norm = kr_inv_norm;
  cudaError_t e = msa::launch_encode_pool(p, dtype, d, sm_count(), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "msa_encode_pool launch");
  return ok();
}

msa_status msa_encode_pool_status(int32_t* code, void* stream) {
  REQUIRE(code, MSA_ERR_INVALID_ARG, "null code");
  int v = 0;
  cudaError_t e = msa::read_encode_status(&v, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "msa_encode_pool_status");
  *code = v;
  if (v != 0) return fail(MSA_ERR_DEVICE, "device status %d recorded by the pooling encode", v);
  return ok();
}

msa_status msa_kr_inv_norm(const void* Kbar_r, int64_t n_chunks, int32_t h_kv, int32_t d,
                           int32_t dtype, float* out, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(n_chunks >= 0, MSA_ERR_INVALID_ARG, "negative n_chunks");
  REQUIRE(n_chunks == 0 || (Kbar_r && out), MSA_ERR_INVALID_ARG, "null tensor");
  cudaError_t e = msa::launch_inv_norm(Kbar_r, n_chunks, h_kv, d, dtype, out, sm_count(),
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "msa_kr_inv_norm launch");
  return ok();
}

size_t msa_route_topk_workspace(int32_t B, int32_t T, int32_t h_qr, int32_t h_kv, int32_t d,
                                int32_t dtype, int64_t n_docs, int64_t n_chunks, int32_t k) {
  if (B < 1 || T < 1 || k < 1 || h_kv < 1 || d < 1) return kHeader;
  size_t tc = kHeader;
  if (dtype == MSA_BF16) {  // the tensor-core scan may serve any bf16 query length
    const msa::TcPlan pl = msa::tc_plan(B, T, h_kv, d, n_docs, n_chunks, k, sm_count());
    if (pl.ok) tc = kHeader + pl.q_bytes + pl.m_bytes + pl.cand_bytes;
  }
  if (T > 16) return tc;
  int bp, passes;
  route_passes(B, T, &bp, &passes);
  const msa::RouteChoice c = msa::route_choose(dtype, bp * T, h_kv * d);
  if (c.R == 0) return kHeader;
  const int grid = msa::route_grid(dtype, c, h_kv * d, h_kv, h_qr, sm_count(), n_chunks);
  if (grid < 1) return tc;
  return std::max(tc, kHeader + (size_t)passes * grid * bp * k * sizeof(unsigned long long));
}

msa_status msa_kr_normalize(const void* Kbar_r, int64_t n_chunks, int32_t h_kv, int32_t d,
                            int32_t dtype, void* out, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(n_chunks >= 0, MSA_ERR_INVALID_ARG, "negative n_chunks");
  REQUIRE(n_chunks == 0 || (Kbar_r && out), MSA_ERR_INVALID_ARG, "null tensor");
  cudaError_t e = msa::launch_kr_normalize(Kbar_r, n_chunks, h_kv, d, dtype, out, sm_count(),
                                           (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "msa_kr_normalize launch");
  return ok();
}

msa_status msa_route_topk(const void* Q_r, int32_t B, int32_t T, int32_t h_qr,
                          const void* Kbar_r, const float* kr_inv_norm, const void* Kbar_r_hat,
                          const int64_t* doc_chunk_off, int64_t n_docs, int64_t n_chunks,
                          int32_t h_kv, int32_t d, int32_t dtype, int32_t k,
                          const uint32_t* exclude_bits, int32_t* top_ids, float* top_scores,
                          float* doc_scores, void* ws, size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && T >= 1 && n_docs >= 1 && n_chunks >= 0, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d T=%d n_docs=%lld n_chunks=%lld)", B, T, (long long)n_docs,
          (long long)n_chunks);
  REQUIRE(h_qr >= 1 && h_qr % h_kv == 0, MSA_ERR_INVALID_ARG, "h_qr %d not a multiple of h_kv %d",
          h_qr, h_kv);
  REQUIRE(k >= 1 && k <= n_docs, MSA_ERR_INVALID_ARG, "k %d outside [1, n_docs=%lld]", k,
          (long long)n_docs);
  REQUIRE(k <= 32, MSA_ERR_UNSUPPORTED, "k %d > 32", k);
  if (T > 16) {
    REQUIRE(T <= 256, MSA_ERR_UNSUPPORTED, "query length T=%d > 256", T);
    REQUIRE(dtype == MSA_BF16, MSA_ERR_UNSUPPORTED,
            "queries with T=%d > 16 use the bf16 tensor-core scan (fp32 banks: T <= 16)", T);
    REQUIRE(Kbar_r_hat != nullptr, MSA_ERR_INVALID_ARG,
            "T=%d > 16 needs the normalised bank Kbar_r_hat (msa_kr_normalize)", T);
  }
  if (B == 0) return ok();
  // the tensor-core scan reads only the normalised bank: Kbar_r and its inverse norms may be
  // null there (a bank prepared for it need not keep K̄_r resident)
  const bool tc_scan = T > 16 || (dtype == MSA_BF16 && Kbar_r_hat != nullptr);
  REQUIRE(Q_r && doc_chunk_off && top_ids && top_scores && (tc_scan || (Kbar_r && kr_inv_norm)),
          MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(tc_scan || aligned16(Kbar_r), MSA_ERR_INVALID_ARG, "Kbar_r must be 16-byte aligned");
  if (tc_scan) {
    REQUIRE(aligned16(Kbar_r_hat) && aligned16(Q_r), MSA_ERR_INVALID_ARG,
            "Kbar_r_hat and Q_r must be 16-byte aligned");
    const msa::TcPlan pl = msa::tc_plan(B, T, h_kv, d, n_docs, n_chunks, k, sm_count());
    REQUIRE(pl.ok, MSA_ERR_UNSUPPORTED, "tensor-core scan: h_kv*d=%d not a multiple of 64",
            h_kv * d);
    const size_t need = kHeader + pl.q_bytes + pl.m_bytes + pl.cand_bytes;
    REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
            MSA_ERR_WORKSPACE, "workspace %zu bytes at %p, need %zu (256-byte aligned)",
            ws_bytes, ws, need);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    // no memset node: the query fold (the call's first kernel) zeroes the header
    unsigned char* base = static_cast<unsigned char*>(ws);
    msa::RouteTcArgs ta{};
    ta.Q_r = Q_r;
    ta.Kr_hat = Kbar_r_hat;
    ta.coff = doc_chunk_off;
    ta.excl = exclude_bits;
    ta.n_docs = n_docs;
    ta.n_chunks = n_chunks;
    ta.B = B;
    ta.T = T;
    ta.h_qr = h_qr;
    ta.h_kv = h_kv;
    ta.d = d;
    ta.k = k;
    ta.dtype = dtype;
    ta.top_ids = top_ids;
    ta.top_scores = top_scores;
    ta.doc_scores = doc_scores;
    ta.q_hat = reinterpret_cast<__nv_bfloat16*>(base + kHeader);
    ta.mscore = nullptr;
    ta.cand = reinterpret_cast<unsigned long long*>(base + kHeader + pl.q_bytes + pl.m_bytes);
    ta.counter = reinterpret_cast<unsigned int*>(base) + 1;
    ta.err = reinterpret_cast<int*>(base);
    ta.wait_limit = msa::device_wait_limit();
    e = msa::launch_route_tc(ta, pl, st);
    if (e != cudaSuccess) return cuda_fail(e, "msa_route_topk (tensor-core scan) launch");
    return ok();
  }
  int bp, passes;
  route_passes(B, T, &bp, &passes);
  REQUIRE(passes <= kMaxPasses, MSA_ERR_UNSUPPORTED, "B=%d needs %d passes (> %d)", B, passes,
          kMaxPasses);
  const int W = h_kv * d;
  const msa::RouteChoice c = msa::route_choose(dtype, bp * T, W);
  REQUIRE(c.R != 0, MSA_ERR_UNSUPPORTED, "router key row h_kv*d=%d not supported", W);
  const int grid = msa::route_grid(dtype, c, W, h_kv, h_qr, sm_count(), n_chunks);
  REQUIRE(grid >= 1, MSA_ERR_CUDA, "occupancy query failed");
  const size_t need = kHeader + (size_t)passes * grid * bp * k * sizeof(unsigned long long);
  REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "workspace %zu bytes at %p, need %zu (256-byte aligned)", ws_bytes,
          ws, need);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, kHeader, st);
  if (e != cudaSuccess) return cuda_fail(e, "workspace header reset");
  unsigned char* base = static_cast<unsigned char*>(ws);
  const int64_t words = (n_docs + 31) / 32;
  const size_t qstride = (size_t)T * h_qr * d * esize(dtype);
  for (int pass = 0; pass < passes; ++pass) {
    const int b0 = pass * bp;
    const int nb = std::min(bp, B - b0);
    if (nb <= 0) break;
    msa::RouteParams p{};
    p.qr = static_cast<const unsigned char*>(Q_r) + (size_t)b0 * qstride;
    p.kr = Kbar_r;
    p.invk = kr_inv_norm;
    p.coff = doc_chunk_off;
    p.excl = exclude_bits ? exclude_bits + (size_t)b0 * words : nullptr;
    p.n_docs = n_docs;
    p.n_chunks = n_chunks;
    p.words = words;
    p.B = nb;
    p.T = T;
    p.h_qr = h_qr;
    p.h_kv = h_kv;
    p.d = d;
    p.k = k;
    p.top_ids = top_ids + (size_t)b0 * k;
    p.top_scores = top_scores + (size_t)b0 * k;
    p.doc_scores = doc_scores ? doc_scores + (size_t)b0 * n_docs : nullptr;
    p.cand = reinterpret_cast<unsigned long long*>(base + kHeader) + (size_t)pass * grid * bp * k;
    p.counter = reinterpret_cast<unsigned int*>(base) + 1 + pass;
    p.err = reinterpret_cast<int*>(base);
    p.inv_bulk = (h_kv % 4 == 0 && aligned16(kr_inv_norm)) ? 1 : 0;
    e = msa::route_launch(dtype, c, p, grid, st);
    if (e != cudaSuccess) return cuda_fail(e, "msa_route_topk launch");
  }
  return ok();
}

msa_status msa_workspace_status(const void* ws, int32_t* code, void* stream) {
  REQUIRE(ws && code, MSA_ERR_INVALID_ARG, "null pointer");
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "msa_workspace_status");
  *code = v;
  if (v != 0) return fail(MSA_ERR_DEVICE, "device status %d recorded in the workspace", v);
  return ok();
}

msa_status msa_gather(const int32_t* top_ids, int32_t B, int32_t k,
                      const int64_t* doc_chunk_off, int64_t n_docs, const void* Kbar,
                      const void* Vbar, int32_t h_kv, int32_t d, int32_t dtype, int32_t max_ctx,
                      int32_t* gather_idx, int32_t* ctx_len, void* ctxK, void* ctxV, void* ws,
                      size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && k >= 1 && k <= 32 && max_ctx >= 0 && n_docs >= 1, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d k=%d max_ctx=%d)", B, k, max_ctx);
  REQUIRE(ws && ws_bytes >= kHeader && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "gather needs a 256-byte aligned workspace of >= 256 bytes");
  if (B == 0) return ok();
  REQUIRE(top_ids && doc_chunk_off && gather_idx && ctx_len && Kbar && Vbar && ctxK && ctxV,
          MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(aligned16(Kbar) && aligned16(Vbar) && aligned16(ctxK) && aligned16(ctxV),
          MSA_ERR_INVALID_ARG, "bank and context must be 16-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
  msa::GatherParams p{top_ids, doc_chunk_off, n_docs, B, k, max_ctx,
                      (int64_t)h_kv * d * (int64_t)esize(dtype), Kbar, Vbar, gather_idx,
                      ctx_len, ctxK, ctxV, static_cast<int*>(ws)};
  e = msa::launch_gather(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_gather launch");
  return ok();
}

// ----------------------------------------------------------------------------- host fetch
struct msa_fetch {
  int32_t max_B = 0, max_k = 0;
  int32_t* ids_host = nullptr;  // pinned
  cudaEvent_t ids_ready = nullptr, copy_done = nullptr;
  int32_t B = 0, k = 0;
  bool pending = false;
};

msa_status msa_fetch_create(int32_t max_B, int32_t max_k, msa_fetch** out) {
  REQUIRE(out && max_B >= 1 && max_k >= 1 && max_k <= 32, MSA_ERR_INVALID_ARG,
          "bad fetch context sizes");
  msa_fetch* f = new msa_fetch();
  f->max_B = max_B;
  f->max_k = max_k;
  cudaError_t e = cudaHostAlloc(&f->ids_host, (size_t)max_B * max_k * sizeof(int32_t),
                                cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f->ids_ready, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f->copy_done, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    msa_fetch_destroy(f);
    return cuda_fail(e, "msa_fetch_create");
  }
  *out = f;
  return ok();
}

void msa_fetch_destroy(msa_fetch* f) {
  if (!f) return;
  if (f->ids_host) cudaFreeHost(f->ids_host);
  if (f->ids_ready) cudaEventDestroy(f->ids_ready);
  if (f->copy_done) cudaEventDestroy(f->copy_done);
  delete f;
}

msa_status msa_fetch_begin(msa_fetch* f, const int32_t* top_ids, int32_t B, int32_t k,
                           const int64_t* doc_chunk_off, int64_t n_docs, int32_t max_ctx,
                           int32_t* gather_idx, int32_t* ctx_len, void* ws, size_t ws_bytes,
                           void* stream) {
  REQUIRE(f, MSA_ERR_INVALID_ARG, "null fetch context");
  REQUIRE(B >= 1 && B <= f->max_B && k >= 1 && k <= f->max_k && max_ctx >= 0 && n_docs >= 1,
          MSA_ERR_INVALID_ARG, "B=%d k=%d outside the context's %d x %d", B, k, f->max_B,
          f->max_k);
  REQUIRE(top_ids && doc_chunk_off && gather_idx && ctx_len, MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(ws && ws_bytes >= kHeader && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "fetch needs a 256-byte aligned workspace of >= 256 bytes");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
  msa::GatherParams p{top_ids, doc_chunk_off, n_docs, B, k, max_ctx, 16, nullptr, nullptr,
                      gather_idx, ctx_len, nullptr, nullptr, static_cast<int*>(ws)};
  e = msa::launch_gather(p, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(f->ids_host, top_ids, (size_t)B * k * sizeof(int32_t),
                        cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaEventRecord(f->ids_ready, st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_fetch_begin");
  f->B = B;
  f->k = k;
  f->pending = true;
  return ok();
}

msa_status msa_fetch_finish(msa_fetch* f, const int64_t* coff, int64_t n_docs,
                            const void* Kbar_host, const void* Vbar_host, int32_t h_kv,
                            int32_t d, int32_t dtype, int32_t max_ctx, void* ctxK, void* ctxV,
                            void* stream, void* copy_stream, int32_t timeout_ms) {
  REQUIRE(f && f->pending, MSA_ERR_INVALID_ARG, "msa_fetch_finish without msa_fetch_begin");
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(coff && Kbar_host && Vbar_host && ctxK && ctxV && max_ctx >= 0, MSA_ERR_INVALID_ARG,
          "null pointer");
  // bounded host wait for the selected ids
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    cudaError_t q = cudaEventQuery(f->ids_ready);
    if (q == cudaSuccess) break;
    if (q != cudaErrorNotReady) return cuda_fail(q, "waiting for the selected ids");
    const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(
                        std::chrono::steady_clock::now() - t0).count();
    if (ms >= timeout_ms)
      return fail(MSA_ERR_TIMEOUT, "selected ids not ready after %d ms", timeout_ms);
    std::this_thread::yield();
  }
  f->pending = false;
  cudaStream_t st = (cudaStream_t)stream, cst = (cudaStream_t)copy_stream;
  cudaError_t e = cudaStreamWaitEvent(cst, f->ids_ready, 0);
  if (e != cudaSuccess) return cuda_fail(e, "copy stream wait");
  const size_t row = (size_t)h_kv * d * esize(dtype);
  const unsigned char* hk = static_cast<const unsigned char*>(Kbar_host);
  const unsigned char* hv = static_cast<const unsigned char*>(Vbar_host);
  unsigned char* dk = static_cast<unsigned char*>(ctxK);
  unsigned char* dv = static_cast<unsigned char*>(ctxV);
  std::vector<int32_t> ids;
  ids.reserve(f->k);
  for (int b = 0; b < f->B; ++b) {
    ids.clear();
    for (int j = 0; j < f->k; ++j) {
      const int32_t id = f->ids_host[b * f->k + j];
      if (id >= 0 && id < n_docs) ids.push_back(id);
    }
    std::sort(ids.begin(), ids.end());
    int64_t off = 0;
    size_t q = 0;
    while (q < ids.size() && off < max_ctx) {
      // merge docs whose chunk ranges are adjacent in the bank into one copy
      int64_t src = coff[ids[q]], end = coff[ids[q] + 1];
      size_t r = q + 1;
      while (r < ids.size() && coff[ids[r]] == end) end = coff[ids[r++] + 1];
      int64_t n = end - src;
      if (off + n > max_ctx) n = max_ctx - off;
      if (n > 0) {
        const size_t dst = ((size_t)b * max_ctx + off) * row;
        e = cudaMemcpyAsync(dk + dst, hk + src * row, n * row, cudaMemcpyHostToDevice, cst);
        if (e == cudaSuccess)
          e = cudaMemcpyAsync(dv + dst, hv + src * row, n * row, cudaMemcpyHostToDevice, cst);
        if (e != cudaSuccess) return cuda_fail(e, "host bank fetch");
      }
      off += n;
      q = r;
    }
  }
  e = cudaEventRecord(f->copy_done, cst);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, f->copy_done, 0);
  if (e != cudaSuccess) return cuda_fail(e, "fetch completion event");
  return ok();
}

// ----------------------------------------------------------------------------- attention
size_t msa_sparse_attend_workspace(int32_t B, int32_t T, int32_t h_q, int32_t h_kv, int32_t d,
                                   int32_t max_ctx, int32_t L_loc) {
  if (B < 1 || T < 1 || h_q < 1 || h_kv < 1 || d < 2 || max_ctx < 0 || L_loc < 1) return kHeader;
  const msa::AttendPlan pl = msa::attend_plan(B, T, h_q, h_kv, d, max_ctx, L_loc, sm_count());
  size_t need = kHeader + pl.cs_bytes + pl.part_o_bytes + pl.part_ml_bytes + pl.ctr_bytes;
  if (h_q % h_kv == 0) {  // the decode kernel (bf16) lays out the same workspace differently
    const msa::DecPlan dp = msa::attend_dec_plan(B, T, h_q, h_kv, d, max_ctx, L_loc, sm_count());
    if (dp.ok)
      need = std::max(need, kHeader + dp.ctr_bytes + dp.part_ml_bytes + dp.part_o_bytes);
    const msa::AtcPlan ap = msa::attend_tc_plan(B, T, h_q, h_kv, d, max_ctx, L_loc);
    if (ap.ok)
      need = std::max(need, kHeader + ap.q_bytes + ap.k_bytes + ap.vl_bytes + ap.vc_bytes);
  }
  return need;
}

msa_status msa_sparse_attend(const void* Q, int32_t B, int32_t T, int32_t h_q,
                             const void* K_loc, const void* V_loc, int32_t L_loc,
                             const void* ctxK, const void* ctxV, const int32_t* ctx_len,
                             int32_t max_ctx, int32_t h_kv, int32_t d, int32_t dtype,
                             int32_t pos0, float rope_base, float scale, void* O, void* ws,
                             size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && T >= 1 && L_loc >= T && max_ctx >= 0, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d T=%d L_loc=%d max_ctx=%d)", B, T, L_loc, max_ctx);
  REQUIRE(h_q >= h_kv && h_q % h_kv == 0, MSA_ERR_INVALID_ARG, "h_q %d not a multiple of h_kv %d",
          h_q, h_kv);
  REQUIRE(pos0 >= 0, MSA_ERR_INVALID_ARG, "pos0 %d", pos0);
  if (B == 0) return ok();
  REQUIRE(Q && K_loc && V_loc && ctx_len && O, MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(max_ctx == 0 || (ctxK && ctxV), MSA_ERR_INVALID_ARG, "null context");
  REQUIRE(aligned16(Q) && aligned16(K_loc) && aligned16(V_loc) &&
              (max_ctx == 0 || (aligned16(ctxK) && aligned16(ctxV))),
          MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  if (dtype == 1) {
    const msa::DecPlan dp = msa::attend_dec_plan(B, T, h_q, h_kv, d, max_ctx, L_loc, sm_count());
    if (dp.ok) {
      const size_t need = kHeader + dp.ctr_bytes + dp.part_ml_bytes + dp.part_o_bytes;
      REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
              MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes,
              need);
      unsigned char* w8 = static_cast<unsigned char*>(ws);
      msa::DecParams q{};
      q.Q = static_cast<const __nv_bfloat16*>(Q);
      q.Kl = static_cast<const __nv_bfloat16*>(K_loc);
      q.Vl = static_cast<const __nv_bfloat16*>(V_loc);
      q.cK = static_cast<const __nv_bfloat16*>(ctxK);
      q.cV = static_cast<const __nv_bfloat16*>(ctxV);
      q.ctx_len = ctx_len;
      q.B = B;
      q.T = T;
      q.h_q = h_q;
      q.h_kv = h_kv;
      q.L = L_loc;
      q.Ls = L_loc;
      q.L_dev = nullptr;
      q.max_ctx = max_ctx;
      q.rope = rope_base > 0.f ? 1 : 0;
      q.pos0 = pos0;
      msa::rope_turns(q.rope ? (double)rope_base : 0.0, 128, q.rope_turns);
      q.scale_log2 = sc * 1.4426950408889634f;
      q.CT = dp.CT;
      q.max_seg = dp.max_seg;
      q.grid = dp.grid;
      q.err = reinterpret_cast<int*>(w8);
      q.part_ml = reinterpret_cast<float*>(w8 + kHeader + dp.ctr_bytes);
      q.part_o = reinterpret_cast<float*>(w8 + kHeader + dp.ctr_bytes + dp.part_ml_bytes);
      q.O = static_cast<__nv_bfloat16*>(O);
      q.start_status = 1;  // no memset node: the attention kernel starts the status word
      cudaStream_t st = (cudaStream_t)stream;
      cudaError_t e = msa::launch_attend_dec(q, dp, st);
      if (e != cudaSuccess) return cuda_fail(e, "msa_sparse_attend launch");
      return ok();
    }
    const msa::AtcPlan ap = msa::attend_tc_plan(B, T, h_q, h_kv, d, max_ctx, L_loc);
    if (ap.ok) {  // long queries: tensor-core attention
      const size_t need = kHeader + ap.q_bytes + ap.k_bytes + ap.vl_bytes + ap.vc_bytes;
      REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
              MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes,
              need);
      unsigned char* w8 = static_cast<unsigned char*>(ws);
      msa::AtcParams a{};
      a.Q = static_cast<const __nv_bfloat16*>(Q);
      a.Kl = static_cast<const __nv_bfloat16*>(K_loc);
      a.Vl = static_cast<const __nv_bfloat16*>(V_loc);
      a.cK = static_cast<const __nv_bfloat16*>(ctxK);
      a.cV = static_cast<const __nv_bfloat16*>(ctxV);
      a.ctx_len = ctx_len;
      a.B = B;
      a.T = T;
      a.h_q = h_q;
      a.h_kv = h_kv;
      a.L = L_loc;
      a.max_ctx = max_ctx;
      a.rope = rope_base > 0.f ? 1 : 0;
      a.pos0 = pos0;
      msa::rope_turns(a.rope ? (double)rope_base : 0.0, 128, a.rope_turns);
      a.scale_log2 = sc * 1.4426950408889634f;
      a.err = reinterpret_cast<int*>(w8);
      a.O = static_cast<__nv_bfloat16*>(O);
      cudaStream_t st = (cudaStream_t)stream;
      cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);  // status word
      if (e == cudaSuccess) e = msa::launch_attend_tc(a, ap, w8 + kHeader, sm_count(), st);
      if (e != cudaSuccess) return cuda_fail(e, "msa_sparse_attend launch");
      return ok();
    }
  }
  const msa::AttendPlan pl = msa::attend_plan(B, T, h_q, h_kv, d, max_ctx, L_loc, sm_count());
  const size_t need = kHeader + pl.cs_bytes + pl.part_o_bytes + pl.part_ml_bytes + pl.ctr_bytes;
  REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, need);
  unsigned char* base = static_cast<unsigned char*>(ws) + kHeader;
  msa::AttendParams p{};
  p.Q = Q;
  p.Kl = K_loc;
  p.Vl = V_loc;
  p.cK = ctxK;
  p.cV = ctxV;
  p.ctx_len = ctx_len;
  p.B = B;
  p.T = T;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.d = d;
  p.L = L_loc;
  p.max_ctx = max_ctx;
  p.rope = rope_base > 0.f ? 1 : 0;
  p.cs = reinterpret_cast<const float2*>(base);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.S = pl.S;
  p.KPS = pl.KPS;
  p.RB = pl.RB;
  p.NRB = pl.NRB;
  p.part_o = reinterpret_cast<float*>(base + pl.cs_bytes);
  p.part_ml = reinterpret_cast<float*>(base + pl.cs_bytes + pl.part_o_bytes);
  p.counters = reinterpret_cast<unsigned int*>(base + pl.cs_bytes + pl.part_o_bytes +
                                               pl.part_ml_bytes);
  p.O = O;
  cudaError_t e = msa::launch_attend(p, dtype, (double)rope_base, pos0, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "msa_sparse_attend launch");
  return ok();
}

// ----------------------------------------------------------------------------- backward
size_t msa_sparse_attend_backward_workspace(int32_t B, int32_t T, int32_t h_q, int32_t h_kv,
                                            int32_t d, int32_t max_ctx, int32_t L_loc) {
  const msa::BwdPlan pl = msa::attend_bwd_plan(B, T, h_q, h_kv, d, max_ctx, L_loc);
  if (!pl.ok) return kHeader;
  return kHeader + pl.fwd_bytes + pl.o_bytes + 2 * pl.lse_bytes;
}

msa_status msa_sparse_attend_backward(const void* Q, int32_t B, int32_t T, int32_t h_q,
                                      const void* K_loc, const void* V_loc, int32_t L_loc,
                                      const void* ctxK, const void* ctxV, const int32_t* ctx_len,
                                      int32_t max_ctx, int32_t h_kv, int32_t d, int32_t dtype,
                                      int32_t pos0, float rope_base, float scale, const void* dO,
                                      float* dQ, float* dK_loc, float* dV_loc, float* dK_ctx,
                                      float* dV_ctx, void* ws, size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && T >= 1 && L_loc >= T && max_ctx >= 0 && h_q >= 1, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d T=%d L_loc=%d max_ctx=%d)", B, T, L_loc, max_ctx);
  REQUIRE(h_q % h_kv == 0, MSA_ERR_INVALID_ARG, "h_q %d not a multiple of h_kv %d", h_q, h_kv);
  REQUIRE(dtype == MSA_BF16 && d == 128, MSA_ERR_UNSUPPORTED,
          "the attention backward runs on bf16 with d = 128");
  const msa::BwdPlan pl = msa::attend_bwd_plan(B, T, h_q, h_kv, d, max_ctx, L_loc);
  REQUIRE(pl.ok, MSA_ERR_UNSUPPORTED, "h_q / h_kv = %d must divide 64", h_q / h_kv);
  if (B == 0) return ok();
  REQUIRE(Q && K_loc && V_loc && ctx_len && dO && dQ && dK_loc && dV_loc, MSA_ERR_INVALID_ARG,
          "null tensor");
  REQUIRE(max_ctx == 0 || (ctxK && ctxV && dK_ctx && dV_ctx), MSA_ERR_INVALID_ARG,
          "null context");
  REQUIRE(aligned16(Q) && aligned16(K_loc) && aligned16(V_loc) && aligned16(dO) &&
              aligned16(dQ) && aligned16(dK_loc) && aligned16(dV_loc) &&
              (max_ctx == 0 || (aligned16(ctxK) && aligned16(ctxV) && aligned16(dK_ctx) &&
                                aligned16(dV_ctx))),
          MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const size_t need = msa_sparse_attend_backward_workspace(B, T, h_q, h_kv, d, max_ctx, L_loc);
  REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, need);
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  unsigned char* w8 = static_cast<unsigned char*>(ws);
  msa::BwdParams p{};
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.Kl = static_cast<const __nv_bfloat16*>(K_loc);
  p.Vl = static_cast<const __nv_bfloat16*>(V_loc);
  p.cK = static_cast<const __nv_bfloat16*>(ctxK);
  p.cV = static_cast<const __nv_bfloat16*>(ctxV);
  p.ctx_len = ctx_len;
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.B = B;
  p.T = T;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.L = L_loc;
  p.max_ctx = max_ctx;
  p.rope = rope_base > 0.f ? 1 : 0;
  p.pos0 = pos0;
  msa::rope_turns(p.rope ? (double)rope_base : 0.0, 128, p.rope_turns);
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.dQ = dQ;
  p.dKl = dK_loc;
  p.dVl = dV_loc;
  p.dKc = dK_ctx;
  p.dVc = dV_ctx;
  p.err = reinterpret_cast<int*>(w8);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);  // status word
  if (e == cudaSuccess) e = msa::launch_attend_bwd(p, pl, w8 + kHeader, sm_count(), st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_sparse_attend_backward launch");
  return ok();
}

msa_status msa_scatter_bank_grad(const int32_t* gather_idx, const int32_t* ctx_len, int32_t B,
                                 int32_t max_ctx, int32_t h_kv, int32_t d, const float* dK_ctx,
                                 const float* dV_ctx, float* dKbar, float* dVbar,
                                 int64_t n_chunks, void* ws, size_t ws_bytes, void* stream) {
  REQUIRE(B >= 0 && max_ctx >= 0 && h_kv >= 1 && (d == 64 || d == 128) && n_chunks >= 0,
          MSA_ERR_INVALID_ARG, "bad sizes (B=%d max_ctx=%d h_kv=%d d=%d)", B, max_ctx, h_kv, d);
  REQUIRE(ws && ws_bytes >= kHeader && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "needs a 256-byte aligned workspace of >= 256 bytes");
  if (B == 0 || max_ctx == 0) return ok();
  REQUIRE(gather_idx && ctx_len && dK_ctx && dV_ctx && dKbar && dVbar, MSA_ERR_INVALID_ARG,
          "null tensor");
  REQUIRE(aligned16(dK_ctx) && aligned16(dV_ctx) && aligned16(dKbar) && aligned16(dVbar),
          MSA_ERR_INVALID_ARG, "gradients must be 16-byte aligned");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e == cudaSuccess)
    e = msa::launch_scatter_bank_grad(gather_idx, ctx_len, B, max_ctx, (int64_t)h_kv * d, dK_ctx,
                                      dV_ctx, dKbar, dVbar, n_chunks,
                                      static_cast<int*>(ws), sm_count(), st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_scatter_bank_grad launch");
  return ok();
}

size_t msa_aux_routing_loss_workspace(int32_t B, int64_t n_chunks) {
  if (B < 1 || n_chunks < 1) return kHeader;
  return kHeader + msa::aux_loss_scratch_bytes(B, n_chunks);
}

msa_status msa_aux_routing_loss(const void* Q_r, int32_t B, int32_t T, int32_t h_qr,
                                const void* Kbar_r, int64_t n_chunks, int32_t h_kv, int32_t d,
                                int32_t dtype, const uint32_t* positive_bits, float tau,
                                float* loss, float* dQ_r, float* dKbar_r, void* ws,
                                size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 1 && T >= 1 && n_chunks >= 1, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d T=%d n_chunks=%lld)", B, T, (long long)n_chunks);
  REQUIRE(h_qr >= 1 && h_qr % h_kv == 0, MSA_ERR_INVALID_ARG, "h_qr %d not a multiple of h_kv %d",
          h_qr, h_kv);
  REQUIRE(tau > 0.f, MSA_ERR_INVALID_ARG, "tau must be positive");
  REQUIRE(Q_r && Kbar_r && positive_bits && loss, MSA_ERR_INVALID_ARG, "null tensor");
  const size_t need = msa_aux_routing_loss_workspace(B, n_chunks);
  REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e == cudaSuccess)
    e = msa::launch_aux_routing_loss(Q_r, B, T, h_qr, Kbar_r, n_chunks, h_kv, d, dtype,
                                     positive_bits, tau, loss, dQ_r, dKbar_r,
                                     static_cast<unsigned char*>(ws) + kHeader, sm_count(), st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_aux_routing_loss launch");
  return ok();
}

// ----------------------------------------------------------------------------- interleave
msa_status msa_assemble_local(int32_t B, int32_t n_seg, const void* const* seg_k,
                              const void* const* seg_v, const int32_t* seg_len, const void* K_q,
                              const void* V_q, int32_t T, int32_t h_kv, int32_t d, int32_t dtype,
                              int64_t L_loc, void* K_out, void* V_out, void* ws, size_t ws_bytes,
                              void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && n_seg >= 0 && n_seg <= 1024 && T >= 0 && L_loc >= T, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d n_seg=%d T=%d L_loc=%lld)", B, n_seg, T, (long long)L_loc);
  REQUIRE(ws && ws_bytes >= kHeader && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "assemble needs a 256-byte aligned workspace of >= 256 bytes");
  if (B == 0 || L_loc == 0) return ok();
  REQUIRE(K_out && V_out && (T == 0 || (K_q && V_q)) && (n_seg == 0 || (seg_k && seg_v && seg_len)),
          MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(aligned16(K_out) && aligned16(V_out) && (T == 0 || (aligned16(K_q) && aligned16(V_q))),
          MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  msa::AssembleParams p{};
  p.B = B;
  p.n_seg = n_seg;
  p.T = T;
  p.L = L_loc;
  p.row_bytes = (int64_t)h_kv * d * (dtype == 1 ? 2 : 4);
  p.seg_k = seg_k;
  p.seg_v = seg_v;
  p.seg_len = seg_len;
  p.K_q = K_q;
  p.V_q = V_q;
  p.K_out = K_out;
  p.V_out = V_out;
  p.err = static_cast<int*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e == cudaSuccess) e = msa::launch_assemble_local(p, st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_assemble_local launch");
  return ok();
}


// ------------------------------------------------------------------------ sparse generation
msa_status msa_kv_append(void* K_cache, void* V_cache, int32_t B, int32_t cap, int32_t* len_dev,
                         const void* K_new, const void* V_new, int32_t T_new, int32_t h_kv,
                         int32_t d, int32_t dtype, int32_t pos0, float rope_base, void* ws,
                         size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && cap >= 1 && T_new >= 0, MSA_ERR_INVALID_ARG, "bad sizes (B=%d cap=%d T_new=%d)",
          B, cap, T_new);
  REQUIRE(T_new <= cap, MSA_ERR_INVALID_ARG, "T_new %d exceeds the capacity %d", T_new, cap);
  REQUIRE(pos0 >= 0, MSA_ERR_INVALID_ARG, "pos0 %d", pos0);
  REQUIRE(ws && ws_bytes >= kHeader && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "append needs a 256-byte aligned workspace of >= 256 bytes");
  if (B == 0 || T_new == 0) return ok();
  REQUIRE(K_cache && V_cache && len_dev && K_new && V_new, MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(aligned16(K_cache) && aligned16(V_cache) && aligned16(K_new) && aligned16(V_new),
          MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  msa::AppendParams p{};
  p.B = B;
  p.T_new = T_new;
  p.cap = cap;
  p.row_bytes = (int64_t)h_kv * d * (int64_t)esize(dtype);
  p.K_cache = K_cache;
  p.V_cache = V_cache;
  p.K_new = K_new;
  p.V_new = V_new;
  p.len = len_dev;
  p.err = static_cast<int*>(ws);
  p.ticket = reinterpret_cast<unsigned int*>(static_cast<unsigned char*>(ws) + 4);
  p.rope = rope_base > 0.f ? 1 : 0;
  p.pos0 = pos0;
  p.d = d;
  p.esize = (int)esize(dtype);
  msa::rope_turns(p.rope ? (double)rope_base : 0.0, d, p.rope_turns);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * sizeof(int32_t), st);  // status word, ticket
  if (e == cudaSuccess) e = msa::launch_kv_append(p, sm_count(), st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_kv_append launch");
  return ok();
}

size_t msa_decode_step_workspace(int32_t B, int32_t T, int32_t h_q, int32_t h_kv, int32_t d,
                                 int32_t max_ctx, int32_t cap) {
  if (B < 1 || T < 1 || h_kv < 1 || h_q % h_kv != 0 || max_ctx < 0 || cap < T) return kHeader;
  const msa::DecPlan dp = msa::attend_dec_plan_cap(B, T, h_q, h_kv, d, max_ctx, cap, sm_count());
  if (!dp.ok) return kHeader;
  return kHeader + dp.ctr_bytes + dp.part_ml_bytes + dp.part_o_bytes;
}

msa_status msa_decode_step(const void* Q, const void* K_new, const void* V_new, int32_t B,
                           int32_t T, int32_t h_q, void* K_cache, void* V_cache, int32_t cap,
                           int32_t* len_dev, const void* ctxK, const void* ctxV,
                           const int32_t* ctx_len, int32_t max_ctx, int32_t h_kv, int32_t d,
                           int32_t dtype, int32_t pos0, float rope_base, float scale, void* O,
                           void* ws, size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(B >= 0 && T >= 1 && cap >= T && max_ctx >= 0, MSA_ERR_INVALID_ARG,
          "bad sizes (B=%d T=%d cap=%d max_ctx=%d)", B, T, cap, max_ctx);
  REQUIRE(h_q >= h_kv && h_q % h_kv == 0, MSA_ERR_INVALID_ARG, "h_q %d not a multiple of h_kv %d",
          h_q, h_kv);
  REQUIRE(pos0 >= 0, MSA_ERR_INVALID_ARG, "pos0 %d", pos0);
  const msa::DecPlan dp = msa::attend_dec_plan_cap(B, T, h_q, h_kv, d, max_ctx, cap, sm_count());
  REQUIRE(dtype == MSA_BF16 && dp.ok, MSA_ERR_UNSUPPORTED,
          "decode step: bf16, d = 128, h_kv in {1, 2, 4, 8}, (h_q / h_kv) * T <= 8");
  const size_t need = kHeader + dp.ctr_bytes + dp.part_ml_bytes + dp.part_o_bytes;
  REQUIRE(ws != nullptr && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, need);
  if (B == 0) return ok();
  REQUIRE(Q && K_new && V_new && K_cache && V_cache && len_dev && ctx_len && O,
          MSA_ERR_INVALID_ARG, "null tensor");
  REQUIRE(max_ctx == 0 || (ctxK && ctxV), MSA_ERR_INVALID_ARG, "null context");
  REQUIRE(aligned16(Q) && aligned16(K_new) && aligned16(V_new) && aligned16(K_cache) &&
              aligned16(V_cache) && (max_ctx == 0 || (aligned16(ctxK) && aligned16(ctxV))),
          MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  unsigned char* w8 = static_cast<unsigned char*>(ws);
  cudaStream_t st = (cudaStream_t)stream;
  // the append is fused into the attention launch: its first CTA starts the status word, the
  // merge kernel advances the length (no memset node, no append kernel per step)
  cudaError_t e = cudaSuccess;
  msa::DecParams q{};
  q.Q = static_cast<const __nv_bfloat16*>(Q);
  q.Kl = static_cast<const __nv_bfloat16*>(K_cache);
  q.Vl = static_cast<const __nv_bfloat16*>(V_cache);
  q.cK = static_cast<const __nv_bfloat16*>(ctxK);
  q.cV = static_cast<const __nv_bfloat16*>(ctxV);
  q.ctx_len = ctx_len;
  q.B = B;
  q.T = T;
  q.h_q = h_q;
  q.h_kv = h_kv;
  q.L = cap;
  q.Ls = cap;
  q.L_dev = len_dev;
  q.skip_on_err = 1;   // an overflowing append leaves O unwritten
  q.keys_rotated = 1;  // the cache holds keys rotated at pos0 + row
  q.K_new = static_cast<const __nv_bfloat16*>(K_new);
  q.V_new = static_cast<const __nv_bfloat16*>(V_new);
  q.L_out = reinterpret_cast<int*>(w8 + 8);
  q.max_ctx = max_ctx;
  q.rope = rope_base > 0.f ? 1 : 0;
  q.pos0 = pos0;
  msa::rope_turns(q.rope ? (double)rope_base : 0.0, 128, q.rope_turns);
  q.scale_log2 = (scale > 0.f ? scale : 1.0f / sqrtf((float)d)) * 1.4426950408889634f;
  q.CT = dp.CT;
  q.max_seg = dp.max_seg;
  q.grid = dp.grid;
  q.err = reinterpret_cast<int*>(w8);
  q.part_ml = reinterpret_cast<float*>(w8 + kHeader + dp.ctr_bytes);
  q.part_o = reinterpret_cast<float*>(w8 + kHeader + dp.ctr_bytes + dp.part_ml_bytes);
  q.O = static_cast<__nv_bfloat16*>(O);
  if (e == cudaSuccess) e = msa::launch_attend_dec(q, dp, st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_decode_step launch");
  return ok();
}

// ------------------------------------------------------------------ encode from hidden states
size_t msa_encode_hidden_workspace(int64_t n_chunks) {
  if (n_chunks < 0) return kHeader;
  return kHeader + (((size_t)n_chunks * 3 * sizeof(int32_t) + 255) & ~(size_t)255);
}

msa_status msa_encode_hidden(const void* H, int64_t n_tok, int32_t D, const void* W_k,
                             const void* W_v, const void* W_r, const int64_t* doc_tok_off_host,
                             int64_t n_docs, int32_t chunk, int32_t h_kv, int32_t d,
                             int32_t dtype, float rope_base, void* Kbar, void* Vbar,
                             void* Kbar_r, int64_t* doc_chunk_off, int64_t n_chunks, void* ws,
                             size_t ws_bytes, void* stream) {
  msa_status s = check_common(h_kv, d, dtype);
  if (s != MSA_OK) return s;
  REQUIRE(dtype == MSA_BF16 && d == 128 && chunk == 64 && h_kv % 2 == 0 && h_kv <= 64,
          MSA_ERR_UNSUPPORTED, "encode from hidden states: bf16, d = 128, chunk = 64, even h_kv");
  REQUIRE(D >= 64 && D % 64 == 0, MSA_ERR_UNSUPPORTED, "hidden size %d (a multiple of 64)", D);
  REQUIRE(n_docs >= 0 && n_tok >= 0 && n_chunks >= 0 && n_tok < (1ll << 31), MSA_ERR_INVALID_ARG,
          "bad sizes (n_tok=%lld n_docs=%lld)", (long long)n_tok, (long long)n_docs);
  REQUIRE(doc_tok_off_host && doc_chunk_off, MSA_ERR_INVALID_ARG, "null offset pointer");
  REQUIRE(doc_tok_off_host[n_docs] == n_tok, MSA_ERR_INVALID_ARG,
          "doc_tok_off[n_docs] = %lld != n_tok %lld", (long long)doc_tok_off_host[n_docs],
          (long long)n_tok);
  const int64_t nc = msa_count_chunks(doc_tok_off_host, n_docs, chunk);
  REQUIRE(nc >= 0, MSA_ERR_INVALID_ARG, "doc_tok_off must start at 0 and not decrease");
  REQUIRE(nc == n_chunks, MSA_ERR_INVALID_ARG, "n_chunks %lld != %lld implied by the offsets",
          (long long)n_chunks, (long long)nc);
  const size_t need = msa_encode_hidden_workspace(n_chunks);
  REQUIRE(ws && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0,
          MSA_ERR_WORKSPACE, "workspace %zu bytes, need %zu (256-byte aligned)", ws_bytes, need);
  if (n_chunks > 0) {
    REQUIRE(H && W_k && W_v && W_r && Kbar && Vbar && Kbar_r, MSA_ERR_INVALID_ARG,
            "null tensor");
    REQUIRE(aligned16(H) && aligned16(W_k) && aligned16(W_v) && aligned16(W_r) &&
                aligned16(Kbar) && aligned16(Vbar) && aligned16(Kbar_r),
            MSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  }
  // chunk table [first token row, valid rows, position of the first row in its document] and
  // the chunk offsets, from the host offsets
  std::vector<int32_t> tab((size_t)n_chunks * 3);
  std::vector<int64_t> coff((size_t)n_docs + 1);
  int64_t c = 0;
  for (int64_t i = 0; i < n_docs; ++i) {
    coff[i] = c;
    for (int64_t s0 = doc_tok_off_host[i]; s0 < doc_tok_off_host[i + 1]; s0 += chunk, ++c) {
      tab[3 * c] = (int32_t)s0;
      tab[3 * c + 1] = (int32_t)std::min<int64_t>(chunk, doc_tok_off_host[i + 1] - s0);
      tab[3 * c + 2] = (int32_t)(s0 - doc_tok_off_host[i]);
    }
  }
  coff[n_docs] = c;
  cudaStream_t st = (cudaStream_t)stream;
  unsigned char* w8 = static_cast<unsigned char*>(ws);
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e == cudaSuccess && n_chunks > 0)
    e = cudaMemcpyAsync(w8 + kHeader, tab.data(), tab.size() * sizeof(int32_t),
                        cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(doc_chunk_off, coff.data(), coff.size() * sizeof(int64_t),
                        cudaMemcpyHostToDevice, st);
  msa::EhParams p{};
  p.n_chunks = n_chunks;
  p.n_tiles = h_kv / 2;
  p.n_units = ((n_chunks + 1) / 2) * 3 * p.n_tiles;
  p.D = D;
  p.h_kv = h_kv;
  p.ctab = reinterpret_cast<const int32_t*>(w8 + kHeader);
  p.rope = rope_base > 0.f ? 1 : 0;
  msa::rope_turns(p.rope ? (double)rope_base : 0.0, d, p.rope_turns);
  p.Kbar = static_cast<__nv_bfloat16*>(Kbar);
  p.Vbar = static_cast<__nv_bfloat16*>(Vbar);
  p.Kbar_r = static_cast<__nv_bfloat16*>(Kbar_r);
  p.err = reinterpret_cast<int*>(w8);
  if (e == cudaSuccess) e = msa::launch_encode_hidden(p, H, n_tok, W_k, W_v, W_r, sm_count(), st);
  // the host tables above are sources of the copies: they must outlive them
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "msa_encode_hidden");
  return ok();
}

}  // extern "C"
