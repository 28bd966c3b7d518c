// libstem C-ABI: argument validation, the host TPD planner, workspace carve-up
// and the entry points declared in include/stem.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "stem_internal.cuh"

namespace stem {
namespace {

thread_local char g_err[512] = "";

stem_status_t fail(stem_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
stem_status_t fail(stem_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

stem_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(STEM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------- TPD planner
// Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍", section
// "TPD：优先级排序": budget decays linearly, end = mu * start, total redistributed.
// k_i(r) = min(i+1, max(m_i, floor(r * w_i))), w_i = (1 - (1-mu) i/(N-1)) (i+1),
// m_i = min(2, i+1).  The plan is the midpoint of the first interval of r on which
// the total reaches T; it is located by bisection on r, then pinned to the exact
// jump values n / w_i that bound that interval.
double tpd_weight(int N, double mu, int i) {
  if (N == 1) return 1.0;
  volatile double t = ((1.0 - mu) * static_cast<double>(i)) / static_cast<double>(N - 1);
  return (1.0 - t) * static_cast<double>(i + 1);
}

struct Planner {
  int N;
  double mu;
  std::vector<double> w;
  Planner(int n, double m) : N(n), mu(m), w(n) {
    for (int i = 0; i < n; ++i) w[i] = tpd_weight(n, m, i);
  }
  int64_t total(double r) const {
    int64_t s = 0;
    for (int i = 0; i < N; ++i) {
      double f = floor(r * w[i]);
      int64_t m = std::min(2, i + 1);
      int64_t k = f < static_cast<double>(m) ? m : (f > static_cast<double>(i + 1) ? i + 1 : static_cast<int64_t>(f));
      s += k;
    }
    return s;
  }
  // smallest jump value strictly greater than x (+inf if none)
  double next_jump(double x) const {
    double best = INFINITY;
    for (int i = 0; i < N; ++i) {
      const int lo_n = std::min(2, i + 1) + 1;
      if (lo_n > i + 1) continue;
      double f = floor(x * w[i]);
      int64_t n = std::max<int64_t>(lo_n, static_cast<int64_t>(f < 0 ? 0 : f));
      while (n > lo_n && static_cast<double>(n - 1) / w[i] > x) --n;
      while (n <= i + 1 && static_cast<double>(n) / w[i] <= x) ++n;
      if (n <= i + 1) best = std::min(best, static_cast<double>(n) / w[i]);
    }
    return best;
  }
  double last_jump() const {
    double best = -INFINITY;
    for (int i = 0; i < N; ++i)
      if (std::min(2, i + 1) + 1 <= i + 1) best = std::max(best, static_cast<double>(i + 1) / w[i]);
    return best;
  }
};

int64_t tpd_target(int N, double keep) {
  const int64_t C = static_cast<int64_t>(N) * (N + 1) / 2;
  int64_t T = static_cast<int64_t>(floor(keep * static_cast<double>(C) + 0.5));
  T = std::min(T, C);
  T = std::max(T, static_cast<int64_t>(2) * N - 1);
  return T;
}

void plan_uncached(int N, double keep, double mu, double* r_out, int64_t* total_out) {
  Planner P(N, mu);
  const int64_t T = tpd_target(N, keep);
  const double first = P.next_jump(0.0);
  if (!std::isfinite(first)) {  // no jumps at all (N <= 2)
    *r_out = 1.0;
    *total_out = P.total(1.0);
    return;
  }
  if (P.total(first / 2.0) >= T) {
    *r_out = first / 2.0;
    *total_out = P.total(*r_out);
    return;
  }
  double lo = 0.0, hi = 2.0 * P.last_jump();
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (P.total(mid) >= T) hi = mid; else lo = mid;
  }
  // Walk the jump values from just below lo: the first interval whose midpoint
  // total reaches T is the plan (midpoints sit far from any rounding-sensitive jump).
  double J = P.next_jump(lo * (1.0 - 1e-12));
  for (;;) {
    const double J2 = P.next_jump(J);
    const double mid = std::isfinite(J2) ? 0.5 * (J + J2) : 2.0 * J;
    if (!std::isfinite(J2) || P.total(mid) >= T) {
      *r_out = mid;
      break;
    }
    J = J2;
  }
  *total_out = P.total(*r_out);
}

std::mutex g_plan_mu;
std::map<std::tuple<int, double, double>, std::pair<double, int64_t>> g_plan_cache;

void plan(int N, double keep, double mu, double* r, int64_t* total) {
  const auto key = std::make_tuple(N, keep, mu);
  {
    std::lock_guard<std::mutex> g(g_plan_mu);
    auto it = g_plan_cache.find(key);
    if (it != g_plan_cache.end()) {
      *r = it->second.first;
      *total = it->second.second;
      return;
    }
  }
  plan_uncached(N, keep, mu, r, total);
  std::lock_guard<std::mutex> g(g_plan_mu);
  if (g_plan_cache.size() > 4096) g_plan_cache.clear();
  g_plan_cache[key] = std::make_pair(*r, *total);
}

// ------------------------------------------------------------- validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

stem_status_t check_problem(const stem_problem_t* pr) {
  if (pr == nullptr) return fail(STEM_ERR_INVALID, "problem is NULL");
  if (pr->num_seqs < 1 || pr->num_seqs > STEM_MAX_SEQS)
    return fail(STEM_ERR_INVALID, "num_seqs %d outside [1, %d]", pr->num_seqs, STEM_MAX_SEQS);
  if (pr->cu_seqlens == nullptr) return fail(STEM_ERR_INVALID, "cu_seqlens is NULL");
  if (pr->cu_seqlens[0] != 0) return fail(STEM_ERR_INVALID, "cu_seqlens[0] must be 0");
  for (int b = 0; b < pr->num_seqs; ++b)
    if (pr->cu_seqlens[b + 1] <= pr->cu_seqlens[b])
      return fail(STEM_ERR_INVALID, "sequence %d has length %d", b, pr->cu_seqlens[b + 1] - pr->cu_seqlens[b]);
  if (pr->num_q_heads < 1 || pr->num_kv_heads < 1 || pr->num_q_heads % pr->num_kv_heads != 0)
    return fail(STEM_ERR_INVALID, "num_q_heads %d must be a positive multiple of num_kv_heads %d", pr->num_q_heads,
                pr->num_kv_heads);
  if (pr->num_q_heads > 256) return fail(STEM_ERR_UNSUPPORTED, "num_q_heads %d > 256", pr->num_q_heads);
  if (pr->head_dim != 64 && pr->head_dim != 128)
    return fail(STEM_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", pr->head_dim);
  if (pr->block_size != 64 && pr->block_size != 128)
    return fail(STEM_ERR_UNSUPPORTED, "block_size %d (supported: 64, 128)", pr->block_size);
  if (pr->dtype != STEM_DT_BF16 && pr->dtype != STEM_DT_FP8_E4M3)
    return fail(STEM_ERR_INVALID, "unknown dtype %d", static_cast<int>(pr->dtype));
  if (pr->dtype == STEM_DT_FP8_E4M3) {
    if (pr->head_dim != 128 || pr->block_size != 128)
      return fail(STEM_ERR_UNSUPPORTED, "FP8 needs head_dim 128 and block_size 128");
    if (!(pr->q_scale > 0.f) || !(pr->k_scale > 0.f) || !(pr->v_scale > 0.f) || !std::isfinite(pr->q_scale) ||
        !std::isfinite(pr->k_scale) || !std::isfinite(pr->v_scale))
      return fail(STEM_ERR_INVALID, "FP8 scales must be finite and positive");
  }
  if (!(pr->keep > 0.0 && pr->keep <= 1.0)) return fail(STEM_ERR_INVALID, "keep %g outside (0, 1]", pr->keep);
  if (!(pr->mu > 0.0 && pr->mu <= 1.0)) return fail(STEM_ERR_INVALID, "mu %g outside (0, 1]", pr->mu);
  if (!std::isfinite(pr->beta)) return fail(STEM_ERR_INVALID, "beta is not finite");
  if (!std::isfinite(pr->softmax_scale)) return fail(STEM_ERR_INVALID, "softmax_scale is not finite");
  if (pr->shared_lists != 0 && pr->shared_lists != 1)
    return fail(STEM_ERR_INVALID, "shared_lists %d must be 0 or 1", pr->shared_lists);
  long long T = pr->cu_seqlens[pr->num_seqs];
  if (T > (1ll << 30)) return fail(STEM_ERR_UNSUPPORTED, "total tokens %lld too large", T);
  for (int b = 0; b < pr->num_seqs; ++b) {
    const int len = pr->cu_seqlens[b + 1] - pr->cu_seqlens[b];
    const int nb = (len + pr->block_size - 1) / pr->block_size;
    if (nb > STEM_MAX_BLOCKS)
      return fail(STEM_ERR_UNSUPPORTED, "sequence %d has %d blocks (max %d)", b, nb, STEM_MAX_BLOCKS);
  }
  return STEM_OK;
}

stem_status_t check_paged(const stem_problem_t* pr, const stem_paged_kv_t* pg) {
  if (pg == nullptr) return STEM_OK;
  if (pg->k_cache == nullptr || pg->v_cache == nullptr || pg->block_table == nullptr)
    return fail(STEM_ERR_INVALID, "paged cache pointers must not be NULL");
  if (!aligned16(pg->k_cache) || !aligned16(pg->v_cache))
    return fail(STEM_ERR_INVALID, "paged caches must be 16-byte aligned");
  if (pg->page_size != STEM_PAGE_SIZE)
    return fail(STEM_ERR_UNSUPPORTED, "page_size %d (supported: %d)", pg->page_size, STEM_PAGE_SIZE);
  if (pg->num_slots < 1) return fail(STEM_ERR_INVALID, "num_slots %d", pg->num_slots);
  for (int b = 0; b < pr->num_seqs; ++b) {
    const int len = pr->cu_seqlens[b + 1] - pr->cu_seqlens[b];
    if ((len + STEM_PAGE_SIZE - 1) / STEM_PAGE_SIZE > pg->max_pages_per_seq)
      return fail(STEM_ERR_INVALID, "sequence %d needs more than max_pages_per_seq=%d pages", b,
                  pg->max_pages_per_seq);
  }
  return STEM_OK;
}

void build_batch(const stem_problem_t* pr, Batch* bt) {
  memset(bt, 0, sizeof(*bt));
  bt->num_seqs = pr->num_seqs;
  bt->block = pr->block_size;
  bt->mu = pr->mu;
  bt->total_tokens = pr->cu_seqlens[pr->num_seqs];
  int rows = 0;
  long long sc = 0, nz = 0;
  for (int b = 0; b < pr->num_seqs; ++b) {
    SeqInfo& s = bt->seq[b];
    s.tok0 = pr->cu_seqlens[b];
    s.len = pr->cu_seqlens[b + 1] - pr->cu_seqlens[b];
    s.nblk = (s.len + pr->block_size - 1) / pr->block_size;
    s.row0 = rows;
    s.score0 = sc;
    s.nnz0 = nz;
    int64_t tot = 0;
    plan(s.nblk, pr->keep, pr->mu, &s.r_start, &tot);
    s.nnz = tot;
    rows += s.nblk;
    sc += static_cast<long long>(s.nblk) * (s.nblk + 1) / 2;
    nz += tot;
  }
  bt->total_rows = rows;
  bt->scores_per_head = sc;
  bt->nnz_per_head = nz;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Lists of one selection: a list per q-head, or per KV group with shared lists.
int list_heads(const stem_problem_t* pr) { return pr->shared_lists ? pr->num_kv_heads : pr->num_q_heads; }
int list_group(const stem_problem_t* pr) { return pr->num_q_heads / list_heads(pr); }

WsLayout layout(const stem_problem_t* pr, const Batch& bt) {
  WsLayout L;
  size_t o = 0;
  L.status = o;
  o += 256;
  const size_t R = static_cast<size_t>(bt.total_rows), d = static_cast<size_t>(pr->head_dim);
  L.qbar = o;
  o = align256(o + static_cast<size_t>(pr->num_q_heads) * R * d * 4);
  L.kbar = o;
  o = align256(o + static_cast<size_t>(pr->num_kv_heads) * R * d * 4);
  L.lbar = o;
  o = align256(o + static_cast<size_t>(pr->num_kv_heads) * R * 4);
  L.scores = o;
  o = align256(o + static_cast<size_t>(pr->num_q_heads) * static_cast<size_t>(bt.scores_per_head) * 4);
  L.row_ptr = o;
  o = align256(o + (R + 1) * 4);
  L.col_idx = o;
  o = align256(o + static_cast<size_t>(list_heads(pr)) * static_cast<size_t>(bt.nnz_per_head) * 4);
  L.total = o;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

float sigma_of(const stem_problem_t* pr) {
  return pr->softmax_scale > 0.f ? pr->softmax_scale : 1.0f / sqrtf(static_cast<float>(pr->head_dim));
}

stem_status_t check_ws(const stem_problem_t* pr, const Batch& bt, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = layout(pr, bt);
  if (ws == nullptr) return fail(STEM_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(STEM_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < L->total)
    return fail(STEM_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, L->total);
  return STEM_OK;
}

// Block means of Q and K and block mean log-norms of V into the workspace (one launch).
stem_status_t do_pool(const stem_problem_t* pr, const Batch& bt, const WsLayout& L, const void* q, const void* k,
                      const void* v, const stem_paged_kv_t* pg, void* ws, cudaStream_t st) {
  const bool fp8 = pr->dtype == STEM_DT_FP8_E4M3;
  PoolSet ps{};
  ps.count = 3;
  ps.t[0] = PoolTensor{q, pr->num_q_heads, 0, fp8 ? pr->q_scale : 1.0f, at<float>(ws, L.qbar), nullptr, 0};
  ps.t[1] = PoolTensor{pg ? pg->k_cache : k, pr->num_kv_heads, pg != nullptr, fp8 ? pr->k_scale : 1.0f,
                       at<float>(ws, L.kbar), nullptr, 0};
  ps.t[2] = PoolTensor{pg ? pg->v_cache : v, pr->num_kv_heads, pg != nullptr, fp8 ? pr->v_scale : 1.0f, nullptr,
                       at<float>(ws, L.lbar), 0};
  ps.block_table = pg ? pg->block_table : nullptr;
  ps.max_pages = pg ? pg->max_pages_per_seq : 0;
  ps.num_slots = pg ? pg->num_slots : 0;
  ps.status = at<uint32_t>(ws, L.status);
  cudaError_t e = launch_pool(bt, ps, pr->head_dim, fp8, st);
  if (e != cudaSuccess) return cuda_fail(e, "pool");
  return STEM_OK;
}

stem_status_t do_score(const stem_problem_t* pr, const Batch& bt, const WsLayout& L, const void* q, const void* k,
                       const void* v, const stem_paged_kv_t* pg, float* scores, void* ws, cudaStream_t st) {
  stem_status_t s = do_pool(pr, bt, L, q, k, v, pg, ws, st);
  if (s != STEM_OK) return s;
  cudaError_t e = launch_score(bt, at<float>(ws, L.qbar), at<float>(ws, L.kbar), at<float>(ws, L.lbar), pr->num_q_heads,
                   pr->num_kv_heads, pr->head_dim, sigma_of(pr), pr->beta, scores, st);
  if (e != cudaSuccess) return cuda_fail(e, "score");
  return STEM_OK;
}

stem_status_t do_bsa(const stem_problem_t* pr, const Batch& bt, const WsLayout& L, const void* q, const void* k,
                     const void* v, const stem_paged_kv_t* pg, const int32_t* row_ptr, const int32_t* col_idx,
                     void* out, float* lse, void* ws, bool dense, cudaStream_t st) {
  BsaArgs a{};
  a.q = q;
  a.k = pg ? pg->k_cache : k;
  a.v = pg ? pg->v_cache : v;
  a.block_table = pg ? pg->block_table : nullptr;
  a.max_pages = pg ? pg->max_pages_per_seq : 0;
  a.kv_rows = pg ? static_cast<long long>(pg->num_slots) * STEM_PAGE_SIZE : bt.total_tokens;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.list_group = list_group(pr);
  a.out = out;
  a.lse = lse;
  a.Hq = pr->num_q_heads;
  a.Hkv = pr->num_kv_heads;
  a.head_dim = pr->head_dim;
  a.sigma = sigma_of(pr);
  a.q_scale = pr->q_scale;
  a.k_scale = pr->k_scale;
  a.v_scale = pr->v_scale;
  cudaError_t e = launch_bsa(bt, a, pr->dtype == STEM_DT_FP8_E4M3, pg != nullptr, dense, at<uint32_t>(ws, L.status), st);
  if (e != cudaSuccess) return cuda_fail(e, dense ? "bsa_dense" : "bsa");
  return STEM_OK;
}

// pool -> scores -> budget + top-k, into row_ptr / col_idx.  fused: the scores are
// computed inside the selection kernel and never stored (stem_score_select); otherwise, and
// for shapes the fused kernel does not cover, the score matrix goes through the workspace
// (the front of stem_attention: on B200 the tiled score GEMM and the selection kernel
// together take less time than the fused kernel, which re-reads a row's block summaries
// for every row).  Both give the same lists bit for bit.
stem_status_t do_front(const stem_problem_t* pr, const Batch& bt, const WsLayout& L, const void* q, const void* k,
                       const void* v, const stem_paged_kv_t* pg, int32_t* row_ptr, int32_t* col_idx, void* ws,
                       cudaStream_t st, bool fused = false) {
  uint32_t* status = at<uint32_t>(ws, L.status);
  if (fused && fused_select_supported(pr->num_q_heads, pr->num_kv_heads, list_group(pr), pr->head_dim)) {
    stem_status_t s = do_pool(pr, bt, L, q, k, v, pg, ws, st);
    if (s != STEM_OK) return s;
    cudaError_t e = launch_select_fused(bt, at<float>(ws, L.qbar), at<float>(ws, L.kbar), at<float>(ws, L.lbar),
                                        pr->num_q_heads, pr->num_kv_heads, list_group(pr), pr->head_dim, sigma_of(pr),
                                        pr->beta, row_ptr, col_idx, status, st);
    if (e != cudaSuccess) return cuda_fail(e, "score_select");
    return STEM_OK;
  }
  stem_status_t s = do_score(pr, bt, L, q, k, v, pg, at<float>(ws, L.scores), ws, st);
  if (s != STEM_OK) return s;
  cudaError_t e = launch_select(bt, at<float>(ws, L.scores), pr->num_q_heads, list_group(pr), row_ptr, col_idx, status,
                                st);
  if (e != cudaSuccess) return cuda_fail(e, "select");
  return STEM_OK;
}

// the selection kept in the workspace, copied out on request
stem_status_t copy_selection(const stem_problem_t* pr, const Batch& bt, const WsLayout& L, void* ws,
                             int32_t* row_ptr_out, int32_t* col_idx_out, cudaStream_t st) {
  cudaError_t e;
  if (row_ptr_out != nullptr) {
    e = cudaMemcpyAsync(row_ptr_out, at<int32_t>(ws, L.row_ptr), (static_cast<size_t>(bt.total_rows) + 1) * 4,
                        cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "copy row_ptr");
  }
  if (col_idx_out != nullptr) {
    e = cudaMemcpyAsync(col_idx_out, at<int32_t>(ws, L.col_idx), static_cast<size_t>(list_heads(pr)) * bt.nnz_per_head * 4,
                        cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "copy col_idx");
  }
  return STEM_OK;
}

// Two non-blocking streams per device for the copies of stem_attention_host (host to
// device, device to host), created on first use and kept for the life of the process.
constexpr int kMaxCopyDevices = 64;
std::mutex g_copy_mu;
cudaStream_t g_copy_streams[kMaxCopyDevices][2] = {};

cudaError_t copy_streams_for_current_device(cudaStream_t* in, cudaStream_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxCopyDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_copy_mu);
  for (int i = 0; i < 2; ++i)
    if (g_copy_streams[dev][i] == nullptr) {
      e = cudaStreamCreateWithFlags(&g_copy_streams[dev][i], cudaStreamNonBlocking);
      if (e != cudaSuccess) return e;
    }
  *in = g_copy_streams[dev][0];
  *out = g_copy_streams[dev][1];
  return cudaSuccess;
}

// CUDA events of one stem_attention_host call, released when the call returns (an event
// whose recorded work is still pending is freed once that work completes).
struct CallEvents {
  std::vector<cudaEvent_t> ev;
  ~CallEvents() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
  cudaError_t record(cudaStream_t on, cudaStream_t waiter) {  // waiter waits for `on`'s work so far
    cudaEvent_t e = nullptr;
    cudaError_t r = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
    if (r != cudaSuccess) return r;
    ev.push_back(e);
    r = cudaEventRecord(e, on);
    return r == cudaSuccess ? cudaStreamWaitEvent(waiter, e, 0) : r;
  }
};

stem_status_t check_qkv(const void* q, const void* k, const void* v, const stem_paged_kv_t* pg) {
  if (q == nullptr || !aligned16(q)) return fail(STEM_ERR_INVALID, "q must be a non-NULL 16-byte aligned pointer");
  if (pg == nullptr) {
    if (k == nullptr || v == nullptr || !aligned16(k) || !aligned16(v))
      return fail(STEM_ERR_INVALID, "k and v must be non-NULL 16-byte aligned pointers");
  }
  return STEM_OK;
}

}  // namespace

std::atomic<int> g_inject{0};
int take_injection() { return g_inject.exchange(0); }
void set_injection(int mode) { g_inject.store(mode); }

stem_status_t set_last_error(stem_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace stem

using namespace stem;

extern "C" {

stem_status_t stem_query_sizes(const stem_problem_t* prob, stem_sizes_t* out) {
  stem_status_t s = check_problem(prob);
  if (s != STEM_OK) return s;
  if (out == nullptr) return fail(STEM_ERR_INVALID, "out is NULL");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L = layout(prob, bt);
  out->num_rows = bt.total_rows;
  out->scores_per_head = bt.scores_per_head;
  out->nnz_per_head = bt.nnz_per_head;
  out->total_tokens = bt.total_tokens;
  out->workspace_bytes = L.total;
  out->list_heads = list_heads(prob);
  return STEM_OK;
}

size_t stem_workspace_size(const stem_problem_t* prob) {
  stem_sizes_t s;
  return stem_query_sizes(prob, &s) == STEM_OK ? s.workspace_bytes : 0;
}

stem_status_t stem_tpd_plan(int n_blocks, double keep, double mu, double* r_start, int64_t* total) {
  if (n_blocks < 1) return fail(STEM_ERR_INVALID, "n_blocks %d < 1", n_blocks);
  if (!(keep > 0.0 && keep <= 1.0)) return fail(STEM_ERR_INVALID, "keep %g outside (0, 1]", keep);
  if (!(mu > 0.0 && mu <= 1.0)) return fail(STEM_ERR_INVALID, "mu %g outside (0, 1]", mu);
  if (r_start == nullptr || total == nullptr) return fail(STEM_ERR_INVALID, "output pointer is NULL");
  plan(n_blocks, keep, mu, r_start, total);
  return STEM_OK;
}

stem_status_t stem_score(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                         const stem_paged_kv_t* paged, float* scores, void* ws, size_t ws_bytes, void* stream) {
  stem_status_t s = check_problem(prob);
  if (s == STEM_OK) s = check_paged(prob, paged);
  if (s == STEM_OK) s = check_qkv(q, k, v, paged);
  if (s != STEM_OK) return s;
  if (scores == nullptr) return fail(STEM_ERR_INVALID, "scores is NULL");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;
  return do_score(prob, bt, L, q, k, v, paged, scores, ws, static_cast<cudaStream_t>(stream));
}

stem_status_t stem_select(const stem_problem_t* prob, const float* scores, int32_t* row_ptr, int32_t* col_idx,
                          void* ws, size_t ws_bytes, void* stream) {
  stem_status_t s = check_problem(prob);
  if (s != STEM_OK) return s;
  if (scores == nullptr || row_ptr == nullptr || col_idx == nullptr)
    return fail(STEM_ERR_INVALID, "scores, row_ptr and col_idx must not be NULL");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;
  cudaError_t e = launch_select(bt, scores, prob->num_q_heads, list_group(prob), row_ptr, col_idx,
                                at<uint32_t>(ws, L.status), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "select");
  return STEM_OK;
}

stem_status_t stem_score_select(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                                const stem_paged_kv_t* paged, int32_t* row_ptr, int32_t* col_idx, void* ws,
                                size_t ws_bytes, void* stream) {
  stem_status_t s = check_problem(prob);
  if (s == STEM_OK) s = check_paged(prob, paged);
  if (s == STEM_OK) s = check_qkv(q, k, v, paged);
  if (s != STEM_OK) return s;
  if (row_ptr == nullptr || col_idx == nullptr) return fail(STEM_ERR_INVALID, "row_ptr and col_idx must not be NULL");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;
  return do_front(prob, bt, L, q, k, v, paged, row_ptr, col_idx, ws, static_cast<cudaStream_t>(stream), true);
}

stem_status_t bsa_prefill(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                          const stem_paged_kv_t* paged, const int32_t* row_ptr, const int32_t* col_idx, void* out,
                          float* lse, void* ws, size_t ws_bytes, void* stream) {
  stem_status_t s = check_problem(prob);
  if (s == STEM_OK) s = check_paged(prob, paged);
  if (s == STEM_OK) s = check_qkv(q, k, v, paged);
  if (s != STEM_OK) return s;
  if (row_ptr == nullptr || col_idx == nullptr) return fail(STEM_ERR_INVALID, "row_ptr and col_idx must not be NULL");
  if (out == nullptr || !aligned16(out)) return fail(STEM_ERR_INVALID, "out must be a non-NULL 16-byte aligned pointer");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;
  return do_bsa(prob, bt, L, q, k, v, paged, row_ptr, col_idx, out, lse, ws, false, static_cast<cudaStream_t>(stream));
}

stem_status_t bsa_dense_prefill(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                                const stem_paged_kv_t* paged, void* out, float* lse, void* ws, size_t ws_bytes,
                                void* stream) {
  stem_status_t s = check_problem(prob);
  if (s == STEM_OK) s = check_paged(prob, paged);
  if (s == STEM_OK) s = check_qkv(q, k, v, paged);
  if (s != STEM_OK) return s;
  if (out == nullptr || !aligned16(out)) return fail(STEM_ERR_INVALID, "out must be a non-NULL 16-byte aligned pointer");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;
  return do_bsa(prob, bt, L, q, k, v, paged, nullptr, nullptr, out, lse, ws, true, static_cast<cudaStream_t>(stream));
}

stem_status_t stem_attention(const stem_problem_t* prob, const void* q, const void* k, const void* v,
                             const stem_paged_kv_t* paged, void* out, float* lse, int32_t* row_ptr_out,
                             int32_t* col_idx_out, void* ws, size_t ws_bytes, void* stream) {
  stem_status_t s = check_problem(prob);
  if (s == STEM_OK) s = check_paged(prob, paged);
  if (s == STEM_OK) s = check_qkv(q, k, v, paged);
  if (s != STEM_OK) return s;
  if (out == nullptr || !aligned16(out)) return fail(STEM_ERR_INVALID, "out must be a non-NULL 16-byte aligned pointer");
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = do_front(prob, bt, L, q, k, v, paged, at<int32_t>(ws, L.row_ptr), at<int32_t>(ws, L.col_idx), ws, st)) !=
      STEM_OK)
    return s;
  if ((s = do_bsa(prob, bt, L, q, k, v, paged, at<int32_t>(ws, L.row_ptr), at<int32_t>(ws, L.col_idx), out, lse, ws,
                  false, st)) != STEM_OK)
    return s;
  return copy_selection(prob, bt, L, ws, row_ptr_out, col_idx_out, st);
}

stem_status_t stem_attention_host(const stem_problem_t* prob, const void* q_host, const void* k_host,
                                  const void* v_host, void* q, void* k, void* v, const stem_paged_kv_t* paged,
                                  void* out_host, void* out, float* lse, int32_t* row_ptr_out, int32_t* col_idx_out,
                                  int out_groups, void* ws, size_t ws_bytes, void* stream) {
  stem_status_t s = check_problem(prob);
  if (s == STEM_OK) s = check_paged(prob, paged);
  if (s == STEM_OK) s = check_qkv(q, k, v, paged);
  if (s != STEM_OK) return s;
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || out_host == nullptr)
    return fail(STEM_ERR_INVALID, "q_host, k_host, v_host and out_host must not be NULL");
  if (out == nullptr || !aligned16(out)) return fail(STEM_ERR_INVALID, "out must be a non-NULL 16-byte aligned pointer");
  if (out_groups < 0) return fail(STEM_ERR_INVALID, "out_groups %d < 0", out_groups);
  Batch bt;
  build_batch(prob, &bt);
  WsLayout L;
  if ((s = check_ws(prob, bt, ws, ws_bytes, &L)) != STEM_OK) return s;

  // Groups of kv-heads: the largest divisor of Hkv not above the request (0: 8).  Every
  // group is a problem of its own (its q-heads, its kv-heads) whose inputs and output
  // are staged contiguously, group after group, in the device buffers.
  const int Hq = prob->num_q_heads, Hkv = prob->num_kv_heads;
  const int want = out_groups > 0 ? out_groups : 8;
  int G = 1;
  for (int c = 1; c <= Hkv; ++c)
    if (Hkv % c == 0 && c <= want) G = c;
  stem_problem_t sub = *prob;
  sub.num_q_heads = Hq / G;
  sub.num_kv_heads = Hkv / G;
  Batch sbt;
  build_batch(&sub, &sbt);
  WsLayout SL;
  if ((s = check_ws(&sub, sbt, ws, ws_bytes, &SL)) != STEM_OK) return s;
  const size_t es = prob->dtype == STEM_DT_FP8_E4M3 ? 1 : 2;
  const size_t d = static_cast<size_t>(prob->head_dim);
  const size_t T = static_cast<size_t>(bt.total_tokens);
  const size_t kv_rows = paged ? static_cast<size_t>(paged->num_slots) * STEM_PAGE_SIZE : T;
  const size_t q_row = static_cast<size_t>(Hq) * d * es, q_grow = static_cast<size_t>(sub.num_q_heads) * d * es;
  const size_t kv_row = static_cast<size_t>(Hkv) * d * es, kv_grow = static_cast<size_t>(sub.num_kv_heads) * d * es;
  const size_t o_row = static_cast<size_t>(Hq) * d * 2, o_grow = static_cast<size_t>(sub.num_q_heads) * d * 2;
  char* qd = static_cast<char*>(q);
  char* kd = static_cast<char*>(paged ? const_cast<void*>(paged->k_cache) : k);
  char* vd = static_cast<char*>(paged ? const_cast<void*>(paged->v_cache) : v);
  char* od = static_cast<char*>(out);
  const int sub_lists = list_heads(&sub);

  cudaStream_t st = static_cast<cudaStream_t>(stream), cin = nullptr, cout = nullptr;
  cudaError_t e = copy_streams_for_current_device(&cin, &cout);
  if (e != cudaSuccess) return cuda_fail(e, "copy streams");
  CallEvents ev;
  // the caller's earlier work on these buffers completes before they are overwritten
  if ((e = ev.record(st, cin)) != cudaSuccess) return cuda_fail(e, "order the input copies");
  // With two or more groups of one kv-head each (per-head lists, q-heads per group a
  // multiple of 4), the first and the last group run as two halves of their q-heads: the
  // copy in front of the first half and the copy behind the last half each move half as
  // much, and those are the two copies no other group's work can hide.
  const bool halves = G >= 2 && sub.num_kv_heads == 1 && !prob->shared_lists && sub.num_q_heads % 4 == 0;
  stem_problem_t half = sub;
  half.num_q_heads = sub.num_q_heads / 2;
  Batch hbt;
  WsLayout HL;
  if (halves) {
    build_batch(&half, &hbt);
    if ((s = check_ws(&half, hbt, ws, ws_bytes, &HL)) != STEM_OK) return s;
  }
  const int half_lists = list_heads(&half);
  for (int g = 0; g < G && s == STEM_OK; ++g) {
    const int parts = halves && (g == 0 || g == G - 1) ? 2 : 1;
    const stem_problem_t* pp = parts == 2 ? &half : &sub;
    const Batch& pbt = parts == 2 ? hbt : sbt;
    const WsLayout& PL = parts == 2 ? HL : SL;
    const size_t q_prow = q_grow / parts, o_prow = o_grow / parts;
    for (int part = 0; part < parts; ++part) {
      // this piece's inputs, host -> device (pitched: its heads out of every token row);
      // the group's K and V come with its first piece
      char* qg = qd + g * T * q_grow + part * T * q_prow;
      e = cudaMemcpy2DAsync(qg, q_prow, static_cast<const char*>(q_host) + g * q_grow + part * q_prow, q_row, q_prow, T,
                            cudaMemcpyHostToDevice, cin);
      if (e == cudaSuccess && part == 0)
        e = cudaMemcpy2DAsync(kd + g * kv_rows * kv_grow, kv_grow, static_cast<const char*>(k_host) + g * kv_grow,
                              kv_row, kv_grow, kv_rows, cudaMemcpyHostToDevice, cin);
      if (e == cudaSuccess && part == 0)
        e = cudaMemcpy2DAsync(vd + g * kv_rows * kv_grow, kv_grow, static_cast<const char*>(v_host) + g * kv_grow,
                              kv_row, kv_grow, kv_rows, cudaMemcpyHostToDevice, cin);
      if (e == cudaSuccess) e = ev.record(cin, st);
      if (e != cudaSuccess) {
        s = cuda_fail(e, "copy inputs to the device");
        break;
      }
      // the path on this piece
      const void* kg = paged ? nullptr : kd + g * kv_rows * kv_grow;
      const void* vg = paged ? nullptr : vd + g * kv_rows * kv_grow;
      stem_paged_kv_t pgg{};
      if (paged) {
        pgg = *paged;
        pgg.k_cache = kd + g * kv_rows * kv_grow;
        pgg.v_cache = vd + g * kv_rows * kv_grow;
      }
      const stem_paged_kv_t* pg = paged ? &pgg : nullptr;
      char* og = od + g * T * o_grow + part * T * o_prow;
      const size_t head0 = static_cast<size_t>(g) * sub.num_q_heads + static_cast<size_t>(part) * pp->num_q_heads;
      float* lg = lse ? lse + head0 * T : nullptr;
      s = do_front(pp, pbt, PL, qg, kg, vg, pg, at<int32_t>(ws, PL.row_ptr), at<int32_t>(ws, PL.col_idx), ws, st);
      if (s == STEM_OK)
        s = do_bsa(pp, pbt, PL, qg, kg, vg, pg, at<int32_t>(ws, PL.row_ptr), at<int32_t>(ws, PL.col_idx), og, lg, ws,
                   false, st);
      const size_t list0 = static_cast<size_t>(g) * sub_lists + static_cast<size_t>(part) * half_lists;
      if (s == STEM_OK)
        s = copy_selection(pp, pbt, PL, ws, g == 0 && part == 0 ? row_ptr_out : nullptr,
                           col_idx_out ? col_idx_out + list0 * pbt.nnz_per_head : nullptr, st);
      if (s != STEM_OK) break;
      // this piece's output, device -> host, while the next pieces compute
      e = ev.record(st, cout);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(static_cast<char*>(out_host) + g * o_grow + part * o_prow, o_row, og, o_prow, o_prow, T,
                              cudaMemcpyDeviceToHost, cout);
      if (e != cudaSuccess) {
        s = cuda_fail(e, "copy output to the host");
        break;
      }
    }
  }
  // the caller's stream covers every copy enqueued (also after an error)
  cudaError_t j = ev.record(cin, st);
  if (j == cudaSuccess) j = ev.record(cout, st);
  if (s != STEM_OK) return s;
  if (j != cudaSuccess) return cuda_fail(j, "join the copy streams");
  return STEM_OK;
}

stem_status_t stem_query_status(void* ws, void* stream) {
  if (ws == nullptr) return fail(STEM_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  e = cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  e = cudaMemset(ws, 0, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  if (word & kStatusTimeout) return fail(STEM_ERR_TIMEOUT, "a device pipeline wait timed out");
  if (word & kStatusBounds) return fail(STEM_ERR_BOUNDS, "a block index outside its sequence was seen");
  return STEM_OK;
}

stem_status_t stem_reset_status(void* ws, void* stream) {
  if (ws == nullptr) return fail(STEM_ERR_WORKSPACE, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reset status");
  return STEM_OK;
}

const char* stem_status_string(stem_status_t s) {
  switch (s) {
    case STEM_OK: return "ok";
    case STEM_ERR_INVALID: return "invalid argument";
    case STEM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case STEM_ERR_WORKSPACE: return "workspace missing or too small";
    case STEM_ERR_CUDA: return "CUDA error";
    case STEM_ERR_TIMEOUT: return "device pipeline wait timed out";
    case STEM_ERR_BOUNDS: return "block index out of range";
  }
  return "unknown status";
}

const char* stem_last_error(void) { return g_err; }

stem_status_t stem_debug_inject(int mode) {
  if (mode != 0 && mode != 1) return fail(STEM_ERR_INVALID, "unknown injection mode %d", mode);
  set_injection(mode);
  return STEM_OK;
}

}  // extern "C"
