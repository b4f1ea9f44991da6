// C ABI of libspattn: plans, workspace layout, argument checks, dispatch.
#include <math.h>
#include <stdlib.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <new>
#include <numeric>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "spattn.h"
#include "common.cuh"
#include "internal.h"

namespace spattn {
cudaError_t launch_attend_mma(const Problem& p, const void* Q, const void* K, const void* V,
                              const int32_t* row_ptr, const int32_t* col_idx, void* O,
                              const Work& w, cudaStream_t s);
cudaError_t launch_attend_tc(const Problem& p, const void* Q, const void* K, const void* V,
                             const int32_t* row_ptr, const int32_t* col_idx, void* O,
                             const Work& w, cudaStream_t s);
bool attend_tc_supported(const Problem& p);
}  // namespace spattn

using spattn::Problem;
using spattn::Work;

namespace {

thread_local char g_err[512] = "";

spattn_status_t fail(spattn_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

spattn_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(SPATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// NVTX range over one library call (host side), so that profilers can group
// the kernels a call enqueues; free when no tool is attached.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

constexpr size_t ALIGN = 256;
inline size_t up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

// Byte offsets of the workspace regions.
struct Layout {
  size_t qp, kp, vp, qbar, kbar, vbar, kbar16, vbar16, counts, lists, row_ptr, col_idx, order,
      ctrl, total;
};

// With a permutation the pooling writes permuted copies of Q, K and V, which
// the attention then reads as whole tiles.  (Gathering the attention's rows
// through the permutation instead, with TMA row gathers, was measured slower
// on B200: at 0.4 % kept blocks the step took 1.65 ms against 1.35 ms, and a
// dense pass over the permuted layer 4.4 times as long.)
bool keeps_copies(const Problem& p) { return p.perm != nullptr; }

Layout make_layout(const Problem& p) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += up(bytes); return o; };
  const size_t tok = (size_t)p.BH * p.N * p.d;
  const size_t cen = (size_t)p.BH * p.nb * p.d;
  const size_t rows = (size_t)p.BH * p.nb;
  const bool perm = keeps_copies(p);
  L.qp = perm ? take(tok * 2) : 0;
  L.kp = perm ? take(tok * 2) : 0;
  L.vp = perm ? take(tok * 2) : 0;
  L.qbar = take(cen * 4);
  L.kbar = take(cen * 4);
  L.vbar = take(cen * 4);
  L.kbar16 = take(cen * 2);
  L.vbar16 = take(cen * 2);
  L.counts = take(rows * 4);
  L.lists = take(rows * p.kcap * 4);
  L.row_ptr = take((rows + 1) * 4);
  L.col_idx = take(rows * p.kcap * 4);
  L.order = take(rows * 4);
  L.ctrl = take(spattn::CTRL_WORDS * 4);
  L.total = off;
  return L;
}

Work bind(const Problem& p, const Layout& L, void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  Work w;
  const bool perm = keeps_copies(p);
  w.qp = perm ? reinterpret_cast<__nv_bfloat16*>(b + L.qp) : nullptr;
  w.kp = perm ? reinterpret_cast<__nv_bfloat16*>(b + L.kp) : nullptr;
  w.vp = perm ? reinterpret_cast<__nv_bfloat16*>(b + L.vp) : nullptr;
  w.qbar = reinterpret_cast<float*>(b + L.qbar);
  w.kbar = reinterpret_cast<float*>(b + L.kbar);
  w.vbar = reinterpret_cast<float*>(b + L.vbar);
  w.kbar16 = reinterpret_cast<__nv_bfloat16*>(b + L.kbar16);
  w.vbar16 = reinterpret_cast<__nv_bfloat16*>(b + L.vbar16);
  w.counts = reinterpret_cast<int32_t*>(b + L.counts);
  w.lists = reinterpret_cast<int32_t*>(b + L.lists);
  w.row_ptr = reinterpret_cast<int32_t*>(b + L.row_ptr);
  w.col_idx = reinterpret_cast<int32_t*>(b + L.col_idx);
  w.order = reinterpret_cast<int32_t*>(b + L.order);
  w.ctrl = reinterpret_cast<int32_t*>(b + L.ctrl);
  return w;
}

// Staging bytes of one tensor of a chunk of c (batch, head) pairs.
size_t chunk_tensor_bytes(const Problem& p, int c) { return up((size_t)c * p.N * p.d * 2); }

// The problem restricted to `c` consecutive (batch, head) pairs: heads are
// independent through the whole path, so a chunk is a problem with B = 1,
// H = c and the same token partition, knobs and permutation.
Problem sub_problem(const Problem& p, int c) {
  Problem q = p;
  q.B = 1; q.H = c; q.BH = c;
  return q;
}

// Heads per chunk of spattn_forward_host.  A chunk's workspace starts at the
// base and must end before the plan's control block, which collects the
// chunks' errors; when rounding makes a smaller chunk reach it (tiny
// problems), the whole problem is one chunk and uses the plan's own layout.
int effective_chunk(const Problem& p, const Layout& L, int chunk_heads) {
  const int c = std::min(chunk_heads, p.BH);
  if (c < p.BH && make_layout(sub_problem(p, c)).total > L.ctrl) return p.BH;
  return c;
}

// Keep the first device error: copy a chunk's error word into the plan's
// word unless that already holds one.
__global__ void merge_error_kernel(int32_t* dst, const int32_t* src) {
  if (src[spattn::CTRL_ERROR] != 0 && dst[spattn::CTRL_ERROR] == 0) {
    dst[spattn::CTRL_ERROR] = src[spattn::CTRL_ERROR];
    dst[spattn::CTRL_ERROR_AUX] = src[spattn::CTRL_ERROR_AUX];
  }
}

}  // namespace

namespace spattn {
void record_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

cudaError_t ensure_dyn_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;  // below the default limit
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> granted;
  std::lock_guard<std::mutex> lock(mu);
  size_t& g = granted[{fn, dev}];
  if (g >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) g = bytes;
  return e;
}
}  // namespace spattn

struct spattn_plan_s {
  Problem p;
  Layout L;
  int32_t* perm_dev = nullptr;
};

namespace {

spattn_status_t check_plan(spattn_plan_t plan) {
  if (!plan) return fail(SPATTN_ERR_INVALID_ARG, "plan is NULL");
  return SPATTN_OK;
}

spattn_status_t check_inputs(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                             const void* ws) {
  if (spattn_status_t st = check_plan(plan)) return st;
  if (!Q || !K || !V) return fail(SPATTN_ERR_INVALID_ARG, "Q, K and V must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
       reinterpret_cast<uintptr_t>(V)) & 15)
    return fail(SPATTN_ERR_INVALID_ARG, "Q, K and V must be 16-byte aligned");
  if (!ws) return fail(SPATTN_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & (ALIGN - 1))
    return fail(SPATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return SPATTN_OK;
}

}  // namespace

extern "C" {

const char* spattn_last_error(void) { return g_err; }

spattn_status_t spattn_plan(spattn_plan_t* out, int B, int H, int N, int d, int b, float tau,
                            int kmin, int kmax, int residual, const int32_t* perm_host,
                            size_t* workspace_bytes) {
  return spattn_plan_ex(out, B, H, N, d, b, tau, kmin, kmax, residual, perm_host,
                        SPATTN_ROUTING_CENTROID, workspace_bytes);
}

spattn_status_t spattn_plan_ex(spattn_plan_t* out, int B, int H, int N, int d, int b, float tau,
                               int kmin, int kmax, int residual, const int32_t* perm_host,
                               int routing, size_t* workspace_bytes) {
  g_err[0] = 0;
  if (!out) return fail(SPATTN_ERR_INVALID_ARG, "out is NULL");
  const int estimate = routing & ~(SPATTN_SELECT_THRESHOLD | SPATTN_SELECT_INLINE);
  if (estimate != SPATTN_ROUTING_CENTROID && estimate != SPATTN_ROUTING_PAMA)
    return fail(SPATTN_ERR_INVALID_ARG, "routing must be SPATTN_ROUTING_CENTROID or SPATTN_ROUTING_PAMA, optionally | SPATTN_SELECT_THRESHOLD | SPATTN_SELECT_INLINE (got %d)", routing);
  if ((routing & SPATTN_SELECT_INLINE) && estimate != SPATTN_ROUTING_CENTROID)
    return fail(SPATTN_ERR_INVALID_ARG, "routing: SPATTN_SELECT_INLINE needs the centroid estimate");
  *out = nullptr;
  if (B < 1 || H < 1 || N < 1) return fail(SPATTN_ERR_INVALID_ARG, "need B, H, N >= 1 (got %d, %d, %d)", B, H, N);
  if (d != 64 && d != 128) return fail(SPATTN_ERR_UNSUPPORTED, "d must be 64 or 128 (got %d)", d);
  if (b != 64 && b != 128) return fail(SPATTN_ERR_UNSUPPORTED, "b must be 64 or 128 (got %d)", b);
  if (!isfinite(tau)) return fail(SPATTN_ERR_INVALID_ARG, "tau must be finite");
  if (kmin < 1 || kmax < kmin) return fail(SPATTN_ERR_INVALID_ARG, "need 1 <= kmin <= kmax (got %d, %d)", kmin, kmax);
  if (residual != 0 && residual != 1) return fail(SPATTN_ERR_INVALID_ARG, "residual must be 0 or 1");
  const long long nb = (N + (long long)b - 1) / b;
  if (nb > 2048) return fail(SPATTN_ERR_UNSUPPORTED, "nb = %lld blocks exceeds 2048", nb);
  if ((long long)B * H * nb > (1LL << 30) || (long long)B * H * (long long)N * d > (1LL << 40))
    return fail(SPATTN_ERR_UNSUPPORTED, "problem too large");
  // the routing kernels index (batch, head) pairs by the grid's y dimension
  if ((long long)B * H > 65535)
    return fail(SPATTN_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535", (long long)B * H);
  // kept-list offsets (CSR row_ptr, per-row list bases) are int32
  if ((long long)B * H * nb * std::min<long long>(kmax, nb) > 0x7FFFFFFFLL)
    return fail(SPATTN_ERR_UNSUPPORTED, "kept-list capacity B*H*nb*min(kmax, nb) = %lld exceeds 2^31 - 1",
                (long long)B * H * nb * std::min<long long>(kmax, nb));
  if (perm_host) {
    std::vector<uint8_t> seen(N, 0);
    for (int n = 0; n < N; ++n) {
      const int32_t v = perm_host[n];
      if (v < 0 || v >= N || seen[v]) return fail(SPATTN_ERR_INVALID_ARG, "perm is not a bijection of [0, N) (entry %d)", n);
      seen[v] = 1;
    }
  }
  spattn_plan_s* P = new (std::nothrow) spattn_plan_s;
  if (!P) return fail(SPATTN_ERR_INVALID_ARG, "out of host memory");
  Problem& p = P->p;
  p.B = B; p.H = H; p.N = N; p.d = d; p.b = b;
  p.nb = (int)nb;
  p.n_last = N - (p.nb - 1) * b;
  p.kcap = std::min(kmax, p.nb);
  p.BH = B * H;
  p.tau = tau; p.kmin = kmin; p.kmax = kmax; p.residual = residual;
  p.perm = nullptr;
  p.routing = estimate == SPATTN_ROUTING_PAMA ? spattn::ROUTING_PAMA : spattn::ROUTING_CENTROID;
  p.threshold = (routing & SPATTN_SELECT_THRESHOLD) ? 1 : 0;
  p.inline_sel = (routing & SPATTN_SELECT_INLINE) ? 1 : 0;
  {
    // tcgen05/TMEM kernel for every supported shape; with SPATTN_ATTN=mma in
    // the environment when the plan is made, the warp-MMA kernel instead
    // (kept only to cross-check the two GPU paths in the tests).
    const char* env = getenv("SPATTN_ATTN");
    p.use_tc = spattn::attend_tc_supported(p) && !(env && strcmp(env, "mma") == 0);
    // the inline selection lives in the tcgen05 kernel
    if (p.inline_sel && !p.use_tc) { delete P; return fail(SPATTN_ERR_UNSUPPORTED, "SPATTN_SELECT_INLINE needs the tcgen05 attention kernel"); }
    // Failure-path test: with SPATTN_TEST_WAIT_TIMEOUT=1 in the environment
    // when the plan is made, the tcgen05 attention's first CTA waits on an
    // mbarrier phase that nothing completes; the bounded wait gives up after
    // its limit (~2 s), the CTA winds down, and spattn_check reports
    // SPATTN_ERR_TIMEOUT.  Nothing faults or hangs.
    const char* st = getenv("SPATTN_TEST_WAIT_TIMEOUT");
    p.test_stall = (st && strcmp(st, "1") == 0) ? 1 : 0;
  }
  if (perm_host) {
    // Failure-path test: with SPATTN_TEST_FAIL_ALLOC=1 in the environment the
    // permutation's device allocation reports out-of-memory without being
    // attempted, so the error path runs without exhausting any memory.
    const char* fa = getenv("SPATTN_TEST_FAIL_ALLOC");
    cudaError_t e = (fa && strcmp(fa, "1") == 0)
                        ? cudaErrorMemoryAllocation
                        : cudaMalloc(&P->perm_dev, sizeof(int32_t) * (size_t)N);
    if (e != cudaSuccess) { delete P; return cuda_fail(e, "cudaMalloc(perm)"); }
    e = cudaMemcpy(P->perm_dev, perm_host, sizeof(int32_t) * (size_t)N, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(P->perm_dev); delete P; return cuda_fail(e, "cudaMemcpy(perm)"); }
    p.perm = P->perm_dev;
  }
  P->L = make_layout(p);
  if (workspace_bytes) *workspace_bytes = P->L.total;
  *out = P;
  return SPATTN_OK;
}

spattn_status_t spattn_plan_destroy(spattn_plan_t plan) {
  if (!plan) return SPATTN_OK;
  cudaError_t e = cudaSuccess;
  if (plan->perm_dev) e = cudaFree(plan->perm_dev);
  delete plan;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree(perm)");
  return SPATTN_OK;
}

spattn_status_t spattn_plan_info(spattn_plan_t plan, int* nb, int64_t* col_capacity) {
  if (spattn_status_t st = check_plan(plan)) return st;
  if (nb) *nb = plan->p.nb;
  if (col_capacity) *col_capacity = (int64_t)plan->p.BH * plan->p.nb * plan->p.kcap;
  return SPATTN_OK;
}

spattn_status_t spattn_pool(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                            void* workspace, void* stream) {
  Range range("spattn_pool");
  if (spattn_status_t st = check_inputs(plan, Q, K, V, workspace)) return st;
  const Work w = bind(plan->p, plan->L, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the pooling kernel also clears the control block
  cudaError_t e = spattn::launch_pool(plan->p, Q, K, V, w, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool kernel");
  return SPATTN_OK;
}

spattn_status_t spattn_route(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                             void* workspace, int32_t* row_ptr, int32_t* col_idx, void* stream) {
  Range range("spattn_route");
  if (spattn_status_t st = check_inputs(plan, Q, K, V, workspace)) return st;
  const Work w = bind(plan->p, plan->L, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the pooling kernel also clears the control block
  cudaError_t e = spattn::launch_pool(plan->p, Q, K, V, w, s);
  if (e != cudaSuccess) return cuda_fail(e, "pool kernel");
  // the warp-MMA attention reads the compact CSR of the workspace
  e = spattn::launch_route(plan->p, w, Q, row_ptr, col_idx, !plan->p.use_tc, s);
  if (e != cudaSuccess) return cuda_fail(e, "route kernels");
  return SPATTN_OK;
}

spattn_status_t spattn_attend(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                              const int32_t* row_ptr, const int32_t* col_idx, void* O,
                              void* workspace, void* stream) {
  Range range("spattn_attend");
  if (spattn_status_t st = check_inputs(plan, Q, K, V, workspace)) return st;
  if (!O) return fail(SPATTN_ERR_INVALID_ARG, "O must be non-NULL");
  if (reinterpret_cast<uintptr_t>(O) & 15) return fail(SPATTN_ERR_INVALID_ARG, "O must be 16-byte aligned");
  if ((row_ptr == nullptr) != (col_idx == nullptr))
    return fail(SPATTN_ERR_INVALID_ARG, "row_ptr and col_idx must both be NULL or both be set");
  const Work w = bind(plan->p, plan->L, workspace);
  if (!row_ptr) { row_ptr = w.row_ptr; col_idx = w.col_idx; }
  cudaError_t e = spattn::launch_attend(plan->p, Q, K, V, row_ptr, col_idx, O, w,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
  return SPATTN_OK;
}

spattn_status_t spattn_forward(spattn_plan_t plan, const void* Q, const void* K, const void* V,
                               void* O, void* workspace, void* stream) {
  Range range("spattn_forward");
  // with inline selection the attention kernel selects from the means: no
  // routing launch
  if (plan && plan->p.inline_sel) {
    if (spattn_status_t st = spattn_pool(plan, Q, K, V, workspace, stream)) return st;
  } else if (spattn_status_t st = spattn_route(plan, Q, K, V, workspace, nullptr, nullptr, stream)) {
    return st;
  }
  return spattn_attend(plan, Q, K, V, nullptr, nullptr, O, workspace, stream);
}

spattn_status_t spattn_host_staging_bytes(spattn_plan_t plan, int chunk_heads, size_t* bytes) {
  if (spattn_status_t st = check_plan(plan)) return st;
  if (chunk_heads < 1) return fail(SPATTN_ERR_INVALID_ARG, "chunk_heads must be >= 1");
  if (!bytes) return fail(SPATTN_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = 8 * chunk_tensor_bytes(plan->p, effective_chunk(plan->p, plan->L, chunk_heads));
  return SPATTN_OK;
}

spattn_status_t spattn_forward_host(spattn_plan_t plan, const void* Q_host, const void* K_host,
                                    const void* V_host, void* O_host, void* workspace,
                                    void* staging, int chunk_heads, void* stream) {
  Range range("spattn_forward_host");
  if (spattn_status_t st = check_plan(plan)) return st;
  if (!Q_host || !K_host || !V_host || !O_host)
    return fail(SPATTN_ERR_INVALID_ARG, "Q_host, K_host, V_host and O_host must be non-NULL");
  if (chunk_heads < 1) return fail(SPATTN_ERR_INVALID_ARG, "chunk_heads must be >= 1");
  if (!workspace) return fail(SPATTN_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) & (ALIGN - 1))
    return fail(SPATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (!staging) return fail(SPATTN_ERR_WORKSPACE, "staging is NULL");
  if (reinterpret_cast<uintptr_t>(staging) & (ALIGN - 1))
    return fail(SPATTN_ERR_WORKSPACE, "staging must be 256-byte aligned");
  const Problem& p = plan->p;
  const int c = effective_chunk(p, plan->L, chunk_heads);
  const int G = (p.BH + c - 1) / c;
  const size_t tb = chunk_tensor_bytes(p, c);
  const size_t head_bytes = (size_t)p.N * p.d * 2;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* ctrl = reinterpret_cast<int32_t*>(ws + plan->L.ctrl);
  auto slot_buf = [&](int slot, int t) { return static_cast<uint8_t*>(staging) + (size_t)(slot * 4 + t) * tb; };
  const uint8_t* src[3] = {static_cast<const uint8_t*>(Q_host), static_cast<const uint8_t*>(K_host),
                           static_cast<const uint8_t*>(V_host)};
  uint8_t* dst = static_cast<uint8_t*>(O_host);

  cudaStream_t s0 = static_cast<cudaStream_t>(stream), s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_end = nullptr, ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};
  cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
  cudaEvent_t* evs[8] = {&ev_start, &ev_end, &ev_in[0], &ev_in[1], &ev_done[0], &ev_done[1],
                         &ev_out[0], &ev_out[1]};
  for (int i = 0; i < 8 && e == cudaSuccess; ++i)
    e = cudaEventCreateWithFlags(evs[i], cudaEventDisableTiming);
  const char* what = "creating streams and events";
  // the plan's error word starts clear; the copy streams start after the
  // caller's earlier work on `stream` (which may still use the staging)
  if (e == cudaSuccess) { what = "clearing the error word"; e = cudaMemsetAsync(ctrl, 0, 2 * sizeof(int32_t), s0); }
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, s0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_start, 0);
  for (int g = 0; g < G && e == cudaSuccess; ++g) {
    const int slot = g & 1, h0 = g * c, cg = std::min(c, p.BH - h0);
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)cg * head_bytes;
    // inputs of chunk g, once chunk g - 2 is done with this slot
    what = "copying a chunk in";
    if (g >= 2) e = cudaStreamWaitEvent(s_in, ev_done[slot], 0);
    for (int t = 0; t < 3 && e == cudaSuccess; ++t)
      e = cudaMemcpyAsync(slot_buf(slot, t), src[t] + off, bytes, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[slot], s_in);
    // the path on chunk g, once its inputs are in and chunk g - 2's output is out
    what = "ordering a chunk";
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, ev_in[slot], 0);
    if (e == cudaSuccess && g >= 2) e = cudaStreamWaitEvent(s0, ev_out[slot], 0);
    if (e != cudaSuccess) break;
    const Problem ps = sub_problem(p, cg);
    const Layout Ls = make_layout(ps);
    const Work w = bind(ps, Ls, workspace);
    const void *q = slot_buf(slot, 0), *k = slot_buf(slot, 1), *v = slot_buf(slot, 2);
    void* o = slot_buf(slot, 3);
    what = "pool kernel";
    e = spattn::launch_pool(ps, q, k, v, w, s0);
    if (e == cudaSuccess && !ps.inline_sel) { what = "route kernels"; e = spattn::launch_route(ps, w, q, nullptr, nullptr, !ps.use_tc, s0); }
    if (e == cudaSuccess) { what = "attention kernel"; e = spattn::launch_attend(ps, q, k, v, w.row_ptr, w.col_idx, o, w, s0); }
    if (e == cudaSuccess && w.ctrl != ctrl) {
      what = "error merge";
      merge_error_kernel<<<1, 1, 0, s0>>>(ctrl, w.ctrl);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_done[slot], s0);
    // output of chunk g
    what = "copying a chunk out";
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_done[slot], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dst + off, o, bytes, cudaMemcpyDeviceToHost, s_out);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out[slot], s_out);
  }
  // the caller's stream sees the last output copy
  if (e == cudaSuccess) { what = "joining the streams"; e = cudaEventRecord(ev_end, s_out); }
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s0, ev_end, 0);
  // resources are released once the enqueued work completes
  for (int i = 0; i < 8; ++i)
    if (*evs[i]) cudaEventDestroy(*evs[i]);
  if (s_in) cudaStreamDestroy(s_in);
  if (s_out) cudaStreamDestroy(s_out);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return SPATTN_OK;
}

spattn_status_t spattn_probe_scratch_bytes(spattn_plan_t plan, int M, size_t* bytes) {
  if (spattn_status_t st = check_plan(plan)) return st;
  if (M < 1) return fail(SPATTN_ERR_INVALID_ARG, "need M >= 1 probe rows (got %d)", M);
  if (!bytes) return fail(SPATTN_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = spattn::probe_scratch_bytes(plan->p, M);
  return SPATTN_OK;
}

spattn_status_t spattn_probe_correct(spattn_plan_t plan, const void* Q, const void* K,
                                     const void* V, void* O, const int32_t* probes, int M,
                                     float lam, int r, void* workspace, void* scratch,
                                     void* stream) {
  Range range("spattn_probe_correct");
  if (spattn_status_t st = check_inputs(plan, Q, K, V, workspace)) return st;
  const Problem& p = plan->p;
  if (!O || (reinterpret_cast<uintptr_t>(O) & 15))
    return fail(SPATTN_ERR_INVALID_ARG, "O must be non-NULL and 16-byte aligned");
  if (!probes) return fail(SPATTN_ERR_INVALID_ARG, "probes is NULL");
  if (M < 1 || (long long)M * p.BH > (1LL << 30))
    return fail(SPATTN_ERR_INVALID_ARG, "need 1 <= M and B*H*M <= 2^30 (got M = %d)", M);
  if (!isfinite(lam) || lam < 0.f) return fail(SPATTN_ERR_INVALID_ARG, "lam must be finite and >= 0");
  if (r < 0 || r > p.d) return fail(SPATTN_ERR_INVALID_ARG, "need 0 <= r <= d (got %d)", r);
  if (p.BH > 65535) return fail(SPATTN_ERR_UNSUPPORTED, "the probe correction takes B*H <= 65535");
  if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & (ALIGN - 1)))
    return fail(SPATTN_ERR_WORKSPACE, "scratch must be non-NULL and 256-byte aligned");
  const Work w = bind(p, plan->L, workspace);
  cudaError_t e = spattn::launch_probe_correct(p, Q, K, V, O, probes, M, lam, r, scratch, w.ctrl,
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "probe correction kernels");
  return SPATTN_OK;
}

spattn_status_t spattn_means(spattn_plan_t plan, const void* workspace, float* Qbar, float* Kbar,
                             float* Vbar, void* stream) {
  if (spattn_status_t st = check_plan(plan)) return st;
  if (!workspace) return fail(SPATTN_ERR_WORKSPACE, "workspace is NULL");
  const Work w = bind(plan->p, plan->L, const_cast<void*>(workspace));
  const size_t bytes = (size_t)plan->p.BH * plan->p.nb * plan->p.d * sizeof(float);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float* src[3] = {w.qbar, w.kbar, w.vbar};
  float* dst[3] = {Qbar, Kbar, Vbar};
  for (int t = 0; t < 3; ++t) {
    if (!dst[t]) continue;
    cudaError_t e = cudaMemcpyAsync(dst[t], src[t], bytes, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(means)");
  }
  return SPATTN_OK;
}

spattn_status_t spattn_check(spattn_plan_t plan, void* workspace, void* stream) {
  if (spattn_status_t st = check_plan(plan)) return st;
  if (!workspace) return fail(SPATTN_ERR_WORKSPACE, "workspace is NULL");
  const Work w = bind(plan->p, plan->L, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(h, w.ctrl, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  e = cudaMemsetAsync(w.ctrl, 0, sizeof(int32_t) * 2, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  if (h[0] == spattn::DEV_BAD_INDEX)
    return fail(SPATTN_ERR_DEVICE, "an index outside its range was skipped: a CSR block index "
                "(work item %d) or a probe token (entry %d of probes)", h[1], h[1]);
  if (h[0] == spattn::DEV_TIMEOUT)
    return fail(SPATTN_ERR_TIMEOUT, "a device-side wait gave up (site %d)", h[1]);
  if (h[0] == spattn::DEV_NUMERIC)
    return fail(SPATTN_ERR_DEVICE, "the probe fit's normal equations were not positive definite "
                "(head %d left uncorrected)", h[1]);
  if (h[0] != 0) return fail(SPATTN_ERR_DEVICE, "device error code %d (aux %d)", h[0], h[1]);
  return SPATTN_OK;
}

// ---- 3D Hilbert order (host, no CUDA) ----
// Skilling's transform, one cell at a time: walk the bit levels from the top,
// at each level either invert the lower bits of axis 0 or swap them with axis
// i, then Gray-encode across the axes; the index reads the three transformed
// words level by level, axis 0 most significant.
static uint64_t hilbert_key3(uint32_t x[3], int bits) {
  const uint32_t top = 1u << (bits - 1);
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
    for (int i = 0; i < 3; ++i) {
      if (x[i] & q) {
        x[0] ^= low;
      } else {
        const uint32_t t = (x[0] ^ x[i]) & low;
        x[0] ^= t;
        x[i] ^= t;
      }
    }
  }
  x[1] ^= x[0];
  x[2] ^= x[1];
  uint32_t flip = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (x[2] & q) flip ^= q - 1;
  for (int i = 0; i < 3; ++i) x[i] ^= flip;
  uint64_t key = 0;
  for (int level = bits - 1; level >= 0; --level)
    for (int i = 0; i < 3; ++i) key = (key << 1) | ((x[i] >> level) & 1u);
  return key;
}

spattn_status_t spattn_hilbert_perm(int T, int Hs, int W, int32_t* perm_host) {
  if (T < 1 || Hs < 1 || W < 1) return fail(SPATTN_ERR_INVALID_ARG, "grid sides must be >= 1");
  if (!perm_host) return fail(SPATTN_ERR_INVALID_ARG, "perm_host is NULL");
  const long long N = (long long)T * Hs * W;
  if (N > (1LL << 31) - 1) return fail(SPATTN_ERR_UNSUPPORTED, "grid too large");
  const int side = std::max(T, std::max(Hs, W));
  // three axes of `bits` bits each must fit the 64-bit curve index
  if (side > (1 << 21)) return fail(SPATTN_ERR_UNSUPPORTED, "grid side %d exceeds 2^21", side);
  int bits = 1;
  while ((1 << bits) < side) ++bits;
  std::vector<uint64_t> key((size_t)N);
  for (int t = 0; t < T; ++t)
    for (int h = 0; h < Hs; ++h)
      for (int w = 0; w < W; ++w) {
        uint32_t x[3] = {(uint32_t)t, (uint32_t)h, (uint32_t)w};
        key[((size_t)t * Hs + h) * W + w] = hilbert_key3(x, bits);
      }
  std::vector<int32_t> idx((size_t)N);
  std::iota(idx.begin(), idx.end(), 0);
  std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) { return key[a] < key[b]; });
  memcpy(perm_host, idx.data(), sizeof(int32_t) * (size_t)N);
  return SPATTN_OK;
}

}  // extern "C"

namespace spattn {
cudaError_t launch_attend(const Problem& p, const void* Q, const void* K, const void* V,
                          const int32_t* row_ptr, const int32_t* col_idx, void* O,
                          const Work& w, cudaStream_t s) {
  if (p.use_tc) return launch_attend_tc(p, Q, K, V, row_ptr, col_idx, O, w, s);
  return launch_attend_mma(p, Q, K, V, row_ptr, col_idx, O, w, s);
}
}  // namespace spattn
