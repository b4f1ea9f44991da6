// spattn_route_static: the routing step (block means of Q and K, proxy
// scores, Top-p selection, CSR) without any device allocation.
//
// Some callers cannot call cudaMalloc: code whose device memory is owned by
// another allocator that forbids side allocations, plug-ins handed only their
// input and output buffers, and loops that must not pay cudaMalloc's implicit
// device synchronisation.  For them this entry point keeps its scratch (the
// fp32 means, per-row budgets and padded kept lists) in one file-scope device
// array of fixed size, allocated when the library's device code is loaded and
// held by every GPU that loads the library until the process exits.
//
// Host code must not use the array's name as a device address (it is a host
// stand-in): the address is looked up once per device with
// cudaGetSymbolAddress, while that device is current, on the first call.
// All calls share the array and it keeps the last call's contents, so every
// call clears the words that must start at zero; calls that overlap on the GPU
// (other streams, other host threads) race on it and must be serialised by
// the caller.  The cached address belongs to the device's current context: a
// cudaDeviceReset invalidates it, so this entry point must not be used across
// one.  Device-side errors (a permutation entry outside [0, N), which the
// pooling skips without reading, or a bounded wait that gave up) are recorded
// only in the array's control block and are not reported to the caller.
#include <math.h>
#include <mutex>
#include <stdarg.h>
#include <stdio.h>

#include "spattn.h"
#include "common.cuh"
#include "internal.h"

namespace spattn {
cudaError_t launch_pool_qk(const Problem& p, const void* Q, const void* K, float* qbar,
                           float* kbar, int32_t* ctrl, cudaStream_t s);
void record_error(const char* msg);  // the message spattn_last_error() returns
}

namespace {

constexpr size_t kScratchBytes = (size_t)SPATTN_ROUTE_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t* g_scratch_dev[kMaxDevices] = {};

spattn_status_t fail(spattn_status_t st, const char* fmt, ...) {
  char msg[256];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof(msg), fmt, ap);
  va_end(ap);
  spattn::record_error(msg);
  return st;
}

inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Device address of the scratch array on the current device (looked up once).
spattn_status_t scratch_address(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SPATTN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SPATTN_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_dev[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_route_scratch);
    if (e != cudaSuccess)
      return fail(SPATTN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_scratch_dev[dev] = static_cast<uint8_t*>(ptr);
  }
  *out = g_scratch_dev[dev];
  return SPATTN_OK;
}

}  // namespace

extern "C" spattn_status_t spattn_route_static(int B, int H, int N, int d, int b, float tau,
                                               int kmin, int kmax, const int32_t* perm,
                                               const void* Q, const void* K, int32_t* row_ptr,
                                               int32_t* col_idx, void* stream) {
  if (B < 1 || H < 1 || N < 1) return fail(SPATTN_ERR_INVALID_ARG, "need B, H, N >= 1");
  if (d != 64 && d != 128) return fail(SPATTN_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (b != 64 && b != 128) return fail(SPATTN_ERR_UNSUPPORTED, "b must be 64 or 128");
  if (!isfinite(tau)) return fail(SPATTN_ERR_INVALID_ARG, "tau must be finite");
  if (kmin < 1 || kmax < kmin) return fail(SPATTN_ERR_INVALID_ARG, "need 1 <= kmin <= kmax");
  const long long nb = (N + (long long)b - 1) / b;
  if (nb > 2048) return fail(SPATTN_ERR_UNSUPPORTED, "nb = %lld blocks exceeds 2048", nb);
  if ((long long)B * H > 65535) return fail(SPATTN_ERR_UNSUPPORTED, "B*H exceeds 65535");
  const int kcap = kmax < nb ? kmax : (int)nb;

  // scratch layout: control block, Qbar, Kbar (fp32), counts, padded lists,
  // order; each region rounded up to 256 bytes.  The size is checked before
  // the pointers, so that a caller can ask whether a shape fits without
  // passing any buffer.
  const size_t rows = (size_t)B * H * nb;
  const size_t cen = rows * d * sizeof(float);
  size_t off = 0;
  const size_t o_ctrl = off; off += up256(spattn::CTRL_WORDS * 4);
  const size_t o_qbar = off; off += up256(cen);
  const size_t o_kbar = off; off += up256(cen);
  const size_t o_counts = off; off += up256(rows * 4);
  const size_t o_lists = off; off += up256(rows * kcap * 4);
  const size_t o_order = off; off += up256(rows * 4);
  if (off > kScratchBytes)
    return fail(SPATTN_ERR_UNSUPPORTED,
                "this problem needs %zu bytes of routing scratch; the static scratch holds %zu "
                "bytes (use spattn_route with a caller workspace)", off, kScratchBytes);

  if (!Q || !K || !row_ptr || !col_idx)
    return fail(SPATTN_ERR_INVALID_ARG, "Q, K, row_ptr and col_idx must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K)) & 15)
    return fail(SPATTN_ERR_INVALID_ARG, "Q and K must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(perm) | reinterpret_cast<uintptr_t>(row_ptr) |
       reinterpret_cast<uintptr_t>(col_idx)) & 3)
    return fail(SPATTN_ERR_INVALID_ARG, "perm, row_ptr and col_idx must be 4-byte aligned");

  spattn::Problem p;
  p.B = B; p.H = H; p.N = N; p.d = d; p.b = b;
  p.nb = (int)nb;
  p.n_last = N - (p.nb - 1) * b;
  p.kcap = kcap;
  p.BH = B * H;
  p.tau = tau; p.kmin = kmin; p.kmax = kmax;
  p.residual = 0;
  p.use_tc = 0;
  p.routing = spattn::ROUTING_CENTROID;
  p.threshold = 0;
  p.inline_sel = 0;
  p.test_stall = 0;
  p.perm = perm;

  uint8_t* base = nullptr;
  if (spattn_status_t st = scratch_address(&base)) return st;
  spattn::Work w = {};
  w.qbar = reinterpret_cast<float*>(base + o_qbar);
  w.kbar = reinterpret_cast<float*>(base + o_kbar);
  w.counts = reinterpret_cast<int32_t*>(base + o_counts);
  w.lists = reinterpret_cast<int32_t*>(base + o_lists);
  w.order = reinterpret_cast<int32_t*>(base + o_order);
  w.ctrl = reinterpret_cast<int32_t*>(base + o_ctrl);
  w.row_ptr = row_ptr;
  w.col_idx = col_idx;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the pooling kernel also clears the control block
  cudaError_t e = spattn::launch_pool_qk(p, Q, K, w.qbar, w.kbar, w.ctrl, s);
  if (e == cudaSuccess) e = spattn::launch_route(p, w, Q, nullptr, nullptr, true, s);
  if (e != cudaSuccess) return fail(SPATTN_ERR_CUDA, "routing kernels: %s", cudaGetErrorString(e));
  return SPATTN_OK;
}
