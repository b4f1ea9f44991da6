// Token gather (optional permutation) fused with block-mean pooling.
//
// Blocks are represented by the mean of their tokens (PARK page, abstract and
// section 4: query and key blocks are compared through their averages).  With a
// permutation, the kernel reads X[perm[n]] and writes the permuted copy Xp[n]
// in the same pass (DFSAttn abstract: Hilbert reordering before blocking), so
// Q/K/V are read from HBM exactly once.
//
// Persistent CTAs (two per SM), each taking a strided share of the units
// (tensor, head, block).  Without a permutation a unit's rows are contiguous
// and stream through a ring of shared-memory tiles filled by one TMA bulk
// copy each (pool_kernel).  With a permutation the rows are gathered with
// 16-byte loads into registers, one unit ahead (pool_gather_kernel), and the
// permuted copy is written from the same registers.  A thread owns one
// 16-byte chunk (8 channels) and sums the rows r0, r0+R, ... of the tile in
// fp32 in a fixed order; the R partial sums are then added in a fixed order,
// so the means are bit-reproducible.
//
// CTA 0 also clears the workspace control block: this is the first kernel of
// the routing chain.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace spattn {
namespace {

constexpr int POOL_THREADS = 256;
constexpr int POOL_STAGES = 3;
constexpr int POOL_CTAS_PER_SM = 2;

struct PoolArgs {
  const __nv_bfloat16* X[3];
  __nv_bfloat16* Xp[3];    // permuted copies, NULL when there is no perm
  float* bar[3];           // fp32 means [BH, nb, d]
  __nv_bfloat16* bar16[3]; // bf16 means (K and V only; NULL for Q)
  const int32_t* perm;
  int32_t* ctrl;           // control block cleared by CTA 0 (NULL: leave it)
  int N, b, nb, n_last, BH, units;
};

template <int D>
struct PoolGeom {
  static constexpr int CH = D / 8;              // 16-byte chunks per row
  static constexpr int R = POOL_THREADS / CH;   // row groups
};

template <int D>
size_t pool_smem_bytes(int b) {
  return (size_t)POOL_STAGES * b * D * 2 + (size_t)PoolGeom<D>::R * (D + 4) * 4 +
         POOL_STAGES * 8 + 16;
}

template <int D>
__global__ void __launch_bounds__(POOL_THREADS, POOL_CTAS_PER_SM) pool_kernel(const PoolArgs a) {
  constexpr int CH = PoolGeom<D>::CH, R = PoolGeom<D>::R;
  extern __shared__ __align__(128) uint8_t smem[];
  const int row_bytes = D * 2, tile_bytes = a.b * row_bytes;
  float(*red)[D + 4] = reinterpret_cast<float(*)[D + 4]>(smem + POOL_STAGES * tile_bytes);
  uint8_t* tail = smem + POOL_STAGES * tile_bytes + R * (D + 4) * 4;
  uint64_t* fullb = reinterpret_cast<uint64_t*>(tail);
  volatile int* abort = reinterpret_cast<volatile int*>(tail + POOL_STAGES * 8);
  const uint32_t ring = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (blockIdx.x == 0 && a.ctrl)
    for (int q = tid; q < CTRL_WORDS; q += POOL_THREADS) a.ctrl[q] = 0;
  if (tid == 0) {
    for (int s = 0; s < POOL_STAGES; ++s) tc::mbar_init(smem_u32(&fullb[s]), 1);
    *abort = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();

  const int per_head = a.nb, per_tensor = a.BH * a.nb;
  auto rows_of = [&](int j) { return j == a.nb - 1 ? a.n_last : a.b; };
  // select by branch, not by indexing the parameter arrays (which would copy
  // them to local memory)
  auto src_of = [&](int t) { return t == 0 ? a.X[0] : t == 1 ? a.X[1] : a.X[2]; };
  const int G = gridDim.x;
  const int mine = a.units > (int)blockIdx.x ? (a.units - 1 - (int)blockIdx.x) / G + 1 : 0;

  // warp 0: fill ring slot k % STAGES with this CTA's k-th unit
  int issued = 0;
  auto issue = [&](int k) {
    ++issued;
    const int u = blockIdx.x + k * G;
    const int t = u / per_tensor, bh = (u % per_tensor) / per_head, j = u % per_head;
    const int n = rows_of(j);
    const uint32_t slot = k % POOL_STAGES;
    const uint32_t fb = smem_u32(&fullb[slot]);
    const uint32_t dst = ring + slot * tile_bytes;
    const __nv_bfloat16* X = src_of(t) + (size_t)bh * a.N * D;
    if (lane == 0) {
      tc::mbar_expect_tx(fb, (uint32_t)(n * row_bytes));
      tc::bulk_load(dst, X + (size_t)j * a.b * D, (uint32_t)(n * row_bytes), fb);
    }
  };
  if (warp == 0)
    for (int k = 0; k < POOL_STAGES && k < mine; ++k) issue(k);

  const int c = tid % CH, r0 = tid / CH;
  for (int k = 0; k < mine; ++k) {
    const int u = blockIdx.x + k * G;
    const int t = u / per_tensor, bh = (u % per_tensor) / per_head, j = u % per_head;
    const int n = rows_of(j);
    const uint32_t slot = k % POOL_STAGES;
    const uint8_t* tile = smem + slot * tile_bytes;
    const bool ok = tc::mbar_wait(smem_u32(&fullb[slot]), (uint32_t)(k / POOL_STAGES) & 1u, abort,
                                  a.ctrl, 20);
    if (!__syncthreads_and(ok)) break;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int r = r0; r < n; r += R) {
      const uint4 v = *reinterpret_cast<const uint4*>(tile + r * row_bytes + c * 16);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][c * 8 + e] = acc[e];
    __syncthreads();
    // the slot has been read: refill it
    if (warp == 0 && k + POOL_STAGES < mine) issue(k + POOL_STAGES);
    if (tid < D) {
      float s = 0.f;
#pragma unroll 8
      for (int q = 0; q < R; ++q) s += red[q][tid];
      const float mean = s / (float)n;
      const size_t o = ((size_t)bh * a.nb + j) * D + tid;
      float* bar = t == 0 ? a.bar[0] : t == 1 ? a.bar[1] : a.bar[2];
      __nv_bfloat16* bar16 = t == 0 ? a.bar16[0] : t == 1 ? a.bar16[1] : a.bar16[2];
      bar[o] = mean;
      if (bar16) bar16[o] = __float2bfloat16_rn(mean);
    }
    __syncthreads();
  }
  if (*abort && warp == 0) {
    // let the copies already issued land before the CTA can exit
    for (int kk = issued > POOL_STAGES ? issued - POOL_STAGES : 0; kk < issued; ++kk)
      tc::mbar_drain(smem_u32(&fullb[kk % POOL_STAGES]), (uint32_t)(kk / POOL_STAGES) & 1u);
  }
}

// Gather form for a permutation: rows are scattered, so each thread loads its
// share of a unit's rows with 16-byte loads straight into registers (no
// per-row copy setup), writes the permuted copy from them and sums them.
// The next unit's rows are loaded before the current unit is reduced, so
// every SM keeps two units of loads in flight.
template <int D>
__global__ void __launch_bounds__(POOL_THREADS, POOL_CTAS_PER_SM) pool_gather_kernel(const PoolArgs a) {
  constexpr int CH = PoolGeom<D>::CH, R = PoolGeom<D>::R;
  constexpr int IT = 128 / R;                 // row passes for a 128-token block
  __shared__ float red[R][D + 4];
  const int tid = threadIdx.x;
  if (blockIdx.x == 0 && a.ctrl)
    for (int q = tid; q < CTRL_WORDS; q += POOL_THREADS) a.ctrl[q] = 0;
  const int per_head = a.nb, per_tensor = a.BH * a.nb;
  const int c = tid % CH, r0 = tid / CH;
  const int G = gridDim.x;
  auto rows_of = [&](int j) { return j == a.nb - 1 ? a.n_last : a.b; };

  uint4 cur[IT], nxt[IT];
  auto load = [&](int u, uint4 (&v)[IT]) {
    const int t = u / per_tensor, bh = (u % per_tensor) / per_head, j = u % per_head;
    const int n = rows_of(j);
    const __nv_bfloat16* X = (t == 0 ? a.X[0] : t == 1 ? a.X[1] : a.X[2]) + (size_t)bh * a.N * D;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int r = r0 + it * R;
      if (r < n) {
        // a permutation entry outside [0, N) (possible only where the
        // caller's device permutation is not checked on the host) is
        // flagged and its row left out, never read through
        const int src = __ldg(a.perm + j * a.b + r);
        if ((unsigned)src < (unsigned)a.N) {
          v[it] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)src * D) + c);
        } else {
          v[it] = make_uint4(0u, 0u, 0u, 0u);
          if (c == 0 && a.ctrl) flag_error(a.ctrl, DEV_BAD_INDEX, j * a.b + r);
        }
      }
    }
  };
  int u = blockIdx.x;
  if (u < a.units) load(u, cur);
  for (; u < a.units; u += G) {
    const int un = u + G;
    if (un < a.units) load(un, nxt);
    const int t = u / per_tensor, bh = (u % per_tensor) / per_head, j = u % per_head;
    const int n = rows_of(j);
    __nv_bfloat16* Xp = t == 0 ? a.Xp[0] : t == 1 ? a.Xp[1] : a.Xp[2];
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int r = r0 + it * R;
      if (r < n) {
        if (Xp) reinterpret_cast<uint4*>(Xp + ((size_t)bh * a.N + (size_t)j * a.b + r) * D)[c] = cur[it];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&cur[it]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0][c * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
#pragma unroll 8
      for (int q = 0; q < R; ++q) s += red[q][tid];
      const float mean = s / (float)n;
      const size_t o = ((size_t)bh * a.nb + j) * D + tid;
      float* bar = t == 0 ? a.bar[0] : t == 1 ? a.bar[1] : a.bar[2];
      __nv_bfloat16* bar16 = t == 0 ? a.bar16[0] : t == 1 ? a.bar16[1] : a.bar16[2];
      bar[o] = mean;
      if (bar16) bar16[o] = __float2bfloat16_rn(mean);
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < IT; ++it) cur[it] = nxt[it];
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

template <int D>
cudaError_t launch_pool_d(const PoolArgs& a, cudaStream_t s) {
  if (a.perm) {
    const int grid = std::max(1, std::min(a.units, POOL_CTAS_PER_SM * sm_count()));
    pool_gather_kernel<D><<<grid, POOL_THREADS, 0, s>>>(a);
    return cudaGetLastError();
  }
  const size_t smem = pool_smem_bytes<D>(a.b);
  cudaError_t e = ensure_dyn_smem((const void*)pool_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(a.units, POOL_CTAS_PER_SM * sm_count()));
  pool_kernel<D><<<grid, POOL_THREADS, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_pool_any(const Problem& p, const PoolArgs& a, cudaStream_t s) {
  return p.d == 128 ? launch_pool_d<128>(a, s) : launch_pool_d<64>(a, s);
}

}  // namespace

cudaError_t launch_pool(const Problem& p, const void* Q, const void* K, const void* V,
                        const Work& w, cudaStream_t s) {
  PoolArgs a;
  a.X[0] = static_cast<const __nv_bfloat16*>(Q);
  a.X[1] = static_cast<const __nv_bfloat16*>(K);
  a.X[2] = static_cast<const __nv_bfloat16*>(V);
  a.Xp[0] = w.qp; a.Xp[1] = w.kp; a.Xp[2] = w.vp;
  a.bar[0] = w.qbar; a.bar[1] = w.kbar; a.bar[2] = w.vbar;
  a.bar16[0] = nullptr; a.bar16[1] = w.kbar16; a.bar16[2] = w.vbar16;
  a.perm = p.perm;
  a.ctrl = w.ctrl;
  a.N = p.N; a.b = p.b; a.nb = p.nb; a.n_last = p.n_last; a.BH = p.BH;
  a.units = 3 * p.BH * p.nb;
  return launch_pool_any(p, a, s);
}

// Means of Q and K only, no bf16 copies and no permuted copies: what the
// routing step needs, for callers that keep no other scratch.
cudaError_t launch_pool_qk(const Problem& p, const void* Q, const void* K, float* qbar,
                           float* kbar, int32_t* ctrl, cudaStream_t s) {
  PoolArgs a;
  a.X[0] = static_cast<const __nv_bfloat16*>(Q);
  a.X[1] = static_cast<const __nv_bfloat16*>(K);
  a.X[2] = nullptr;
  a.Xp[0] = a.Xp[1] = a.Xp[2] = nullptr;
  a.bar[0] = qbar; a.bar[1] = kbar; a.bar[2] = nullptr;
  a.bar16[0] = a.bar16[1] = a.bar16[2] = nullptr;
  a.perm = p.perm;
  a.ctrl = ctrl;
  a.N = p.N; a.b = p.b; a.nb = p.nb; a.n_last = p.n_last; a.BH = p.BH;
  a.units = 2 * p.BH * p.nb;
  return launch_pool_any(p, a, s);
}

}  // namespace spattn
