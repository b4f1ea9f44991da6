// Token gather (optional permutation) fused with block-mean pooling.
//
// Blocks are represented by the mean of their tokens (PARK page, abstract and
// section 4: "averaged representations of query and key blocks").  With a
// permutation, the kernel reads X[perm[n]] and writes the permuted copy Xp[n]
// in the same pass (DFSAttn abstract: Hilbert reordering before blocking), so
// Q/K/V are read from HBM exactly once.
//
// One CTA per (block j, head bh, tensor); 256 threads.  A thread owns one
// 16-byte chunk (8 channels) of the row and walks the rows r0, r0+R, ... of
// the block, accumulating in fp32 in a fixed order; the R partial sums are
// then reduced in a fixed order too, so the means are bit-reproducible.
#include "common.cuh"
#include "internal.h"

namespace spattn {
namespace {

struct PoolArgs {
  const __nv_bfloat16* X[3];
  __nv_bfloat16* Xp[3];    // permuted copies, NULL when there is no perm
  float* bar[3];           // fp32 means [BH, nb, d]
  __nv_bfloat16* bar16[3]; // bf16 means (K and V only; NULL for Q)
  const int32_t* perm;
  int N, b, nb, n_last;
};

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(PoolArgs a) {
  constexpr int CH = D / 8;          // 16-byte chunks per row
  constexpr int R = 256 / CH;        // rows in flight per CTA pass
  constexpr int IT = 128 / R;        // passes for the largest block (b = 128)
  __shared__ float red[R][D + 4];

  const int j = blockIdx.x, bh = blockIdx.y, t = blockIdx.z;
  const int n = (j == a.nb - 1) ? a.n_last : a.b;
  const size_t head = (size_t)bh * a.N * D;
  // select by branch, not by indexing the parameter arrays (which would copy
  // them to local memory)
  const __nv_bfloat16* X = (t == 0 ? a.X[0] : t == 1 ? a.X[1] : a.X[2]) + head;
  __nv_bfloat16* Xp0 = t == 0 ? a.Xp[0] : t == 1 ? a.Xp[1] : a.Xp[2];
  __nv_bfloat16* Xp = Xp0 ? Xp0 + head : nullptr;
  float* bar = t == 0 ? a.bar[0] : t == 1 ? a.bar[1] : a.bar[2];
  __nv_bfloat16* bar16 = t == 0 ? a.bar16[0] : t == 1 ? a.bar16[1] : a.bar16[2];
  const int c = threadIdx.x % CH, r0 = threadIdx.x / CH;

  uint4 v[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int r = r0 + it * R;
    if (r < n) {
      const int tok = j * a.b + r;
      const int src = a.perm ? __ldg(a.perm + tok) : tok;
      v[it] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)src * D) + c);
    }
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int r = r0 + it * R;
    if (r < n) {
      if (Xp) reinterpret_cast<uint4*>(Xp + (size_t)(j * a.b + r) * D)[c] = v[it];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[it]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[r0][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int q = 0; q < R; ++q) s += red[q][threadIdx.x];
    const float mean = s / (float)n;
    const size_t o = ((size_t)bh * a.nb + j) * D + threadIdx.x;
    bar[o] = mean;
    if (bar16) bar16[o] = __float2bfloat16_rn(mean);
  }
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
  a.N = p.N; a.b = p.b; a.nb = p.nb; a.n_last = p.n_last;
  dim3 grid(p.nb, p.BH, 3);
  if (p.d == 128) pool_kernel<128><<<grid, 256, 0, s>>>(a);
  else pool_kernel<64><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// Means of Q and K only (grid z = 2), no bf16 copies and no permuted copies:
// what the routing step needs, for callers that keep no other scratch.
cudaError_t launch_pool_qk(const Problem& p, const void* Q, const void* K, float* qbar,
                           float* kbar, cudaStream_t s) {
  PoolArgs a;
  a.X[0] = static_cast<const __nv_bfloat16*>(Q);
  a.X[1] = static_cast<const __nv_bfloat16*>(K);
  a.X[2] = nullptr;
  a.Xp[0] = a.Xp[1] = a.Xp[2] = nullptr;
  a.bar[0] = qbar; a.bar[1] = kbar; a.bar[2] = nullptr;
  a.bar16[0] = a.bar16[1] = a.bar16[2] = nullptr;
  a.perm = p.perm;
  a.N = p.N; a.b = p.b; a.nb = p.nb; a.n_last = p.n_last;
  dim3 grid(p.nb, p.BH, 2);
  if (p.d == 128) pool_kernel<128><<<grid, 256, 0, s>>>(a);
  else pool_kernel<64><<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace spattn
