// Probe-fitted residual correction of a routed attention output.
//
// SparsePR page, section 2B: a few query rows (probes) are evaluated exactly;
// their residual R = O_dense - O_sparse is modelled as an affine function of
// the sparse output, R ~ b + x B, fitted per attention call by ridge
// regression; the fitted correction is restricted to the span of the r
// leading right singular vectors of the probe residuals and added to every
// row's sparse output.  Probe rows take their exact output.
//
// One head at a time (every (batch, head) pair is its own attention call):
//
//   probe_gather_kernel the probe queries into whole 128-row tiles, then the
//                       tcgen05 attention kernel in its dense mode: exact
//                       softmax attention of those rows over all N keys, fp32
//                       output (bf16 operands, fp32 accumulation, as every
//                       attention row of this library);
//   probe_fit_kernel    normal equations of the ridge fit on [1, x]:
//                       G = A^T A + lam * diag(0, 1, ..., 1), C = A^T R, then
//                       a Cholesky factorisation of G and two triangular
//                       solves for W = [b; B] (one CTA per head);
//   probe_eig_kernel    R^T R, its eigenvectors by the cyclic Jacobi method
//                       with a round-robin pairing (d/2 disjoint rotations per
//                       step), the projector P = V_r V_r^T on the r largest
//                       eigenvalues (the r leading right singular vectors of
//                       R), and B P, b P (one CTA per head);
//   probe_apply_kernel  O <- O + O (B P) + b P for every row, bf16 out;
//   probe_set_kernel    probe rows <- their exact output.
//
// All arithmetic is fp32.  A probe index outside [0, N) is skipped and
// flagged (DEV_BAD_INDEX); normal equations that are not positive definite
// leave that head uncorrected and are flagged (DEV_NUMERIC).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace spattn {
namespace {

constexpr int PB_THREADS = 256;
constexpr int PF_CHUNK = 32;               // probe rows per accumulation chunk
constexpr int PA_ROWS = 64;                // output rows per apply CTA
constexpr int JACOBI_MAX_SWEEPS = 16;

struct ProbeArgs {
  const __nv_bfloat16 *q, *k, *v;  // [BH, N, D], original token order
  __nv_bfloat16* o;                // [BH, N, D], in: routed output, out: corrected
  const int32_t* probes;           // [BH, M] token indices
  float* od;                       // [BH, M, D] exact probe rows
  float* w;                        // [BH, D + 1, D] ridge solution, row 0 = b
  float* wp;                       // [BH, D, D] B P
  float* cp;                       // [BH, D] b P
  int32_t* ctrl;                   // error word
  int N, M, BH, r;
  float lam;
};

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int probe_token(const ProbeArgs& a, int bh, int m) {
  const int tok = __ldg(a.probes + (size_t)bh * a.M + m);
  return (tok >= 0 && tok < a.N) ? tok : -1;
}

// ---- exact rows ------------------------------------------------------------
// The probe queries are gathered into a [BH, Mpad, D] bf16 buffer (rows past M
// zero); the tcgen05 attention kernel then runs them as dense query tiles over
// all N keys with an fp32 output (launch_dense_rows_tc).

template <int D>
__global__ void __launch_bounds__(PB_THREADS) probe_gather_kernel(const ProbeArgs a, int m_alloc,
                                                                  __nv_bfloat16* qg) {
  constexpr int CH = D / 8;   // 16-byte chunks per row
  const int bh = blockIdx.y;
  const int e = blockIdx.x * PB_THREADS + threadIdx.x;
  const int m = e / CH, c = e % CH;
  if (m >= m_alloc) return;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (m < a.M) {
    const int tok = probe_token(a, bh, m);
    if (tok >= 0) {
      v = __ldg(reinterpret_cast<const uint4*>(a.q + ((size_t)bh * a.N + tok) * D) + c);
    } else if (c == 0) {
      flag_error(a.ctrl, DEV_BAD_INDEX, bh * a.M + m);
    }
  }
  reinterpret_cast<uint4*>(qg + ((size_t)bh * m_alloc + m) * D)[c] = v;
}

// ---- ridge fit -------------------------------------------------------------

template <int D>
size_t fit_smem_bytes() {
  constexpr int DA = D + 1;
  return ((size_t)DA * DA + (size_t)DA * D + (size_t)PF_CHUNK * DA + (size_t)PF_CHUNK * D + 4) *
         sizeof(float);
}

// Rows m0 .. m0 + PF_CHUNK - 1 of A = [1, x] and R = x_exact - x into shared
// memory (rows past M, or with a bad probe index, are zero and add nothing).
template <int D>
__device__ void load_probe_chunk(const ProbeArgs& a, int bh, int m0, float* xa, float* rc) {
  constexpr int DA = D + 1;
  for (int e = threadIdx.x; e < PF_CHUNK * D; e += PB_THREADS) {
    const int rr = e / D, c = e % D, m = m0 + rr;
    const int tok = m < a.M ? probe_token(a, bh, m) : -1;
    float x = 0.f, res = 0.f;
    if (tok >= 0) {
      x = __bfloat162float(a.o[((size_t)bh * a.N + tok) * D + c]);
      res = a.od[((size_t)bh * a.M + m) * D + c] - x;
    }
    xa[rr * DA + 1 + c] = x;
    rc[rr * D + c] = res;
    if (c == 0) xa[rr * DA] = tok >= 0 ? 1.f : 0.f;
  }
}

template <int D>
__global__ void __launch_bounds__(PB_THREADS) probe_fit_kernel(const ProbeArgs a) {
  constexpr int DA = D + 1;
  extern __shared__ float psm[];
  float* G = psm;                  // [DA][DA]
  float* C = G + DA * DA;          // [DA][D], then the solution W
  float* xa = C + DA * D;          // [PF_CHUNK][DA]
  float* rc = xa + PF_CHUNK * DA;  // [PF_CHUNK][D]
  int* bad = reinterpret_cast<int*>(rc + PF_CHUNK * D);
  const int bh = blockIdx.x, tid = threadIdx.x;
  for (int e = tid; e < DA * DA; e += PB_THREADS) G[e] = 0.f;
  for (int e = tid; e < DA * D; e += PB_THREADS) C[e] = 0.f;
  if (tid == 0) *bad = 0;
  for (int m0 = 0; m0 < a.M; m0 += PF_CHUNK) {
    __syncthreads();
    load_probe_chunk<D>(a, bh, m0, xa, rc);
    __syncthreads();
    for (int e = tid; e < DA * DA; e += PB_THREADS) {
      const int i = e / DA, j = e % DA;
      float s = G[e];
      for (int rr = 0; rr < PF_CHUNK; ++rr) s = fmaf(xa[rr * DA + i], xa[rr * DA + j], s);
      G[e] = s;
    }
    for (int e = tid; e < DA * D; e += PB_THREADS) {
      const int i = e / D, c = e % D;
      float s = C[e];
      for (int rr = 0; rr < PF_CHUNK; ++rr) s = fmaf(xa[rr * DA + i], rc[rr * D + c], s);
      C[e] = s;
    }
  }
  __syncthreads();
  for (int i = 1 + tid; i < DA; i += PB_THREADS) G[i * DA + i] += a.lam;   // the bias is not penalised
  __syncthreads();
  // Cholesky, lower triangle in place: G = L L^T
  for (int k = 0; k < DA; ++k) {
    if (tid == 0) {
      const float dkk = G[k * DA + k];
      if (!(dkk > 0.f) || !isfinite(dkk)) *bad = 1;
      G[k * DA + k] = sqrtf(fmaxf(dkk, 1e-30f));
    }
    __syncthreads();
    const float lkk = G[k * DA + k];
    for (int i = k + 1 + tid; i < DA; i += PB_THREADS) G[i * DA + k] /= lkk;
    __syncthreads();
    const int n = DA - k - 1;   // trailing block (k, DA) x (k, DA), lower part
    for (int e = tid; e < n * n; e += PB_THREADS) {
      const int i = k + 1 + e / n, j = k + 1 + e % n;
      if (j <= i) G[i * DA + j] = fmaf(-G[i * DA + k], G[j * DA + k], G[i * DA + j]);
    }
    __syncthreads();
  }
  // L Y = C, then L^T W = Y: one right-hand side (output channel) per thread
  for (int c = tid; c < D; c += PB_THREADS) {
    for (int i = 0; i < DA; ++i) {
      float s = C[i * D + c];
      for (int k = 0; k < i; ++k) s = fmaf(-G[i * DA + k], C[k * D + c], s);
      C[i * D + c] = s / G[i * DA + i];
    }
    for (int i = DA - 1; i >= 0; --i) {
      float s = C[i * D + c];
      for (int k = i + 1; k < DA; ++k) s = fmaf(-G[k * DA + i], C[k * D + c], s);
      C[i * D + c] = s / G[i * DA + i];
    }
  }
  __syncthreads();
  const bool failed = *bad != 0;
  if (failed && tid == 0) flag_error(a.ctrl, DEV_NUMERIC, bh);
  float* w = a.w + (size_t)bh * DA * D;
  for (int e = tid; e < DA * D; e += PB_THREADS) w[e] = failed ? 0.f : C[e];
}

// ---- residual subspace and the folded correction --------------------------

template <int D>
size_t eig_smem_bytes() {
  return ((size_t)2 * D * (D + 1) + (size_t)PF_CHUNK * D + (size_t)PF_CHUNK * (D + 1) +
          (size_t)2 * (D / 2) + 2 * D + 4) * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(PB_THREADS) probe_eig_kernel(const ProbeArgs a) {
  constexpr int DP = D + 1;        // padded row: column updates hit distinct banks
  constexpr int H = D / 2;
  extern __shared__ float psm[];
  float* S = psm;                  // [D][DP]: R^T R, rotated towards diagonal; later P
  float* V = S + D * DP;           // [D][DP]: eigenvectors (columns); later B
  float* xa = V + D * DP;          // [PF_CHUNK][D + 1]
  float* rc = xa + PF_CHUNK * (D + 1);   // [PF_CHUNK][D]
  float* rot_c = rc + PF_CHUNK * D;      // [H]
  float* rot_s = rot_c + H;              // [H]
  float* lam = rot_s + H;                // [D] eigenvalues
  float* sel = lam + D;                  // [D] 1 for the r largest, else 0
  int* flags = reinterpret_cast<int*>(sel + D);
  __shared__ int pp[H], qq[H];
  const int bh = blockIdx.x, tid = threadIdx.x;
  const float* wfit = a.w + (size_t)bh * (D + 1) * D;
  float* wp = a.wp + (size_t)bh * D * D;
  float* cp = a.cp + (size_t)bh * D;

  if (a.r <= 0 || a.r >= D) {
    // P = 0 (no correction) or P = I (the whole output space)
    const bool full = a.r >= D;
    for (int e = tid; e < D * D; e += PB_THREADS) wp[e] = full ? wfit[D + e] : 0.f;
    for (int c = tid; c < D; c += PB_THREADS) cp[c] = full ? wfit[c] : 0.f;
    return;
  }
  for (int e = tid; e < D * DP; e += PB_THREADS) S[e] = 0.f;
  for (int m0 = 0; m0 < a.M; m0 += PF_CHUNK) {
    __syncthreads();
    load_probe_chunk<D>(a, bh, m0, xa, rc);
    __syncthreads();
    for (int e = tid; e < D * D; e += PB_THREADS) {
      const int i = e / D, j = e % D;
      float s = S[i * DP + j];
      for (int rr = 0; rr < PF_CHUNK; ++rr) s = fmaf(rc[rr * D + i], rc[rr * D + j], s);
      S[i * DP + j] = s;
    }
  }
  for (int e = tid; e < D * DP; e += PB_THREADS) V[e] = (e % DP == e / DP) ? 1.f : 0.f;
  __syncthreads();

  // cyclic Jacobi, round-robin pairing: in step t of a sweep, pair 0 is
  // (t, D - 1) and pair k > 0 is ((t + k) mod (D - 1), (t - k) mod (D - 1));
  // every unordered pair meets once per sweep of D - 1 steps
  for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS; ++sweep) {
    // stop when the off-diagonal mass is negligible against the diagonal
    if (tid < 32) {
      float off = 0.f, dia = 0.f;
      for (int e = tid; e < D * D; e += 32) {
        const int i = e / D, j = e % D;
        const float x = S[i * DP + j];
        if (i == j) dia += x * x; else off += x * x;
      }
      off = warp_sum_f(off);
      dia = warp_sum_f(dia);
      if (tid == 0) flags[0] = off <= 1e-12f * dia ? 1 : 0;
    }
    __syncthreads();
    if (flags[0]) break;
    for (int t = 0; t < D - 1; ++t) {
      if (tid < H) {
        int p, q;
        if (tid == 0) {
          p = t; q = D - 1;
        } else {
          p = (t + tid) % (D - 1);
          q = (t - tid + (D - 1)) % (D - 1);
        }
        if (p > q) { const int x = p; p = q; q = x; }
        const float apq = S[p * DP + q], app = S[p * DP + p], aqq = S[q * DP + q];
        float c = 1.f, s = 0.f;
        if (fabsf(apq) > 1e-30f) {
          const float theta = (aqq - app) / (2.f * apq);
          const float tt = copysignf(1.f, theta) / (fabsf(theta) + sqrtf(fmaf(theta, theta, 1.f)));
          c = rsqrtf(fmaf(tt, tt, 1.f));
          s = tt * c;
        }
        pp[tid] = p; qq[tid] = q; rot_c[tid] = c; rot_s[tid] = s;
      }
      __syncthreads();
      // columns: S <- S J, V <- V J
      for (int e = tid; e < H * D; e += PB_THREADS) {
        const int k = e / D, i = e % D;
        const int p = pp[k], q = qq[k];
        const float c = rot_c[k], s = rot_s[k];
        const float sp = S[i * DP + p], sq = S[i * DP + q];
        S[i * DP + p] = c * sp - s * sq;
        S[i * DP + q] = s * sp + c * sq;
        const float vp = V[i * DP + p], vq = V[i * DP + q];
        V[i * DP + p] = c * vp - s * vq;
        V[i * DP + q] = s * vp + c * vq;
      }
      __syncthreads();
      // rows: S <- J^T S
      for (int e = tid; e < H * D; e += PB_THREADS) {
        const int k = e / D, j = e % D;
        const int p = pp[k], q = qq[k];
        const float c = rot_c[k], s = rot_s[k];
        const float sp = S[p * DP + j], sq = S[q * DP + j];
        S[p * DP + j] = c * sp - s * sq;
        S[q * DP + j] = s * sp + c * sq;
      }
      __syncthreads();
    }
  }
  // eigenvalues; the r largest (ties: lower index) span the subspace
  for (int i = tid; i < D; i += PB_THREADS) lam[i] = S[i * DP + i];
  __syncthreads();
  for (int i = tid; i < D; i += PB_THREADS) {
    int rank = 0;
    for (int j = 0; j < D; ++j) rank += (lam[j] > lam[i] || (lam[j] == lam[i] && j < i)) ? 1 : 0;
    sel[i] = rank < a.r ? 1.f : 0.f;
  }
  __syncthreads();
  // P = V diag(sel) V^T into S
  for (int e = tid; e < D * D; e += PB_THREADS) {
    const int i = e / D, j = e % D;
    float s = 0.f;
    for (int k = 0; k < D; ++k) s = fmaf(sel[k] * V[i * DP + k], V[j * DP + k], s);
    S[i * DP + j] = s;
  }
  __syncthreads();
  // B into V's space, then B P and b P
  for (int e = tid; e < D * D; e += PB_THREADS) V[(e / D) * DP + e % D] = wfit[D + e];
  __syncthreads();
  for (int e = tid; e < D * D; e += PB_THREADS) {
    const int i = e / D, j = e % D;
    float s = 0.f;
    for (int k = 0; k < D; ++k) s = fmaf(V[i * DP + k], S[k * DP + j], s);
    wp[e] = s;
  }
  for (int j = tid; j < D; j += PB_THREADS) {
    float s = 0.f;
    for (int k = 0; k < D; ++k) s = fmaf(wfit[k], S[k * DP + j], s);
    cp[j] = s;
  }
}

// ---- apply -----------------------------------------------------------------

template <int D>
size_t apply_smem_bytes() {
  return ((size_t)D * D + D + (size_t)PA_ROWS * D) * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(PB_THREADS) probe_apply_kernel(const ProbeArgs a) {
  constexpr int RPT = PA_ROWS * D / PB_THREADS;   // rows per thread (one column each)
  extern __shared__ float psm[];
  float* W = psm;                 // [D][D] B P
  float* cvec = W + D * D;        // [D]    b P
  float* X = cvec + D;            // [PA_ROWS][D] sparse output rows
  const int bh = blockIdx.y, n0 = blockIdx.x * PA_ROWS, tid = threadIdx.x;
  const float* wp = a.wp + (size_t)bh * D * D;
  for (int e = tid; e < D * D; e += PB_THREADS) W[e] = wp[e];
  for (int c = tid; c < D; c += PB_THREADS) cvec[c] = a.cp[(size_t)bh * D + c];
  __nv_bfloat16* orows = a.o + ((size_t)bh * a.N + n0) * D;
  for (int e = tid; e < PA_ROWS * D; e += PB_THREADS) {
    const int rr = e / D;
    X[e] = n0 + rr < a.N ? __bfloat162float(orows[e]) : 0.f;
  }
  __syncthreads();
  const int j = tid % D, r0 = (tid / D) * RPT;
  float acc[RPT];
#pragma unroll
  for (int t = 0; t < RPT; ++t) acc[t] = X[(r0 + t) * D + j] + cvec[j];
  for (int i = 0; i < D; ++i) {
    const float w = W[i * D + j];
#pragma unroll
    for (int t = 0; t < RPT; ++t) acc[t] = fmaf(X[(r0 + t) * D + i], w, acc[t]);
  }
#pragma unroll
  for (int t = 0; t < RPT; ++t)
    if (n0 + r0 + t < a.N) orows[(size_t)(r0 + t) * D + j] = __float2bfloat16_rn(acc[t]);
}

template <int D>
__global__ void __launch_bounds__(D) probe_set_kernel(const ProbeArgs a) {
  const int m = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const int tok = probe_token(a, bh, m);
  if (tok < 0) return;
  a.o[((size_t)bh * a.N + tok) * D + c] = __float2bfloat16_rn(a.od[((size_t)bh * a.M + m) * D + c]);
}

template <int D>
cudaError_t launch_probe_d(const Problem& p, const ProbeArgs& a, int m_alloc, __nv_bfloat16* qg,
                           cudaStream_t s) {
  cudaError_t e;
  if ((e = ensure_dyn_smem((const void*)probe_fit_kernel<D>, fit_smem_bytes<D>())) != cudaSuccess) return e;
  if ((e = ensure_dyn_smem((const void*)probe_eig_kernel<D>, eig_smem_bytes<D>())) != cudaSuccess) return e;
  if ((e = ensure_dyn_smem((const void*)probe_apply_kernel<D>, apply_smem_bytes<D>())) != cudaSuccess) return e;
  const int gather_blocks = (m_alloc * (D / 8) + PB_THREADS - 1) / PB_THREADS;
  probe_gather_kernel<D><<<dim3(gather_blocks, a.BH), PB_THREADS, 0, s>>>(a, m_alloc, qg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_dense_rows_tc(p, qg, m_alloc, a.M, a.k, a.v, a.od, a.ctrl, s)) != cudaSuccess) return e;
  probe_fit_kernel<D><<<a.BH, PB_THREADS, fit_smem_bytes<D>(), s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  probe_eig_kernel<D><<<a.BH, PB_THREADS, eig_smem_bytes<D>(), s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  probe_apply_kernel<D><<<dim3((a.N + PA_ROWS - 1) / PA_ROWS, a.BH), PB_THREADS, apply_smem_bytes<D>(), s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  probe_set_kernel<D><<<dim3(a.M, a.BH), D, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

// Probe queries are gathered into whole 128-row tiles.
inline int probe_rows_alloc(int M) { return (M + 127) / 128 * 128; }

size_t probe_scratch_bytes(const Problem& p, int M) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t BH = (size_t)p.BH, d = (size_t)p.d;
  return up(BH * M * d * 4) + up(BH * (d + 1) * d * 4) + up(BH * d * d * 4) + up(BH * d * 4) +
         up(BH * probe_rows_alloc(M) * d * 2);
}

cudaError_t launch_probe_correct(const Problem& p, const void* Q, const void* K, const void* V,
                                 void* O, const int32_t* probes, int M, float lam, int r,
                                 void* scratch, int32_t* ctrl, cudaStream_t s) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t BH = (size_t)p.BH, d = (size_t)p.d;
  uint8_t* b = static_cast<uint8_t*>(scratch);
  ProbeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(Q);
  a.k = static_cast<const __nv_bfloat16*>(K);
  a.v = static_cast<const __nv_bfloat16*>(V);
  a.o = static_cast<__nv_bfloat16*>(O);
  a.probes = probes;
  size_t off = 0;
  a.od = reinterpret_cast<float*>(b + off); off += up(BH * M * d * 4);
  a.w = reinterpret_cast<float*>(b + off);  off += up(BH * (d + 1) * d * 4);
  a.wp = reinterpret_cast<float*>(b + off); off += up(BH * d * d * 4);
  a.cp = reinterpret_cast<float*>(b + off); off += up(BH * d * 4);
  __nv_bfloat16* qg = reinterpret_cast<__nv_bfloat16*>(b + off);
  a.ctrl = ctrl;
  a.N = p.N; a.M = M; a.BH = p.BH; a.r = r; a.lam = lam;
  const int m_alloc = probe_rows_alloc(M);
  return p.d == 128 ? launch_probe_d<128>(p, a, m_alloc, qg, s)
                    : launch_probe_d<64>(p, a, m_alloc, qg, s);
}

}  // namespace spattn
