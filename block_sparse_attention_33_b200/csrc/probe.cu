// Probe-fitted residual correction of a routed attention output.
//
// SparsePR page, section 2B: a few query rows (probes) are evaluated exactly;
// their residual R = O_dense - O_sparse is modelled as an affine function of
// the sparse output, R ~ b + x B, fitted per attention call by ridge
// regression; the fitted correction is restricted to the span of the r
// leading right singular vectors of the probe residuals and added to every
// row's sparse output.  Probe rows take their exact output.
//
// Per (batch, head) pair (every pair is its own attention call):
//
//   probe_gather_kernel the probe queries into whole 128-row tiles, then the
//                       tcgen05 attention kernel in its dense mode: exact
//                       softmax attention of those rows over all N keys, fp32
//                       output (bf16 operands, fp32 accumulation, as every
//                       attention row of this library);
//   probe_gram_kernel   the Gram matrix of the probe rows [1, x, R] (one CTA
//                       per 128 probe rows and head, partial sums per slab):
//                       its blocks are A^T A, A^T R and R^T R for A = [1, x];
//   probe_solve_kernel  role 0, the ridge fit: G = A^T A + lam diag(0, 1,
//                       ..., 1), C = A^T R, Cholesky and two triangular solves
//                       for W = [b; B]; role 1, the r leading eigenvectors of
//                       R^T R (the leading right singular vectors of R) by
//                       block subspace iteration with a Rayleigh-Ritz step, or
//                       cyclic Jacobi on the whole matrix for large r;
//   probe_fold_kernel   B P and b P with P = U U^T;
//   then the tcgen05 apply (launch_probe_apply_tc): O <- O + O (B P) + b P
//                       for every row, bf16 out;
//   probe_set_kernel    probe rows <- their exact output.
//
// The fit and the subspace are fp32; B P enters the tensor-core apply in
// bf16 (the correction it makes is about a thousandth of the output).  A
// probe index outside [0, N) is skipped and flagged (DEV_BAD_INDEX); normal
// equations that are not positive definite leave that head uncorrected and
// are flagged (DEV_NUMERIC).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace spattn {
namespace {

constexpr int PB_THREADS = 256;
constexpr int JACOBI_MAX_SWEEPS = 16;

struct ProbeArgs {
  const __nv_bfloat16 *q, *k, *v;  // [BH, N, D], original token order
  __nv_bfloat16* o;                // [BH, N, D], in: routed output, out: corrected
  const int32_t* probes;           // [BH, M] token indices
  float* od;                       // [BH, M, D] exact probe rows
  float* w;                        // [BH, D + 1, D] ridge solution, row 0 = b
  __nv_bfloat16* wt;               // [BH, D, D] (B P)^T, bf16
  float* cp;                       // [BH, D] b P
  float* pu;                       // [BH, D, D] leading eigenvectors of R^T R (first r columns)
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

// ---- Gram matrix of the probe rows -----------------------------------------
// Every quantity of the fit comes from the Gram matrix of the rows
// Z = [1, x, R] (x the sparse output of a probe row, R = exact - x): with
// A = [1, x], G = A^T A, C = A^T R and S = R^T R are its blocks.  The rows of
// one head are cut into slabs of GR_ROWS; one CTA per (slab, head) adds up
// the upper-triangle 4 x 4 tiles of its slab's Gram matrix (register tiles,
// rows staged in shared memory 32 at a time) and writes them to its own
// partial buffer; the solve kernel adds the partials in slab order.

constexpr int GR_ROWS = 128;      // probe rows per Gram CTA
constexpr int GR_THREADS = 768;
constexpr int GR_CHUNK = 32;      // rows staged at a time
constexpr int SV_THREADS = 1024;  // solve kernel
constexpr int SUB_ITERS = 16;     // subspace iterations
constexpr int SUB_EXTRA = 16;     // subspace columns beyond r
constexpr int SUB_MAXQ = 64;      // subspace iteration for r + SUB_EXTRA <= 64, else Jacobi

template <int D>
struct GramGeom {
  static constexpr int ZC = 1 + 2 * D;                // columns of Z
  static constexpr int NT = (ZC + 3) / 4;             // 4-wide column tiles
  static constexpr int ZW = 4 * NT;                   // padded row width
  static constexpr int TILES = NT * (NT + 1) / 2;     // upper-triangle tiles
  static constexpr int PER = (TILES + GR_THREADS - 1) / GR_THREADS;
};

inline int gram_slabs(int M) { return (M + GR_ROWS - 1) / GR_ROWS; }

// tile index e (row-major over the upper triangle, ti <= tj) -> (ti, tj)
__device__ __forceinline__ void upper_tile(int e, int nt, int& ti, int& tj) {
  int i = 0, rowlen = nt;
  while (e >= rowlen) { e -= rowlen; ++i; --rowlen; }
  ti = i;
  tj = i + e;
}

template <int D>
__global__ void __launch_bounds__(GR_THREADS) probe_gram_kernel(const ProbeArgs a, float* gp,
                                                                int slabs) {
  using G = GramGeom<D>;
  __shared__ __align__(16) float Zs[GR_CHUNK][G::ZW];
  const int slab = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  int ti[G::PER], tj[G::PER];
  float acc[G::PER][16];
#pragma unroll
  for (int u = 0; u < G::PER; ++u) {
    const int e = tid + u * GR_THREADS;
    if (e < G::TILES) upper_tile(e, G::NT, ti[u], tj[u]); else ti[u] = tj[u] = -1;
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[u][k] = 0.f;
  }
  const int m_lo = slab * GR_ROWS, m_hi = min(a.M, m_lo + GR_ROWS);
  for (int m0 = m_lo; m0 < m_hi; m0 += GR_CHUNK) {
    __syncthreads();
    // Z rows m0 .. m0 + 31 (zero past the slab, or for a bad probe index)
    for (int e = tid; e < GR_CHUNK * G::ZW; e += GR_THREADS) {
      const int rr = e / G::ZW, c = e % G::ZW, m = m0 + rr;
      const int tok = m < m_hi ? probe_token(a, bh, m) : -1;
      float z = 0.f;
      if (tok >= 0) {
        if (c == 0) {
          z = 1.f;
        } else if (c <= D) {
          z = __bfloat162float(a.o[((size_t)bh * a.N + tok) * D + c - 1]);
        } else if (c <= 2 * D) {
          const int cc = c - D - 1;
          z = a.od[((size_t)bh * a.M + m) * D + cc] -
              __bfloat162float(a.o[((size_t)bh * a.N + tok) * D + cc]);
        }
      }
      Zs[rr][c] = z;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < G::PER; ++u) {
      if (ti[u] < 0) continue;
      for (int rr = 0; rr < GR_CHUNK; ++rr) {
        const float4 x = *reinterpret_cast<const float4*>(&Zs[rr][4 * ti[u]]);
        const float4 y = *reinterpret_cast<const float4*>(&Zs[rr][4 * tj[u]]);
        const float xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[u][4 * p + q] = fmaf(xs[p], ys[q], acc[u][4 * p + q]);
      }
    }
  }
  float* out = gp + ((size_t)bh * slabs + slab) * G::ZW * G::ZW;
#pragma unroll
  for (int u = 0; u < G::PER; ++u) {
    if (ti[u] < 0) continue;
#pragma unroll
    for (int p = 0; p < 4; ++p)
      *reinterpret_cast<float4*>(out + (size_t)(4 * ti[u] + p) * G::ZW + 4 * tj[u]) =
          make_float4(acc[u][4 * p], acc[u][4 * p + 1], acc[u][4 * p + 2], acc[u][4 * p + 3]);
  }
}

// Entry (i, j) of a head's Gram matrix: the slabs' partials added in order
// (only upper-triangle tiles are stored, so (i, j) is read from the tile side).
template <int D>
__device__ __forceinline__ float gram_at(const float* gph, int slabs, int i, int j) {
  using G = GramGeom<D>;
  if ((i >> 2) > (j >> 2)) { const int t = i; i = j; j = t; }
  float s = 0.f;
  for (int k = 0; k < slabs; ++k) s += gph[(size_t)k * G::ZW * G::ZW + (size_t)i * G::ZW + j];
  return s;
}

// ---- solve: ridge fit (role 0) and residual subspace (role 1) ---------------

template <int D>
constexpr size_t solve_smem_bytes() {
  constexpr size_t DA = D + 1;
  constexpr size_t fit = (DA * DA + DA * D + 8) * sizeof(float);
  constexpr size_t jac = (2 * (size_t)D * (D + 1) + 4 * (size_t)D + 8) * sizeof(float);
  constexpr size_t sub = ((size_t)D * (D + 4) + 2 * (size_t)D * SUB_MAXQ +
                          2 * (size_t)SUB_MAXQ * (SUB_MAXQ + 1) + 4 * (size_t)SUB_MAXQ + 8) *
                         sizeof(float);
  return fit > jac ? (fit > sub ? fit : sub) : (jac > sub ? jac : sub);
}

// In-place Cholesky of the n x n matrix A (row stride ld, lower triangle
// used) by the whole CTA; a pivot that is not positive and finite sets *bad
// (and is replaced by a tiny one so the factorisation still completes).
__device__ void cholesky_cta(float* A, int n, int ld, int* bad) {
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int k = 0; k < n; ++k) {
    if (tid == 0) {
      const float dkk = A[k * ld + k];
      if (!(dkk > 0.f) || !isfinite(dkk)) *bad = 1;
      A[k * ld + k] = sqrtf(fmaxf(dkk, 1e-30f));
    }
    __syncthreads();
    const float lkk = A[k * ld + k];
    for (int i = k + 1 + tid; i < n; i += nt) A[i * ld + k] /= lkk;
    __syncthreads();
    const int m = n - k - 1;   // trailing block, lower part
    for (int e = tid; e < m * m; e += nt) {
      const int i = k + 1 + e / m, j = k + 1 + e % m;
      if (j <= i) A[i * ld + j] = fmaf(-A[i * ld + k], A[j * ld + k], A[i * ld + j]);
    }
    __syncthreads();
  }
}

// Cyclic Jacobi on the symmetric n x n matrix S (row stride ld, n even),
// round-robin pairing (n / 2 disjoint rotations per step; every pair meets
// once in a sweep of n - 1 steps), accumulating the rotations into V (row
// stride ld, starts at the identity).  Stops when the off-diagonal mass is
// negligible against the diagonal.  rc, rs: n / 2 floats; pq: n ints; flag: 1.
__device__ void jacobi_cta(float* S, float* V, int n, int ld, float* rc, float* rs, int* pq,
                           int* flag) {
  const int tid = threadIdx.x, nt = blockDim.x, h = n / 2;
  for (int e = tid; e < n * ld; e += nt) V[e] = (e % ld == e / ld) ? 1.f : 0.f;
  __syncthreads();
  for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS; ++sweep) {
    if (tid < 32) {
      float off = 0.f, dia = 0.f;
      for (int e = tid; e < n * n; e += 32) {
        const int i = e / n, j = e % n;
        const float x = S[i * ld + j];
        if (i == j) dia += x * x; else off += x * x;
      }
      off = warp_sum_f(off);
      dia = warp_sum_f(dia);
      // 1e-9: the off-diagonal elements are then about 3e-5 of the diagonal's
      // scale; fp32 rounding alone keeps a converged matrix near 1e-11, so a
      // tighter test would never stop before the sweep limit
      if (tid == 0) *flag = off <= 1e-9f * dia ? 1 : 0;
    }
    __syncthreads();
    if (*flag) break;
    for (int t = 0; t < n - 1; ++t) {
      if (tid < h) {
        int p, q;
        if (tid == 0) {
          p = t; q = n - 1;
        } else {
          p = (t + tid) % (n - 1);
          q = (t - tid + (n - 1)) % (n - 1);
        }
        if (p > q) { const int x = p; p = q; q = x; }
        const float apq = S[p * ld + q], app = S[p * ld + p], aqq = S[q * ld + q];
        float c = 1.f, s = 0.f;
        if (fabsf(apq) > 1e-30f) {
          const float theta = (aqq - app) / (2.f * apq);
          const float tt = copysignf(1.f, theta) / (fabsf(theta) + sqrtf(fmaf(theta, theta, 1.f)));
          c = rsqrtf(fmaf(tt, tt, 1.f));
          s = tt * c;
        }
        pq[2 * tid] = p; pq[2 * tid + 1] = q; rc[tid] = c; rs[tid] = s;
      }
      __syncthreads();
      for (int e = tid; e < h * n; e += nt) {   // columns: S <- S J, V <- V J
        const int k = e / n, i = e % n;
        const int p = pq[2 * k], q = pq[2 * k + 1];
        const float c = rc[k], s = rs[k];
        const float sp = S[i * ld + p], sq = S[i * ld + q];
        S[i * ld + p] = c * sp - s * sq;
        S[i * ld + q] = s * sp + c * sq;
        const float vp = V[i * ld + p], vq = V[i * ld + q];
        V[i * ld + p] = c * vp - s * vq;
        V[i * ld + q] = s * vp + c * vq;
      }
      __syncthreads();
      for (int e = tid; e < h * n; e += nt) {   // rows: S <- J^T S
        const int k = e / n, j = e % n;
        const int p = pq[2 * k], q = pq[2 * k + 1];
        const float c = rc[k], s = rs[k];
        const float sp = S[p * ld + j], sq = S[q * ld + j];
        S[p * ld + j] = c * sp - s * sq;
        S[q * ld + j] = s * sp + c * sq;
      }
      __syncthreads();
    }
  }
}

// Columns of the r largest eigenvalues (diagonal of S after jacobi_cta; ties
// to the lower index), copied from V into U (row stride D) in rank order.
__device__ void top_vectors(const float* S, const float* V, int n, int ld, int r, float* U,
                            int D, int* rank) {
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int i = tid; i < n; i += nt) {
    const float li = S[i * ld + i];
    int k = 0;
    for (int j = 0; j < n; ++j) {
      const float lj = S[j * ld + j];
      k += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    rank[i] = k;
  }
  __syncthreads();
  for (int e = tid; e < n * n; e += nt) {
    const int row = e / n, col = e % n;
    if (rank[col] < r) U[row * D + rank[col]] = V[row * ld + col];
  }
}

template <int D>
__global__ void __launch_bounds__(SV_THREADS) probe_solve_kernel(const ProbeArgs a, const float* gp,
                                                                 int slabs) {
  using G = GramGeom<D>;
  constexpr int DA = D + 1;
  extern __shared__ __align__(16) float psm[];
  const int bh = blockIdx.x, role = blockIdx.y, tid = threadIdx.x, nt = blockDim.x;
  const float* gph = gp + (size_t)bh * slabs * G::ZW * G::ZW;
  if (role == 0) {
    // ---- ridge fit: (A^T A + lam diag(0, 1, ..., 1)) W = A^T R, W = [b; B]
    float* Gm = psm;               // [DA][DA]
    float* Cm = Gm + DA * DA;      // [DA][D], then Y, then W
    int* bad = reinterpret_cast<int*>(Cm + DA * D);
    for (int e = tid; e < DA * DA; e += nt) {
      const int i = e / DA, j = e % DA;
      Gm[e] = gram_at<D>(gph, slabs, i, j) + ((i == j && i > 0) ? a.lam : 0.f);
    }
    for (int e = tid; e < DA * D; e += nt) Cm[e] = gram_at<D>(gph, slabs, e / D, DA + e % D);
    if (tid == 0) *bad = 0;
    __syncthreads();
    cholesky_cta(Gm, DA, DA, bad);
    // L Y = C, then L^T W = Y, one row at a time; (column c, part) threads
    // add strided parts of each row's sum, reduced over 8 lanes
    const int c = tid >> 3, part = tid & 7;
    const bool live = c < D;
    for (int i = 0; i < DA; ++i) {
      float s = 0.f;
      if (live)
        for (int k = part; k < i; k += 8) s = fmaf(Gm[i * DA + k], Cm[k * D + c], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (live && part == 0) Cm[i * D + c] = (Cm[i * D + c] - s) / Gm[i * DA + i];
      __syncthreads();
    }
    for (int i = DA - 1; i >= 0; --i) {
      float s = 0.f;
      if (live)
        for (int k = i + 1 + part; k < DA; k += 8) s = fmaf(Gm[k * DA + i], Cm[k * D + c], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (live && part == 0) Cm[i * D + c] = (Cm[i * D + c] - s) / Gm[i * DA + i];
      __syncthreads();
    }
    const bool failed = *bad != 0;
    if (failed && tid == 0) flag_error(a.ctrl, DEV_NUMERIC, bh);
    float* w = a.w + (size_t)bh * DA * D;
    for (int e = tid; e < DA * D; e += nt) w[e] = failed ? 0.f : Cm[e];
    return;
  }
  // ---- residual subspace: the r leading eigenvectors of S = R^T R (the
  // leading right singular vectors of R) into U [D][D] (first r columns)
  const int r = a.r;
  if (r <= 0 || r >= D) return;   // P = 0 or P = I: the fold needs no U
  float* U = a.pu + (size_t)bh * D * D;
  constexpr int DP = D + 1;
  const int q = r + SUB_EXTRA;
  if (((q + 7) & ~7) > SUB_MAXQ || q >= D) {
    // Jacobi on the whole D x D matrix
    float* S = psm;               // [D][DP]
    float* V = S + D * DP;        // [D][DP]
    float* rc = V + D * DP;       // [D / 2]
    float* rs = rc + D / 2;       // [D / 2]
    int* pq = reinterpret_cast<int*>(rs + D / 2);   // [D]
    int* rank = pq + D;                              // [D]
    int* flag = rank + D;
    for (int e = tid; e < D * D; e += nt) S[(e / D) * DP + e % D] = gram_at<D>(gph, slabs, DA + e / D, DA + e % D);
    __syncthreads();
    jacobi_cta(S, V, D, DP, rc, rs, pq, flag);
    top_vectors(S, V, D, DP, r, U, D, rank);
    return;
  }
  // block subspace iteration with a Rayleigh-Ritz step: X (D x q, orthonormal
  // columns) <- orth(S X), SUB_ITERS times from a fixed +-1 start; then the
  // q x q matrix T = X^T S X is diagonalised by Jacobi and the r leading Ritz
  // vectors X W are the basis.  The subspace error decays like
  // (lambda_{q+1} / lambda_r)^SUB_ITERS.  q = r + SUB_EXTRA rounded up to a
  // multiple of 8, so that the products run on 4 x 4 register tiles of
  // float4 rows (S is symmetric: row j of S is column j).
  constexpr int QM = SUB_MAXQ, QP = SUB_MAXQ + 1, DS = D + 4;
  const int qn = (q + 7) & ~7;   // q > SUB_MAXQ was sent to Jacobi above; qn <= SUB_MAXQ
  float* S = psm;                 // [D][DS]
  float* X = S + D * DS;          // [D][QM]
  float* Y = X + D * QM;          // [D][QM]
  float* T = Y + D * QM;          // [QM][QP]: Gram of Y, L^-1, Rayleigh quotient
  float* W = T + QM * QP;         // [QM][QP]: Cholesky factor, Jacobi vectors
  float* rc = W + QM * QP;        // [QM / 2]
  float* rs = rc + QM / 2;        // [QM / 2]
  int* pq = reinterpret_cast<int*>(rs + QM / 2);  // [QM]
  int* rank = pq + QM;                             // [QM]
  int* flag = rank + QM;
  for (int e = tid; e < D * D; e += nt) S[(e / D) * DS + e % D] = gram_at<D>(gph, slabs, DA + e / D, DA + e % D);
  for (int e = tid; e < D * qn; e += nt) {
    const int i = e / qn, c = e % qn;
    // a fixed +-1 pattern from a multiplicative hash of (i, c): full column
    // rank (an xor of per-row and per-column bits would give rank 1)
    unsigned h = (unsigned)i * 0x9E3779B1u + (unsigned)c * 0x85EBCA77u;
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 12;
    X[i * QM + c] = (h >> 31) ? 1.f : -1.f;
  }
  __syncthreads();
  const int qb = qn / 4;          // 4-column blocks
  // C (D x qn) = A (D x D, rows of stride lda, symmetric) x Bm (D x qn)
  auto mul_tiles = [&](const float* A, int lda, const float* Bm, float* C) {
    for (int t = tid; t < (D / 4) * qb; t += nt) {
      const int ib = t / qb, cb = t % qb;
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
      for (int j = 0; j < D; ++j) {
        const float4 a4 = *reinterpret_cast<const float4*>(A + j * lda + 4 * ib);   // A[4ib..][j]
        const float4 b4 = *reinterpret_cast<const float4*>(Bm + j * QM + 4 * cb);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(C + (4 * ib + u) * QM + 4 * cb) =
            make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
  };
  // T (qn x qn) = A^T Bm for A, Bm (D x qn)
  auto gram_tiles = [&](const float* A, const float* Bm) {
    for (int t = tid; t < qb * qb; t += nt) {
      const int ib = t / qb, cb = t % qb;
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
      for (int k = 0; k < D; ++k) {
        const float4 a4 = *reinterpret_cast<const float4*>(A + k * QM + 4 * ib);
        const float4 b4 = *reinterpret_cast<const float4*>(Bm + k * QM + 4 * cb);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) T[(4 * ib + u) * QP + 4 * cb + v] = acc[u][v];
    }
    __syncthreads();
  };
  // X <- Y L^-T with Y^T Y = L L^T (Cholesky QR); a column that has become
  // dependent (tiny pivot) is set to zero
  auto orth = [&]() {
    gram_tiles(Y, Y);
    if (tid < 32) {   // one warp: Cholesky into W (lower), then L^-1 into T (lower)
      float scale = 0.f;
      for (int k = tid; k < qn; k += 32) scale = fmaxf(scale, T[k * QP + k]);
      scale = warp_max_f(scale);
      for (int e = tid; e < qn * qn; e += 32) W[(e / qn) * QP + e % qn] = T[(e / qn) * QP + e % qn];
      __syncwarp();
      for (int k = 0; k < qn; ++k) {
        const float dkk = W[k * QP + k];
        const bool dead = !(dkk > 1e-12f * fmaxf(scale, 1e-30f));
        const float lkk = dead ? 0.f : sqrtf(dkk);
        __syncwarp();
        for (int i = k + 1 + tid; i < qn; i += 32) W[i * QP + k] = dead ? 0.f : W[i * QP + k] / lkk;
        if (tid == 0) W[k * QP + k] = lkk;
        __syncwarp();
        for (int e = tid; e < (qn - k - 1) * (qn - k - 1); e += 32) {
          const int i = k + 1 + e / (qn - k - 1), j = k + 1 + e % (qn - k - 1);
          if (j <= i) W[i * QP + j] = fmaf(-W[i * QP + k], W[j * QP + k], W[i * QP + j]);
        }
        __syncwarp();
      }
      // L^-1, one column per lane (columns of a dead pivot stay zero)
      for (int c = tid; c < qn; c += 32) {
        for (int i = 0; i < qn; ++i) {
          float v = 0.f;
          if (i >= c) {
            float sum = (i == c) ? 1.f : 0.f;
            for (int k = c; k < i; ++k) sum = fmaf(-W[i * QP + k], T[k * QP + c], sum);
            v = W[i * QP + i] > 0.f ? sum / W[i * QP + i] : 0.f;
          }
          T[i * QP + c] = v;   // rows of column c are written in order, reads are rows < i
        }
      }
    }
    __syncthreads();
    // X = Y (L^-1)^T: X[i][c] = sum_k Y[i][k] Linv[c][k]
    for (int t = tid; t < (D / 4) * qb; t += nt) {
      const int ib = t / qb, cb = t % qb;
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
      for (int k = 0; k < qn; ++k) {
        float av[4], bv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) av[u] = Y[(4 * ib + u) * QM + k];
#pragma unroll
        for (int v = 0; v < 4; ++v) bv[v] = T[(4 * cb + v) * QP + k];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(X + (4 * ib + u) * QM + 4 * cb) =
            make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
  };
  for (int it = 0; it < SUB_ITERS; ++it) {
    mul_tiles(S, DS, X, Y);
    orth();
  }
  mul_tiles(S, DS, X, Y);   // Y = S X; T = X^T Y
  gram_tiles(X, Y);
  // symmetrise (the pairing of Jacobi needs an even size; qn is a multiple of 8)
  for (int e = tid; e < qn * qn; e += nt) {
    const int i = e / qn, j = e % qn;
    if (i < j) {
      const float v = 0.5f * (T[i * QP + j] + T[j * QP + i]);
      T[i * QP + j] = v;
      T[j * QP + i] = v;
    }
  }
  __syncthreads();
  jacobi_cta(T, W, qn, QP, rc, rs, pq, flag);
  __syncthreads();
  // rank the Ritz values; U[:, k] = X W[:, col of rank k], k < r
  for (int i = tid; i < qn; i += nt) {
    const float li = T[i * QP + i];
    int k = 0;
    for (int j = 0; j < qn; ++j) {
      const float lj = T[j * QP + j];
      k += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    rank[i] = k;
  }
  __syncthreads();
  for (int e = tid; e < D * qn; e += nt) {
    const int row = e / qn, col = e % qn;
    if (rank[col] < r) {
      float sacc = 0.f;
      for (int k = 0; k < qn; ++k) sacc = fmaf(X[row * QM + k], W[k * QP + col], sacc);
      U[row * D + rank[col]] = sacc;
    }
  }
}

// B P and b P with P = U U^T (U: the first r columns), or P = 0 / I for
// r = 0 / r >= D; one CTA per head.  B P goes out transposed in bf16 (row n
// holds column n: the K-major operand of the tensor-core apply; the
// correction is about a thousandth of the output, so bf16 rounding of it is
// far below the output's own rounding), b P in fp32.
template <int D>
size_t fold_smem_bytes(int r) {
  const int rr = (r > 0 && r < D) ? r : 0;
  return ((size_t)(D + 1) * D + (size_t)D * rr + (size_t)(D + 1) * rr) * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(PB_THREADS) probe_fold_kernel(const ProbeArgs a) {
  extern __shared__ __align__(16) float psm[];
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int r = a.r;
  float* Ws = psm;                  // [D + 1][D]: row 0 = b, rows 1.. = B
  const float* wfit = a.w + (size_t)bh * (D + 1) * D;
  __nv_bfloat16* wt = a.wt + (size_t)bh * D * D;
  float* cp = a.cp + (size_t)bh * D;
  for (int e = tid; e < (D + 1) * D; e += PB_THREADS) Ws[e] = wfit[e];
  __syncthreads();
  if (r <= 0 || r >= D) {
    const bool full = r >= D;
    for (int e = tid; e < D * D; e += PB_THREADS) {
      const int n = e / D, k = e % D;   // W^T[n][k] = B[k][n]
      wt[e] = __float2bfloat16_rn(full ? Ws[(k + 1) * D + n] : 0.f);
    }
    for (int c = tid; c < D; c += PB_THREADS) cp[c] = full ? Ws[c] : 0.f;
    return;
  }
  float* Us = Ws + (D + 1) * D;     // [D][r]
  float* BU = Us + D * r;           // [D + 1][r]: row 0 = b U, rows 1.. = B U
  const float* U = a.pu + (size_t)bh * D * D;
  for (int e = tid; e < D * r; e += PB_THREADS) Us[e] = U[(e / r) * D + e % r];
  __syncthreads();
  for (int e = tid; e < (D + 1) * r; e += PB_THREADS) {
    const int i = e / r, k = e % r;
    float s = 0.f;
    for (int j = 0; j < D; ++j) s = fmaf(Ws[i * D + j], Us[j * r + k], s);
    BU[e] = s;
  }
  __syncthreads();
  for (int e = tid; e < (D + 1) * D; e += PB_THREADS) {
    const int i = e / D, j = e % D;   // (B P)[i - 1][j], or (b P)[j] for i = 0
    float s = 0.f;
    for (int k = 0; k < r; ++k) s = fmaf(BU[i * r + k], Us[j * r + k], s);
    if (i == 0) cp[j] = s; else wt[(size_t)j * D + (i - 1)] = __float2bfloat16_rn(s);
  }
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
                           float* gp, cudaStream_t s) {
  cudaError_t e;
  if ((e = ensure_dyn_smem((const void*)probe_solve_kernel<D>, solve_smem_bytes<D>())) != cudaSuccess) return e;
  if ((e = ensure_dyn_smem((const void*)probe_fold_kernel<D>, fold_smem_bytes<D>(D - 1))) != cudaSuccess) return e;
  const int gather_blocks = (m_alloc * (D / 8) + PB_THREADS - 1) / PB_THREADS;
  probe_gather_kernel<D><<<dim3(gather_blocks, a.BH), PB_THREADS, 0, s>>>(a, m_alloc, qg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_dense_rows_tc(p, qg, m_alloc, a.M, a.k, a.v, a.od, a.ctrl, s)) != cudaSuccess) return e;
  const int slabs = gram_slabs(a.M);
  probe_gram_kernel<D><<<dim3(slabs, a.BH), GR_THREADS, 0, s>>>(a, gp, slabs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  probe_solve_kernel<D><<<dim3(a.BH, 2), SV_THREADS, solve_smem_bytes<D>(), s>>>(a, gp, slabs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  probe_fold_kernel<D><<<a.BH, PB_THREADS, fold_smem_bytes<D>(a.r), s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_probe_apply_tc(p, a.o, a.wt, a.cp, a.ctrl, s)) != cudaSuccess) return e;
  probe_set_kernel<D><<<dim3(a.M, a.BH), D, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

// Probe queries are gathered into whole 128-row tiles.
inline int probe_rows_alloc(int M) { return (M + 127) / 128 * 128; }

// Padded width of a head's Gram matrix of [1, x, R] (a multiple of 4).
inline size_t gram_width(int d) { return (size_t)(1 + 2 * d + 3) / 4 * 4; }

size_t probe_scratch_bytes(const Problem& p, int M) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t BH = (size_t)p.BH, d = (size_t)p.d, zw = gram_width(p.d);
  return up(BH * M * d * 4) + up(BH * (d + 1) * d * 4) + up(BH * d * d * 4) + up(BH * d * 4) +
         up(BH * probe_rows_alloc(M) * d * 2) + up(BH * d * d * 4) +
         up(BH * (size_t)gram_slabs(M) * zw * zw * 4);
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
  a.wt = reinterpret_cast<__nv_bfloat16*>(b + off); off += up(BH * d * d * 4);
  a.cp = reinterpret_cast<float*>(b + off); off += up(BH * d * 4);
  const int m_alloc = probe_rows_alloc(M);
  __nv_bfloat16* qg = reinterpret_cast<__nv_bfloat16*>(b + off); off += up(BH * m_alloc * d * 2);
  a.pu = reinterpret_cast<float*>(b + off); off += up(BH * d * d * 4);
  float* gp = reinterpret_cast<float*>(b + off);
  a.ctrl = ctrl;
  a.N = p.N; a.M = M; a.BH = p.BH; a.r = r; a.lam = lam;
  return p.d == 128 ? launch_probe_d<128>(p, a, m_alloc, qg, gp, s)
                    : launch_probe_d<64>(p, a, m_alloc, qg, gp, s);
}

}  // namespace spattn
