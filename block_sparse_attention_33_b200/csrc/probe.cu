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
//                       attention row of this library), the keys cut into
//                       ranges put together afterwards when the tiles are
//                       too few to fill the GPU;
//   probe_gram_kernel   the Gram matrix of the probe rows [1, x, R] (one CTA
//                       per pair of 64-column blocks and head, all probe rows
//                       in order): its blocks are A^T A, A^T R and R^T R for
//                       A = [1, x];
//   probe_solve_kernel  role 0, the ridge fit: G = A^T A + lam diag(0, 1,
//                       ..., 1), C = A^T R, G^-1 by Gauss-Jordan elimination
//                       in registers, W = [b; B] = G^-1 C; role 1, the r
//                       leading eigenvectors of R^T R (the leading right
//                       singular vectors of R) by block subspace iteration
//                       with a Rayleigh-Ritz step, or cyclic Jacobi on the
//                       whole matrix for large r;
//   probe_fold_kernel   B P and b P with P = U U^T (eight CTAs per head);
//   then the tcgen05 apply (launch_probe_apply_tc): O <- O + O (B P) + b P
//                       for every row, bf16 out;
//   probe_set_kernel    probe rows <- their exact output.
//
// The fit and the subspace are fp32; B P enters the tensor-core apply in
// bf16 (the correction it makes is about a thousandth of the output).  A
// probe index outside [0, N) is skipped and flagged (DEV_BAD_INDEX); normal
// equations that are not positive definite, or a fit or residual basis that
// is not finite, leave that head uncorrected and are flagged (DEV_NUMERIC).
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
// A = [1, x], G = A^T A, C = A^T R and S = R^T R are its blocks.  The 2D
// columns [x, R] are cut into blocks of 64; one CTA per (pair of blocks
// I <= J, head) runs over all probe rows, 32 at a time (the next rows'
// loads in flight while the current ones are multiplied), and writes its
// 64 x 64 block and the mirror image.  The diagonal CTAs also write their
// columns' sums (the products with the constant column) and CTA (0, 0) the
// number of valid rows.  Every entry is one thread's sum in row order: no
// partial sums, no atomics.  Layout per head: [zw][zw] floats, index 0 the
// constant column, 1 .. D the x columns, D + 1 .. 2D the R columns.

constexpr int GR_THREADS = 256;
constexpr int GR_BLK = 64;     // columns per block
constexpr int GR_CHUNK = 32;   // rows staged at a time

template <int D>
__host__ __device__ constexpr int gram_w() { return (1 + 2 * D + 3) / 4 * 4; }

template <int D>
constexpr int gram_pairs() { return (2 * D / GR_BLK) * (2 * D / GR_BLK + 1) / 2; }

// 8 consecutive columns (from col0, inside one block) of probe row m, token tok
template <int D>
__device__ __forceinline__ void z_cols(const ProbeArgs& a, int bh, int m, int tok, int col0,
                                       float* z) {
  if (tok < 0) {
#pragma unroll
    for (int c = 0; c < 8; ++c) z[c] = 0.f;
    return;
  }
  const int cx = col0 < D ? col0 : col0 - D;
  const uint4 ov = __ldg(reinterpret_cast<const uint4*>(a.o + ((size_t)bh * a.N + tok) * D + cx));
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
  float x[8];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float2 f = __bfloat1622float2(o2[c]);
    x[2 * c] = f.x;
    x[2 * c + 1] = f.y;
  }
  if (col0 < D) {
#pragma unroll
    for (int c = 0; c < 8; ++c) z[c] = x[c];
  } else {
    const float4* e = reinterpret_cast<const float4*>(a.od + ((size_t)bh * a.M + m) * D + cx);
    const float4 e0 = e[0], e1 = e[1];
    z[0] = e0.x - x[0]; z[1] = e0.y - x[1]; z[2] = e0.z - x[2]; z[3] = e0.w - x[3];
    z[4] = e1.x - x[4]; z[5] = e1.y - x[5]; z[6] = e1.z - x[6]; z[7] = e1.w - x[7];
  }
}

template <int D>
__global__ void __launch_bounds__(GR_THREADS) probe_gram_kernel(const ProbeArgs a, float* gram) {
  constexpr int NB = 2 * D / GR_BLK, ZW = gram_w<D>();
  __shared__ __align__(16) float Zi[GR_CHUNK][GR_BLK];
  __shared__ __align__(16) float Zj[GR_CHUNK][GR_BLK];
  __shared__ int cnt_s;
  int I = 0, rem = blockIdx.x, len = NB;   // pair -> (I, J), row-major over I <= J
  while (rem >= len) { rem -= len; ++I; --len; }
  const int J = I + rem;
  const bool diag = I == J;
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int sr = tid >> 3, sc = (tid & 7) * 8;   // staging: row, first of 8 columns
  const int ty = tid >> 4, tx = tid & 15;        // 4 x 4 output tile
  float acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
  float csum = 0.f;
  int cnt = 0;
  float zi[8], zj[8];
  auto load = [&](int m0) {
    const int m = m0 + sr;
    const int tok = m < a.M ? probe_token(a, bh, m) : -1;
    if (sc == 0 && tok >= 0) ++cnt;
    z_cols<D>(a, bh, m, tok, I * GR_BLK + sc, zi);
    if (!diag) z_cols<D>(a, bh, m, tok, J * GR_BLK + sc, zj);
  };
  if (tid == 0) cnt_s = 0;
  load(0);
  for (int m0 = 0; m0 < a.M; m0 += GR_CHUNK) {
    __syncthreads();   // the previous rows are no longer read
    *reinterpret_cast<float4*>(&Zi[sr][sc]) = make_float4(zi[0], zi[1], zi[2], zi[3]);
    *reinterpret_cast<float4*>(&Zi[sr][sc + 4]) = make_float4(zi[4], zi[5], zi[6], zi[7]);
    if (!diag) {
      *reinterpret_cast<float4*>(&Zj[sr][sc]) = make_float4(zj[0], zj[1], zj[2], zj[3]);
      *reinterpret_cast<float4*>(&Zj[sr][sc + 4]) = make_float4(zj[4], zj[5], zj[6], zj[7]);
    }
    __syncthreads();
    if (m0 + GR_CHUNK < a.M) load(m0 + GR_CHUNK);
    const float (*Zb)[GR_BLK] = diag ? Zi : Zj;
#pragma unroll 4
    for (int rr = 0; rr < GR_CHUNK; ++rr) {
      const float4 x = *reinterpret_cast<const float4*>(&Zi[rr][4 * ty]);
      const float4 y = *reinterpret_cast<const float4*>(&Zb[rr][4 * tx]);
      const float xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(xs[u], ys[v], acc[u][v]);
    }
    if (diag && tid < GR_BLK)
      for (int rr = 0; rr < GR_CHUNK; ++rr) csum += Zi[rr][tid];
  }
  float* out = gram + (size_t)bh * ZW * ZW;
  const int gi = 1 + I * GR_BLK + 4 * ty, gj = 1 + J * GR_BLK + 4 * tx;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) out[(size_t)(gi + u) * ZW + gj + v] = acc[u][v];
  if (!diag) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) out[(size_t)(gj + v) * ZW + gi + u] = acc[u][v];
  }
  if (diag && tid < GR_BLK) {
    const int c = 1 + I * GR_BLK + tid;
    out[c] = csum;
    out[(size_t)c * ZW] = csum;
  }
  if (I == 0 && J == 0) {
    if (cnt) atomicAdd(&cnt_s, cnt);   // integer count: any order gives the same sum
    __syncthreads();
    if (tid == 0) out[0] = (float)cnt_s;
  }
}

// ---- solve: ridge fit (role 0) and residual subspace (role 1) ---------------

constexpr int SV_THREADS = 256;   // solve kernel
constexpr int GJ_G = 16;          // Gauss-Jordan: 16 x 16 threads over the matrix
constexpr int SUB_ITERS = 12;     // subspace iterations
constexpr int SUB_EXTRA = 16;     // subspace columns beyond r

// Columns of the subspace iteration: r + SUB_EXTRA rounded up to 32 or 64;
// 0 means the whole-matrix Jacobi path (no room for the extra columns).
__host__ __device__ constexpr int sub_cols(int r, int d) {
  return (r + SUB_EXTRA <= 32 && 32 < d) ? 32 : (r + SUB_EXTRA <= 64 && 64 < d) ? 64 : 0;
}

template <int D>
struct FitGeom {
  static constexpr int N = D + 1;                    // rows of W = [b; B]
  static constexpr int NS = (N + GJ_G - 1) / GJ_G;   // register slots per thread and dimension
  static constexpr int NP = NS * GJ_G;               // padded order
  static constexpr int LDA = (N + 3) / 4 * 4;        // row stride of the inverse in shared memory
  static constexpr size_t smem =
      ((size_t)N * LDA + (size_t)N * D + 4 * (size_t)NP + 8) * sizeof(float);
};

template <int D, int QN>
constexpr size_t subspace_smem() {
  return ((size_t)D * (D + 4) + 2 * (size_t)D * QN + 2 * (size_t)QN * (QN + 1) + 4 * (size_t)QN +
          64 + 16 * (size_t)SV_THREADS) * sizeof(float);
}

template <int D>
constexpr size_t jacobi_smem() {
  return (2 * (size_t)D * (D + 1) + 4 * (size_t)D + 64) * sizeof(float);
}


__device__ __forceinline__ float block_sum(float v, float* red) {
  const int tid = threadIdx.x, nw = blockDim.x >> 5;
  v = warp_sum_f(v);
  __syncthreads();
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < nw; ++w) s += red[w];
  return s;
}

// Pair k of step t of the round-robin order on n indices (n even): (t, n - 1)
// for k = 0, else (t + k, t - k) mod n - 1; returned with p < q.
__device__ __forceinline__ void rr_pair(int t, int k, int n, int& p, int& q) {
  if (k == 0) {
    p = t; q = n - 1;
  } else {
    p = t + k;
    if (p >= n - 1) p -= n - 1;
    q = t - k + (n - 1);
    if (q >= n - 1) q -= n - 1;
  }
  if (p > q) { const int x = p; p = q; q = x; }
}

// The Jacobi rotation (c, s) that zeroes S[p][q] in J^T S J, J = [[c, s], [-s, c]]
// on columns p, q.  Fast divides: c and s are a rotation whatever t's rounding.
__device__ __forceinline__ void jacobi_rot(const float* S, int ld, int p, int q, float& c, float& s) {
  const float apq = S[p * ld + q], app = S[p * ld + p], aqq = S[q * ld + q];
  c = 1.f;
  s = 0.f;
  if (fabsf(apq) > 1e-30f) {
    const float theta = __fdividef(aqq - app, 2.f * apq);
    float tt;
    if (fabsf(theta) > 1e18f) {
      tt = __fdividef(0.5f, theta);   // theta^2 would overflow: t = 1 / (2 theta) to first order
    } else {
      const float h2 = fmaf(theta, theta, 1.f);   // sqrt(h2) = h2 rsqrt(h2), h2 < 1e37
      tt = __fdividef(copysignf(1.f, theta), fabsf(theta) + h2 * rsqrtf(h2));
    }
    c = rsqrtf(fmaf(tt, tt, 1.f));
    s = tt * c;
  }
}

// Cyclic Jacobi on the symmetric n x n matrix S (n a power of two, row
// stride ld), round-robin pairing: every step rotates n / 2 disjoint pairs,
// every pair meets once in a sweep of n - 1 steps.  A step applies all its
// rotations at once: each thread takes 2 x 2 blocks (rows of one pair,
// columns of another) of J^T S J and pairs of columns of V J.  V (row stride
// ld) starts at the identity.  Stops when the off-diagonal squares are below
// 1e-9 of the diagonal's: the off-diagonal elements are then about 3e-5 of
// the diagonal's scale, and fp32 rounding alone keeps a converged matrix
// near 1e-11, so a tighter test would never stop before the sweep limit.
__device__ void jacobi_cta(float* S, float* V, int n, int ld, float* rc, float* rs, int* pq,
                           float* red) {
  const int tid = threadIdx.x, nt = blockDim.x, h = n >> 1;
  const int lgn = 31 - __clz(n), lgh = lgn - 1;
  for (int e = tid; e < n * n; e += nt) {
    const int i = e >> lgn, j = e & (n - 1);
    V[i * ld + j] = i == j ? 1.f : 0.f;
  }
  for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS; ++sweep) {
    float off = 0.f, dia = 0.f;
    for (int e = tid; e < n * n; e += nt) {
      const int i = e >> lgn, j = e & (n - 1);
      const float x = S[i * ld + j];
      if (i == j) dia += x * x; else off += x * x;
    }
    off = block_sum(off, red);
    dia = block_sum(dia, red + 32);
    if (off <= 1e-9f * dia) break;   // the same sums in every thread: a uniform exit
    for (int t = 0; t < n - 1; ++t) {
      if (tid < h) {
        int p, q;
        float c, s;
        rr_pair(t, tid, n, p, q);
        jacobi_rot(S, ld, p, q, c, s);
        pq[2 * tid] = p; pq[2 * tid + 1] = q; rc[tid] = c; rs[tid] = s;
      }
      __syncthreads();
      for (int e = tid; e < h * h; e += nt) {   // S <- J^T S J, one 2 x 2 block
        const int k1 = e >> lgh, k2 = e & (h - 1);
        const int p1 = pq[2 * k1], q1 = pq[2 * k1 + 1], p2 = pq[2 * k2], q2 = pq[2 * k2 + 1];
        const float c1 = rc[k1], s1 = rs[k1], c2 = rc[k2], s2 = rs[k2];
        const float b00 = S[p1 * ld + p2], b01 = S[p1 * ld + q2];
        const float b10 = S[q1 * ld + p2], b11 = S[q1 * ld + q2];
        const float r00 = c2 * b00 - s2 * b01, r01 = s2 * b00 + c2 * b01;
        const float r10 = c2 * b10 - s2 * b11, r11 = s2 * b10 + c2 * b11;
        S[p1 * ld + p2] = c1 * r00 - s1 * r10;
        S[p1 * ld + q2] = c1 * r01 - s1 * r11;
        S[q1 * ld + p2] = s1 * r00 + c1 * r10;
        S[q1 * ld + q2] = s1 * r01 + c1 * r11;
      }
      for (int e = tid; e < n * h; e += nt) {   // V <- V J
        const int i = e >> lgh, k = e & (h - 1);
        const int p = pq[2 * k], q = pq[2 * k + 1];
        const float c = rc[k], s = rs[k];
        const float vp = V[i * ld + p], vq = V[i * ld + q];
        V[i * ld + p] = c * vp - s * vq;
        V[i * ld + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
  __syncthreads();
}

// The same Jacobi for n = 32 with 256 threads: thread (k1, k2) computes the
// rotations of pairs k1 and k2 itself, its 2 x 2 block of J^T S J and rows
// k1 and k1 + 16 of V J on pair k2's columns.  S alternates between S and S2
// (the step reads one and writes the other), so one barrier per step
// suffices; each V element is read and written by the same thread.  Returns
// the buffer that holds the result.
__device__ float* jacobi32(float* S, float* S2, float* V, int ld, float* red) {
  constexpr int n = 32, h = 16;
  const int tid = threadIdx.x, k1 = tid >> 4, k2 = tid & 15;
  for (int e = tid; e < n * n; e += SV_THREADS) V[(e >> 5) * ld + (e & 31)] = (e >> 5) == (e & 31) ? 1.f : 0.f;
  for (int sweep = 0; sweep < JACOBI_MAX_SWEEPS; ++sweep) {
    float off = 0.f, dia = 0.f;
    for (int e = tid; e < n * n; e += SV_THREADS) {
      const float x = S[(e >> 5) * ld + (e & 31)];
      if ((e >> 5) == (e & 31)) dia += x * x; else off += x * x;
    }
    off = block_sum(off, red);
    dia = block_sum(dia, red + 32);
    if (off <= 1e-9f * dia) break;   // the same sums in every thread: a uniform exit
    for (int t = 0; t < n - 1; ++t) {   // n - 1 is odd: a sweep ends in the other buffer
      int p1, q1, p2, q2;
      float c1, s1, c2, s2;
      rr_pair(t, k1, n, p1, q1);
      rr_pair(t, k2, n, p2, q2);
      jacobi_rot(S, ld, p1, q1, c1, s1);
      jacobi_rot(S, ld, p2, q2, c2, s2);
      const float b00 = S[p1 * ld + p2], b01 = S[p1 * ld + q2];
      const float b10 = S[q1 * ld + p2], b11 = S[q1 * ld + q2];
      const float r00 = c2 * b00 - s2 * b01, r01 = s2 * b00 + c2 * b01;
      const float r10 = c2 * b10 - s2 * b11, r11 = s2 * b10 + c2 * b11;
      S2[p1 * ld + p2] = c1 * r00 - s1 * r10;
      S2[p1 * ld + q2] = c1 * r01 - s1 * r11;
      S2[q1 * ld + p2] = s1 * r00 + c1 * r10;
      S2[q1 * ld + q2] = s1 * r01 + c1 * r11;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int i = k1 + m * h;
        const float vp = V[i * ld + p2], vq = V[i * ld + q2];
        V[i * ld + p2] = c2 * vp - s2 * vq;
        V[i * ld + q2] = s2 * vp + c2 * vq;
      }
      float* x = S; S = S2; S2 = x;
      __syncthreads();   // this step's S complete; the other buffer's readers done
    }
  }
  __syncthreads();
  return S;
}

// Rank of each of the n diagonal entries of S (descending, ties to the
// lower index) into rank[]; then U[:, rank] (row stride D, first r columns)
// = B[:, j] (rows nrow, row stride ldb) times the eigenvector columns of V.
__device__ void rank_values(const float* S, int n, int ld, int* rank) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float li = S[i * ld + i];
    int k = 0;
    for (int j = 0; j < n; ++j) {
      const float lj = S[j * ld + j];
      k += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    rank[i] = k;
  }
  __syncthreads();
}

// A residual basis that is not finite: the head's correction is left out
// (its first r columns of U zeroed, so B P = 0) and flagged.  Every thread
// of the CTA calls this after writing its share of U.
template <int D>
__device__ void basis_check(float* U, int r, int nonfinite, int32_t* ctrl, int bh) {
  if (__syncthreads_or(nonfinite)) {
    if (threadIdx.x == 0) flag_error(ctrl, DEV_NUMERIC, bh);
    for (int e = threadIdx.x; e < D * r; e += blockDim.x) U[(e / r) * D + e % r] = 0.f;
  }
}

// role 0: W = (G + lam diag(0, 1, ..., 1))^-1 C.  The inverse is taken in
// place by Gauss-Jordan elimination without pivoting (the matrix is
// symmetric positive definite), the matrix held in registers: thread
// (ty, tx) of a 16 x 16 grid owns rows ty + 16 a and columns tx + 16 b.
// Step k needs row k and column k as they stand; their owners publish them
// to shared memory before the step's barrier (two buffers, one barrier per
// step) and clear them in registers, so that every element takes the same
// update  A <- A - u v^T  with u = column k (-1 at k) and v = row k / A_kk
// (1 / A_kk at k).  Pad rows and columns are the identity and never pivot.
template <int D>
__device__ void fit_role(const ProbeArgs& a, const float* gh, int bh, float* sm) {
  using F = FitGeom<D>;
  constexpr int N = F::N, NS = F::NS, NP = F::NP, LDA = F::LDA, ZW = gram_w<D>();
  float* Ai = sm;                 // [N][LDA] the inverse
  float* Cm = Ai + N * LDA;       // [N][D]
  float* rowb = Cm + N * D;       // [2][NP]
  float* colb = rowb + 2 * NP;    // [2][NP]
  float* pivb = colb + 2 * NP;    // [2]
  int* badp = reinterpret_cast<int*>(pivb + 2);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
#pragma unroll 8
  for (int e = tid; e < N * D; e += SV_THREADS) Cm[e] = gh[(size_t)(e / D) * ZW + N + e % D];
  float A[NS][NS];
#pragma unroll
  for (int s = 0; s < NS; ++s)
#pragma unroll
    for (int b = 0; b < NS; ++b) {
      const int i = ty + GJ_G * s, j = tx + GJ_G * b;
      A[s][b] = (i < N && j < N) ? gh[(size_t)i * ZW + j] + ((i == j && i > 0) ? a.lam : 0.f)
                                 : (i == j ? 1.f : 0.f);
    }
  if (tid == 0) *badp = 0;
  for (int k = 0; k < N; ++k) {
    const int buf = k & 1, ks = k >> 4, kl = k & 15;
    // the owners publish row k and column k as step k - 1 left them, then
    // clear them (buffer k & 1 was last read in step k - 2, before the
    // barrier of step k - 1)
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      if (s != ks) continue;   // the same slot in every thread
      if (ty == kl) {
        if (tx == kl) pivb[buf] = A[s][s];
#pragma unroll
        for (int b = 0; b < NS; ++b) {
          const int j = tx + GJ_G * b;
          rowb[buf * NP + j] = j == k ? 1.f : A[s][b];
        }
      }
      if (tx == kl) {
#pragma unroll
        for (int b = 0; b < NS; ++b) {
          const int i = ty + GJ_G * b;
          colb[buf * NP + i] = i == k ? -1.f : A[b][s];
        }
      }
      if (ty == kl) {
#pragma unroll
        for (int b = 0; b < NS; ++b) A[s][b] = 0.f;
      }
      if (tx == kl) {
#pragma unroll
        for (int b = 0; b < NS; ++b) A[b][s] = 0.f;
      }
    }
    __syncthreads();
    const float pk = pivb[buf];
    if (tid == 0 && !(pk > 0.f && pk < INFINITY)) *badp = 1;
    const float piv = 1.f / pk;
    float u[NS], v[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) u[s] = colb[buf * NP + ty + GJ_G * s];
#pragma unroll
    for (int b = 0; b < NS; ++b) v[b] = rowb[buf * NP + tx + GJ_G * b] * piv;
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
      for (int b = 0; b < NS; ++b) A[s][b] = fmaf(-u[s], v[b], A[s][b]);
  }
  int nonfinite = 0;
#pragma unroll
  for (int s = 0; s < NS; ++s)
#pragma unroll
    for (int b = 0; b < NS; ++b) {
      const int i = ty + GJ_G * s, j = tx + GJ_G * b;
      if (i < N && j < LDA) Ai[i * LDA + j] = j < N ? A[s][b] : 0.f;
      nonfinite |= !isfinite(A[s][b]);
    }
  for (int e = tid; e < N * D; e += SV_THREADS) nonfinite |= !isfinite(Cm[e]);
  // a pivot that was not positive, or an inverse or right-hand side that is
  // not finite: the head is left uncorrected (W = 0) and flagged
  const bool failed = __syncthreads_or(nonfinite) || *badp != 0;
  if (failed && tid == 0) flag_error(a.ctrl, DEV_NUMERIC, bh);
  float* w = a.w + (size_t)bh * N * D;
  // W = Ai C on 4 x 4 tiles; the inverse is symmetric, so its row j serves as
  // column j
  constexpr int TI = (N + 3) / 4, TC = D / 4;
  for (int t = tid; t < TI * TC; t += SV_THREADS) {
    const int ti = t / TC, tc = t % TC;
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
    for (int j = 0; j < N; ++j) {
      const float4 x = *reinterpret_cast<const float4*>(Ai + j * LDA + 4 * ti);
      const float4 c = *reinterpret_cast<const float4*>(Cm + j * D + 4 * tc);
      const float xs[4] = {x.x, x.y, x.z, x.w}, cs[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(xs[u], cs[v], acc[u][v]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = 4 * ti + u;
      if (i < N)
        *reinterpret_cast<float4*>(w + (size_t)i * D + 4 * tc) =
            failed ? make_float4(0.f, 0.f, 0.f, 0.f)
                   : make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
  }
}

// role 1, r + SUB_EXTRA <= QN < D: block subspace iteration with a
// Rayleigh-Ritz step.  X (D x QN, orthonormal columns) <- orth(S X),
// SUB_ITERS times from a fixed +-1 start; orth is Cholesky QR: T = Y^T Y =
// L L^T, X = Y L^-T.  Then T = X^T S X is diagonalised by Jacobi and the r
// leading Ritz vectors X W are the basis.  The subspace error decays like
// (lambda_{QN+1} / lambda_r)^SUB_ITERS.  Products on 4 x 4 register tiles of
// float4 rows (S is symmetric: row j of S is column j); the QN x QN Cholesky
// in the registers of one warp (QN / 32 rows per lane, columns of L passed
// by shuffles); the triangular solve one thread per row of Y.
template <int D, int QN>
__device__ void subspace_role(const float* gh, int r, float* U, float* sm, int32_t* ctrl, int bh) {
  constexpr int DS = D + 4, TP = QN + 1, QB = QN / 4, ZW = gram_w<D>();
  constexpr int TILES = QB * QB, SL = SV_THREADS / TILES > 1 ? SV_THREADS / TILES : 1;
  static_assert(QN % 32 == 0 && QN < D, "subspace width");
  float* S = sm;                  // [D][DS]
  float* X = S + D * DS;          // [D][QN]
  float* Y = X + D * QN;          // [D][QN]
  float* T = Y + D * QN;          // [QN][TP]: Gram of Y, then the Rayleigh quotient
  float* L = T + QN * TP;         // [QN][TP]: Cholesky factor, then Jacobi vectors
  float* rinv = L + QN * TP;      // [QN]
  float* rc = rinv + QN;          // [QN / 2]
  float* rs = rc + QN / 2;        // [QN / 2]
  int* pq = reinterpret_cast<int*>(rs + QN / 2);   // [QN]
  int* rank = pq + QN;                              // [QN]
  float* red = reinterpret_cast<float*>(rank + QN); // [64]
  float* Pp = red + 64;                             // [SL][16][TILES] partial tiles; Cholesky columns
  static_assert((D * DS + 2 * D * QN + 2 * QN * TP + QN + QN + 2 * QN + 64) % 4 == 0,
                "16-byte aligned partial buffer");
  const int tid = threadIdx.x;
#pragma unroll 8
  for (int e = tid; e < D * D; e += SV_THREADS)
    S[(e / D) * DS + e % D] = gh[(size_t)(D + 1 + e / D) * ZW + D + 1 + e % D];
  for (int e = tid; e < D * QN; e += SV_THREADS) {
    const int i = e / QN, c = e % QN;
    // a fixed +-1 pattern from a multiplicative hash of (i, c): full column
    // rank (an xor of per-row and per-column bits would give rank 1)
    unsigned h = (unsigned)i * 0x9E3779B1u + (unsigned)c * 0x85EBCA77u;
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 12;
    X[e] = (h >> 31) ? 1.f : -1.f;
  }
  __syncthreads();
  // Y = S X
  auto mul = [&]() {
    for (int t = tid; t < (D / 4) * QB; t += SV_THREADS) {
      const int ib = t / QB, cb = t % QB;
      float acc[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
#pragma unroll 4
      for (int j = 0; j < D; ++j) {
        const float4 a4 = *reinterpret_cast<const float4*>(S + j * DS + 4 * ib);
        const float4 b4 = *reinterpret_cast<const float4*>(X + j * QN + 4 * cb);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(Y + (4 * ib + u) * QN + 4 * cb) =
            make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
    }
    __syncthreads();
  };
  // T = A^T B for A, B (D x QN): 4 x 4 tiles; with fewer tiles than threads
  // the row range is split into SL slices (a warp's lanes share one slice),
  // whose partial tiles are added in slice order through shared memory
  auto gram = [&](const float* A, const float* B) {
    const int tile = tid % TILES, sl = tid / TILES;
    const int ib = tile / QB, cb = tile % QB;
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
    if (sl < SL) {
#pragma unroll 4
      for (int k = sl * (D / SL); k < (sl + 1) * (D / SL); ++k) {
        const float4 a4 = *reinterpret_cast<const float4*>(A + k * QN + 4 * ib);
        const float4 b4 = *reinterpret_cast<const float4*>(B + k * QN + 4 * cb);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
      }
    }
    if (SL == 1) {
      if (sl == 0)
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) T[(4 * ib + u) * TP + 4 * cb + v] = acc[u][v];
    } else {
      if (sl < SL)
#pragma unroll
        for (int e = 0; e < 16; ++e) Pp[(sl * 16 + e) * TILES + tile] = acc[e >> 2][e & 3];
      __syncthreads();
      if (tid < TILES) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float s = 0.f;
#pragma unroll
          for (int q = 0; q < SL; ++q) s += Pp[(q * 16 + e) * TILES + tid];
          T[(4 * ib + (e >> 2)) * TP + 4 * cb + (e & 3)] = s;
        }
      }
    }
    __syncthreads();
  };
  // X = Y L^-T with Y^T Y = L L^T; a column whose pivot is tiny against the
  // largest diagonal entry (dependent) gets L column 0 and X column 0
  auto orth = [&]() {
    gram(Y, Y);
    if (tid < 32) {
      constexpr int RPL = QN / 32;
      const int lane = tid;
      float scale = 0.f;
#pragma unroll
      for (int u = 0; u < RPL; ++u) scale = fmaxf(scale, T[(lane + 32 * u) * TP + lane + 32 * u]);
      scale = warp_max_f(scale);
      const float tiny = 1e-12f * fmaxf(scale, 1e-30f);
      float c[RPL][QN];
#pragma unroll
      for (int u = 0; u < RPL; ++u)
#pragma unroll
        for (int j = 0; j < QN; ++j) c[u][j] = T[(lane + 32 * u) * TP + j];
      if constexpr (QN == 32) {
#pragma unroll
      for (int k = 0; k < QN; ++k) {
        // column k of L goes to shared memory (two buffers: a lane that
        // writes buffer k & 1 has passed step k - 1's warp barrier, so every
        // lane has finished reading it in step k - 2) and comes back as
        // broadcast float4 reads
        float* colk = Pp + (k & 1) * QN;
        const float dkk = __shfl_sync(0xffffffffu, c[k >> 5][k], k & 31);
        const bool dead = !(dkk > tiny && dkk < INFINITY);
        const float rk = dead ? 0.f : rsqrtf(dkk);   // approximate: the next step re-orthonormalises
        const float lkk = dkk * rk;
#pragma unroll
        for (int u = 0; u < RPL; ++u) {
          const int i = lane + 32 * u;
          if (i > k) c[u][k] *= rk;
          else if (i == k) c[u][k] = lkk;
          colk[i] = c[u][k];
        }
        if (lane == 0) rinv[k] = rk;
        __syncwarp();
#pragma unroll
        for (int m = 0; m < QN / 4; ++m) {
          if (4 * m + 3 <= k) continue;   // all four columns j <= k
          const float4 l4 = *reinterpret_cast<const float4*>(colk + 4 * m);
          const float lj[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * m + e;
            if (j <= k) continue;
#pragma unroll
            for (int u = 0; u < RPL; ++u)
              if (lane + 32 * u >= j) c[u][j] = fmaf(-c[u][k], lj[e], c[u][j]);
          }
        }
      }
      } else {
#pragma unroll
      for (int k = 0; k < QN; ++k) {   // QN = 64: columns of L passed by shuffles
        const float dkk = __shfl_sync(0xffffffffu, c[k >> 5][k], k & 31);
        const bool dead = !(dkk > tiny && dkk < INFINITY);
        const float rk = dead ? 0.f : rsqrtf(dkk);
        const float lkk = dkk * rk;
#pragma unroll
        for (int u = 0; u < RPL; ++u) {
          const int i = lane + 32 * u;
          if (i > k) c[u][k] *= rk;
          else if (i == k) c[u][k] = lkk;
        }
        if (lane == 0) rinv[k] = rk;
#pragma unroll
        for (int j = 1; j < QN; ++j) {   // j > k (a constant trip count unrolls fully)
          if (j <= k) continue;
          const float ljk = __shfl_sync(0xffffffffu, c[j >> 5][k], j & 31);
#pragma unroll
          for (int u = 0; u < RPL; ++u)
            if (lane + 32 * u >= j) c[u][j] = fmaf(-c[u][k], ljk, c[u][j]);
        }
      }
      }
#pragma unroll
      for (int u = 0; u < RPL; ++u)
#pragma unroll
        for (int j = 0; j < QN; ++j) L[(lane + 32 * u) * TP + j] = j <= lane + 32 * u ? c[u][j] : 0.f;
    }
    __syncthreads();
    if (tid < D) {   // row tid of X: x L^T = y, column by column
      float y[QN];
#pragma unroll
      for (int c4 = 0; c4 < QB; ++c4) {
        const float4 v = *reinterpret_cast<const float4*>(Y + tid * QN + 4 * c4);
        y[4 * c4] = v.x; y[4 * c4 + 1] = v.y; y[4 * c4 + 2] = v.z; y[4 * c4 + 3] = v.w;
      }
#pragma unroll
      for (int k = 0; k < QN; ++k) {
        const float x = y[k] * rinv[k];
        y[k] = x;
#pragma unroll
        for (int c = 1; c < QN; ++c)
          if (c > k) y[c] = fmaf(-L[c * TP + k], x, y[c]);
      }
#pragma unroll
      for (int c4 = 0; c4 < QB; ++c4)
        *reinterpret_cast<float4*>(X + tid * QN + 4 * c4) =
            make_float4(y[4 * c4], y[4 * c4 + 1], y[4 * c4 + 2], y[4 * c4 + 3]);
    }
    __syncthreads();
  };
  for (int it = 0; it < SUB_ITERS; ++it) {
    mul();
    orth();
  }
  mul();         // Y = S X
  gram(X, Y);    // T = X^T S X
  for (int e = tid; e < QN * QN; e += SV_THREADS) {   // symmetrise
    const int i = e / QN, j = e % QN;
    if (i < j) {
      const float v = 0.5f * (T[i * TP + j] + T[j * TP + i]);
      T[i * TP + j] = v;
      T[j * TP + i] = v;
    }
  }
  __syncthreads();
  float* Td = T;   // the diagonalised Rayleigh quotient
  if constexpr (QN == 32) Td = jacobi32(T, Y, L, TP, red);   // Y is free: its second buffer
  else jacobi_cta(T, L, QN, TP, rc, rs, pq, red);
  rank_values(Td, QN, TP, rank);
  int nonfinite = 0;
  for (int e = tid; e < D * QN; e += SV_THREADS) {
    const int row = e / QN, col = e % QN;
    if (rank[col] < r) {
      float acc = 0.f;
      for (int k = 0; k < QN; ++k) acc = fmaf(X[row * QN + k], L[k * TP + col], acc);
      U[row * D + rank[col]] = acc;
      nonfinite |= !isfinite(acc);
    }
  }
  basis_check<D>(U, r, nonfinite, ctrl, bh);
}

// role 1 without room for the extra columns: Jacobi on the whole D x D matrix.
template <int D>
__device__ void eigen_role(const float* gh, int r, float* U, float* sm, int32_t* ctrl, int bh) {
  constexpr int DP = D + 1, ZW = gram_w<D>();
  float* S = sm;                  // [D][DP]
  float* V = S + D * DP;          // [D][DP]
  float* rc = V + D * DP;         // [D / 2]
  float* rs = rc + D / 2;         // [D / 2]
  int* pq = reinterpret_cast<int*>(rs + D / 2);    // [D]
  int* rank = pq + D;                               // [D]
  float* red = reinterpret_cast<float*>(rank + D);  // [64]
  const int tid = threadIdx.x;
#pragma unroll 8
  for (int e = tid; e < D * D; e += SV_THREADS)
    S[(e / D) * DP + e % D] = gh[(size_t)(D + 1 + e / D) * ZW + D + 1 + e % D];
  __syncthreads();
  jacobi_cta(S, V, D, DP, rc, rs, pq, red);
  rank_values(S, D, DP, rank);
  int nonfinite = 0;
  for (int e = tid; e < D * D; e += SV_THREADS) {
    const int row = e / D, col = e % D;
    if (rank[col] < r) {
      U[row * D + rank[col]] = V[row * DP + col];
      nonfinite |= !isfinite(V[row * DP + col]);
    }
  }
  basis_check<D>(U, r, nonfinite, ctrl, bh);
}

// One instantiation per subspace width QN = sub_cols(r, D) (0: the whole-
// matrix Jacobi), so that each gets its own register allocation.
template <int D, int QN>
__global__ void __launch_bounds__(SV_THREADS) probe_solve_kernel(const ProbeArgs a, const float* gram) {
  extern __shared__ __align__(16) float psm[];
  const int bh = blockIdx.x, role = blockIdx.y;
  const int r = a.r;
  const float* gh = gram + (size_t)bh * gram_w<D>() * gram_w<D>();
  if (r <= 0) return;   // P = 0: no correction, the fold writes zeros
  if (role == 0) {
    fit_role<D>(a, gh, bh, psm);
    return;
  }
  if (r >= D) return;   // P = I: the fold needs no U
  float* U = a.pu + (size_t)bh * D * D;
  if constexpr (QN > 0) subspace_role<D, QN>(gh, r, U, psm, a.ctrl, bh);
  else eigen_role<D>(gh, r, U, psm, a.ctrl, bh);
}

template <int D, int QN>
cudaError_t launch_solve(const ProbeArgs& a, const float* gp, cudaStream_t s) {
  constexpr size_t f = FitGeom<D>::smem;
  constexpr size_t g = QN > 0 ? subspace_smem<D, QN>() : jacobi_smem<D>();
  constexpr size_t smem = f > g ? f : g;
  cudaError_t e = ensure_dyn_smem((const void*)probe_solve_kernel<D, QN>, smem);
  if (e != cudaSuccess) return e;
  probe_solve_kernel<D, QN><<<dim3(a.BH, 2), SV_THREADS, smem, s>>>(a, gp);
  return cudaGetLastError();
}

// B P and b P with P = U U^T (U: the first r columns), or P = 0 / I for
// r = 0 / r >= D.  B P goes out transposed in bf16 (row n holds column n: the
// K-major operand of the tensor-core apply; the correction is about a
// thousandth of the output, so bf16 rounding of it is far below the output's
// own rounding), b P in fp32.  FOLD_SPLIT CTAs per head, each taking a range
// of rows of W = [b; B]: W U for its rows (one thread per (row, k)), then
// (W U) U^T with the output row across lanes.  The solve kernel has already
// zeroed W or U where the fit or the basis was not finite.
constexpr int FOLD_SPLIT = 8;

template <int D>
constexpr int fold_rows() { return (D + 1 + FOLD_SPLIT - 1) / FOLD_SPLIT; }

template <int D>
size_t fold_smem_bytes(int r) {
  const int rr = (r > 0 && r < D) ? r : 0;
  return ((size_t)fold_rows<D>() * D + (size_t)D * (rr + 1) + (size_t)fold_rows<D>() * (rr + 1)) *
         sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(PB_THREADS) probe_fold_kernel(const ProbeArgs a) {
  extern __shared__ __align__(16) float psm[];
  constexpr int RW = fold_rows<D>();
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int i0 = blockIdx.y * RW, i1 = min(D + 1, i0 + RW), nr = i1 - i0;   // rows of W
  if (nr <= 0) return;
  const int r = a.r;
  float* Ws = psm;                  // [nr][D]: rows i0 .. i1 - 1 of W (row 0 = b, rows 1.. = B)
  const float* wfit = a.w + (size_t)bh * (D + 1) * D;
  __nv_bfloat16* wt = a.wt + (size_t)bh * D * D;
  float* cp = a.cp + (size_t)bh * D;
  // output element (j, row i) of B P (i >= 1: W^T row j, column i - 1) or b P (i = 0)
  auto put = [&](int j, int i, float v) {
    if (i == 0) cp[j] = v; else wt[(size_t)j * D + (i - 1)] = __float2bfloat16_rn(v);
  };
  if (r <= 0) {
    for (int e = tid; e < D * nr; e += PB_THREADS) put(e / nr, i0 + e % nr, 0.f);
    return;
  }
  for (int e = tid; e < nr * D / 4; e += PB_THREADS)
    reinterpret_cast<float4*>(Ws)[e] = reinterpret_cast<const float4*>(wfit + (size_t)i0 * D)[e];
  __syncthreads();
  if (r >= D) {
    for (int e = tid; e < D * nr; e += PB_THREADS) {
      const int j = e / nr, q = e % nr;   // (B P)[i - 1][j] = B[i - 1][j]
      put(j, i0 + q, Ws[q * D + j]);
    }
    return;
  }
  const int rp = r + 1;
  float* Us = Ws + RW * D;          // [D][r + 1]
  float* BU = Us + D * rp;          // [nr][r + 1]
  const float* U = a.pu + (size_t)bh * D * D;
  for (int e = tid; e < D * r; e += PB_THREADS) Us[(e / r) * rp + e % r] = U[(e / r) * D + e % r];
  __syncthreads();
  // four interleaved partial sums (channels j mod 4), added in a fixed order
  for (int e = tid; e < nr * r; e += PB_THREADS) {
    const int q = e / r, k = e % r;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int j = 0; j < D; j += 4)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[c] = fmaf(Ws[q * D + j + c], Us[(j + c) * rp + k], s[c]);
    BU[q * rp + k] = (s[0] + s[1]) + (s[2] + s[3]);
  }
  __syncthreads();
  for (int e = tid; e < D * nr; e += PB_THREADS) {
    const int j = e / nr, q = e % nr;
    float s = 0.f;
    for (int k = 0; k < r; ++k) s = fmaf(BU[q * rp + k], Us[j * rp + k], s);
    put(j, i0 + q, s);
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
                           float* gp, float* part, float* lse, cudaStream_t s) {
  cudaError_t e;
  if ((e = ensure_dyn_smem((const void*)probe_fold_kernel<D>, fold_smem_bytes<D>(D - 1))) != cudaSuccess) return e;
  const int gather_blocks = (m_alloc * (D / 8) + PB_THREADS - 1) / PB_THREADS;
  probe_gather_kernel<D><<<dim3(gather_blocks, a.BH), PB_THREADS, 0, s>>>(a, m_alloc, qg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_dense_rows_tc(p, qg, m_alloc, a.M, a.k, a.v, a.od, part, lse, a.ctrl, s)) != cudaSuccess)
    return e;
  probe_gram_kernel<D><<<dim3(gram_pairs<D>(), a.BH), GR_THREADS, 0, s>>>(a, gp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int qn = sub_cols(a.r, D);
  if (qn == 32) e = launch_solve<D, 32>(a, gp, s);
  else if (qn == 64) e = launch_solve<D, (64 < D ? 64 : 0)>(a, gp, s);
  else e = launch_solve<D, 0>(a, gp, s);
  if (e != cudaSuccess) return e;
  probe_fold_kernel<D><<<dim3(a.BH, FOLD_SPLIT), PB_THREADS, fold_smem_bytes<D>(a.r), s>>>(a);
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
         up(BH * probe_rows_alloc(M) * d * 2) + up(BH * d * d * 4) + up(BH * zw * zw * 4) +
         up(DENSE_MAX_SPLITS * BH * M * d * 4) + up(DENSE_MAX_SPLITS * BH * M * 4);
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
  float* gp = reinterpret_cast<float*>(b + off); off += up(BH * gram_width(p.d) * gram_width(p.d) * 4);
  float* part = reinterpret_cast<float*>(b + off); off += up(DENSE_MAX_SPLITS * BH * M * d * 4);
  float* lse = reinterpret_cast<float*>(b + off);
  a.ctrl = ctrl;
  a.N = p.N; a.M = M; a.BH = p.BH; a.r = r; a.lam = lam;
  return p.d == 128 ? launch_probe_d<128>(p, a, m_alloc, qg, gp, part, lse, s)
                    : launch_probe_d<64>(p, a, m_alloc, qg, gp, part, lse, s);
}

}  // namespace spattn
