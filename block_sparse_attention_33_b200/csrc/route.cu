// Proxy logits, block softmax, Top-p selection, kept lists of every query
// block, work order, CSR.
//
// Block importance (PARK page 3.2): p_ij = softmax_j(Qbar_i . Kbar_j / sqrt(d)
// + ln n_j), the centroid estimate of the block log-mass (PARK D.2).  Blocks
// are taken in descending p until the cumulative mass reaches tau (PARK 3.2,
// Top-p), ties to the lower block index, budget clamped to [kmin, kmax]
// (Sol-Attn abstract: dynamic but controllable budgets).  The proxy map never
// leaves shared memory.  pama_kernel computes p_i instead by per-query
// attention-mass aggregation (PARK page 5.1) and shares the selection.
//
// With a threshold instead (Sol-Attn abstract: blocks are selected by comparing
// their proxy scores with a threshold; read as p_ij >= theta).  The selection
// itself (a sort-free search on the float bits of p) is in select.cuh, shared
// with the attention kernel's inline selection.
//
// route_kernel: one CTA per (ROWS query blocks, head), ROWS = 4, 8 or 16 by
// the number of blocks so that small problems still fill the GPU; 8 warps.
// The proxy tile S[ROWS][nb] is computed with fp32 FMAs, not TF32/BF16: a
// logit error of 1e-2 would move the cumulative mass by more than the 1e-4
// comparison margin.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace spattn {
namespace {

constexpr int RT_THREADS = 256;

// query blocks per routing CTA
inline int route_rows_per_cta(int nb) { return nb <= 128 ? 4 : (nb <= 512 ? 8 : 16); }

struct RouteArgs {
  const float* qbar;
  const float* kbar;
  int32_t* counts;
  int32_t* lists;
  int nb, b, n_last, kcap, kmin;
  float tau;      // Top-p mass, or the per-block threshold theta
  int threshold;  // 1: keep p_ij >= tau (Sol-Attn on-the-fly thresholding)
};

// One warp: the selection of probability row p[0..nb) (shared memory), then
// the kept blocks of query row `row` emitted in ascending j into the padded
// lists, and their count.
__device__ void select_emit(const float* p, const RouteArgs& a, int row) {
  const int lane = threadIdx.x & 31;
  const sel::Cut c = sel::cut_row(p, a.nb, a.tau, a.threshold, a.kmin, a.kcap);
  int32_t* out = a.lists + (size_t)row * a.kcap;
  int base = 0;
  sel::walk_kept(p, a.nb, c, [&](int j0, bool keep, unsigned km) {
    if (keep) out[base + __popc(km & ((1u << lane) - 1u))] = j0 + lane;
    base += __popc(km);
  });
  if (lane == 0) a.counts[row] = c.k;
}


// Proxy logits S[r][j] = Qbar_r . Kbar_j / sqrt(d) + ln n_j of a routing
// CTA's rows.  Split form: a group of TPJ threads owns key block j (all
// rows), each thread a strided share of the channels, reduced with shuffles;
// TPJ = 256 / nb (at most 32) keeps every thread busy when nb is small.
template <int D, int RT_ROWS>
__device__ __forceinline__ void proxy_split(const float* Qs, const float* kbar, float* S, int nbp,
                                            const RouteArgs& a, float inv_sqrt_d, int tpj) {
  const int sub = threadIdx.x % tpj, grp = threadIdx.x / tpj, ngrp = RT_THREADS / tpj;
  for (int j0 = 0; j0 < a.nb; j0 += ngrp) {
    const int j = j0 + grp;
    const bool live = j < a.nb;
    float acc[RT_ROWS];
#pragma unroll
    for (int r = 0; r < RT_ROWS; ++r) acc[r] = 0.f;
    if (live) {
      const float4* kr = reinterpret_cast<const float4*>(kbar + (size_t)j * D);
#pragma unroll 4
      for (int k4 = sub; k4 < D / 4; k4 += tpj) {
        const float4 kv = __ldg(kr + k4);
#pragma unroll
        for (int r = 0; r < RT_ROWS; ++r) {
          const float4 q = reinterpret_cast<const float4*>(Qs + r * D)[k4];
          acc[r] = fmaf(q.x, kv.x, acc[r]);
          acc[r] = fmaf(q.y, kv.y, acc[r]);
          acc[r] = fmaf(q.z, kv.z, acc[r]);
          acc[r] = fmaf(q.w, kv.w, acc[r]);
        }
      }
    }
    // fixed-order tree over the group's lanes (groups are aligned within a warp)
    for (int o = 1; o < tpj; o <<= 1)
#pragma unroll
      for (int r = 0; r < RT_ROWS; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
    if (live && sub == 0) {
      const int nj = (j == a.nb - 1) ? a.n_last : a.b;
      const float lnn = logf((float)nj);
#pragma unroll
      for (int r = 0; r < RT_ROWS; ++r) S[r * nbp + j] = fmaf(acc[r], inv_sqrt_d, lnn);
    }
  }
}

// Tiled form, one thread per block (nb >= 256): a thread takes JT blocks, so
// that each mean row of Q read from shared memory feeds JT dot products;
// every dot product is still one fma chain over the channels in order, the
// arithmetic of the split form with TPJ = 1.  (Spreading a warp's quarters
// over different rows instead, so that each shared-memory read serves one
// quarter, measured slower on B200: the key rows' global reads then feed
// too few FMAs each.)
template <int D, int RT_ROWS>
__device__ __forceinline__ void proxy_tiled(const float* Qs, const float* kbar, float* S, int nbp,
                                            const RouteArgs& a, float inv_sqrt_d) {
  constexpr int JT = RT_ROWS >= 16 ? 2 : 4;   // 32 accumulators a thread
  for (int j0 = 0; j0 < a.nb; j0 += JT * RT_THREADS) {
    float acc[JT][RT_ROWS];
    const float4* kr[JT];
    bool live[JT];
#pragma unroll
    for (int u = 0; u < JT; ++u) {
      const int j = j0 + u * RT_THREADS + threadIdx.x;
      live[u] = j < a.nb;
      kr[u] = reinterpret_cast<const float4*>(kbar + (size_t)(live[u] ? j : 0) * D);
#pragma unroll
      for (int r = 0; r < RT_ROWS; ++r) acc[u][r] = 0.f;
    }
#pragma unroll 2
    for (int k4 = 0; k4 < D / 4; ++k4) {
      float4 kv[JT];
#pragma unroll
      for (int u = 0; u < JT; ++u) kv[u] = live[u] ? __ldg(kr[u] + k4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < RT_ROWS; ++r) {
        const float4 q = reinterpret_cast<const float4*>(Qs + r * D)[k4];
#pragma unroll
        for (int u = 0; u < JT; ++u) {
          acc[u][r] = fmaf(q.x, kv[u].x, acc[u][r]);
          acc[u][r] = fmaf(q.y, kv[u].y, acc[u][r]);
          acc[u][r] = fmaf(q.z, kv[u].z, acc[u][r]);
          acc[u][r] = fmaf(q.w, kv[u].w, acc[u][r]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < JT; ++u) {
      const int j = j0 + u * RT_THREADS + threadIdx.x;
      if (live[u]) {
        const int nj = (j == a.nb - 1) ? a.n_last : a.b;
        const float lnn = logf((float)nj);
#pragma unroll
        for (int r = 0; r < RT_ROWS; ++r) S[r * nbp + j] = fmaf(acc[u][r], inv_sqrt_d, lnn);
      }
    }
  }
}

template <int D, int RT_ROWS>
__global__ void __launch_bounds__(RT_THREADS, RT_ROWS >= 8 ? 2 : 1) route_kernel(RouteArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int nbp = (a.nb + 31) & ~31;
  float* Qs = sm;                       // [RT_ROWS][D]
  float* S = sm + RT_ROWS * D;          // [RT_ROWS][nbp]
  const int bh = blockIdx.y, i0 = blockIdx.x * RT_ROWS;
  const int rows = min(RT_ROWS, a.nb - i0);
  const float* qbar = a.qbar + ((size_t)bh * a.nb + i0) * D;
  const float* kbar = a.kbar + (size_t)bh * a.nb * D;

  for (int e = threadIdx.x; e < RT_ROWS * D; e += RT_THREADS)
    Qs[e] = (e / D < rows) ? qbar[e] : 0.f;
  __syncthreads();

  // ---- proxy logits (nb >= 256 means at least 8 rows a CTA: only those
  // instantiations carry the tiled form) ----
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  const int tpj = sel::proxy_threads_per_block(a.nb);
  if constexpr (RT_ROWS >= 8) {
    if (tpj == 1) proxy_tiled<D, RT_ROWS>(Qs, kbar, S, nbp, a, inv_sqrt_d);
    else proxy_split<D, RT_ROWS>(Qs, kbar, S, nbp, a, inv_sqrt_d, tpj);
  } else {
    proxy_split<D, RT_ROWS>(Qs, kbar, S, nbp, a, inv_sqrt_d, tpj);
  }
  __syncthreads();

  // ---- per query block: softmax, selection, emission (one warp per row) ----
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < rows; r += RT_THREADS / 32) {
    float* p = S + r * nbp;
    sel::softmax_row(p, a.nb);
    select_emit(p, a, bh * a.nb + i0 + r);
  }
}

// PAMA block importance (PARK page 5.1): every query token of block i keeps
// its own softmax over the key blocks of the centroid logit
// q . Kbar_j / sqrt(d) + ln n_j, and p_i is the mean of the n_i tokens'
// rows; then the same Top-p selection.  One CTA per (query block, head),
// 256 threads: thread t owns tokens t % 64 and t % 64 + 64 and quarter
// t / 64 of each chunk of 32 key blocks (2 x 8 dot products, fp32 FMAs over
// the channels, each centroid value read from shared memory feeding two
// tokens).  Pass 1 runs an online (max, sum) per token over all chunks;
// pass 2 recomputes the logits, forms each token's probabilities and sums
// them over the tokens (shuffle tree inside a warp, then the two warps of a
// quarter).  Tokens are read through the permutation when there is one.
constexpr int PAMA_THREADS = 256;
constexpr int PAMA_CHUNK = 32;

template <int D>
size_t pama_smem_bytes(int nb) {
  const int nbp = (nb + 31) & ~31;
  return ((size_t)(128 + PAMA_CHUNK) * (D + 4) + nbp + 4 * 128 * 2 + 8 * 8) * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(PAMA_THREADS, 2) pama_kernel(RouteArgs a,
                                                              const __nv_bfloat16* qtok,
                                                              const int32_t* perm, int N) {
  constexpr int QS = D + 4;   // padded fp32 row stride (float4-aligned)
  extern __shared__ __align__(16) float sm[];
  const int nbp = (a.nb + 31) & ~31;
  float* Qs = sm;                          // [128][QS]
  float* Ks = Qs + 128 * QS;               // [PAMA_CHUNK][QS]
  float* p = Ks + PAMA_CHUNK * QS;         // [nbp]
  float* ml = p + nbp;                     // [4 quarters][128 tokens][m, l]
  float* part = ml + 4 * 128 * 2;          // [8 warps][8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int ni = (i == a.nb - 1) ? a.n_last : a.b;

  // tokens of query block i, fp32; rows past n_i are zero (masked below)
  const __nv_bfloat16* qh = qtok + (size_t)bh * N * D;
  for (int e = tid; e < 128 * (D / 8); e += PAMA_THREADS) {
    const int r = e / (D / 8), c8 = e % (D / 8);
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = 0.f;
    if (r < ni) {
      const int tok = i * a.b + r;
      const int src = perm ? __ldg(perm + tok) : tok;
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qh + (size_t)src * D) + c8);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h[k]);
        v[2 * k] = f.x;
        v[2 * k + 1] = f.y;
      }
    }
    float4* dst = reinterpret_cast<float4*>(Qs + r * QS + c8 * 8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }

  const float* kbar = a.kbar + (size_t)bh * a.nb * D;
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  const float lg_b = logf((float)a.b), lg_last = logf((float)a.n_last);
  const int ra = tid & 63, rb = ra + 64, qq = tid >> 6;
  const int nch = (a.nb + PAMA_CHUNK - 1) / PAMA_CHUNK;

  auto load_chunk = [&](int c) {
    __syncthreads();   // the previous chunk's readers are done
    for (int e = tid; e < PAMA_CHUNK * (D / 4); e += PAMA_THREADS) {
      const int jj = e / (D / 4), k4 = e % (D / 4);
      const int j = c * PAMA_CHUNK + jj;
      const float4 v = j < a.nb ? __ldg(reinterpret_cast<const float4*>(kbar + (size_t)j * D) + k4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(Ks + jj * QS)[k4] = v;
    }
    __syncthreads();
  };
  // logits of tokens ra, rb against blocks qq*8 .. qq*8+7 of chunk c
  auto logits = [&](int c, float (&sa)[8], float (&sb)[8]) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) sa[jj] = sb[jj] = 0.f;
    const float4* qa4 = reinterpret_cast<const float4*>(Qs + ra * QS);
    const float4* qb4 = reinterpret_cast<const float4*>(Qs + rb * QS);
#pragma unroll 2
    for (int k4 = 0; k4 < D / 4; ++k4) {
      const float4 qa = qa4[k4], qb = qb4[k4];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const float4 kv = reinterpret_cast<const float4*>(Ks + (qq * 8 + jj) * QS)[k4];
        sa[jj] = fmaf(qa.x, kv.x, sa[jj]);
        sa[jj] = fmaf(qa.y, kv.y, sa[jj]);
        sa[jj] = fmaf(qa.z, kv.z, sa[jj]);
        sa[jj] = fmaf(qa.w, kv.w, sa[jj]);
        sb[jj] = fmaf(qb.x, kv.x, sb[jj]);
        sb[jj] = fmaf(qb.y, kv.y, sb[jj]);
        sb[jj] = fmaf(qb.z, kv.z, sb[jj]);
        sb[jj] = fmaf(qb.w, kv.w, sb[jj]);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = c * PAMA_CHUNK + qq * 8 + jj;
      const float bias = j == a.nb - 1 ? lg_last : lg_b;
      sa[jj] = j < a.nb ? fmaf(sa[jj], inv_sqrt_d, bias) : -INFINITY;
      sb[jj] = j < a.nb ? fmaf(sb[jj], inv_sqrt_d, bias) : -INFINITY;
    }
  };
  auto online = [&](const float (&sv)[8], float& m, float& l) {
    float cm = sv[0];
#pragma unroll
    for (int jj = 1; jj < 8; ++jj) cm = fmaxf(cm, sv[jj]);
    const float mn = fmaxf(m, cm);
    if (mn > -INFINITY) {
      float add = 0.f;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) add += expf(sv[jj] - mn);
      l = l * expf(m - mn) + add;
      m = mn;
    }
  };

  // pass 1: per token, running max and sum over this thread's quarter of every chunk
  float ma = -INFINITY, la = 0.f, mb = -INFINITY, lb = 0.f;
  for (int c = 0; c < nch; ++c) {
    load_chunk(c);
    float sa[8], sb[8];
    logits(c, sa, sb);
    online(sa, ma, la);
    online(sb, mb, lb);
  }
  ml[(qq * 128 + ra) * 2] = ma;
  ml[(qq * 128 + ra) * 2 + 1] = la;
  ml[(qq * 128 + rb) * 2] = mb;
  ml[(qq * 128 + rb) * 2 + 1] = lb;
  __syncthreads();
  auto combine = [&](int r, float& M, float& invL) {
    M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q) M = fmaxf(M, ml[(q * 128 + r) * 2]);
    float L = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float mq = ml[(q * 128 + r) * 2];
      if (mq > -INFINITY) L += ml[(q * 128 + r) * 2 + 1] * expf(mq - M);
    }
    invL = (r < ni && L > 0.f) ? 1.f / L : 0.f;   // padding rows contribute nothing
  };
  float Ma, iLa, Mb, iLb;
  combine(ra, Ma, iLa);
  combine(rb, Mb, iLb);

  // pass 2: probabilities, summed over the block's tokens
  for (int c = 0; c < nch; ++c) {
    load_chunk(c);
    float sa[8], sb[8];
    logits(c, sa, sb);
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      float w = (sa[jj] > -INFINITY ? expf(sa[jj] - Ma) * iLa : 0.f) +
                (sb[jj] > -INFINITY ? expf(sb[jj] - Mb) * iLb : 0.f);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
      if (lane == 0) part[warp * 8 + jj] = w;
    }
    __syncthreads();
    if (tid < PAMA_CHUNK) {
      // block tid of the chunk: quarter tid / 8, summed over its two warps
      const int q = tid >> 3, jj = tid & 7;
      const float t = part[(2 * q) * 8 + jj] + part[(2 * q + 1) * 8 + jj];
      const int j = c * PAMA_CHUNK + tid;
      if (j < a.nb) p[j] = t / (float)ni;
    }
  }
  __syncthreads();
  if (warp == 0) select_emit(p, a, bh * a.nb + i);
}

template <int D>
cudaError_t launch_pama_d(const RouteArgs& a, const void* Q, const int32_t* perm, int N, int BH,
                          cudaStream_t s) {
  const size_t smem = pama_smem_bytes<D>(a.nb);
  cudaError_t e = ensure_dyn_smem((const void*)pama_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nb, BH);
  pama_kernel<D><<<grid, PAMA_THREADS, smem, s>>>(a, static_cast<const __nv_bfloat16*>(Q), perm, N);
  return cudaGetLastError();
}

// Exclusive scan of the per-row counts into row_ptr (single CTA), total in
// ctrl[CTRL_NNZ]; also the work order of the attention grid: rows grouped by
// consecutive heads (group_rows rows per group, sized so one group's K and V
// stay resident in L2 while its rows run), longest budget first inside a
// group.  The order is a counting sort on the key
// group * (kcap + 1) + (kcap - count).
constexpr int SCAN_THREADS = 1024;
constexpr size_t SCAN_SMEM_MAX = 200 * 1024;   // histogram plus staged counts

// Exclusive prefix sum over the CTA's threads (SCAN_THREADS = 32 warps):
// shuffle scans inside each warp, one warp scans the warp totals.  `part`
// holds 32 ints; the trailing barrier lets the caller reuse it at once.
__device__ __forceinline__ int block_exclusive_scan(int v, int* part) {
  static_assert(SCAN_THREADS == 1024, "one warp scans the 32 warp totals");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) part[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = part[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    part[lane] = wi - w;
  }
  __syncthreads();
  const int ex = part[warp] + x - v;
  __syncthreads();
  return ex;
}

__global__ void __launch_bounds__(SCAN_THREADS) scan_kernel(const int32_t* counts_g, int rows,
                                                            int kcap, int group_rows, int stage,
                                                            int32_t* row_ptr, int32_t* order,
                                                            int32_t* ctrl) {
  __shared__ int part[32];
  extern __shared__ int hist[];  // [ngroups * (kcap + 1)], then the counts when staged
  const int ngroups = (rows + group_rows - 1) / group_rows;
  const int nbins = ngroups * (kcap + 1);
  // every thread reads a contiguous range of counts three times: from shared
  // memory when they fit (one coalesced pass over global memory)
  const int32_t* counts = counts_g;
  if (stage) {
    int* cs = hist + nbins;
    for (int q = threadIdx.x; q < rows; q += SCAN_THREADS) cs[q] = counts_g[q];
    counts = cs;
    __syncthreads();   // (stage is the same for every thread)
  }
  auto key = [&](int q) { return (q / group_rows) * (kcap + 1) + (kcap - min(counts[q], kcap)); };
  const int per = (rows + SCAN_THREADS - 1) / SCAN_THREADS;
  const int lo = threadIdx.x * per, hi = min(rows, lo + per);
  for (int q = threadIdx.x; q < nbins; q += SCAN_THREADS) hist[q] = 0;
  int s = 0;
  for (int q = lo; q < hi; ++q) s += counts[q];
  int run = block_exclusive_scan(s, part);
  if (threadIdx.x == SCAN_THREADS - 1) {
    row_ptr[rows] = run + s;
    ctrl[CTRL_NNZ] = run + s;
  }
  for (int q = lo; q < hi; ++q) {
    row_ptr[q] = run;
    run += counts[q];
  }
  // (the scan's barriers also order the zeroing of hist before the counts)
  for (int q = lo; q < hi; ++q) atomicAdd(&hist[key(q)], 1);
  __syncthreads();
  // exclusive offsets of the bins in ascending key order
  const int bper = (nbins + SCAN_THREADS - 1) / SCAN_THREADS;
  const int blo = threadIdx.x * bper, bhi = min(nbins, blo + bper);
  int bs = 0;
  for (int q = blo; q < bhi; ++q) bs += hist[q];
  int acc = block_exclusive_scan(bs, part);
  for (int q = blo; q < bhi; ++q) {
    const int c = hist[q];
    hist[q] = acc;
    acc += c;
  }
  __syncthreads();
  for (int q = lo; q < hi; ++q) order[atomicAdd(&hist[key(q)], 1)] = q;
}

// Copy the padded per-row lists into the compact CSR (one warp per row).
__global__ void __launch_bounds__(256) compact_kernel(const int32_t* counts, const int32_t* lists,
                                                      const int32_t* row_ptr, int rows, int kcap,
                                                      int32_t* col_idx, int32_t* row_ptr_out,
                                                      int32_t* col_idx_out) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row < rows) {
    const int c = counts[row], o = row_ptr[row];
    const int32_t* src = lists + (size_t)row * kcap;
    for (int q = lane; q < c; q += 32) {
      const int32_t v = src[q];
      col_idx[o + q] = v;
      if (col_idx_out) col_idx_out[o + q] = v;
    }
    if (row_ptr_out && lane == 0) {
      row_ptr_out[row] = o;
      if (row == rows - 1) row_ptr_out[rows] = o + c;
    }
  }
}

}  // namespace

size_t route_smem_bytes(int d, int nb, int rows) {
  const int nbp = (nb + 31) & ~31;
  return (size_t)rows * (d + nbp) * sizeof(float);
}

template <int D, int ROWS>
cudaError_t launch_route_rows(const RouteArgs& a, int nb, int BH, cudaStream_t s) {
  const size_t smem = route_smem_bytes(D, nb, ROWS);
  cudaError_t e = ensure_dyn_smem((const void*)route_kernel<D, ROWS>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((nb + ROWS - 1) / ROWS, BH);
  route_kernel<D, ROWS><<<grid, RT_THREADS, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_route_d(const RouteArgs& a, int nb, int BH, cudaStream_t s) {
  switch (route_rows_per_cta(nb)) {
    case 4: return launch_route_rows<D, 4>(a, nb, BH, s);
    case 8: return launch_route_rows<D, 8>(a, nb, BH, s);
    default: return launch_route_rows<D, 16>(a, nb, BH, s);
  }
}

// Rows per work-order group: whole heads, as many as keep the group's K and V
// (bf16) within a third of the device's L2, and few enough groups that the
// scan's histogram fits its shared-memory budget.
static int scan_group_rows(const Problem& p) {
  static std::atomic<long long> l2_cache[64];
  long long l2 = 126ll << 20;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    long long c = l2_cache[dev].load(std::memory_order_relaxed);
    if (c == 0) {
      int v = 0;
      if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) == cudaSuccess && v > 0) c = v;
      else c = l2;
      l2_cache[dev].store(c, std::memory_order_relaxed);
    }
    l2 = c;
  }
  const long long head_bytes = 2ll * p.N * p.d * 2;  // K and V of one head
  int heads = (int)std::max(1ll, (l2 / 3) / std::max(1ll, head_bytes));
  heads = std::min(heads, p.BH);
  constexpr long long HIST_BUDGET = 96 * 1024;
  const long long max_groups = std::max(1ll, HIST_BUDGET / ((long long)(p.kcap + 1) * 4));
  while ((p.BH + heads - 1) / heads > max_groups) ++heads;
  return heads * p.nb;
}

cudaError_t launch_route(const Problem& p, const Work& w, const void* Q, int32_t* row_ptr_out,
                         int32_t* col_idx_out, bool need_csr, cudaStream_t s) {
  RouteArgs a;
  a.qbar = w.qbar; a.kbar = w.kbar; a.counts = w.counts; a.lists = w.lists;
  a.nb = p.nb; a.b = p.b; a.n_last = p.n_last; a.kcap = p.kcap; a.kmin = p.kmin;
  a.tau = p.tau;
  a.threshold = p.threshold;
  cudaError_t e;
  if (p.routing == ROUTING_PAMA) {
    // tokens in blocked order: the pooling's permuted copy when there is
    // one, else the queries read through the permutation
    const void* q = w.qp ? (const void*)w.qp : Q;
    const int32_t* perm = w.qp ? nullptr : p.perm;
    e = p.d == 128 ? launch_pama_d<128>(a, q, perm, p.N, p.BH, s)
                   : launch_pama_d<64>(a, q, perm, p.N, p.BH, s);
  } else {
    e = p.d == 128 ? launch_route_d<128>(a, p.nb, p.BH, s) : launch_route_d<64>(a, p.nb, p.BH, s);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int rows = p.BH * p.nb;
  const int group_rows = scan_group_rows(p);
  const size_t hist_bytes =
      (size_t)((rows + group_rows - 1) / group_rows) * (p.kcap + 1) * sizeof(int);
  const size_t staged = hist_bytes + (size_t)rows * sizeof(int);
  const int stage = staged <= SCAN_SMEM_MAX ? 1 : 0;
  const size_t smem = stage ? staged : hist_bytes;
  if ((e = ensure_dyn_smem((const void*)scan_kernel, smem)) != cudaSuccess) return e;
  scan_kernel<<<1, SCAN_THREADS, smem, s>>>(w.counts, rows, p.kcap, group_rows, stage, w.row_ptr,
                                            w.order, w.ctrl);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (!need_csr && !row_ptr_out && !col_idx_out) return cudaSuccess;
  compact_kernel<<<(rows + 7) / 8, 256, 0, s>>>(w.counts, w.lists, w.row_ptr, rows, p.kcap,
                                                w.col_idx, row_ptr_out, col_idx_out);
  return cudaGetLastError();
}

}  // namespace spattn
