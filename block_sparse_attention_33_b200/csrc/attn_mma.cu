// Routed attention on the legacy warp-MMA path (mma.sync m16n8k16, bf16 -> fp32).
//
// This is the simple, portable form of the routed attention: it is kept as
// the baseline the tcgen05 kernel is measured against and as a second,
// independently written GPU path for cross-checks.
//
// Each CTA owns one work item = (head, query block i) of b query rows
// (b/16 warps, 16 rows per warp).  Per query token it runs one online
// softmax (Sol-Attn abstract: one online-softmax sweep over the selection) over
//   * the exact tokens of every kept key block (CSR row i), in 64-token
//     sub-tiles; tokens past n_j of the partial last block are masked;
//   * in residual mode, the block centroids as pseudo-keys: tile c holds
//     Kbar_j, Vbar_j for j in [64c, 64c+64) with logit bias ln n_j for a
//     dropped block and -inf for a kept one (Sol-Attn abstract: skipped
//     blocks approximated from the router's scores).
// The epilogue divides by the softmax sum and scatters rows back through the
// permutation (O[perm[n]] = Op[n]).
#include "common.cuh"
#include "internal.h"

namespace spattn {
namespace {

constexpr int KT = 64;  // key tokens per sub-tile

struct AttnArgs {
  const __nv_bfloat16 *q, *k, *v;        // blocked (permuted) inputs [BH, N, D]
  const __nv_bfloat16 *kbar, *vbar;      // bf16 centroids [BH, nb, D]
  const int32_t *row_ptr, *col_idx, *order;
  const int32_t* perm;
  __nv_bfloat16* o;                      // [BH, N, D], original token order
  int32_t* ctrl;
  int N, b, nb, n_last, residual;
  float sl2;                             // log2(e) / sqrt(d)
};

template <int D, int BQ>
__global__ void __launch_bounds__(BQ * 2, 1) attn_mma_kernel(AttnArgs a) {
  constexpr int NW = BQ / 16;
  constexpr int NT = NW * 32;
  constexpr int RB = D * 2;           // row bytes
  constexpr int CPR = RB / 16;        // 16-byte chunks per row
  constexpr int KK = D / 16;          // k-steps over the head dim
  constexpr int DN = D / 8;           // n-tiles over the head dim
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;                              // [BQ][D]
  uint8_t* sK = sQ + BQ * RB;                      // 2 x [KT][D]
  uint8_t* sV = sK + 2 * KT * RB;                  // 2 x [KT][D]
  uint32_t* kept_bits = reinterpret_cast<uint32_t*>(sV + 2 * KT * RB);  // [nb/32]

  const int item = a.order ? a.order[blockIdx.x] : blockIdx.x;
  const int bh = item / a.nb, i = item % a.nb;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t head = (size_t)bh * a.N * D;
  const int r_lo = __ldg(a.row_ptr + item), r_hi = __ldg(a.row_ptr + item + 1);
  const int nkept = r_hi - r_lo;
  const int subs = a.b / KT;  // sub-tiles per key block
  const int ntiles_res = a.residual ? (a.nb + KT - 1) / KT : 0;
  const int ntasks = nkept * subs + ntiles_res;

  const int nwords = (a.nb + 31) / 32;
  for (int q = tid; q < nwords; q += NT) kept_bits[q] = 0;
  __syncthreads();
  for (int q = r_lo + tid; q < r_hi; q += NT) {
    const int j = __ldg(a.col_idx + q);
    if (j >= 0 && j < a.nb) atomicOr(&kept_bits[j >> 5], 1u << (j & 31));
    else flag_error(a.ctrl, DEV_BAD_INDEX, item);
  }

  // ---- Q tile ----
  {
    const int rows_valid = (i == a.nb - 1) ? a.n_last : a.b;
    for (int c = tid; c < BQ * CPR; c += NT) {
      const int r = c / CPR, ch = c % CPR;
      const int rr = min(r, rows_valid - 1);
      cp_async16(smem_u32(sQ + swz(r, ch, RB)), a.q + head + (size_t)(i * a.b + rr) * D + ch * 8);
    }
    cp_async_commit();
  }

  // task t -> source rows; returns number of valid rows (0 = nothing to do)
  auto task_rows = [&](int t, const __nv_bfloat16*& kp, const __nv_bfloat16*& vp, int& row0,
                       int& nvalid, int& jres) {
    if (t < nkept * subs) {
      const int j = __ldg(a.col_idx + r_lo + t / subs), s = t % subs;
      jres = -1;
      if (j < 0 || j >= a.nb) { nvalid = 0; return; }
      const int nj = (j == a.nb - 1) ? a.n_last : a.b;
      nvalid = min(KT, nj - s * KT);
      row0 = j * a.b + s * KT;
      kp = a.k + head; vp = a.v + head;
    } else {
      const int c = t - nkept * subs;
      jres = c * KT;
      row0 = c * KT;
      nvalid = min(KT, a.nb - row0);
      kp = a.kbar + (size_t)bh * a.nb * D; vp = a.vbar + (size_t)bh * a.nb * D;
    }
  };
  auto load_task = [&](int t, int buf) {
    const __nv_bfloat16 *kp, *vp;
    int row0, nvalid, jres;
    task_rows(t, kp, vp, row0, nvalid, jres);
    if (nvalid <= 0) return;
    uint8_t* dk = sK + buf * KT * RB;
    uint8_t* dv = sV + buf * KT * RB;
    for (int c = tid; c < KT * CPR; c += NT) {
      const int r = c / CPR, ch = c % CPR;
      const int rr = row0 + min(r, nvalid - 1);
      cp_async16(smem_u32(dk + swz(r, ch, RB)), kp + (size_t)rr * D + ch * 8);
      cp_async16(smem_u32(dv + swz(r, ch, RB)), vp + (size_t)rr * D + ch * 8);
    }
  };

  if (ntasks > 0) load_task(0, 0);
  cp_async_commit();
  cp_async_wait<1>();  // Q landed
  __syncthreads();

  // Q fragments for this warp's 16 rows stay in registers
  uint32_t qf[KK][4];
#pragma unroll
  for (int kk = 0; kk < KK; ++kk) {
    const int mi = lane >> 3;
    const int r = warp * 16 + (mi & 1) * 8 + (lane & 7);
    const int ch = kk * 2 + (mi >> 1);
    ldmatrix_x4(qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], smem_u32(sQ + swz(r, ch, RB)));
  }

  float o[DN][4];
#pragma unroll
  for (int n = 0; n < DN; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int g = lane >> 2, tq = lane & 3;

  for (int t = 0; t < ntasks; ++t) {
    if (t + 1 < ntasks) load_task(t + 1, (t + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const __nv_bfloat16 *kp, *vp;
    int row0, nvalid, jres;
    task_rows(t, kp, vp, row0, nvalid, jres);
    bool skip = nvalid <= 0;
    if (!skip && jres >= 0) {
      // residual tile: skip when every centroid in it is kept
      bool any = false;
      for (int c = 0; c < nvalid; c += 32) {
        const int j = jres + c;
        const uint32_t w = kept_bits[j >> 5];
        const int cnt = min(32, nvalid - c);
        const uint32_t mask = cnt == 32 ? 0xffffffffu : ((1u << cnt) - 1u);
        if ((~w) & mask) any = true;
      }
      skip = !any;
    }
    if (!skip) {
      const uint8_t* bk = sK + (t & 1) * KT * RB;
      const uint8_t* bv = sV + (t & 1) * KT * RB;
      float s[KT / 8][4];
#pragma unroll
      for (int n = 0; n < KT / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
        for (int n = 0; n < KT / 8; n += 2) {
          const int mi = lane >> 3;
          const int r = n * 8 + (mi >> 1) * 8 + (lane & 7);
          const int ch = kk * 2 + (mi & 1);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(b0, b1, b2, b3, smem_u32(bk + swz(r, ch, RB)));
          mma_bf16_16816(s[n], qf[kk], b0, b1);
          mma_bf16_16816(s[n + 1], qf[kk], b2, b3);
        }
      }
      // scale to log2 units, add the column bias, masked columns -> -inf
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < KT / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = n * 8 + 2 * tq + (e & 1);
          float bias;
          if (jres < 0) {
            bias = col < nvalid ? 0.f : -INFINITY;
          } else {
            const int j = jres + col;
            const bool dropped = col < nvalid && !((kept_bits[j >> 5] >> (j & 31)) & 1u);
            bias = dropped ? log2f((float)((j == a.nb - 1) ? a.n_last : a.b)) : -INFINITY;
          }
          const float x = fmaf(s[n][e], a.sl2, bias);
          s[n][e] = x;
          mx[e >> 1] = fmaxf(mx[e >> 1], x);
        }
      }
      float alpha[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float m_new = fmaxf(m_r[h], mx[h]);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        alpha[h] = exp2f(m_r[h] - m_use);
        m_r[h] = m_new;
        mx[h] = m_use;
        l_r[h] *= alpha[h];
      }
#pragma unroll
      for (int n = 0; n < DN; ++n) {
        o[n][0] *= alpha[0]; o[n][1] *= alpha[0];
        o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
      }
      uint32_t pf[KT / 16][4];
#pragma unroll
      for (int n = 0; n < KT / 8; ++n) {
        const float p0 = exp2f(s[n][0] - mx[0]), p1 = exp2f(s[n][1] - mx[0]);
        const float p2 = exp2f(s[n][2] - mx[1]), p3 = exp2f(s[n][3] - mx[1]);
        l_r[0] += p0 + p1;
        l_r[1] += p2 + p3;
        pf[n >> 1][(n & 1) * 2 + 0] = pack_bf16x2(p0, p1);
        pf[n >> 1][(n & 1) * 2 + 1] = pack_bf16x2(p2, p3);
      }
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
#pragma unroll
        for (int n = 0; n < DN; n += 2) {
          const int mi = lane >> 3;
          const int r = kk * 16 + (mi & 1) * 8 + (lane & 7);
          const int ch = n + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(b0, b1, b2, b3, smem_u32(bv + swz(r, ch, RB)));
          mma_bf16_16816(o[n], pf[kk], b0, b1);
          mma_bf16_16816(o[n + 1], pf[kk], b2, b3);
        }
      }
    }
    __syncthreads();
  }

  // ---- epilogue: normalise and scatter rows back ----
  const int rows_valid = (i == a.nb - 1) ? a.n_last : a.b;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l = l_r[h];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int r = warp * 16 + g + h * 8;
    if (r < rows_valid) {
      const int tok = i * a.b + r;
      const int dst = a.perm ? __ldg(a.perm + tok) : tok;
      __nv_bfloat16* orow = a.o + head + (size_t)dst * D;
#pragma unroll
      for (int n = 0; n < DN; ++n) {
        *reinterpret_cast<uint32_t*>(orow + n * 8 + 2 * tq) =
            pack_bf16x2(o[n][2 * h] * inv, o[n][2 * h + 1] * inv);
      }
    }
  }
}

template <int D, int BQ>
cudaError_t launch_one(const AttnArgs& a, int items, cudaStream_t s) {
  const size_t smem = (size_t)BQ * D * 2 + 4 * KT * D * 2 + (2048 / 32) * 4;
  cudaError_t e = ensure_dyn_smem((const void*)attn_mma_kernel<D, BQ>, smem);
  if (e != cudaSuccess) return e;
  attn_mma_kernel<D, BQ><<<items, BQ * 2, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_mma(const Problem& p, const void* Q, const void* K, const void* V,
                              const int32_t* row_ptr, const int32_t* col_idx, void* O,
                              const Work& w, cudaStream_t s) {
  AttnArgs a;
  a.q = w.qp ? w.qp : static_cast<const __nv_bfloat16*>(Q);
  a.k = w.kp ? w.kp : static_cast<const __nv_bfloat16*>(K);
  a.v = w.vp ? w.vp : static_cast<const __nv_bfloat16*>(V);
  a.kbar = w.kbar16; a.vbar = w.vbar16;
  a.row_ptr = row_ptr; a.col_idx = col_idx;
  a.order = (row_ptr == w.row_ptr) ? w.order : nullptr;
  a.perm = p.perm;
  a.o = static_cast<__nv_bfloat16*>(O);
  a.ctrl = w.ctrl;
  a.N = p.N; a.b = p.b; a.nb = p.nb; a.n_last = p.n_last; a.residual = p.residual;
  a.sl2 = 1.4426950408889634f / sqrtf((float)p.d);
  const int items = p.BH * p.nb;
  if (p.d == 128) return p.b == 128 ? launch_one<128, 128>(a, items, s) : launch_one<128, 64>(a, items, s);
  return p.b == 128 ? launch_one<64, 128>(a, items, s) : launch_one<64, 64>(a, items, s);
}

}  // namespace spattn
