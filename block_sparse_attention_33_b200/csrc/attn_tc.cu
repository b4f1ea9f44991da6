// Routed block-sparse attention on Blackwell tensor cores, with
// the residual pseudo-keys folded into the same online softmax.
//
// One CTA per work item (head bh, query block i of 128 tokens); items are
// launched longest budget first (the counting sort of the routing step), two
// CTAs per SM so that one CTA's softmax overlaps the other's MMAs.  Warp roles:
//
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  For every
//              task it reads the 128 fp32 logits of its row from TMEM, adds the
//              column bias, updates the running max (rescaling O in TMEM only
//              when the max grows by more than 2^8), writes P as packed bf16
//              back into the first 64 TMEM columns of S, and finally
//              normalises O and stores its row (scattered through perm).
//   warp 4     producer: TMA loads of the Q tile and, per task, the K and V
//              tiles (128 tokens x d, 128-byte swizzle, no multicast).
//   warp 5     MMA: S = Q K^T (both operands in shared memory) and
//              O += P V (P from TMEM, V from shared memory) with tcgen05.mma,
//              accumulators in TMEM (S: 128 columns, O: d columns).
//
// Tasks of an item: its kept key blocks (CSR row; Sol-Attn: "a single
// online-softmax pass" over the selected blocks), then, in residual mode,
// every 128-row tile of the bf16 block centroids Kbar/Vbar as pseudo-keys
// with logit bias ln n_j for a dropped block and -inf for a kept one
// (Sol-Attn: reuse the proxy scores of unselected blocks).  Tokens past n_j
// of a partial last block are masked; TMA zero-fills rows past N.
//
// Every mbarrier wait is bounded (tc::mbar_wait): on a timeout the CTA
// records DEV_TIMEOUT, every role leaves its loop, in-flight copies and MMAs
// are drained with a further bounded wait, and TMEM is freed before exit.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace spattn {
namespace {

// One pair of exponentials in every SPATTN_EXP_EMU pairs runs on the FMA pipe
// (tc::ex2_fma) instead of the MUFU unit; 0 keeps every exponential on MUFU.
#ifndef SPATTN_EXP_EMU
#define SPATTN_EXP_EMU 0
#endif

constexpr int TC_THREADS = 192;
constexpr int TILE_ROWS = 128;
constexpr uint32_t TMEM_COLS = 256;  // S/P: columns [0,128), O: [128, 128+d)

enum : int { B_QFULL, B_KFULL, B_VFULL, B_KEMPTY, B_VEMPTY, B_SFULL, B_PREADY, B_OFULL,
             B_DRAIN, B_COUNT };

struct TcArgs {
  const int32_t *row_ptr, *col_idx, *order, *perm;
  __nv_bfloat16* o;
  int32_t* ctrl;
  int N, nb, n_last, residual;
  float sl2;  // log2(e) / sqrt(d)
};

struct __align__(8) TcCtrl {
  uint64_t bar[B_COUNT];
  uint32_t tmem_base;
  int abort;
  uint32_t kept[64];  // kept-block bitmap of this query block (nb <= 2048)
  uint32_t bad[64];   // tasks whose CSR block index is out of range (caller CSR)
  int tail_task;      // task index of the partial last key block, -1 if none
};

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                   const __grid_constant__ CUtensorMap tmVb, const TcArgs a) {
  constexpr int TILE_BYTES = TILE_ROWS * D * 2;
  constexpr int NCH = D / 64;           // 64-channel (128-byte) chunks per row
  constexpr int CHUNK_BYTES = TILE_ROWS * 128;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base, sK = base + TILE_BYTES, sV = base + 2 * TILE_BYTES;
  TcCtrl* cs = reinterpret_cast<TcCtrl*>(gbase + 3 * TILE_BYTES);
  const uint32_t bar0 = smem_u32(&cs->bar[0]);
  auto bar = [&](int k) { return bar0 + 8u * (uint32_t)k; };
  volatile int* abort = &cs->abort;

  const int item = a.order ? a.order[blockIdx.x] : blockIdx.x;
  const int bh = item / a.nb, i = item % a.nb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_lo = __ldg(a.row_ptr + item);
  const int nkept = max(0, __ldg(a.row_ptr + item + 1) - r_lo);
  const int nres = a.residual ? (a.nb + TILE_ROWS - 1) / TILE_ROWS : 0;
  const int T = nkept + nres;

  if (threadIdx.x == 0) {
    for (int k = 0; k < B_COUNT; ++k) tc::mbar_init(bar(k), k == B_PREADY ? 128u : 1u);
    cs->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(smem_u32(&cs->tmem_base), TMEM_COLS);
    tc::tc_fence_before();
  }
  if (warp < 4) {
    for (int q = threadIdx.x; q < 64; q += 128) {
      cs->kept[q] = 0;
      cs->bad[q] = 0;
    }
    if (threadIdx.x == 0) cs->tail_task = -1;
  }
  __syncthreads();
  if (warp < 4) {
    for (int t = threadIdx.x; t < nkept; t += 128) {
      const int j = __ldg(a.col_idx + r_lo + t);
      if (j >= 0 && j < a.nb) {
        atomicOr(&cs->kept[j >> 5], 1u << (j & 31));
        if (j == a.nb - 1 && a.n_last < TILE_ROWS) cs->tail_task = t;
      } else if (t < 2048) {
        atomicOr(&cs->bad[t >> 5], 1u << (t & 31));
      }
    }
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = cs->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 4) {
    // ---------------------------------------------------------- producer
    if (lane == 0 && T > 0) {
      tc::mbar_expect_tx(bar(B_QFULL), TILE_BYTES);
#pragma unroll
      for (int c = 0; c < NCH; ++c)
        tc::tma_load_3d(sQ + c * CHUNK_BYTES, &tmQ, bar(B_QFULL), c * 64, i * TILE_ROWS, bh);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const CUtensorMap* mk;
        const CUtensorMap* mv;
        int row;
        if (t < nkept) {
          int j = __ldg(a.col_idx + r_lo + t);
          if (j < 0 || j >= a.nb) {
            flag_error(a.ctrl, DEV_BAD_INDEX, item);
            j = 0;  // load something valid; the softmax masks the whole task
          }
          mk = &tmK; mv = &tmV; row = j * TILE_ROWS;
        } else {
          mk = &tmKb; mv = &tmVb; row = (t - nkept) * TILE_ROWS;
        }
        const uint32_t par = ((uint32_t)t & 1u) ^ 1u;
        if (!tc::mbar_wait(bar(B_KEMPTY), par, abort, a.ctrl, 1)) break;
        tc::mbar_expect_tx(bar(B_KFULL), TILE_BYTES);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tc::tma_load_3d(sK + c * CHUNK_BYTES, mk, bar(B_KFULL), c * 64, row, bh);
        issued = 2 * t + 1;
        if (!tc::mbar_wait(bar(B_VEMPTY), par, abort, a.ctrl, 2)) break;
        tc::mbar_expect_tx(bar(B_VFULL), TILE_BYTES);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tc::tma_load_3d(sV + c * CHUNK_BYTES, mv, bar(B_VFULL), c * 64, row, bh);
        issued = 2 * t + 2;
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        tc::mbar_drain(bar(B_QFULL), 0);
        if (issued > 0) tc::mbar_drain(bar(B_KFULL), (uint32_t)((issued - 1) / 2) & 1u);
        if (issued > 1) tc::mbar_drain(bar(B_VFULL), (uint32_t)((issued - 2) / 2) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idO = tc::idesc_bf16_f32(128, D, true);
      bool ok = tc::mbar_wait(bar(B_QFULL), 0, abort, a.ctrl, 3);
      for (int t = 0; ok && t < T; ++t) {
        const uint32_t par = (uint32_t)t & 1u;
        if (!(ok = tc::mbar_wait(bar(B_KFULL), par, abort, a.ctrl, 4))) break;
        tc::tc_fence_after();
        // S = Q K^T: M = 128 queries, N = 128 keys, K = d in steps of 16
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
          tc::umma_ss(tS, tc::sdesc_sw128(sQ + off, 16, 1024), tc::sdesc_sw128(sK + off, 16, 1024),
                      idS, kk > 0);
        }
        tc::umma_commit(bar(B_KEMPTY));
        tc::umma_commit(bar(B_SFULL));
        if (!(ok = tc::mbar_wait(bar(B_PREADY), par, abort, a.ctrl, 5))) break;
        if (!(ok = tc::mbar_wait(bar(B_VFULL), par, abort, a.ctrl, 6))) break;
        tc::tc_fence_after();
        // O += P V: M = 128 queries, N = d, K = 128 keys in steps of 16;
        // P is bf16 packed two per TMEM column, V is MN-major (d contiguous)
#pragma unroll
        for (int kk = 0; kk < TILE_ROWS / 16; ++kk) {
          tc::umma_ts(tO, tS + kk * 8, tc::sdesc_sw128(sV + kk * 2048, CHUNK_BYTES, 1024), idO,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc::umma_commit(bar(B_VEMPTY));
      }
      if (ok) {
        tc::umma_commit(bar(B_OFULL));
      } else {
        tc::umma_commit(bar(B_DRAIN));
        tc::mbar_drain(bar(B_DRAIN), 0);
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- softmax
    const int r = threadIdx.x;                       // row / TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int rows_valid = (i == a.nb - 1) ? a.n_last : TILE_ROWS;
    const float lg_b = log2f((float)TILE_ROWS), lg_last = log2f((float)a.n_last);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!(ok = tc::mbar_wait(bar(B_SFULL), (uint32_t)t & 1u, abort, a.ctrl, 7))) break;
      tc::tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]);
        tc::tmem_ld32(tS + lane_off + 32 * c, chunk);
      }
      tc::tmem_wait_ld();
      // Key tiles: the max is taken on the raw scores (the scale is > 0) and
      // columns past n_j of the partial last block (or a whole tile with a
      // bad index) are set to -inf.  Centroid tiles: the log2-scaled logit
      // plus the bias log2 n_j (dropped) / -inf (kept) is formed up front.
      float scale = a.sl2;
      if (t < nkept) {
        const bool bad = t < 2048 && ((cs->bad[t >> 5] >> (t & 31)) & 1u);
        const int nvalid = bad ? 0 : (t == cs->tail_task ? a.n_last : TILE_ROWS);
        if (nvalid < TILE_ROWS) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nvalid) s[c] = __float_as_uint(-INFINITY);
        }
      } else {
        const int jres = (t - nkept) * TILE_ROWS;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int j = jres + c;
          const bool dropped = j < a.nb && !((cs->kept[j >> 5] >> (j & 31)) & 1u);
          const float bias = dropped ? (j == a.nb - 1 ? lg_last : lg_b) : -INFINITY;
          s[c] = __float_as_uint(fmaf(__uint_as_float(s[c]), a.sl2, bias));
        }
        scale = 1.f;
      }
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = __uint_as_float(s[e]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mx[c & 7] = fmaxf(mx[c & 7], __uint_as_float(s[c]));
#pragma unroll
      for (int e = 0; e < 4; ++e) mx[e] = fmaxf(mx[e], mx[e + 4]);
      const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale;
      // lazy rescale: a row moves its reference max only when the new max
      // exceeds it by more than 2^8; the TMEM read-modify-write of O is done
      // by the whole warp (tcgen05.ld/st are warp-collective), scale 1 for
      // rows that keep their max
      const bool grow = rmax > m + 8.0f;
      float sc = 1.f;
      if (grow) {
        sc = tc::ex2(m - rmax);
        l *= sc;
        m = rmax;
      }
      const float nmu = (m == -INFINITY) ? 0.f : -m;
      float ls[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ls[e] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        // 32 logits -> 16 packed bf16 pairs -> TMEM columns [16c, 16c+16)
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = fmaf(__uint_as_float(s[32 * c + 2 * e]), scale, nmu);
          const float x1 = fmaf(__uint_as_float(s[32 * c + 2 * e + 1]), scale, nmu);
          float p0, p1;
          if (SPATTN_EXP_EMU > 0 && (e % (SPATTN_EXP_EMU > 0 ? SPATTN_EXP_EMU : 1)) == 0) {
            p0 = tc::ex2_fma(x0);
            p1 = tc::ex2_fma(x1);
          } else {
            p0 = tc::ex2(x0);
            p1 = tc::ex2(x1);
          }
          ls[(2 * e) & 7] += p0;
          ls[(2 * e + 1) & 7] += p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        tc::tmem_st16(tS + lane_off + 16 * c, pk);
      }
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      if (t > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tc::tmem_ld32(tO + lane_off + 32 * c, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * sc);
          tc::tmem_st32(tO + lane_off + 32 * c, ov);
        }
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(bar(B_PREADY));
    }
    if (ok && T > 0) ok = tc::mbar_wait(bar(B_OFULL), 0, abort, a.ctrl, 8);
    if (ok) {
      tc::tc_fence_after();
      const int tok = i * TILE_ROWS + r;
      const bool store = r < rows_valid;
      const int dst = store ? (a.perm ? __ldg(a.perm + tok) : tok) : 0;
      uint4* orow = reinterpret_cast<uint4*>(a.o + ((size_t)bh * a.N + dst) * D);
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (T > 0) {  // CTA-uniform: every lane of the warp takes part in the load
          tc::tmem_ld32(tO + lane_off + 32 * c, ov);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0u;
        }
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
            orow[c * 4 + q] = v;
          }
        }
      }
    }
    tc::tc_fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---- host side: tensor maps ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [BH, rows, D] bf16 tensor, box = 64 channels x 128 rows x 1, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int D, int rows, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)TILE_ROWS, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc(const CUtensorMap* maps, const TcArgs& a, int items, cudaStream_t s) {
  const size_t smem = 3 * (size_t)TILE_ROWS * D * 2 + sizeof(TcCtrl) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<D><<<items, TC_THREADS, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], a);
  return cudaGetLastError();
}

}  // namespace

bool attend_tc_supported(const Problem& p) { return p.b == TILE_ROWS && (p.d == 64 || p.d == 128); }

cudaError_t launch_attend_tc(const Problem& p, const void* Q, const void* K, const void* V,
                             const int32_t* row_ptr, const int32_t* col_idx, void* O,
                             const Work& w, cudaStream_t s) {
  const void* q = w.qp ? (const void*)w.qp : Q;
  const void* k = w.kp ? (const void*)w.kp : K;
  const void* v = w.vp ? (const void*)w.vp : V;
  CUtensorMap maps[5];
  if (!make_map(&maps[0], q, p.d, p.N, p.BH) || !make_map(&maps[1], k, p.d, p.N, p.BH) ||
      !make_map(&maps[2], v, p.d, p.N, p.BH) || !make_map(&maps[3], w.kbar16, p.d, p.nb, p.BH) ||
      !make_map(&maps[4], w.vbar16, p.d, p.nb, p.BH))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.row_ptr = row_ptr; a.col_idx = col_idx;
  a.order = (row_ptr == w.row_ptr) ? w.order : nullptr;
  a.perm = p.perm;
  a.o = static_cast<__nv_bfloat16*>(O);
  a.ctrl = w.ctrl;
  a.N = p.N; a.nb = p.nb; a.n_last = p.n_last; a.residual = p.residual;
  a.sl2 = 1.4426950408889634f / sqrtf((float)p.d);
  const int items = p.BH * p.nb;
  return p.d == 128 ? launch_tc<128>(maps, a, items, s) : launch_tc<64>(maps, a, items, s);
}

}  // namespace spattn
