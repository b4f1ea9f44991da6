// Routed block-sparse attention on Blackwell tensor cores, with the residual
// pseudo-keys folded into the same online softmax.
//
// One CTA per work item (head bh, query block i of 128 tokens), one CTA per
// SM; items are launched longest budget first (the counting sort of the
// routing step).  TMEM (512 columns) holds two S buffers, the O accumulator
// and two P buffers, so the MMA of task t+1 runs while the softmax of task t
// is computed and the tensor core is fed back to back.  Warp roles:
//
//   warps 0-7  softmax.  Warp w owns TMEM lane quarter w % 4 (query rows
//              32(w%4) .. +31) and key-column half w / 4 of every S tile.  Both
//              warps of a quarter read the whole 128-column row to form the
//              same row maximum, then each exponentiates its 64 columns and
//              writes them as packed bf16 into the P buffer.  The running max
//              moves only when it grows by more than 2^8 (then O and the
//              partial sums are rescaled).  The epilogue normalises O and
//              stores each row, scattered through perm.
//   warp 8     producer: TMA loads of the Q tile and of the K and V tiles
//              (128 tokens x d, 128-byte swizzle, no multicast) through one
//              ring of shared-memory slots, in the order the MMA consumes them.
//   warp 9     MMA issuer: S = Q K^T (both operands in shared memory) into
//              S buffer t & 1, and O += P V (P from TMEM, V from shared memory),
//              tcgen05.mma with fp32 accumulation in TMEM.
//
// Tasks of an item: its kept key blocks (CSR row; Sol-Attn: "a single
// online-softmax pass" over the selected blocks), then, in residual mode,
// every 128-row tile of the bf16 block centroids Kbar/Vbar that holds a
// dropped block, as pseudo-keys with logit bias ln n_j for a dropped block and
// -inf for a kept one (Sol-Attn: reuse the proxy scores of unselected
// blocks).  Tokens past n_j of a partial last block are masked; TMA
// zero-fills rows past N.
//
// Every mbarrier wait is bounded (tc::mbar_wait): on a timeout the CTA
// records DEV_TIMEOUT, every role leaves its loop, in-flight copies and MMAs
// are drained with a further bounded wait, and TMEM is freed before exit.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace spattn {
namespace {

// One pair of exponentials in every SPATTN_EXP_EMU pairs runs on the FMA pipe
// (tc::ex2_fma2) instead of the MUFU unit; 0 keeps every exponential on MUFU.
#ifndef SPATTN_EXP_EMU
#define SPATTN_EXP_EMU 0
#endif

constexpr int NUM_SOFTMAX_WARPS = 8;
constexpr int WARP_PRODUCER = 8, WARP_MMA = 9;
constexpr int TC_THREADS = 32 * 10;
constexpr int TILE_ROWS = 128;
constexpr uint32_t TMEM_COLS = 512;
// TMEM column map: S buffers [0,128) and [128,256), O [256, 256+d),
// P buffers [384, 448) and [448, 512) (bf16 packed two per column).
constexpr uint32_t COL_O = 256, COL_P = 384;
constexpr int MAX_STAGES = 10;

template <int D>
struct TcCfg {
  static constexpr int TILE_BYTES = TILE_ROWS * D * 2;
  static constexpr int STAGES = D == 128 ? 5 : 10;   // K/V ring slots
};

// mbarrier indices
enum : int {
  B_QFULL = 0,
  B_SFULL0, B_SFULL1,      // S buffer b holds S(t) (MMA commit)
  B_SUSED0, B_SUSED1,      // S buffer b has been read by all softmax warps
  B_PREADY,                // P(t) written by all softmax warps (one phase per task)
  B_PVDONE,                // PV(t) complete (one phase per task)
  B_OFULL, B_DRAIN,
  B_RING,                  // full[s] at B_RING + s, empty[s] at B_RING + STAGES + s
};

struct TcArgs {
  const int32_t *row_ptr, *col_idx, *order, *perm;
  __nv_bfloat16* o;
  int32_t* ctrl;
  int N, nb, n_last, residual;
  float sl2;  // log2(e) / sqrt(d)
};

struct __align__(8) TcCtrl {
  uint64_t bar[B_RING + 2 * MAX_STAGES];
  uint32_t tmem_base;
  int abort;
  uint32_t kept[64];  // kept-block bitmap of this query block (nb <= 2048)
  uint32_t bad[64];   // tasks whose CSR block index is out of range (caller CSR)
  int tail_task;      // task index of the partial last key block, -1 if none
  float lsum[2][TILE_ROWS];  // partial row sums of the two column halves
};

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                   const __grid_constant__ CUtensorMap tmVb, const TcArgs a) {
  constexpr int TILE_BYTES = TcCfg<D>::TILE_BYTES;
  constexpr int STAGES = TcCfg<D>::STAGES;
  constexpr int NCH = D / 64;           // 64-channel (128-byte) chunks per row
  constexpr int CHUNK_BYTES = TILE_ROWS * 128;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base, sRing = base + TILE_BYTES;
  TcCtrl* cs = reinterpret_cast<TcCtrl*>(gbase + (1 + STAGES) * TILE_BYTES);
  const uint32_t bar0 = smem_u32(&cs->bar[0]);
  auto bar = [&](int k) { return bar0 + 8u * (uint32_t)k; };
  auto full = [&](int s) { return bar(B_RING + s); };
  auto empty = [&](int s) { return bar(B_RING + STAGES + s); };
  volatile int* abort = &cs->abort;

  const int item = a.order ? a.order[blockIdx.x] : blockIdx.x;
  const int bh = item / a.nb, i = item % a.nb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_lo = __ldg(a.row_ptr + item);
  const int nkept = max(0, __ldg(a.row_ptr + item + 1) - r_lo);

  if (threadIdx.x == 0) {
    tc::mbar_init(bar(B_QFULL), 1);
    tc::mbar_init(bar(B_SFULL0), 1);
    tc::mbar_init(bar(B_SFULL1), 1);
    tc::mbar_init(bar(B_SUSED0), NUM_SOFTMAX_WARPS);
    tc::mbar_init(bar(B_SUSED1), NUM_SOFTMAX_WARPS);
    tc::mbar_init(bar(B_PREADY), NUM_SOFTMAX_WARPS);
    tc::mbar_init(bar(B_PVDONE), 1);
    tc::mbar_init(bar(B_OFULL), 1);
    tc::mbar_init(bar(B_DRAIN), 1);
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full(s), 1);
      tc::mbar_init(empty(s), 1);
    }
    cs->abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tc::tmem_alloc(smem_u32(&cs->tmem_base), TMEM_COLS);
    tc::tc_fence_before();
  }
  if (warp < NUM_SOFTMAX_WARPS) {
    for (int q = threadIdx.x; q < 64; q += 32 * NUM_SOFTMAX_WARPS) {
      cs->kept[q] = 0;
      cs->bad[q] = 0;
    }
    if (threadIdx.x == 0) cs->tail_task = -1;
  }
  __syncthreads();
  if (warp < NUM_SOFTMAX_WARPS) {
    for (int t = threadIdx.x; t < nkept; t += 32 * NUM_SOFTMAX_WARPS) {
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
  // Centroid tiles that hold at least one dropped block; every role derives
  // the same task list from the shared bitmap.
  uint32_t res_tiles = 0;
  if (a.residual) {
    const int ntiles = (a.nb + TILE_ROWS - 1) / TILE_ROWS;
    for (int c = 0; c < ntiles; ++c) {
      bool any = false;
      for (int q = 0; q < TILE_ROWS / 32; ++q) {
        const int j0 = c * TILE_ROWS + q * 32;
        if (j0 >= a.nb) break;
        const int cnt = min(32, a.nb - j0);
        const uint32_t valid = cnt == 32 ? 0xffffffffu : ((1u << cnt) - 1u);
        any |= (~cs->kept[j0 >> 5] & valid) != 0u;
      }
      if (any) res_tiles |= 1u << c;
    }
  }
  const int T = nkept + __popc(res_tiles);
  // tile of the r-th residual task
  auto res_tile = [&](int r) { return (int)__fns(res_tiles, 0, r + 1); };

  if (warp == WARP_PRODUCER) {
    // ---------------------------------------------------------- producer
    // load order = consumption order: K(0), K(1), then per task t: V(t),
    // K(t+2)
    if (lane == 0 && T > 0) {
      tc::mbar_expect_tx(bar(B_QFULL), TILE_BYTES);
#pragma unroll
      for (int c = 0; c < NCH; ++c)
        tc::tma_load_3d(sQ + c * CHUNK_BYTES, &tmQ, bar(B_QFULL), c * 64, i * TILE_ROWS, bh);
      int li = 0;  // loads issued
      auto issue = [&](int t, bool is_v) -> bool {
        const CUtensorMap* m;
        int row;
        if (t < nkept) {
          int j = __ldg(a.col_idx + r_lo + t);
          if (j < 0 || j >= a.nb) {
            flag_error(a.ctrl, DEV_BAD_INDEX, item);
            j = 0;  // load something valid; the softmax masks the whole task
          }
          m = is_v ? &tmV : &tmK;
          row = j * TILE_ROWS;
        } else {
          m = is_v ? &tmVb : &tmKb;
          row = res_tile(t - nkept) * TILE_ROWS;
        }
        const int s = li % STAGES;
        if (!tc::mbar_wait_fast(empty(s), ((uint32_t)(li / STAGES) & 1u) ^ 1u, abort, a.ctrl, 1))
          return false;
        tc::mbar_expect_tx(full(s), TILE_BYTES);
        const uint32_t dst = sRing + s * TILE_BYTES;
#pragma unroll
        for (int c = 0; c < NCH; ++c) tc::tma_load_3d(dst + c * CHUNK_BYTES, m, full(s), c * 64, row, bh);
        ++li;
        return true;
      };
      bool ok = issue(0, false);
      if (ok && T > 1) ok = issue(1, false);
      for (int t = 0; ok && t < T; ++t) {
        ok = issue(t, true);
        if (ok && t + 2 < T) ok = issue(t + 2, false);
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        tc::mbar_drain(bar(B_QFULL), 0);
        for (int k = (li > STAGES ? li - STAGES : 0); k < li; ++k)
          tc::mbar_drain(full(k % STAGES), (uint32_t)(k / STAGES) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // --------------------------------------------------------------- MMA
    if (lane == 0 && T > 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idO = tc::idesc_bf16_f32(128, D, true);
      // loop-invariant descriptors; k-step and slot offsets are added to the
      // address field (bits 0-13, 16-byte units)
      const uint64_t dQ = tc::sdesc_sw128(sQ, 16, 1024);
      const uint64_t dK = tc::sdesc_sw128(sRing, 16, 1024);
      const uint64_t dV = tc::sdesc_sw128(sRing, CHUNK_BYTES, 1024);
      int li = 0;  // loads consumed
      auto issue_s = [&](int t) -> bool {
        const int s = li % STAGES;
        if (!tc::mbar_wait_fast(full(s), (uint32_t)(li / STAGES) & 1u, abort, a.ctrl, 4)) return false;
        tc::tc_fence_after();
        const uint64_t slot16 = (uint64_t)(s * TILE_BYTES / 16);
        const uint32_t dS = tmem + 128u * (uint32_t)(t & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32) >> 4;
          tc::umma_ss(dS, dQ + off16, dK + slot16 + off16, idS, kk > 0);
        }
        tc::umma_commit(empty(s));
        tc::umma_commit(bar(B_SFULL0 + (t & 1)));
        ++li;
        return true;
      };
      bool ok = tc::mbar_wait_fast(bar(B_QFULL), 0, abort, a.ctrl, 3);
      if (ok) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int t = 0; ok && t < T; ++t) {
        if (!(ok = tc::mbar_wait_fast(bar(B_PREADY), (uint32_t)t & 1u, abort, a.ctrl, 5))) break;
        const int s = li % STAGES;
        if (!(ok = tc::mbar_wait_fast(full(s), (uint32_t)(li / STAGES) & 1u, abort, a.ctrl, 6))) break;
        tc::tc_fence_after();
        // O += P V: M = 128 queries, N = d, K = 128 keys in steps of 16; P is
        // bf16 packed two per TMEM column, V is MN-major (d contiguous)
        const uint64_t slot16 = (uint64_t)(s * TILE_BYTES / 16);
        const uint32_t tP = tmem + COL_P + 64u * (uint32_t)(t & 1);
#pragma unroll
        for (int kk = 0; kk < TILE_ROWS / 16; ++kk)
          tc::umma_ts(tmem + COL_O, tP + kk * 8, dV + slot16 + (uint64_t)(kk * 2048 / 16), idO,
                      (t > 0 || kk > 0) ? 1u : 0u);
        tc::umma_commit(empty(s));
        tc::umma_commit(bar(B_PVDONE));
        ++li;
        if (t + 2 < T) {
          // S buffer t & 1 is free once every softmax warp has read S(t)
          if (!(ok = tc::mbar_wait_fast(bar(B_SUSED0 + (t & 1)), (uint32_t)(t >> 1) & 1u, abort,
                                        a.ctrl, 9)))
            break;
          if (!(ok = issue_s(t + 2))) break;
        }
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
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;                 // row / TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int rows_valid = (i == a.nb - 1) ? a.n_last : TILE_ROWS;
    const float lg_b = log2f((float)TILE_ROWS), lg_last = log2f((float)a.n_last);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int b = t & 1;
      if (!(ok = tc::mbar_wait_fast(bar(B_SFULL0 + b), (uint32_t)(t >> 1) & 1u, abort, a.ctrl, 7)))
        break;
      tc::tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]);
        tc::tmem_ld32(tmem + lane_off + 128u * b + 32 * c, chunk);
      }
      tc::tmem_wait_ld();
      // S(t) is in registers: the MMA may overwrite the buffer with S(t+2)
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_SUSED0 + b));
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
        const int jres = res_tile(t - nkept) * TILE_ROWS;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int j = jres + c;
          const bool dropped = j < a.nb && !((cs->kept[j >> 5] >> (j & 31)) & 1u);
          const float bias = dropped ? (j == a.nb - 1 ? lg_last : lg_b) : -INFINITY;
          s[c] = __float_as_uint(fmaf(__uint_as_float(s[c]), a.sl2, bias));
        }
        scale = 1.f;
      }
      // row max over all 128 columns (both halves compute the same value):
      // 8 independent chains of 3-input max
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = __uint_as_float(s[e]);
#pragma unroll
      for (int c = 8; c < 128; c += 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          mx[e] = tc::fmax3(mx[e], __uint_as_float(s[c + e]), __uint_as_float(s[c + e + 8]));
      }
      const float rmax = tc::fmax3(tc::fmax3(mx[0], mx[1], mx[2]), tc::fmax3(mx[3], mx[4], mx[5]),
                                   fmaxf(mx[6], mx[7])) * scale;
      // lazy rescale: a row moves its reference max only when the new max
      // exceeds it by more than 2^8
      const bool grow = rmax > m + 8.0f;
      float sc = 1.f;
      if (grow) {
        sc = tc::ex2(m - rmax);
        l *= sc;
        m = rmax;
      }
      const float nmu = (m == -INFINITY) ? 0.f : -m;
      // this warp's 64 columns: p = 2^(s * scale - m), paired arithmetic; the
      // column half is a template argument so that s[] stays in registers
      const uint64_t sc2 = tc::f2_pack(scale, scale), nmu2 = tc::f2_pack(nmu, nmu);
      uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[32];
      auto exps = [&](auto H) {
        constexpr int c0 = 64 * decltype(H)::value;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint64_t x2 = tc::f2_fma(
              tc::f2_pack(__uint_as_float(s[c0 + 2 * e]), __uint_as_float(s[c0 + 2 * e + 1])), sc2,
              nmu2);
          float p0, p1;
          if (SPATTN_EXP_EMU > 0 && (e % (SPATTN_EXP_EMU > 0 ? SPATTN_EXP_EMU : 1)) == 0) {
            tc::f2_unpack(tc::ex2_fma2(x2), p0, p1);
          } else {
            float x0, x1;
            tc::f2_unpack(x2, x0, x1);
            p0 = tc::ex2(x0);
            p1 = tc::ex2(x1);
          }
          ls2[e & 3] = tc::f2_add(ls2[e & 3], tc::f2_pack(p0, p1));
          pk[e] = pack_bf16x2(p0, p1);
        }
      };
      if (half == 0) exps(std::integral_constant<int, 0>());
      else exps(std::integral_constant<int, 1>());
      tc::tmem_st32(tmem + lane_off + COL_P + 64u * b + 32u * half, pk);
      {
        const uint64_t t2 = tc::f2_add(tc::f2_add(ls2[0], ls2[1]), tc::f2_add(ls2[2], ls2[3]));
        float lo, hi;
        tc::f2_unpack(t2, lo, hi);
        l += lo + hi;
      }
      if (t > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds PV(0..t-1) once PV(t-1) is done; this warp rescales its half
        // of the head dimension (scale 1 on rows that keep their max)
        if (!(ok = tc::mbar_wait_fast(bar(B_PVDONE), (uint32_t)(t - 1) & 1u, abort, a.ctrl, 10)))
          break;
        tc::tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t ov[32];
          const uint32_t col = tmem + lane_off + COL_O + (uint32_t)(half * (D / 2) + 32 * c);
          tc::tmem_ld32(col, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * sc);
          tc::tmem_st32(col, ov);
        }
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_PREADY));
    }
    if (ok && T > 0) ok = tc::mbar_wait(bar(B_OFULL), 0, abort, a.ctrl, 8);
    // both halves of a row combine their partial sums (named barrier per
    // lane quarter, 64 threads)
    cs->lsum[half][r] = l;
    named_sync(1 + quarter, 64);
    const float ltot = cs->lsum[0][r] + cs->lsum[1][r];
    if (ok) {
      tc::tc_fence_after();
      const int tok = i * TILE_ROWS + r;
      const bool store = r < rows_valid;
      const int dst = store ? (a.perm ? __ldg(a.perm + tok) : tok) : 0;
      uint4* orow = reinterpret_cast<uint4*>(a.o + ((size_t)bh * a.N + dst) * D + half * (D / 2));
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[32];
        if (T > 0) {  // CTA-uniform: every lane of the warp takes part in the load
          tc::tmem_ld32(tmem + lane_off + COL_O + (uint32_t)(half * (D / 2) + 32 * c), ov);
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
  if (warp == WARP_MMA) {
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
size_t tc_smem_bytes() {
  return (size_t)(1 + TcCfg<D>::STAGES) * TcCfg<D>::TILE_BYTES + sizeof(TcCtrl) + 1024;
}

template <int D>
cudaError_t launch_tc(const CUtensorMap* maps, const TcArgs& a, int items, cudaStream_t s) {
  const size_t smem = tc_smem_bytes<D>();
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
