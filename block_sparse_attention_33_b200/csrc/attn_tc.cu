// Routed block-sparse attention on Blackwell tensor cores, with the residual
// pseudo-keys folded into the same online softmax.
//
// Persistent: one CTA per SM loops over work items (head bh, query block i
// of 128 tokens) taken from a device ticket counter in the routing step's
// order (heads grouped so their K/V stay in L2, longest budget first); the
// last CTA to retire resets the counter.  TMEM (512 columns) holds two S
// buffers and two O accumulators, one per 64-key half of every key tile, so
// the MMA of task t+1 runs while the softmax of task t is computed.  Warp
// roles:
//
//   warps 0-7  softmax.  Warp w owns TMEM lane quarter w % 4 (query rows
//              32(w%4) .. +31) and key half h = w / 4 of every S tile, and runs
//              its own online softmax over those keys with its own reference
//              maximum m and sum l; O_h accumulates P_h V_h.  The softmax is
//              max-free: m is the row maximum of the first tile, after which
//              p = 2^(s * scale - m) is computed directly and the tile's
//              partial sum tells when m must move (sum > 2^16: m moves up by
//              the integer part of log2 of the sum, an exact power-of-two
//              rescale of l and O_h; sum > 2^60 or not finite: the tile is
//              recomputed against its own maximum).  Optionally a fixed
//              share of the exponentials runs on the FMA pipe (tc::ex2_fma2);
//              measured on B200 the MUFU-only form is faster for this
//              structure, so the share defaults to zero.  P(t) is written as
//              packed bf16 over the warp's own, already read, columns of S(t).  The epilogue merges the two
//              halves of each row, normalises and stores the row, scattered
//              through perm.
//   warp 8     producer: takes the next ticket and describes the item
//              (kept bitmap, residual tiles) in a second slot, then issues
//              TMA loads of the Q tile and of the K and V tiles (128 tokens x
//              d, 128-byte swizzle, no multicast) through one ring of
//              shared-memory slots, in the order the MMA consumes them.
//   warp 9     MMA issuer: S = Q K^T (both operands in shared memory) into
//              S buffer t & 1, and O_h += P_h V_h for both halves (P from
//              TMEM, V from shared memory), tcgen05.mma with fp32
//              accumulation in TMEM.
//
// 64-token blocks use the same 128-row tiles: an item is the pair of query
// blocks 2i and 2i + 1 (rows 0-63 and 64-127 of the Q tile), and its key
// tiles walk the union of the two kept sets in ascending order, two blocks
// per tile (two 64-row TMA boxes).  The softmax warps of lane quarters 0-1
// belong to the first query block, those of quarters 2-3 to the second, and
// each key half holds one key block, so a warp masks a whole half when its
// query block did not keep that key block; the residual bias of a warp
// likewise follows its own query block's kept set.
//
// Tasks of an item: its kept key blocks (one online-softmax sweep over the
// selected blocks, as in the Sol-Attn abstract), then, in residual mode,
// every 128-row tile of the bf16 block centroids Kbar/Vbar that holds a
// dropped block, as pseudo-keys with logit bias ln n_j for a dropped block and
// -inf for a kept one (Sol-Attn abstract: skipped blocks approximated from the router's
// scores).  Tokens past n_j of a partial last block are masked; TMA
// zero-fills rows past N.
//
// Every mbarrier wait is bounded (tc::mbar_wait): on a timeout the CTA
// records DEV_TIMEOUT, every role leaves its loop, in-flight copies and MMAs
// are drained with a further bounded wait, and TMEM is freed before exit.
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace spattn {
namespace {

// SPATTN_EXP_EMU of every 8 pairs of exponentials run on the FMA pipe
// (tc::ex2_fma2) instead of the MUFU unit (0: all on MUFU, the fastest
// setting measured for this kernel).
#ifndef SPATTN_EXP_EMU
#define SPATTN_EXP_EMU 0
#endif

constexpr int NUM_SOFTMAX_WARPS = 8;
constexpr int WARP_PRODUCER = 8, WARP_MMA = 9;
constexpr int TC_THREADS = 32 * 10;
constexpr int TILE_ROWS = 128;
constexpr uint32_t TMEM_COLS = 512;
// TMEM column map: S buffers [0,128) and [128,256); O_0 [256, 256+d) and
// O_1 [384, 384+d).  P(t) (bf16, two per column) of key half h lives in
// columns [64h, 64h+32) of S buffer t & 1.
constexpr uint32_t COL_O = 256;
constexpr int MAX_STAGES = 10;

template <int D>
struct TcCfg {
  static constexpr int TILE_BYTES = TILE_ROWS * D * 2;
  static constexpr int STAGES = D == 128 ? 5 : 10;   // K/V ring slots
};

// mbarrier indices
enum : int {
  B_QFULL = 0, B_QEMPTY,   // Q tile loaded / its last S MMA complete
  B_SFULL0, B_SFULL1,      // S buffer b holds S(g) (MMA commit)
  B_PREADY,                // P(g) written by all softmax warps (one phase per task)
  B_PVDONE,                // PV(g) complete (one phase per task)
  B_OFULL,                 // last PV of an item complete (one phase per item with tasks)
  B_DRAIN,
  B_INFO_FULL0, B_INFO_FULL1,    // item slot s described by the producer warp
  B_INFO_EMPTY0, B_INFO_EMPTY1,  // item slot s released by the MMA and softmax warps
  B_XREADY,                // + 4 * slot + quarter: both key halves of a lane quarter merged
  B_RING = B_XREADY + 8,   // full[s] at B_RING + s, empty[s] at B_RING + STAGES + s
};

struct TcArgs {
  // kept blocks of an item: the compact CSR (row_ptr, col_idx), or, with
  // counts set, the padded per-row lists of the routing step
  // (counts[item] entries at col_idx + item * kcap)
  const int32_t *row_ptr, *col_idx, *counts, *order, *perm;
  int kcap;
  __nv_bfloat16* o;           // bf16 output [BH, q_rows, D], scattered through perm
  float* o32;                 // or, when set, fp32 output [BH, q_rows, D] in tile order
  int q_rows;                 // query (and output) rows per (batch, head)
  int dense;                  // every key tile of the N keys, no residual (exact rows)
  // dense rows only: the key tiles cut into `splits` ranges, one item each
  // (item = tile item * splits + range); range c writes its normalised rows
  // to o32 + c * BH * q_rows * D and their log2 mass to lse[c][BH][q_rows]
  int splits;
  float* lse;
  int32_t* ctrl;
  int N, nb, n_last, residual, items;
  // inline selection (Sol-Attn abstract: blocks chosen inside the attention
  // pass, no stored proxy map and no routing launch): the producer scores
  // each query block against every key block from the fp32 means and cuts
  // the row itself, with the routing kernel's arithmetic
  int inline_sel;
  const float *qbar, *kbar;  // fp32 means [BH, nb, d]
  float tau;                 // Top-p mass, or the per-block threshold theta
  int threshold, kmin;
  int b64;         // 64-token blocks: a tile holds two query (key) blocks
  int nq;          // query tiles per (batch, head): nb (b = 128) or ceil(nb / 2) (b = 64)
  int blk;         // block size b
  int test_stall;  // failure-path test (see Problem::test_stall)
  float sl2;       // log2(e) / sqrt(d)
};

// One work item as described by the producer warp.  Two slots: the producer
// builds item n+1 (and starts its loads) while item n is still in the
// softmax and epilogue.
struct ItemInfo {
  int item;            // bh * nq + query tile; -1 once the work is exhausted
  int nkept;           // key-tile tasks (b = 128: the CSR row length)
  int T;               // tasks: the key tiles, then residual centroid tiles
  int tail_task;       // b = 128: task index of the partial last key block, -1 if none
  int nunion;          // b = 64: blocks kept by either query block of the tile
  uint32_t res_tiles;  // bit c: centroid tile c holds a dropped block
  uint32_t kept[2][64];  // kept-block bitmaps (nb <= 2048) of the tile's query block(s):
                         // [1] is the second query block with b = 64
  uint32_t bad[64];    // b = 128: tasks whose CSR block index is out of range (caller CSR)
  uint16_t ublk[2048]; // b = 64: the union of both kept sets, ascending; key tile t
                       // holds blocks ublk[2t] (rows 0-63) and ublk[2t + 1] (rows 64-127)
};

struct __align__(8) TcCtrl {
  uint64_t bar[B_RING + 2 * MAX_STAGES];
  uint32_t tmem_base;
  int abort;
  ItemInfo info[2];
  alignas(16) float selp[2048];  // inline selection: the proxy / probability row
  alignas(16) float selq[128];   // inline selection: the query block's mean (float4 access)
  float xm[2][2][TILE_ROWS];  // epilogue, per item slot: reference max of each key half
  float xl[2][2][TILE_ROWS];  // epilogue, per item slot: sum of each key half
};

// Inline selection of query row `row` (bh * nb + query block) into the kept
// bitmap km (one whole warp; selp and selq are shared-memory scratch): the
// centroid proxy logits against every key block, split over the lanes
// exactly as the routing kernel splits them, the block softmax and the cut.
// Kept out of line so that its registers do not add to the softmax warps'.
struct SelArgs {
  const float *qbar, *kbar;
  int nb, n_last, blk, threshold, kmin, kcap;
  float tau;
};

template <int D>
__device__ __noinline__ void select_inline(const SelArgs a, int row, uint32_t* km, float* selp,
                                           float* selq) {
  const int lane = threadIdx.x & 31;
  const float4* qrow = reinterpret_cast<const float4*>(a.qbar + (size_t)row * D);
  for (int c4 = lane; c4 < D / 4; c4 += 32) reinterpret_cast<float4*>(selq)[c4] = __ldg(qrow + c4);
  __syncwarp();
  const float* kb = a.kbar + (size_t)(row / a.nb) * a.nb * D;
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  const int tpj = sel::proxy_threads_per_block(a.nb);
  const int sub = lane % tpj, grp = lane / tpj, ngrp = 32 / tpj;
  // two key blocks per lane at a time and an unrolled channel loop, so that
  // a lane keeps many independent loads of Kbar in flight (one warp reads the
  // whole Kbar of the head); each block's sum keeps the routing kernel's order
  const float4* q4 = reinterpret_cast<const float4*>(selq);
  for (int j0 = 0; j0 < a.nb; j0 += 2 * ngrp) {
    const int ja = j0 + grp, jb = ja + ngrp;
    const bool la = ja < a.nb, lb = jb < a.nb;
    const float4* ka = reinterpret_cast<const float4*>(kb + (size_t)(la ? ja : 0) * D);
    const float4* kc = reinterpret_cast<const float4*>(kb + (size_t)(lb ? jb : 0) * D);
    float acc_a = 0.f, acc_b = 0.f;
#pragma unroll 8
    for (int k4 = sub; k4 < D / 4; k4 += tpj) {
      const float4 va = __ldg(ka + k4), vb = __ldg(kc + k4);
      const float4 q = q4[k4];
      acc_a = fmaf(q.x, va.x, acc_a);
      acc_a = fmaf(q.y, va.y, acc_a);
      acc_a = fmaf(q.z, va.z, acc_a);
      acc_a = fmaf(q.w, va.w, acc_a);
      acc_b = fmaf(q.x, vb.x, acc_b);
      acc_b = fmaf(q.y, vb.y, acc_b);
      acc_b = fmaf(q.z, vb.z, acc_b);
      acc_b = fmaf(q.w, vb.w, acc_b);
    }
    for (int o = 1; o < tpj; o <<= 1) {
      acc_a += __shfl_xor_sync(0xffffffffu, acc_a, o);
      acc_b += __shfl_xor_sync(0xffffffffu, acc_b, o);
    }
    if (sub == 0) {
      if (la) selp[ja] = fmaf(acc_a, inv_sqrt_d, logf((float)(ja == a.nb - 1 ? a.n_last : a.blk)));
      if (lb) selp[jb] = fmaf(acc_b, inv_sqrt_d, logf((float)(jb == a.nb - 1 ? a.n_last : a.blk)));
    }
  }
  __syncwarp();
  sel::softmax_row(selp, a.nb);
  const sel::Cut c = sel::cut_row(selp, a.nb, a.tau, a.threshold, a.kmin, a.kcap);
  sel::walk_kept(selp, a.nb, c, [&](int j0, bool, unsigned w) {
    if (lane == 0) km[j0 >> 5] = w;
  });
  __syncwarp();
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
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A wait made by all 32 lanes of a warp, with a warp-uniform result (one
  // lane may see the phase complete while another sees an abort first).
  auto wait_warp = [&](uint32_t b, uint32_t parity, int site) {
    return __all_sync(0xffffffffu, tc::mbar_wait_fast(b, parity, abort, a.ctrl, site));
  };

  if (threadIdx.x == 0) {
    tc::mbar_init(bar(B_QFULL), 1);
    tc::mbar_init(bar(B_QEMPTY), 1);
    tc::mbar_init(bar(B_SFULL0), 1);
    tc::mbar_init(bar(B_SFULL1), 1);
    tc::mbar_init(bar(B_PREADY), NUM_SOFTMAX_WARPS);
    tc::mbar_init(bar(B_PVDONE), 1);
    tc::mbar_init(bar(B_OFULL), 1);
    tc::mbar_init(bar(B_DRAIN), 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(B_INFO_FULL0 + s), 32);
      tc::mbar_init(bar(B_INFO_EMPTY0 + s), 1 + NUM_SOFTMAX_WARPS);
    }
    for (int q = 0; q < 8; ++q) tc::mbar_init(bar(B_XREADY + q), 64);
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
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = cs->tmem_base;
  const int ntiles = (a.nb + TILE_ROWS - 1) / TILE_ROWS;   // centroid tiles (<= 16)
  // centroid tile of the r-th residual task
  auto res_tile = [](uint32_t tiles, int r) { return (int)__fns(tiles, 0, r + 1); };

  if (warp == WARP_PRODUCER) {
    // ---------------------------------------------------------- producer
    // Per item: take a ticket from the device work counter, describe the
    // item (whole warp), then TMA loads (lane 0) in consumption order:
    // Q, K(0), K(1), then per task t: V(t), K(t+2).
    int n = 0, qn = 0, li = 0;  // items taken, items with tasks (Q loads), K/V loads issued
    bool ok = true;
    for (;; ++n) {
      const int slot = n & 1;
      if (n >= 2 && !(ok = wait_warp(bar(B_INFO_EMPTY0 + slot), (uint32_t)((n - 2) >> 1) & 1u, 11)))
        break;
      int ticket = 0;
      if (lane == 0) ticket = atomicAdd(a.ctrl + CTRL_WORK, 1);
      ticket = __shfl_sync(0xffffffffu, ticket, 0);
      ItemInfo& inf = cs->info[slot];
      if ((unsigned)ticket >= (unsigned)a.items) {   // also a counter left invalid
        if (lane == 0) inf.item = -1;
        __syncwarp();
        tc::mbar_arrive(bar(B_INFO_FULL0 + slot));
        break;
      }
      const int item = a.order ? __ldg(a.order + ticket) : ticket;
      const int tile_item = item / a.splits, range = item % a.splits;
      const int bh = tile_item / a.nq, i = tile_item % a.nq;
      int r_lo = 0, nkept = 0, t0 = 0;
      inf.kept[0][lane] = 0u;
      inf.kept[0][lane + 32] = 0u;
      inf.kept[1][lane] = 0u;
      inf.kept[1][lane + 32] = 0u;
      inf.bad[lane] = 0u;
      inf.bad[lane + 32] = 0u;
      if (lane == 0) inf.tail_task = -1;
      __syncwarp();
      const bool pair2 = a.b64 && 2 * i + 1 < a.nb;   // the tile holds a second query block
      if (a.dense) {
        // exact rows: every key tile of this item's range, in order
        const int per = (a.nb + a.splits - 1) / a.splits;
        t0 = range * per;
        const int t1 = min(a.nb, t0 + per);
        nkept = max(0, t1 - t0);
        if (lane == 0 && t1 == a.nb && nkept > 0 && a.n_last < TILE_ROWS) inf.tail_task = nkept - 1;
        __syncwarp();
      } else if (a.inline_sel) {
        const SelArgs sa{a.qbar, a.kbar, a.nb, a.n_last, a.blk, a.threshold, a.kmin, a.kcap, a.tau};
        select_inline<D>(sa, a.b64 ? bh * a.nb + 2 * i : item, inf.kept[0], cs->selp, cs->selq);
        if (pair2) select_inline<D>(sa, bh * a.nb + 2 * i + 1, inf.kept[1], cs->selp, cs->selq);
      } else if (!a.b64) {
        r_lo = a.counts ? item * a.kcap : __ldg(a.row_ptr + item);
        nkept = a.counts ? __ldg(a.counts + item) : max(0, __ldg(a.row_ptr + item + 1) - r_lo);
        for (int t = lane; t < nkept; t += 32) {
          const int j = __ldg(a.col_idx + r_lo + t);
          if (j >= 0 && j < a.nb) {
            atomicOr(&inf.kept[0][j >> 5], 1u << (j & 31));
            if (j == a.nb - 1 && a.n_last < TILE_ROWS) inf.tail_task = t;
          } else if (t < 2048) {
            atomicOr(&inf.bad[t >> 5], 1u << (t & 31));
          }
        }
        __syncwarp();
      } else {
        // 64-token blocks: query blocks 2i and 2i + 1 share the tile; their
        // kept sets go into two bitmaps (a block index out of range is
        // skipped and flagged), and the key tiles walk the union in
        // ascending order, two blocks per tile
        for (int qb = 0; qb < (pair2 ? 2 : 1); ++qb) {
          const int row = bh * a.nb + 2 * i + qb;
          const int lo = a.counts ? row * a.kcap : __ldg(a.row_ptr + row);
          const int nk = a.counts ? __ldg(a.counts + row) : max(0, __ldg(a.row_ptr + row + 1) - lo);
          uint32_t* km = inf.kept[qb];
          for (int t = lane; t < nk; t += 32) {
            const int j = __ldg(a.col_idx + lo + t);
            if (j >= 0 && j < a.nb) atomicOr(&km[j >> 5], 1u << (j & 31));
            else flag_error(a.ctrl, DEV_BAD_INDEX, row);
          }
        }
        __syncwarp();
      }
      if (a.b64 || a.inline_sel) {
        // the kept blocks (the union of both bitmaps with b = 64) as an
        // ascending list
        const uint32_t w0 = inf.kept[0][2 * lane] | inf.kept[1][2 * lane];
        const uint32_t w1 = inf.kept[0][2 * lane + 1] | inf.kept[1][2 * lane + 1];
        const int c = __popc(w0) + __popc(w1);
        int x = c;   // inclusive scan of the per-lane counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        int pos = x - c;
        for (uint32_t m = w0; m; m &= m - 1u) inf.ublk[pos++] = (uint16_t)(64 * lane + __ffs(m) - 1);
        for (uint32_t m = w1; m; m &= m - 1u) inf.ublk[pos++] = (uint16_t)(64 * lane + 32 + __ffs(m) - 1);
        const int nunion = __shfl_sync(0xffffffffu, x, 31);
        if (a.b64) {
          nkept = (nunion + 1) / 2;
        } else {
          nkept = nunion;
          // the partial last block, when kept, is the last entry
          if (lane == 0 && a.n_last < TILE_ROWS && ((inf.kept[0][(a.nb - 1) >> 5] >> ((a.nb - 1) & 31)) & 1u))
            inf.tail_task = nunion - 1;
        }
        if (lane == 0) inf.nunion = nunion;
        __syncwarp();
      }
      // centroid tiles that hold at least one dropped block (of either query
      // block of the tile, with b = 64)
      bool any = false;
      if (a.residual && lane < ntiles) {
        for (int q = 0; q < TILE_ROWS / 32; ++q) {
          const int j0 = lane * TILE_ROWS + q * 32;
          if (j0 >= a.nb) break;
          const int cnt = min(32, a.nb - j0);
          const uint32_t valid = cnt == 32 ? 0xffffffffu : ((1u << cnt) - 1u);
          any |= (~inf.kept[0][j0 >> 5] & valid) != 0u;
          if (pair2) any |= (~inf.kept[1][j0 >> 5] & valid) != 0u;
        }
      }
      const uint32_t res_tiles = __ballot_sync(0xffffffffu, any);
      const int T = nkept + __popc(res_tiles);
      if (lane == 0) {
        inf.item = item;
        inf.nkept = nkept;
        inf.T = T;
        inf.res_tiles = res_tiles;
      }
      __syncwarp();
      tc::mbar_arrive(bar(B_INFO_FULL0 + slot));   // every lane: releases its own writes
      if (T == 0) continue;
      // Loads: lane 0 makes every wait, sets every transaction count and
      // issues the TMA boxes; the other lanes follow its verdicts.
      // task_rows: first token of the key tile of task t < nkept (and, with
      // b = 64, of its second block)
      auto task_rows = [&](int t, int& row, int& row2) {
        row2 = -1;
        if (a.b64) {
          // an absent second block repeats the first (valid data, masked
          // by the softmax)
          const int j0 = inf.ublk[2 * t];
          const int j1 = 2 * t + 1 < inf.nunion ? inf.ublk[2 * t + 1] : j0;
          row = j0 * 64;
          row2 = j1 * 64;
        } else if (a.dense) {
          row = (t0 + t) * TILE_ROWS;
        } else if (a.inline_sel) {
          row = inf.ublk[t] * TILE_ROWS;
        } else {
          int j = __ldg(a.col_idx + r_lo + t);
          if (j < 0 || j >= a.nb) {
            if (lane == 0) flag_error(a.ctrl, DEV_BAD_INDEX, item);
            j = 0;  // load something valid; the softmax masks the whole task
          }
          row = j * TILE_ROWS;
        }
      };
      if (lane == 0 && qn > 0)
        ok = tc::mbar_wait_fast(bar(B_QEMPTY), (uint32_t)(qn - 1) & 1u, abort, a.ctrl, 12);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok && lane == 0) {
        tc::mbar_expect_tx(bar(B_QFULL), TILE_BYTES);
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          tc::tma_load_3d(sQ + c * CHUNK_BYTES, &tmQ, bar(B_QFULL), c * 64, i * TILE_ROWS, bh);
      }
      auto issue = [&](int t, bool is_v) -> bool {
        const CUtensorMap* m;
        int row = 0, row2 = -1;
        if (t < nkept) {
          m = is_v ? &tmV : &tmK;
          task_rows(t, row, row2);
        } else {
          m = is_v ? &tmVb : &tmKb;
          row = res_tile(res_tiles, t - nkept) * TILE_ROWS;
        }
        const int s = li % STAGES;
        bool free_slot = true;
        if (lane == 0)
          free_slot = tc::mbar_wait_fast(empty(s), ((uint32_t)(li / STAGES) & 1u) ^ 1u, abort, a.ctrl, 1);
        if (!__shfl_sync(0xffffffffu, free_slot, 0)) return false;
        if (lane == 0) {
          tc::mbar_expect_tx(full(s), TILE_BYTES);
          const uint32_t dst = sRing + s * TILE_BYTES;
          if (row2 < 0) {
#pragma unroll
            for (int c = 0; c < NCH; ++c) tc::tma_load_3d(dst + c * CHUNK_BYTES, m, full(s), c * 64, row, bh);
          } else {
            // two 64-row boxes: rows 0-63 and 64-127 of every 128-byte chunk
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
              tc::tma_load_3d(dst + c * CHUNK_BYTES, m, full(s), c * 64, row, bh);
              tc::tma_load_3d(dst + c * CHUNK_BYTES + 64 * 128, m, full(s), c * 64, row2, bh);
            }
          }
        }
        ++li;
        return true;
      };
      if (ok) ok = issue(0, false);
      if (ok && T > 1) ok = issue(1, false);
      for (int t = 0; ok && t < T; ++t) {
        ok = issue(t, true);
        if (ok && t + 2 < T) ok = issue(t + 2, false);
      }
      ++qn;
      if (!ok) break;
    }
    if (lane == 0) {
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        if (qn > 0) tc::mbar_drain(bar(B_QFULL), (uint32_t)(qn - 1) & 1u);
        for (int k = (li > STAGES ? li - STAGES : 0); k < li; ++k)
          tc::mbar_drain(full(k % STAGES), (uint32_t)(k / STAGES) & 1u);
        // take the remaining tickets so the retirement count below holds
        while (atomicAdd(a.ctrl + CTRL_WORK, 1) < a.items) {
        }
      }
      // The last CTA to retire resets the work counter for the next launch
      // (every CTA has drawn its final ticket before it retires).
      __threadfence();
      if (atomicAdd(a.ctrl + CTRL_DONE, 1) == (int)gridDim.x - 1) {
        atomicExch(a.ctrl + CTRL_WORK, 0);
        atomicExch(a.ctrl + CTRL_DONE, 0);
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idO = tc::idesc_bf16_f32(128, D, true);
      // loop-invariant descriptors; k-step and slot offsets are added to the
      // address field (bits 0-13, 16-byte units)
      const uint64_t dQ = tc::sdesc_sw128(sQ, 16, 1024);
      const uint64_t dK = tc::sdesc_sw128(sRing, 16, 1024);
      const uint64_t dV = tc::sdesc_sw128(sRing, CHUNK_BYTES, 1024);
      int n = 0, qn = 0, gt = 0, li = 0;  // items, items with tasks, tasks before this item, loads consumed
      bool ok = true;
      // S(g) = Q K^T into S buffer g & 1
      auto issue_s = [&](int g) -> bool {
        const int s = li % STAGES;
        if (!tc::mbar_wait_fast(full(s), (uint32_t)(li / STAGES) & 1u, abort, a.ctrl, 4)) return false;
        tc::tc_fence_after();
        const uint64_t slot16 = (uint64_t)(s * TILE_BYTES / 16);
        const uint32_t dS = tmem + 128u * (uint32_t)(g & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32) >> 4;
          tc::umma_ss(dS, dQ + off16, dK + slot16 + off16, idS, kk > 0);
        }
        tc::umma_commit(empty(s));
        tc::umma_commit(bar(B_SFULL0 + (g & 1)));
        ++li;
        return true;
      };
      for (;; ++n) {
        const int slot = n & 1;
        if (!(ok = tc::mbar_wait_fast(bar(B_INFO_FULL0 + slot), (uint32_t)(n >> 1) & 1u, abort, a.ctrl, 13)))
          break;
        const int item = cs->info[slot].item;
        if (item < 0) break;
        const int T = cs->info[slot].T;
        if (T > 0) {
          ok = tc::mbar_wait_fast(bar(B_QFULL), (uint32_t)qn & 1u, abort, a.ctrl, 3);
          if (ok) ok = issue_s(gt);
          if (ok && T > 1) ok = issue_s(gt + 1);
          if (ok && T <= 2) tc::umma_commit(bar(B_QEMPTY));
          for (int t = 0; ok && t < T; ++t) {
            const int g = gt + t;
            if (!(ok = tc::mbar_wait_fast(bar(B_PREADY), (uint32_t)g & 1u, abort, a.ctrl, 5))) break;
            const int s = li % STAGES;
            if (!(ok = tc::mbar_wait_fast(full(s), (uint32_t)(li / STAGES) & 1u, abort, a.ctrl, 6))) break;
            tc::tc_fence_after();
            // O_h += P_h V_h for both key halves: M = 128 queries, N = d,
            // K = 64 keys in steps of 16; P is bf16 packed two per TMEM
            // column, V is MN-major (d contiguous), rows 64h .. 64h+63 of the
            // tile
            const uint64_t slot16 = (uint64_t)(s * TILE_BYTES / 16);
            const uint32_t tP = tmem + 128u * (uint32_t)(g & 1);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc::umma_ts(tmem + COL_O + 128u * h, tP + 64u * h + 8u * kk,
                            dV + slot16 + (uint64_t)((64 * h + 16 * kk) * 128 / 16), idO,
                            (t > 0 || kk > 0) ? 1u : 0u);
            tc::umma_commit(empty(s));
            tc::umma_commit(bar(B_PVDONE));
            ++li;
            // S buffer g & 1 (S(g), then P(g)) is free once PV(g) has run;
            // the tensor core executes in issue order
            if (t + 2 < T) {
              if (!(ok = issue_s(g + 2))) break;
              if (t + 3 == T) tc::umma_commit(bar(B_QEMPTY));   // Q's last use
            }
          }
          if (ok) tc::umma_commit(bar(B_OFULL));
          gt += T;
          ++qn;
        }
        if (!ok) break;
        tc::mbar_arrive(bar(B_INFO_EMPTY0 + slot));
      }
      if (!ok) {
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
    const uint32_t tOh = tmem + lane_off + COL_O + 128u * (uint32_t)half;  // this half's O
    const float lg_b = log2f((float)a.blk), lg_last = log2f((float)a.n_last);
    // b = 64: rows 0-63 of a tile are the first query block, rows 64-127 the
    // second, so lane quarters 2 and 3 test the second block's kept set
    const int qsel = a.b64 ? (quarter >> 1) : 0;
    int n = 0, qn = 0, gt = 0;  // items, items with tasks, tasks before this item
    bool ok = true;

    auto rescale_o = [&](float f) {
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tc::tmem_ld32(tOh + 32u * c, ov);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
        tc::tmem_st32(tOh + 32u * c, ov);
      }
    };

    for (;; ++n) {
      const int slot = n & 1;
      if (!(ok = wait_warp(bar(B_INFO_FULL0 + slot), (uint32_t)(n >> 1) & 1u, 14))) break;
      const ItemInfo& inf = cs->info[slot];
      const int item = inf.item;
      if (item < 0) break;
      const int T = inf.T, nkept = inf.nkept, tail_task = inf.tail_task;
      const uint32_t res_tiles = inf.res_tiles;
      // m: reference maximum of this row's key half (log2 units); l: sum of
      // p at that reference; owe: factor O_h owes once PV(g-1) is done.
      float m = -INFINITY, l = 0.f, owe = 1.f;

      // failure-path test: phase 0 of the drain barrier completes only after
      // an abort, so this bounded wait runs out and aborts the CTA
      if (a.test_stall && blockIdx.x == 0 && n == 0 && T > 0 && !(ok = wait_warp(bar(B_DRAIN), 0u, 15)))
        break;
      for (int t = 0; t < T; ++t) {
        const int g = gt + t, b = g & 1;
        if (!(ok = wait_warp(bar(B_SFULL0 + b), (uint32_t)(g >> 1) & 1u, 7))) break;
        tc::tc_fence_after();
        // this warp's 64 columns of S(g).  Key tiles: columns past n_j of the
        // partial last block (or a whole tile with a bad index; with b = 64,
        // a whole half whose block this warp's query block did not keep) are
        // set to -inf.  Centroid tiles: the log2-scaled logit plus the bias
        // log2 n_j (dropped) / -inf (kept) is formed up front.
        uint32_t u[64];
        const uint32_t scol = tmem + lane_off + 128u * (uint32_t)b + 64u * (uint32_t)half;
        const float scale = t < nkept ? a.sl2 : 1.f;
        // the task's mask, looked up before S is loaded (fewer live registers
        // next to S): key tiles, the count of valid columns of this half;
        // centroid tiles, the first block of this half and the kept bits of
        // its 64 blocks
        int nvalid = 64, jres = 0;
        uint32_t kw0 = 0u, kw1 = 0u;
        if (t < nkept) {
          if (a.b64) {
            const int e = 2 * t + half;
            const int j = e < inf.nunion ? (int)inf.ublk[e] : -1;
            const bool mine = j >= 0 && ((inf.kept[qsel][j >> 5] >> (j & 31)) & 1u);
            nvalid = mine ? (j == a.nb - 1 ? a.n_last : 64) : 0;
          } else {
            const bool bad = t < 2048 && ((inf.bad[t >> 5] >> (t & 31)) & 1u);
            nvalid = (bad ? 0 : (t == tail_task ? a.n_last : TILE_ROWS)) - 64 * half;
          }
        } else {
          jres = res_tile(res_tiles, t - nkept) * TILE_ROWS + 64 * half;
          if (jres < a.nb) kw0 = inf.kept[qsel][jres >> 5];
          if (jres + 32 < a.nb) kw1 = inf.kept[qsel][(jres >> 5) + 1];
        }
        auto load_s = [&]() {
          tc::tmem_ld32(scol, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tc::tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tc::tmem_wait_ld();
          if (t < nkept) {
            if (nvalid < 64) {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                if (c >= nvalid) u[c] = __float_as_uint(-INFINITY);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int j = jres + c;
              const uint32_t kw = c < 32 ? kw0 : kw1;
              const bool dropped = j < a.nb && !((kw >> (c & 31)) & 1u);
              const float bias = dropped ? (j == a.nb - 1 ? lg_last : lg_b) : -INFINITY;
              u[c] = __float_as_uint(fmaf(__uint_as_float(u[c]), a.sl2, bias));
            }
          }
        };
        load_s();
        auto tile_max = [&]() {
          float mx[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            mx[e] = tc::fmax3(__uint_as_float(u[e]), __uint_as_float(u[e + 8]), __uint_as_float(u[e + 16]));
#pragma unroll
          for (int c = 24; c < 64; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              mx[e] = c + 8 + e < 64 ? tc::fmax3(mx[e], __uint_as_float(u[c + e]), __uint_as_float(u[c + e + 8]))
                                     : fmaxf(mx[e], __uint_as_float(u[c + e]));
          return tc::fmax3(tc::fmax3(mx[0], mx[1], mx[2]), tc::fmax3(mx[3], mx[4], mx[5]),
                           fmaxf(mx[6], mx[7])) * scale;
        };
        // a row without a reference yet (first tile, or only masked keys so
        // far) takes this tile's maximum
        if (__any_sync(0xffffffffu, m == -INFINITY)) {
          if (m == -INFINITY) m = tile_max();
        }
        uint32_t pk[32];
        float lt;
        auto exps = [&]() {
          const float nmu = (m == -INFINITY) ? 0.f : -m;
          const uint64_t sc2 = tc::f2_pack(scale, scale), nmu2 = tc::f2_pack(nmu, nmu);
          uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint64_t x2 = tc::f2_fma(
                tc::f2_pack(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), sc2, nmu2);
            float p0, p1;
            if ((e & 7) < SPATTN_EXP_EMU) {
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
          const uint64_t t2 = tc::f2_add(tc::f2_add(ls2[0], ls2[1]), tc::f2_add(ls2[2], ls2[3]));
          float lo, hi;
          tc::f2_unpack(t2, lo, hi);
          lt = lo + hi;
        };
        exps();
        // A tile far above the reference is recomputed against its own
        // maximum, so every p stays below 2^60 (bf16 P and fp32 O cannot
        // overflow); O_h then owes the factor before PV(g).
        const bool over = !(lt <= 1.152921504606847e18f);   // 2^60; also catches inf / NaN
        if (__any_sync(0xffffffffu, over)) {
          load_s();   // S(g) is still in TMEM: reload rather than keep u live
          if (over) {
            const float mn = fmaxf(m, tile_max());
            const float f = tc::ex2(m - mn);
            l *= f;
            owe *= f;
            m = mn;
          }
          exps();
        }
        tc::tmem_st32(scol, pk);   // P(g) over this warp's own, already read, columns
        l += lt;
        // O_h owes `owe` once PV(g-1) is done (factor 1 on rows owing
        // nothing).  Every phase of the PV barrier inside an item is waited
        // for, and the item's first task follows the previous item's OFULL,
        // so the parity always names the one PV in question.
        if (t > 0) {
          if (!(ok = wait_warp(bar(B_PVDONE), (uint32_t)(g - 1) & 1u, 10))) break;
          if (__any_sync(0xffffffffu, owe != 1.f)) {
            tc::tc_fence_after();
            rescale_o(owe);
          }
        }
        owe = 1.f;
        // keep p moderate: when this tile's sum passes 2^16 the reference
        // moves up by the integer part of log2(sum), an exact power-of-two
        // rescale (l now; O_h after PV(g), in the next step)
        if (lt > 65536.f) {
          const int e = ((int)(__float_as_uint(lt) >> 23) & 0xFF) - 127;
          const float f = __int_as_float((127 - e) << 23);   // 2^-e
          l *= f;
          owe = f;
          m += (float)e;
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(B_PREADY));
      }
      if (ok && T > 0)
        ok = __all_sync(0xffffffffu, tc::mbar_wait(bar(B_OFULL), (uint32_t)qn & 1u, abort, a.ctrl, 8));
      if (ok && __any_sync(0xffffffffu, owe != 1.f)) {
        tc::tc_fence_after();
        rescale_o(owe);
        tc::tmem_wait_st();
      }
      // merge the two key halves of each row (the two warps of a lane
      // quarter meet on an mbarrier; a bounded wait, so an aborting partner
      // cannot strand this warp)
      cs->xm[slot][half][r] = m;
      cs->xl[slot][half][r] = l;
      tc::tc_fence_before();
      tc::mbar_arrive(bar(B_XREADY + 4 * slot + quarter));
      if (ok) ok = wait_warp(bar(B_XREADY + 4 * slot + quarter), (uint32_t)(n >> 1) & 1u, 9);
      if (ok) {
        tc::tc_fence_after();
        const float m0 = cs->xm[slot][0][r], m1 = cs->xm[slot][1][r];
        const float M = fmaxf(m0, m1);
        const float a0 = m0 == -INFINITY ? 0.f : tc::ex2(m0 - M);
        const float a1 = m1 == -INFINITY ? 0.f : tc::ex2(m1 - M);
        const float L = a0 * cs->xl[slot][0][r] + a1 * cs->xl[slot][1][r];
        // query tile and output head (key range c of a split dense item
        // writes its own copy, c * (batch, head) pairs further on)
        const int it = item / a.splits;
        const int obh = (item % a.splits) * (a.items / (a.splits * a.nq)) + it / a.nq;
        const int tok = (it % a.nq) * TILE_ROWS + r;
        const bool store = tok < a.q_rows;   // rows past the last query are padding
        const int dst = store ? (a.perm ? __ldg(a.perm + tok) : tok) : 0;
        const size_t obase = ((size_t)obh * a.q_rows + dst) * D + half * (D / 2);
        const float inv = L > 0.f ? 1.f / L : 0.f;
        if (a.lse && store && half == 0)   // log2 of the row's mass: sum of 2^(s sl2) = 2^M L
          a.lse[(size_t)obh * a.q_rows + dst] =
              L > 0.f ? M + __log2f(L) : -INFINITY;
        const float w0 = a0 * inv, w1 = a1 * inv;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o0[32], o1[32];
          if (T > 0) {  // warp-uniform: every lane takes part in the loads
            const uint32_t col = (uint32_t)(half * (D / 2) + 32 * c);
            tc::tmem_ld32(tmem + lane_off + COL_O + col, o0);
            tc::tmem_ld32(tmem + lane_off + COL_O + 128u + col, o1);
            tc::tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o0[e] = o1[e] = 0u;
          }
          if (store) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                v[e] = __uint_as_float(o0[8 * q + e]) * w0 + __uint_as_float(o1[8 * q + e]) * w1;
              if (a.o32) {
                float4* orow32 = reinterpret_cast<float4*>(a.o32 + obase);
                orow32[c * 8 + 2 * q] = make_float4(v[0], v[1], v[2], v[3]);
                orow32[c * 8 + 2 * q + 1] = make_float4(v[4], v[5], v[6], v[7]);
              } else {
                uint4 pv;
                pv.x = pack_bf16x2(v[0], v[1]);
                pv.y = pack_bf16x2(v[2], v[3]);
                pv.z = pack_bf16x2(v[4], v[5]);
                pv.w = pack_bf16x2(v[6], v[7]);
                reinterpret_cast<uint4*>(a.o + obase)[c * 4 + q] = pv;
              }
            }
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (!ok) break;
      if (lane == 0) tc::mbar_arrive(bar(B_INFO_EMPTY0 + slot));
      gt += T;
      if (T > 0) ++qn;
    }
    // a role that left early (abort) may still have TMEM accesses in flight
    tc::tmem_wait_ld();
    tc::tmem_wait_st();
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

// [BH, rows, D] bf16 tensor, box = 64 channels x box_rows rows x 1, 128-byte
// swizzle.
bool encode_map(CUtensorMap* m, const void* ptr, int D, int rows, int BH, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A tensor map depends only on (pointer, D, rows, BH, box rows): the last few
// encoded maps of each host thread are kept so repeated calls on the same
// buffers skip the driver's encode.
struct MapKey {
  const void* ptr;
  int D, rows, BH, box;
};
struct MapEntry {
  MapKey k;
  CUtensorMap m;
  bool used;
};

bool make_map(CUtensorMap* m, const void* ptr, int D, int rows, int BH, int box = TILE_ROWS) {
  constexpr int SLOTS = 16;
  thread_local MapEntry cache[SLOTS] = {};
  thread_local int next = 0;
  for (int c = 0; c < SLOTS; ++c) {
    const MapEntry& e = cache[c];
    if (e.used && e.k.ptr == ptr && e.k.D == D && e.k.rows == rows && e.k.BH == BH &&
        e.k.box == box) {
      *m = e.m;
      return true;
    }
  }
  if (!encode_map(m, ptr, D, rows, BH, box)) return false;
  MapEntry& e = cache[next];
  next = (next + 1) % SLOTS;
  e.k = MapKey{ptr, D, rows, BH, box};
  e.m = *m;
  e.used = true;
  return true;
}

// the control block starts 1024-byte aligned (after the tiles); the members
// read or written as float4 must sit on 16-byte offsets inside it
static_assert(offsetof(TcCtrl, selq) % 16 == 0 && offsetof(TcCtrl, selp) % 16 == 0,
              "float4 scratch of the inline selection must be 16-byte aligned");

template <int D>
constexpr size_t tc_smem_bytes() {
  return (size_t)(1 + TcCfg<D>::STAGES) * TcCfg<D>::TILE_BYTES + sizeof(TcCtrl) + 1024;
}
// 227 KB of shared memory per CTA at most
static_assert(tc_smem_bytes<128>() <= 232448 && tc_smem_bytes<64>() <= 232448,
              "attention tiles and control block exceed the shared memory of one CTA");

template <int D>
cudaError_t launch_tc(const CUtensorMap* maps, const TcArgs& a, cudaStream_t s) {
  const size_t smem = tc_smem_bytes<D>();
  cudaError_t e = ensure_dyn_smem((const void*)attn_tc_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (shared memory and TMEM admit one), at most
  // one per work item
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int grid = std::max(1, std::min(a.items, sms));
  attn_tc_kernel<D><<<grid, TC_THREADS, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], a);
  return cudaGetLastError();
}

}  // namespace

bool attend_tc_supported(const Problem& p) {
  return (p.b == TILE_ROWS || p.b == TILE_ROWS / 2) && (p.d == 64 || p.d == 128);
}

cudaError_t launch_attend_tc(const Problem& p, const void* Q, const void* K, const void* V,
                             const int32_t* row_ptr, const int32_t* col_idx, void* O,
                             const Work& w, cudaStream_t s) {
  // with a permutation, the workspace's permuted copies (blocked order)
  const void* q = w.qp ? (const void*)w.qp : Q;
  const void* k = w.kp ? (const void*)w.kp : K;
  const void* v = w.vp ? (const void*)w.vp : V;
  // K and V tiles: one 128-row box, or two 64-row boxes (one per block) with
  // 64-token blocks
  const bool b64 = p.b == TILE_ROWS / 2;
  CUtensorMap maps[5];
  if (!make_map(&maps[0], q, p.d, p.N, p.BH) || !make_map(&maps[1], k, p.d, p.N, p.BH, p.b) ||
      !make_map(&maps[2], v, p.d, p.N, p.BH, p.b) || !make_map(&maps[3], w.kbar16, p.d, p.nb, p.BH) ||
      !make_map(&maps[4], w.vbar16, p.d, p.nb, p.BH))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.inline_sel = (row_ptr == w.row_ptr && p.inline_sel) ? 1 : 0;
  a.qbar = w.qbar; a.kbar = w.kbar;
  a.tau = p.tau; a.threshold = p.threshold; a.kmin = p.kmin;
  if (a.inline_sel) {
    // the producer selects from the workspace means: no lists, plain order
    a.row_ptr = nullptr; a.col_idx = nullptr; a.counts = nullptr; a.kcap = p.kcap;
    a.order = nullptr;
  } else if (row_ptr == w.row_ptr) {
    // the workspace's own routing result: padded lists, longest-first order
    // (the order is per query block: with 64-token blocks the tiles run in
    // plain order)
    a.row_ptr = nullptr; a.col_idx = w.lists; a.counts = w.counts; a.kcap = p.kcap;
    a.order = b64 ? nullptr : w.order;
  } else {
    a.row_ptr = row_ptr; a.col_idx = col_idx; a.counts = nullptr; a.kcap = 0;
    a.order = nullptr;
  }
  a.perm = p.perm;
  a.o = static_cast<__nv_bfloat16*>(O);
  a.o32 = nullptr;
  a.q_rows = p.N;
  a.dense = 0;
  a.splits = 1;
  a.lse = nullptr;
  a.ctrl = w.ctrl;
  a.N = p.N; a.nb = p.nb; a.n_last = p.n_last; a.residual = p.residual;
  a.b64 = b64 ? 1 : 0;
  a.blk = p.b;
  a.nq = b64 ? (p.nb + 1) / 2 : p.nb;
  a.sl2 = 1.4426950408889634f / sqrtf((float)p.d);
  a.items = p.BH * a.nq;
  a.test_stall = p.test_stall;
  // The work counter resets itself at the end of every launch; it starts
  // from zero after the routing call's control-block clear.  A caller CSR
  // may come with a workspace that was never routed: clear the error word
  // and the counters.
  if (row_ptr != w.row_ptr) {
    static_assert(CTRL_ERROR == 0 && CTRL_ERROR_AUX == 1 && CTRL_WORK == 2 && CTRL_DONE == 3,
                  "control words cleared together");
    cudaError_t e = cudaMemsetAsync(w.ctrl, 0, 4 * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  return p.d == 128 ? launch_tc<128>(maps, a, s) : launch_tc<64>(maps, a, s);
}

// ---- probe correction apply on the tensor cores ----------------------------
// O <- O + O (B P) + b P for every row of a head (SparsePR page, section 2B),
// one CTA per 128-row tile: the O tile and W^T = (B P)^T (bf16 [d][d], row n
// holds column n of B P, i.e. a K-major operand) come in by TMA, one group of
// tcgen05 MMAs puts O W into TMEM, and four warps add O (read back from the
// swizzled shared tile) and b P in fp32 and store bf16.

constexpr int AP_THREADS = 128;

template <int D>
constexpr size_t apply_tc_smem_bytes() {
  return (size_t)2 * TILE_ROWS * D * 2 + 64 + 1024;
}

template <int D>
__global__ void __launch_bounds__(AP_THREADS) probe_apply_tc_kernel(
    const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmW,
    __nv_bfloat16* o, const float* cp, int N, int32_t* ctrl) {
  constexpr int NCH = D / 64;
  constexpr int CHUNK_A = TILE_ROWS * 128;   // bytes of one 64-channel chunk of the O tile
  constexpr int CHUNK_B = D * 128;           // of W^T (D rows)
  constexpr int TILE_A = TILE_ROWS * D * 2, TILE_B = D * D * 2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sA = base, sB = base + TILE_A;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + TILE_A + TILE_B);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar_load = smem_u32(&bars[0]), bar_mma = smem_u32(&bars[1]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, bh = blockIdx.y;
  if (threadIdx.x == 0) {
    tc::mbar_init(bar_load, 1);
    tc::mbar_init(bar_mma, 1);
    *abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(tmem_slot), D < 32 ? 32 : D);
    tc::tc_fence_before();
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (threadIdx.x == 0) {
    tc::mbar_expect_tx(bar_load, TILE_A + TILE_B);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      tc::tma_load_3d(sA + c * CHUNK_A, &tmO, bar_load, c * 64, tile * TILE_ROWS, bh);
      tc::tma_load_3d(sB + c * CHUNK_B, &tmW, bar_load, c * 64, 0, bh);
    }
    ok = tc::mbar_wait(bar_load, 0, abort, ctrl, 30);
    if (ok) {
      tc::tc_fence_after();
      const uint64_t dA = tc::sdesc_sw128(sA, 16, 1024), dB = tc::sdesc_sw128(sB, 16, 1024);
      constexpr uint32_t idesc = tc::idesc_bf16_f32(128, D, false);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t offA = ((kk >> 2) * CHUNK_A + (kk & 3) * 32) >> 4;
        const uint32_t offB = ((kk >> 2) * CHUNK_B + (kk & 3) * 32) >> 4;
        tc::umma_ss(tmem, dA + offA, dB + offB, idesc, kk > 0);
      }
      tc::umma_commit(bar_mma);
    }
  }
  ok = __syncthreads_and(ok);
  if (ok) ok = __syncthreads_and(tc::mbar_wait(bar_mma, 0, abort, ctrl, 31));
  if (ok) {
    tc::tc_fence_after();
    const int r = warp * 32 + lane;              // tile row = TMEM lane
    const int tok = tile * TILE_ROWS + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float* cph = cp + (size_t)bh * D;
    uint4* orow = reinterpret_cast<uint4*>(o + ((size_t)bh * N + (tok < N ? tok : 0)) * D);
#pragma unroll
    for (int c32 = 0; c32 < D / 32; ++c32) {
      uint32_t acc[32];
      tc::tmem_ld32(tmem + lane_off + 32u * c32, acc);
      tc::tmem_wait_ld();
      if (tok < N) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // 8 channels per 16-byte piece
          const int ch = c32 * 32 + q * 8;
          const int chunk = ch >> 6, piece = (ch & 63) >> 3;
          const uint4 xv = *reinterpret_cast<const uint4*>(
              gbase + chunk * CHUNK_A + r * 128 + ((piece ^ (r & 7)) << 4));
          const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv);
          float v[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x2 = __bfloat1622float2(xh[e]);
            v[2 * e] = x2.x + (__uint_as_float(acc[q * 8 + 2 * e]) + __ldg(cph + ch + 2 * e));
            v[2 * e + 1] = x2.y + (__uint_as_float(acc[q * 8 + 2 * e + 1]) + __ldg(cph + ch + 2 * e + 1));
          }
          uint4 pv;
          pv.x = pack_bf16x2(v[0], v[1]);
          pv.y = pack_bf16x2(v[2], v[3]);
          pv.z = pack_bf16x2(v[4], v[5]);
          pv.w = pack_bf16x2(v[6], v[7]);
          orow[ch / 8] = pv;
        }
      }
    }
  } else if (threadIdx.x == 0) {
    // let copies and MMAs in flight land before the CTA can exit
    tc::mbar_drain(bar_load, 0);
    tc::mbar_drain(bar_mma, 0);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, D < 32 ? 32 : D);
  }
}

template <int D>
cudaError_t launch_apply_tc_d(const Problem& p, void* O, const void* Wt, const float* cp,
                              int32_t* ctrl, cudaStream_t s) {
  CUtensorMap mo, mw;
  if (!make_map(&mo, O, D, p.N, p.BH) || !make_map(&mw, Wt, D, D, p.BH, D)) return cudaErrorInvalidValue;
  constexpr size_t smem = apply_tc_smem_bytes<D>();
  cudaError_t e = ensure_dyn_smem((const void*)probe_apply_tc_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + TILE_ROWS - 1) / TILE_ROWS, p.BH);
  probe_apply_tc_kernel<D><<<grid, AP_THREADS, smem, s>>>(mo, mw, static_cast<__nv_bfloat16*>(O), cp,
                                                         p.N, ctrl);
  return cudaGetLastError();
}

// Rows of split key ranges put together: range c holds each row normalised
// over its own keys plus the log2 of its mass, so the full row is the
// mass-weighted mean of the ranges.  One warp per row, a float4 per lane.
__global__ void __launch_bounds__(256) dense_combine_kernel(const float* part, const float* lse,
                                                            float* out, int rows, int splits, int d) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  float mx = -INFINITY;
  for (int c = 0; c < splits; ++c) mx = fmaxf(mx, lse[(size_t)c * rows + row]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  const int d4 = d / 4;
  for (int c = 0; c < splits; ++c) {
    const float lc = lse[(size_t)c * rows + row];
    const float w = lc == -INFINITY ? 0.f : exp2f(lc - mx);
    wsum += w;
    if (lane < d4) {
      const float4 v = reinterpret_cast<const float4*>(part + ((size_t)c * rows + row) * d)[lane];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  if (lane < d4)
    reinterpret_cast<float4*>(out + (size_t)row * d)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// Key ranges per dense tile item: the count (at most DENSE_MAX_SPLITS, at
// most one range per key tile) whose waves of items over the SMs finish
// soonest, in units of one unsplit item; the fewest ranges on a tie.
static int dense_splits(int items, int nb, int sms) {
  int best = 1;
  double best_t = std::ceil((double)items / sms);
  for (int s = 2; s <= std::min(DENSE_MAX_SPLITS, nb); ++s) {
    const double tm = std::ceil((double)items * s / sms) / s;
    if (tm < best_t) { best_t = tm; best = s; }
  }
  return best;
}

// Exact (dense) softmax attention of gathered query rows, fp32 out: Qg holds
// q_alloc rows per (batch, head) (a multiple of 128, zero past q_rows), every
// one of the N keys of K and V is attended, and rows [0, q_rows) of each head
// are written to out [BH, q_rows, d].  The probe correction's exact rows.
// When there are too few 128-row tiles to fill the GPU, each tile's keys are
// cut into ranges (part: DENSE_MAX_SPLITS x [BH, q_rows, d] fp32, lse:
// DENSE_MAX_SPLITS x [BH, q_rows]) put together by dense_combine_kernel.
cudaError_t launch_dense_rows_tc(const Problem& p, const void* Qg, int q_alloc, int q_rows,
                                 const void* K, const void* V, float* out, float* part, float* lse,
                                 int32_t* ctrl, cudaStream_t s) {
  const int nb = (p.N + TILE_ROWS - 1) / TILE_ROWS;
  CUtensorMap maps[5];
  if (!make_map(&maps[0], Qg, p.d, q_alloc, p.BH) || !make_map(&maps[1], K, p.d, p.N, p.BH) ||
      !make_map(&maps[2], V, p.d, p.N, p.BH))
    return cudaErrorInvalidValue;
  maps[3] = maps[1];   // no residual tiles: the centroid maps are never read
  maps[4] = maps[2];
  int dev = 0, sms = 148;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  TcArgs a{};
  a.dense = 1;
  a.o = nullptr;
  a.q_rows = q_rows;
  a.ctrl = ctrl;
  a.N = p.N; a.nb = nb; a.n_last = p.N - (nb - 1) * TILE_ROWS; a.residual = 0;
  a.b64 = 0;
  a.blk = TILE_ROWS;
  a.nq = q_alloc / TILE_ROWS;
  a.kcap = nb;
  a.sl2 = 1.4426950408889634f / sqrtf((float)p.d);
  a.splits = (part && lse) ? dense_splits(p.BH * a.nq, nb, sms) : 1;
  a.o32 = a.splits > 1 ? part : out;
  a.lse = a.splits > 1 ? lse : nullptr;
  a.items = p.BH * a.nq * a.splits;
  // the work ticket and retirement count start from zero (the workspace may
  // never have run an attention); the error word is left as it is
  static_assert(CTRL_DONE == CTRL_WORK + 1, "ticket words cleared together");
  if ((e = cudaMemsetAsync(ctrl + CTRL_WORK, 0, 2 * sizeof(int32_t), s)) != cudaSuccess) return e;
  if ((e = p.d == 128 ? launch_tc<128>(maps, a, s) : launch_tc<64>(maps, a, s)) != cudaSuccess) return e;
  if (a.splits == 1) return cudaSuccess;
  const int rows = p.BH * q_rows;
  dense_combine_kernel<<<(rows + 7) / 8, 256, 0, s>>>(part, lse, out, rows, a.splits, p.d);
  return cudaGetLastError();
}

// O <- O + O W + c per head on the tensor cores (the probe correction's
// folded apply); Wt: bf16 [BH, d, d] with row n = column n of W; c: fp32 [BH, d].
cudaError_t launch_probe_apply_tc(const Problem& p, void* O, const void* Wt, const float* c,
                                  int32_t* ctrl, cudaStream_t s) {
  return p.d == 128 ? launch_apply_tc_d<128>(p, O, Wt, c, ctrl, s)
                    : launch_apply_tc_d<64>(p, O, Wt, c, ctrl, s);
}

}  // namespace spattn
