// Block selection shared by the routing kernels and the attention kernel's
// inline selection: the centroid proxy row of one query block, its softmax,
// and the Top-p (or per-block threshold) cut with the budget clamp, all on
// one warp, so that every kernel that selects takes the same decision bit for
// bit.
//
// Top-p (PARK page 3.2): blocks in descending p, ties to the lower block
// index, the shortest prefix whose mass reaches tau, budget clamped to
// [kmin, kcap] (Sol-Attn abstract: dynamic but controllable budgets).
// Threshold (Sol-Attn abstract: blocks whose proxy score passes a threshold;
// read as p_ij >= theta): the cut is bits(theta) - 1, and only a binding
// clamp needs the search.
//
// Selection without a sort: with p >= 0 the float bit pattern orders p, and
// the mass G(u) = sum of p_j whose bits exceed u is monotone in u.  The kept
// prefix is {p_j > v} plus the first few blocks with p_j == v (ascending j),
// where v is the smallest value whose strictly-larger mass is < tau.  A
// search over the bit patterns finds v: 32-way for rows of at most 128
// blocks (each lane evaluates one candidate over the whole row), binary with
// one warp reduction per step otherwise (the row held in registers up to 1024
// blocks).  The same search on the count
// #{p_j > u} yields the top-k set when the clamp binds.  Kept blocks are then
// walked in ascending j with warp ballots.
#pragma once

#include <stdint.h>

namespace spattn {
namespace sel {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Mass of the blocks whose probability bits exceed u.
__device__ __forceinline__ float mass_above(const float* p, int nb, uint32_t u) {
  float s = 0.f;
  for (int j = threadIdx.x & 31; j < nb; j += 32) {
    const float x = p[j];
    if (__float_as_uint(x) > u) s += x;
  }
  return warp_sum(s);
}
__device__ __forceinline__ int count_above(const float* p, int nb, uint32_t u) {
  int c = 0;
  for (int j = threadIdx.x & 31; j < nb; j += 32) c += (__float_as_uint(p[j]) > u) ? 1 : 0;
  return warp_sum_i(c);
}
__device__ __forceinline__ int count_equal(const float* p, int nb, uint32_t u) {
  int c = 0;
  for (int j = threadIdx.x & 31; j < nb; j += 32) c += (__float_as_uint(p[j]) == u) ? 1 : 0;
  return warp_sum_i(c);
}

// Smallest u in [lo, hi] with pred(u) true, for pred monotone in u (false
// ... false true ... true) and pred(hi) true; warp-uniform result.  Each
// round the 32 lanes test 32 evenly spaced candidates and the range shrinks
// 32-fold, so 2^30 candidates need 6 rounds.  pred is evaluated by one lane
// alone (a full pass over the row), which suits short rows.
template <typename Pred>
__device__ __forceinline__ uint32_t search32(uint32_t lo, uint32_t hi, Pred pred) {
  const int lane = threadIdx.x & 31;
  while (lo < hi) {
    const uint32_t span = hi - lo;                    // candidates lo .. hi - 1 undecided
    const uint32_t step = span / 32 + 1;
    const uint32_t u = lo + (uint32_t)lane * step;
    const bool in = u < hi;
    const unsigned yes = __ballot_sync(0xffffffffu, in && pred(u));
    const unsigned cand = __ballot_sync(0xffffffffu, in);
    if (yes == 0u) {
      // every tested candidate is false: the answer is above the last one
      const int last = 31 - __clz(cand);
      lo = lo + (uint32_t)last * step + 1;
    } else {
      const int first = __ffs(yes) - 1;
      const uint32_t uf = lo + (uint32_t)first * step;
      if (first == 0) return uf;                      // pred(lo) holds
      lo = lo + (uint32_t)(first - 1) * step + 1;
      hi = uf;
    }
  }
  return lo;
}

// Mass / count of the blocks whose probability bits exceed u, by one lane.
__device__ __forceinline__ float mass_above_1(const float* p, int nb, uint32_t u) {
  float s = 0.f;
  for (int j = 0; j < nb; ++j) {
    const float x = p[j];
    s += (__float_as_uint(x) > u) ? x : 0.f;
  }
  return s;
}
__device__ __forceinline__ int count_above_1(const float* p, int nb, uint32_t u) {
  int c = 0;
  for (int j = 0; j < nb; ++j) c += (__float_as_uint(p[j]) > u) ? 1 : 0;
  return c;
}

// rows with at most this many blocks use the 32-way search
constexpr int SEARCH32_MAX_NB = 128;
// longer rows up to this many blocks run the binary search on registers
constexpr int REG_MAX_NB = 1024;

// A row in registers: lane l holds p[l + 32 i] in pv[i], +0 past the row
// (bits 0: never above any u, so the mass and count below skip it).  The
// sums run in the order of mass_above / count_above (i ascending per lane,
// then the same xor tree), so they are the same numbers.
__device__ __forceinline__ void row_to_regs(const float* p, int nb, float (&pv)[REG_MAX_NB / 32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < REG_MAX_NB / 32; ++i) {
    const int j = lane + 32 * i;
    pv[i] = j < nb ? p[j] : 0.f;
  }
}
__device__ __forceinline__ float mass_above_r(const float (&pv)[REG_MAX_NB / 32], uint32_t u) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < REG_MAX_NB / 32; ++i)
    if (__float_as_uint(pv[i]) > u) s += pv[i];
  return warp_sum(s);
}
__device__ __forceinline__ int count_above_r(const float (&pv)[REG_MAX_NB / 32], uint32_t u) {
  int c = 0;
#pragma unroll
  for (int i = 0; i < REG_MAX_NB / 32; ++i) c += (__float_as_uint(pv[i]) > u) ? 1 : 0;
  return warp_sum_i(c);
}

// The cut of one probability row: keep {bits(p) > thr} plus the first `ties`
// blocks (ascending j) with bits(p) == thr, or every block when `all`; k is
// the clamped budget.
struct Cut {
  uint32_t thr;
  int ties;
  int k;
  bool all;
};

// One warp: the cut of p[0..nb) (shared memory) under Top-p mass tau, or the
// per-block threshold tau when `threshold`, clamped to [kmin, kcap].
__device__ __forceinline__ Cut cut_row(const float* p, int nb, float tau, int threshold, int kmin,
                                       int kcap) {
  uint32_t thr = 0;
  int ties = 0, kstar = 0;
  bool by_mass = false;
  if (threshold) {
    // p >= theta: for theta > 0 the bits order p, so the critical set is
    // {bits(p) > bits(theta) - 1}, a prefix of the (p desc, j asc) order;
    // theta <= 0 keeps every block
    if (tau <= 0.0f) {
      kstar = nb;
    } else {
      thr = __float_as_uint(tau) - 1u;
      kstar = count_above(p, nb, thr);
      by_mass = true;  // the cut is set: the clamp search runs only if it binds
    }
  } else if (tau >= 1.0f) {
    kstar = nb;               // tau >= 1 keeps every block
  } else if (tau > 0.0f) {
    if (nb <= SEARCH32_MAX_NB) {
      thr = search32(0u, 0x3F800000u, [&](uint32_t u) { return mass_above_1(p, nb, u) < tau; });
    } else if (nb <= REG_MAX_NB) {
      float pv[REG_MAX_NB / 32];
      row_to_regs(p, nb, pv);
      uint32_t lo = 0, hi = 0x3F800000u;  // p <= 1, so nothing is above hi
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (mass_above_r(pv, mid) < tau) hi = mid; else lo = mid + 1;
      }
      thr = lo;
    } else {
      uint32_t lo = 0, hi = 0x3F800000u;
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (mass_above(p, nb, mid) < tau) hi = mid; else lo = mid + 1;
      }
      thr = lo;
    }
    // the same summation as the search's predicate
    const float g = nb <= SEARCH32_MAX_NB ? mass_above_1(p, nb, thr) : mass_above(p, nb, thr);
    const int gt = count_above(p, nb, thr);
    const int eq = count_equal(p, nb, thr);
    const float v = __uint_as_float(thr);
    float e = g;
    int keep = 0;
    while (keep < eq && e < tau) { e += v; ++keep; }
    ties = keep;
    kstar = gt + keep;
    by_mass = true;
  }
  const int k = min(max(kstar, kmin), kcap);
  const bool all = (k >= nb);
  if (!all && !(by_mass && k == kstar)) {
    // the clamp binds (or tau <= 0): top-k in (p desc, j asc) order
    if (nb <= SEARCH32_MAX_NB) {
      thr = search32(0u, 0x3F800000u, [&](uint32_t u) { return count_above_1(p, nb, u) < k; });
    } else if (nb <= REG_MAX_NB) {
      float pv[REG_MAX_NB / 32];
      row_to_regs(p, nb, pv);
      uint32_t lo = 0, hi = 0x3F800000u;
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (count_above_r(pv, mid) < k) hi = mid; else lo = mid + 1;
      }
      thr = lo;
    } else {
      uint32_t lo = 0, hi = 0x3F800000u;
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (count_above(p, nb, mid) < k) hi = mid; else lo = mid + 1;
      }
      thr = lo;
    }
    ties = k - count_above(p, nb, thr);
  }
  return Cut{thr, ties, k, all};
}

// One warp: walk the kept blocks of a cut in ascending j, 32 at a time;
// f(j0, keep, km) is called by every lane for the blocks j0 .. j0 + 31
// (keep: this lane's block j0 + lane is kept; km: the warp's ballot of keep).
template <typename F>
__device__ __forceinline__ void walk_kept(const float* p, int nb, const Cut& c, F&& f) {
  const int lane = threadIdx.x & 31;
  int seen_eq = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < nb;
    const uint32_t u = valid ? __float_as_uint(p[j]) : 0u;
    const bool eq = valid && !c.all && u == c.thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = seen_eq + __popc(eqm & ((1u << lane) - 1u));
    seen_eq += __popc(eqm);
    const bool keep = valid && (c.all || u > c.thr || (eq && eq_rank < c.ties));
    const unsigned km = __ballot_sync(0xffffffffu, keep);
    f(j0, keep, km);
  }
}

// One warp: p[0..nb) <- softmax of the logits in p (max-subtracted, expf,
// lane-strided sums reduced by a fixed xor tree, then one division).
__device__ __forceinline__ void softmax_row(float* p, int nb) {
  const int lane = threadIdx.x & 31;
  float mx = -INFINITY;
  for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, p[j]);
  mx = warp_max(mx);
  float sum = 0.f;
  for (int j = lane; j < nb; j += 32) {
    const float e = expf(p[j] - mx);
    p[j] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  for (int j = lane; j < nb; j += 32) p[j] = p[j] / sum;
  __syncwarp();
}

// Threads sharing one key block's dot product in the proxy: each takes a
// strided share of the channels (in float4 steps), then a fixed xor tree adds
// the shares; more threads per block when nb is small.  Every kernel that
// computes a proxy logit uses this split, so the logits agree bit for bit.
__host__ __device__ __forceinline__ int proxy_threads_per_block(int nb) {
  return nb >= 256 ? 1 : (nb >= 128 ? 2 : (nb >= 64 ? 4 : (nb >= 32 ? 8 : 16)));
}

}  // namespace sel
}  // namespace spattn
