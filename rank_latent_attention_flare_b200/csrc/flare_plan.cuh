// Length-proportional work plans (calls with sequence lengths on the
// tensor-core path), computed on the device by one block.
//
// With lengths, a chunk plan sized for N leaves the CTAs of short heads idle
// while those of the longest heads set the kernel's time.  The plan sizes
// the work by the tiles each head really has: head bh (cnt tiles) gets
// max(1, ceil(cnt / per)) near-equal units, one CTA each, and `per` is the
// one that minimises  waves x (per + set-up)  among the plans with at most
// 1, 2 or 3 waves of resident CTAs, or the units available.  A plan of two
// kinds is written: the 48-token encode (two CTAs per SM) and the 128-token
// decode and backward passes (one per SM).
//
// The body runs in one block of NT threads: the standalone plan kernel
// (forward), or one extra block of the backward's preparation kernel, which
// runs before every kernel that reads the plan.
#pragma once

#include "flare_internal.cuh"

namespace flare {

struct PlanKind {
  int tile;         // tokens per tile
  int slots;        // CTAs resident at once
  float setup;      // a CTA's set-up, in tiles
  int n;            // units available
  int4* units;      // [n]
  int2* heads;      // [B H]
};

// Everything a plan block needs (lens NULL: no plan to compute; k0.units
// NULL: the encode's plan is not needed, only the 128-token one is written).
struct PlanArgs {
  const int32_t* lens = nullptr;
  int64_t B = 0, H = 0, N = 0;
  PlanKind k0{}, k1{};
  uint32_t* err = nullptr;
  __host__ __device__ bool on() const { return lens != nullptr; }
};

constexpr int kPlanCaps = 4;    // plans of at most 1, 2, 3 waves, and of the units available
constexpr int kPlanWarpB = 32;  // batches up to this size: one lane per batch element

__device__ __forceinline__ int64_t plan_warp_sum64(int64_t v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Units of a head of cnt tiles with `per` tiles per unit at most (a head
// has at least one; tile counts and per stay below 2^31).
__device__ __forceinline__ uint32_t units_of(uint32_t cnt, uint32_t per) {
  return cnt > per ? (cnt + per - 1) / per : 1u;
}

// Units of the plan with `per` tiles per unit at most (a warp's sum; cnt
// holds lane b's tiles when B <= 32, else they are read per element).
__device__ __forceinline__ int64_t plan_units(const int32_t* __restrict__ lens, int64_t B,
                                              int64_t H, int64_t N, int tile, uint32_t cnt,
                                              uint32_t per, int lane) {
  int64_t u = 0;
  if (B <= kPlanWarpB) {
    if (lane < B) u = H * units_of(cnt, per);
  } else {
    for (int64_t b = lane; b < B; b += 32)
      u += H * units_of((uint32_t)tiles_of(seq_len(lens, b, N), tile), per);
  }
  return plan_warp_sum64(u);
}

// Writes head bh's table entry and its c units: cnt tiles split evenly, the
// first cnt mod c units one tile longer.
__device__ __forceinline__ void plan_head(const PlanKind& k, int64_t bh, int64_t first, uint32_t c,
                                          uint32_t cnt) {
  k.heads[bh] = make_int2((int)first, (int)c);
  const uint32_t q = cnt / c, r = cnt % c;
  uint32_t t0 = 0;
  for (uint32_t j = 0; j < c; ++j) {
    const uint32_t len = q + (j < r ? 1u : 0u);
    k.units[first + j] = make_int4((int)bh, (int)t0, (int)len, 0);
    t0 += len;
  }
}

// The plan, computed by the NT threads of one block (every thread calls it;
// NT a multiple of 64, at most 1024).  Also records kErrSeqLen for a length
// outside [0, N].
template <int NT>
__device__ void var_plan_body(const PlanArgs& a) {
  static_assert(NT % 64 == 0 && NT <= 1024, "whole warps, two at least");
  constexpr int NW = NT / 32;
  __shared__ double s_cost[2][kPlanCaps];
  __shared__ int64_t s_per[2][kPlanCaps];
  __shared__ int64_t s_scan[2][NW];
  __shared__ int64_t s_best[2], s_used[2];
  __shared__ int64_t s_first[2][kPlanWarpB];
  __shared__ uint32_t s_c[2][kPlanWarpB], s_cnt[2][kPlanWarpB];
  const int32_t* __restrict__ lens = a.lens;
  const int64_t B = a.B, H = a.H, N = a.N;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t BH = B * H;
  const int kind0 = a.k0.units ? 0 : 1;   // the first kind to plan
  for (int64_t b = tid; b < B; b += NT)
    if (lens[b] < 0 || (int64_t)lens[b] > N) record_error(a.err, kErrSeqLen);

  // one warp per (kind, cap) at a time: the smallest per whose plan fits the cap
  for (int wc = kind0 * kPlanCaps + warp; wc < 2 * kPlanCaps; wc += NW) {
    const int kind = wc / kPlanCaps, ci = wc % kPlanCaps;
    const PlanKind& k = kind ? a.k1 : a.k0;
    const int64_t cap = (ci + 1 < kPlanCaps) ? imin64((int64_t)(ci + 1) * k.slots, k.n) : k.n;
    const uint32_t cnt =
        (B <= kPlanWarpB && lane < B) ? (uint32_t)tiles_of(seq_len(lens, lane, N), k.tile) : 0u;
    double cost = INFINITY;
    int64_t per = 1;
    if (cap >= BH) {
      int64_t total = 0, maxc = 0;
      if (B <= kPlanWarpB) {
        total = H * cnt;
        maxc = cnt;
      } else {
        for (int64_t b = lane; b < B; b += 32) {
          const int64_t c = tiles_of(seq_len(lens, b, N), k.tile);
          total += H * c;
          maxc = imax64(maxc, c);
        }
      }
      total = plan_warp_sum64(total);
      for (int o = 16; o > 0; o >>= 1) maxc = imax64(maxc, __shfl_xor_sync(0xffffffffu, maxc, o));
      // per = max(1, maxc) gives one unit per head (BH <= cap); below
      // ceil(total / cap) no plan fits
      int64_t hi = imax64(1, maxc);
      int64_t lo = imin64(imax64(1, (total + cap - 1) / cap), hi);
      while (lo < hi) {
        const int64_t mid = (lo + hi) / 2;
        if (plan_units(lens, B, H, N, k.tile, cnt, (uint32_t)mid, lane) <= cap)
          hi = mid;
        else
          lo = mid + 1;
      }
      per = lo;
      const int64_t u = plan_units(lens, B, H, N, k.tile, cnt, (uint32_t)per, lane);
      cost = (double)((u + k.slots - 1) / k.slots) * ((double)per + k.setup);
    }
    if (lane == 0) {
      s_cost[kind][ci] = cost;
      s_per[kind][ci] = per;
    }
  }
  __syncthreads();
  if (tid < 2 && tid >= kind0) {
    int best = 0;
    for (int ci = 1; ci < kPlanCaps; ++ci)
      if (s_cost[tid][ci] < s_cost[tid][best]) best = ci;
    s_best[tid] = s_per[tid][best];
  }
  __syncthreads();

  if (B <= kPlanWarpB) {
    // warp k scans kind k over the batch (lane b: batch element b); then
    // every thread writes heads, one (kind, head) at a time
    if (warp < 2 && warp >= kind0) {
      const PlanKind& k = warp ? a.k1 : a.k0;
      const uint32_t cnt = lane < B ? (uint32_t)tiles_of(seq_len(lens, lane, N), k.tile) : 0u;
      const uint32_t c = units_of(cnt, (uint32_t)s_best[warp]);
      const int64_t mine = lane < B ? H * c : 0;
      int64_t incl = mine;
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      s_first[warp][lane] = incl - mine;
      s_c[warp][lane] = c;
      s_cnt[warp][lane] = cnt;
      if (lane == 31) s_used[warp] = incl;
    }
    __syncthreads();
    for (int64_t x = kind0 * BH + tid; x < 2 * BH; x += NT) {
      const int kind = x >= BH;
      const int64_t bh = x - (kind ? BH : 0), b = bh / H, h = bh % H;
      const uint32_t c = s_c[kind][b];
      plan_head(kind ? a.k1 : a.k0, bh, s_first[kind][b] + h * c, c, s_cnt[kind][b]);
    }
  } else {
    // both kinds at once: an exclusive scan over the batch of H units(b),
    // each thread taking a contiguous run of batch elements
    const int64_t run = (B + NT - 1) / NT;
    const int64_t b0 = imin64((int64_t)tid * run, B), b1 = imin64(b0 + run, B);
    int64_t mine[2] = {0, 0}, incl[2] = {0, 0};
    for (int kind = kind0; kind < 2; ++kind) {
      const PlanKind& k = kind ? a.k1 : a.k0;
      for (int64_t b = b0; b < b1; ++b)
        mine[kind] += H * units_of((uint32_t)tiles_of(seq_len(lens, b, N), k.tile),
                                   (uint32_t)s_best[kind]);
      incl[kind] = mine[kind];
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, incl[kind], o);
        if (lane >= o) incl[kind] += v;
      }
      if (lane == 31) s_scan[kind][warp] = incl[kind];
    }
    __syncthreads();
    if (warp < 2 && warp >= kind0) {
      const int64_t t = lane < NW ? s_scan[warp][lane] : 0;
      int64_t ti = t;
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t v = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) ti += v;
      }
      if (lane < NW) s_scan[warp][lane] = ti - t;   // exclusive over the warps
      if (lane == NW - 1) s_used[warp] = ti;
    }
    __syncthreads();
    for (int kind = kind0; kind < 2; ++kind) {
      const PlanKind& k = kind ? a.k1 : a.k0;
      const uint32_t per = (uint32_t)s_best[kind];
      int64_t first = s_scan[kind][warp] + incl[kind] - mine[kind];
      for (int64_t b = b0; b < b1; ++b) {
        const uint32_t cnt = (uint32_t)tiles_of(seq_len(lens, b, N), k.tile);
        const uint32_t c = units_of(cnt, per);
        for (int64_t h = 0; h < H; ++h) plan_head(k, b * H + h, first + h * c, c, cnt);
        first += H * c;
      }
    }
  }
  __syncthreads();
  // the units past the plan's stay empty
  for (int kind = kind0; kind < 2; ++kind) {
    const PlanKind& k = kind ? a.k1 : a.k0;
    for (int64_t u = s_used[kind] + tid; u < k.n; u += NT) k.units[u] = make_int4(-1, 0, 0, 0);
  }
}

// Launches the standalone plan kernel for a plan whose block no other
// kernel runs (no-op when !a.on()).
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t st);

}  // namespace flare
