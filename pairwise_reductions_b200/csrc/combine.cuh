// combine.cuh -- the fixed order in which split partials are summed.
//
// A pass split over S column ranges leaves S partial sums per output element,
// S apart by `stride`.  They are added in one fixed order, whoever does it (the
// combine kernel, or an epilogue that reads the partials directly): lane l of
// kCombineLanes takes splits l, l + kCombineLanes, ... in turn from 0, then the
// lane sums are added in lane order.  Results therefore do not depend on which
// kernel combined them, or on the timing of a run.
#pragma once
#include <cstdint>

namespace gs {

constexpr int kCombineLanes = 8;

// Lane l's sum (sequential, starting from 0).  A plain loop: the compiler
// keeps several of its loads in flight with few registers (measured faster
// than explicit batches of four or eight loads, whose extra registers cost
// resident warps).
__device__ __forceinline__ float split_lane_sum(const float* __restrict__ p, int lane_l, int splits,
                                                int64_t stride) {
  float s = 0.f;
  for (int k = lane_l; k < splits; k += kCombineLanes) s += p[k * stride];
  return s;
}

// The whole fixed-order sum by one thread: the first kCombineLanes splits are
// loaded together (one per lane sum, so the loads are in flight at once), the
// rest added to their lane sums in turn, then the lane sums in lane order --
// the same operations as split_lane_sum for each lane, then their sum.
__device__ __forceinline__ float split_sum(const float* __restrict__ p, int splits, int64_t stride) {
  float t[kCombineLanes];
#pragma unroll
  for (int l = 0; l < kCombineLanes; ++l) t[l] = (l < splits) ? 0.f + p[l * stride] : 0.f;
#pragma unroll
  for (int l = 0; l < kCombineLanes; ++l)
    for (int k = l + kCombineLanes; k < splits; k += kCombineLanes) t[l] += p[k * stride];
  float s = t[0];
#pragma unroll
  for (int l = 1; l < kCombineLanes; ++l) s += t[l];
  return s;
}

}  // namespace gs
