// route.cuh -- warp-per-token selection on one row of logits.
//
// Method ("Kolibri Pre-Training from Scratch", section 6.1 routing
// equations, section 7.1 token bias; "Kolibri 1 im Detail", routing steps):
//   B_t,e   = Z_t,e + beta_e                 (fp32, round to nearest even)
//   I_t     = the K largest B_t,e            (ties: lower expert id first)
//   alpha_t = -(the (K+1)-th largest B_t,e)  (= -Q_K(Z_t,: + beta))
//
// Layout: one warp owns one row.  Lane l holds experts
//   e = 128*q + 4*l + i,  q = 0..Q-1, i = 0..3   (slot j = 4q + i)
// loaded as Q float4 vectors (each warp-wide load is 512 contiguous bytes).
//
// Selection in three steps, exact for every input:
//  1. threshold: the lanes are cut into G groups (G >= K+1); each group's
//     maximum is a distinct element, so the (K+1)-th largest group maximum T
//     (or the smallest one when G = 8) is a lower bound of the (K+1)-th
//     largest score: any element below T is beaten by at least K+1 others;
//  2. candidates: the elements with score >= T (usually ~3% of the row);
//  3. K+1 rounds over candidates only: the warp maximum key (redux.sync),
//     ties to the lowest id (a second redux.sync); the owning lane drops that
//     candidate and rescans its own few candidates.
// Scores are compared as order-preserving keys in step 3; steps 1-2 use
// plain float compares, which only ever admit extra candidates.
#pragma once

#include "common.cuh"

namespace kolibri {

constexpr uint32_t kNoId = 0xffffffffu;

__device__ __forceinline__ uint32_t slot_expert(int lane, int j) {
  return static_cast<uint32_t>(128 * (j >> 2) + 4 * lane + (j & 3));
}

// Lane-major position of expert e's value in a row buffer laid out as
// buf[lane * 4Q + j].
template <int Q>
__device__ __forceinline__ int buffer_pos(uint32_t e) {
  const int q = static_cast<int>(e >> 7), r = static_cast<int>(e & 127);
  return (r >> 2) * (4 * Q) + 4 * q + (r & 3);
}

template <int Q>
__device__ __forceinline__ void load_row(const float* __restrict__ zrow, int E, int lane,
                                         float (&z)[4 * Q]) {
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    int e0 = 128 * q + 4 * lane;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e0 < E) v = __ldg(reinterpret_cast<const float4*>(zrow + e0));
    z[4 * q + 0] = v.x;
    z[4 * q + 1] = v.y;
    z[4 * q + 2] = v.z;
    z[4 * q + 3] = v.w;
  }
}

// Float lower bound T of the (K+1)-th largest of the lanes' values.
// lane_max is this lane's maximum (-inf if it holds no expert).
__device__ __forceinline__ float threshold_from_groups(float lane_max, int K) {
  const unsigned full = 0xffffffffu;
  if (K + 1 <= 8) {
    // 8 groups of 4 lanes; T = smallest group maximum
    float g = fmaxf(lane_max, __shfl_xor_sync(full, lane_max, 1));
    g = fmaxf(g, __shfl_xor_sync(full, g, 2));
    float t = fminf(g, __shfl_xor_sync(full, g, 4));
    t = fminf(t, __shfl_xor_sync(full, t, 8));
    t = fminf(t, __shfl_xor_sync(full, t, 16));
    return t;
  }
  // 16 groups of 2 lanes (K+1 <= 16) or 32 groups of 1 lane: bitonic sort of
  // the group maxima across lanes (descending), then take the (K+1)-th.
  const int lane = threadIdx.x & 31;
  float v = lane_max;
  int stride_lo = 1;
  if (K + 1 <= 16) {
    v = fmaxf(v, __shfl_xor_sync(full, v, 1));
    stride_lo = 2;  // lanes 2g, 2g+1 hold group g
  }
  // sort over the lane bits >= stride_lo, descending in the group index
  for (int size = 2 * stride_lo; size <= 32; size <<= 1) {
    for (int stride = size >> 1; stride >= stride_lo; stride >>= 1) {
      float o = __shfl_xor_sync(full, v, stride);
      bool up = ((lane & size) == 0);          // descending blocks
      bool lower = ((lane & stride) == 0);
      bool take_max = (lower == up);
      v = take_max ? fmaxf(v, o) : fminf(v, o);
    }
  }
  return __shfl_sync(full, v, K * stride_lo);
}

}  // namespace kolibri
