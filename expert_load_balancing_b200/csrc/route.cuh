// route.cuh -- warp-per-token selection on one row of logits.
//
// Method ("Kolibri Pre-Training from Scratch", section 6.1 routing
// equations, section 7.1 token bias; "Kolibri 1 im Detail", routing steps):
//   B_t,e   = Z_t,e + beta_e                 (fp32, round to nearest even)
//   I_t     = the K largest B_t,e            (ties: lower expert id first)
//   alpha_t = -(the (K+1)-th largest B_t,e)  (= -Q_K(Z_t,: + beta))
//
// Layout: one warp owns one row.  Lane l holds experts
//   e = 128*q + 4*l + i,  q = 0..Q-1, i = 0..3
// loaded as Q float4 vectors (each warp-wide load is 512 contiguous bytes).
//
// Selection: each lane keeps the two best (key, slot) of its own values.
// Round r (r = 0..K) takes the warp maximum key with one redux.sync, breaks
// ties with a redux.sync minimum over expert ids, and the owning lane pops
// its head.  A lane popped a second time rescans its values below the last
// popped (key, id) to refill its two best, so every round is exact.  After
// K+1 rounds lane r holds the r-th (key, id) of the row.
#pragma once

#include "common.cuh"

namespace kolibri {

constexpr uint32_t kNoId = 0xffffffffu;

template <int Q>
struct RowSlots {
  float z[4 * Q];       // raw logits (0 for slots past E)
  uint32_t key[4 * Q];  // order key of z + beta (0 = absent; finite scores never map to 0)
};

__device__ __forceinline__ uint32_t slot_expert(int lane, int j) {
  return static_cast<uint32_t>(128 * (j >> 2) + 4 * lane + (j & 3));
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

// Biased keys of one row.  beta_lane holds beta for this lane's slots (or
// nothing when has_bias is false: then B = Z exactly).
template <int Q>
__device__ __forceinline__ void row_keys(const float (&z)[4 * Q], const float (&beta_lane)[4 * Q],
                                         bool has_bias, int E, int lane, uint32_t (&key)[4 * Q]) {
#pragma unroll
  for (int j = 0; j < 4 * Q; ++j) {
    float b = has_bias ? __fadd_rn(z[j], beta_lane[j]) : z[j];
    key[j] = (static_cast<int>(slot_expert(lane, j)) < E) ? order_key(b) : 0u;
  }
}

// Two best (key desc, id asc) among this lane's slots that rank strictly
// below (below_key, below_id) in that order.  Pass below_key = ~0u and
// below_id = kNoId... for "no bound" use has_bound = false.
template <int Q>
__device__ __forceinline__ void lane_top2(const uint32_t (&key)[4 * Q], int lane, bool has_bound,
                                          uint32_t below_key, uint32_t below_id, uint32_t& k1,
                                          int& j1, uint32_t& k2, int& j2) {
  k1 = 0u;
  j1 = -1;
  k2 = 0u;
  j2 = -1;
#pragma unroll
  for (int j = 0; j < 4 * Q; ++j) {
    uint32_t k = key[j];
    bool ok = k != 0u;
    if (has_bound) {
      uint32_t e = slot_expert(lane, j);
      ok = ok && (k < below_key || (k == below_key && e > below_id));
    }
    // slots ascend in expert id inside a lane, so strict '>' keeps the
    // lower id ahead on equal keys
    bool gt1 = ok && k > k1;
    bool gt2 = ok && k > k2;
    k2 = gt1 ? k1 : (gt2 ? k : k2);
    j2 = gt1 ? j1 : (gt2 ? j : j2);
    k1 = gt1 ? k : k1;
    j1 = gt1 ? j : j1;
  }
}

// Exact top-(K+1) of the row.  On return lane r (r <= K) holds the r-th
// best key in out_key and its expert id in out_id; other lanes hold junk.
template <int Q>
__device__ __forceinline__ void warp_topk(const uint32_t (&key)[4 * Q], int K, int lane,
                                          uint32_t& out_key, uint32_t& out_id) {
  uint32_t k1, k2;
  int j1, j2;
  lane_top2<Q>(key, lane, false, 0u, 0u, k1, j1, k2, j2);
  bool second_known = true;  // k2/j2 valid
  out_key = 0u;
  out_id = kNoId;
  for (int r = 0; r <= K; ++r) {
    uint32_t M = __reduce_max_sync(0xffffffffu, k1);
    uint32_t my_id = (k1 == M && j1 >= 0) ? slot_expert(lane, j1) : kNoId;
    uint32_t I = __reduce_min_sync(0xffffffffu, my_id);
    if (lane == r) {
      out_key = M;
      out_id = I;
    }
    if (my_id == I) {  // exactly one owner: ids are distinct
      if (second_known) {
        k1 = k2;
        j1 = j2;
        second_known = false;
      } else {
        lane_top2<Q>(key, lane, true, M, I, k1, j1, k2, j2);
        second_known = true;
      }
    }
  }
}

}  // namespace kolibri
