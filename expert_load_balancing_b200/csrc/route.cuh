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
//  2. candidates: the elements with score >= T (a few percent of the row),
//     compacted to at most one per lane through a per-warp buffer;
//  3. K+1 rounds: the warp maximum key (redux.sync), ties to the lowest id
//     (a second redux.sync); the owning lane records its rank and drops out.
// Scores are compared as order-preserving keys in step 3; steps 1-2 use
// plain float compares, which only ever admit extra candidates.  Rows with
// more than 32 candidates (heavy ties) take a slower exact path in which
// each round's owner rescans its own candidates.
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

template <int Q, bool kFull>
__device__ __forceinline__ void load_row(const float* __restrict__ zrow, int E, int lane,
                                         float (&z)[4 * Q]) {
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    const int e0 = 128 * q + 4 * lane;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kFull || e0 < E) v = __ldg(reinterpret_cast<const float4*>(zrow + e0));
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
  for (int size = 2 * stride_lo; size <= 32; size <<= 1) {
    for (int stride = size >> 1; stride >= stride_lo; stride >>= 1) {
      const float o = __shfl_xor_sync(full, v, stride);
      const bool up = ((lane & size) == 0);
      const bool lower = ((lane & stride) == 0);
      v = (lower == up) ? fmaxf(v, o) : fminf(v, o);
    }
  }
  return __shfl_sync(full, v, K * stride_lo);
}

template <bool kBias>
__device__ __forceinline__ float b_of(float z, const float* __restrict__ beta_s, uint32_t e) {
  return kBias ? __fadd_rn(z, beta_s[e]) : z;
}

// Per-warp shared scratch used by the selection.
template <int Q>
struct RowScratch {
  float row[128 * Q];   // this row's raw logits, lane-major
  uint32_t ckey[32];    // compacted candidates: key and expert id
  uint32_t cid[32];
};

// Exact top-(K+1) of one row.  z: this lane's raw logits; beta_s: beta in
// shared memory (ignored without kBias).  On return:
//   rank   = r if this lane holds the r-th best (r <= K), else -1
//   key/id = that element's order key and expert id (rank >= 0)
// except on the slow path (over 32 candidates), where lane r holds the r-th
// best instead (rank = r for lanes r <= K).
template <int Q, bool kFull, bool kBias>
__device__ __forceinline__ void warp_select_row(const float (&z)[4 * Q],
                                                const float* __restrict__ beta_s, uint32_t valid,
                                                int K, int lane, RowScratch<Q>& sc, int& rank,
                                                uint32_t& key, uint32_t& id) {
  constexpr int V = 4 * Q;
  float b[V];
  float lane_max = -INFINITY;
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    float4 bq = make_float4(0.f, 0.f, 0.f, 0.f);
    if (kBias && (kFull || (valid & (1u << (4 * q)))))
      bq = *reinterpret_cast<const float4*>(&beta_s[128 * q + 4 * lane]);
    const float bv[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 4 * q + i;
      b[j] = kBias ? __fadd_rn(z[j], bv[i]) : z[j];
      if (kFull || (valid & (1u << j))) lane_max = fmaxf(lane_max, b[j]);
    }
  }
  const float T = threshold_from_groups(lane_max, K);
  uint32_t cand = 0u;
#pragma unroll
  for (int j = 0; j < V; ++j) cand |= (b[j] >= T) ? (1u << j) : 0u;
  if (!kFull) cand &= valid;
  __syncwarp();
#pragma unroll
  for (int q = 0; q < Q; ++q)
    *reinterpret_cast<float4*>(&sc.row[lane * V + 4 * q]) =
        make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
  const int c = __popc(cand);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  rank = -1;
  key = 0u;
  id = kNoId;
  if (total <= 32) {
    // ---- compact to at most one candidate per lane
    int pos = incl - c;
    uint32_t m = cand;
    while (m) {
      const int j = __ffs(m) - 1;
      m &= m - 1u;
      const uint32_t e = slot_expert(lane, j);
      const float bb = b_of<kBias>(sc.row[lane * V + j], beta_s, e);
      sc.ckey[pos] = order_key(bb);
      sc.cid[pos] = e;
      ++pos;
    }
    __syncwarp();
    uint32_t k = lane < total ? sc.ckey[lane] : 0u;
    uint32_t i = lane < total ? sc.cid[lane] : kNoId;
    for (int r = 0; r <= K; ++r) {
      const uint32_t M = __reduce_max_sync(0xffffffffu, k);
      const uint32_t mine = (k == M) ? i : kNoId;
      const uint32_t I = __reduce_min_sync(0xffffffffu, mine);
      if (i == I && I != kNoId) {  // the owner (ids are distinct)
        rank = r;
        key = k;
        id = i;
        k = 0u;
        i = kNoId;
      }
    }
  } else {
    // ---- heavy ties: K+1 rounds in which each owner rescans its candidates
    __syncwarp();
    auto lane_best = [&](uint32_t mm, uint32_t& bk, uint32_t& bid) {
      bk = 0u;
      bid = kNoId;
      while (mm) {
        const int j = __ffs(mm) - 1;
        mm &= mm - 1u;
        const uint32_t e = slot_expert(lane, j);
        const uint32_t kk = order_key(b_of<kBias>(sc.row[lane * V + j], beta_s, e));
        if (kk > bk) {  // slots ascend in id: strict '>' keeps the lower id
          bk = kk;
          bid = e;
        }
      }
    };
    uint32_t bk, bid;
    lane_best(cand, bk, bid);
    for (int r = 0; r <= K; ++r) {
      const uint32_t M = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t mine = (bk == M) ? bid : kNoId;
      const uint32_t I = __reduce_min_sync(0xffffffffu, mine);
      if (lane == r) {
        rank = r;
        key = M;
        id = I;
      }
      if (bid == I && I != kNoId) {
        cand &= ~(1u << (4 * static_cast<int>(I >> 7) + static_cast<int>(I & 3)));
        lane_best(cand, bk, bid);
      }
    }
  }
}

}  // namespace kolibri
