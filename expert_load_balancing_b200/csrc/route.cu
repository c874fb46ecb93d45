// route.cu -- row-wise kernels over the logits Z [N, E] fp32:
//   * selection: bias add, top-K ids, sigmoid gates, token bias alpha
//     ("Kolibri Pre-Training from Scratch" 6.1 and 7.1; "Kolibri 1 im
//     Detail", routing steps 1-2);
//   * the two row passes of the exact EQB quantile (7.1, 7.3): the keys of
//     Z + alpha at sampled rows, and the full pass that counts keys above a
//     per-expert bracket and gathers the keys inside it.  The full pass can
//     run inside the selection kernel, so Z is streamed from HBM once for
//     routing and balancing together.
//
// One warp per row (see route.cuh for the selection); each block runs its
// warps over consecutive rows and stages bracketed keys in shared memory,
// flushing them to the per-expert gather buffer once per batch of rows with
// one global atomic per expert.
#include "launch.h"
#include "route.cuh"
#include "pdl.cuh"

namespace kolibri {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / kWarp;
constexpr int kRowsPerWarp = 32;     // most rows per warp between gather flushes
constexpr int kStageSlots = 16;      // staged bracket keys per expert per block
constexpr int kRowPrefetch = 2;      // rows ahead that the EQB pass prefetches into L2

struct RouteParams {
  const float* z;
  const float* beta;  // may be null
  int64_t N;
  int E, K;
  int rows_per_warp;  // 1 .. kRowsPerWarp: small batches spread one row per warp
  // selection outputs
  int32_t* ids;
  float* gates;
  float* alpha_out;
  const float* alpha_in;
  // bracketed full pass
  const uint32_t* lo;
  const uint32_t* hi;
  uint32_t* above;
  uint32_t* cand_cnt;
  uint32_t* cand;
  int64_t cap;
};

template <int Q>
struct WarpScratch {
  RowScratch<Q> sel;    // selection scratch (row buffer, compacted candidates)
  float gz[32];         // gate inputs waiting for a batched evaluation
  uint32_t gidx[32];    // their output positions
};

// Shared-memory layout (dynamic): beta[E] | lo[E] | hi[E] | above[E] |
// stage_n[E] | stage[E][kStageSlots] | WarpScratch[kWarps]
struct SmemLayout {
  int off_beta, off_lo, off_hi, off_above, off_stage_n, off_stage, off_warp, total;
};

template <int Q, bool kWindow>
__host__ __device__ SmemLayout smem_layout(int E) {
  SmemLayout L;
  int o = 0;
  L.off_beta = o;
  o += 4 * E;
  const int w = kWindow ? 1 : 0;
  L.off_lo = o;
  o += 4 * E * w;
  L.off_hi = o;
  o += 4 * E * w;
  L.off_above = o;
  o += 4 * E * w;
  L.off_stage_n = o;
  o += 4 * E * w;
  L.off_stage = o;
  o += 4 * E * kStageSlots * w;
  o = (o + 15) & ~15;
  L.off_warp = o;
  o += static_cast<int>(sizeof(WarpScratch<Q>)) * kWarps;
  L.total = o;
  return L;
}

// Evaluate the staged gates (lanes < n) and store them.
__device__ __forceinline__ void flush_gates(float* __restrict__ gates, const float* gz,
                                            const uint32_t* gidx, int n, int lane) {
  if (lane < n) gates[gidx[lane]] = gate_sigmoid(gz[lane]);
}

// Append one bracketed key of expert e: block staging, or the global gather
// buffer directly when the block's slots for e are full.
__device__ __forceinline__ void stage_bracket_key(uint32_t e, uint32_t k, uint32_t* stage_n,
                                                  uint32_t* stage, uint32_t* __restrict__ cand_cnt,
                                                  uint32_t* __restrict__ cand, int64_t cap) {
  const uint32_t pos = atomicAdd(&stage_n[e], 1u);
  if (pos < kStageSlots) {
    stage[e * kStageSlots + pos] = k;
  } else {
    const uint32_t g = atomicAdd(cand_cnt + e, 1u);
    if (g < cap) cand[static_cast<int64_t>(e) * cap + g] = k;
  }
}

template <int Q, bool kFull, bool kBias, bool kRoute, bool kAlphaOut, bool kAlphaIn, bool kWindow>
__global__ void __launch_bounds__(kThreads, kAlphaIn ? 4 : 3) route_rows_kernel(const RouteParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int V = 4 * Q;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E = p.E, K = p.K;
  const SmemLayout L = smem_layout<Q, kWindow>(E);
  float* beta_s = reinterpret_cast<float*>(smem + L.off_beta);
  uint32_t* lo_s = reinterpret_cast<uint32_t*>(smem + L.off_lo);
  uint32_t* hi_s = reinterpret_cast<uint32_t*>(smem + L.off_hi);
  uint32_t* above_s = reinterpret_cast<uint32_t*>(smem + L.off_above);
  uint32_t* stage_n = reinterpret_cast<uint32_t*>(smem + L.off_stage_n);
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem + L.off_stage);
  WarpScratch<Q>& ws = reinterpret_cast<WarpScratch<Q>*>(smem + L.off_warp)[warp];
  pdl_wait();       // Z comes from the kernel before this one
  pdl_trigger();

  for (int e = threadIdx.x; e < E; e += kThreads) {
    if constexpr (kBias) beta_s[e] = p.beta[e];
    if constexpr (kWindow) {
      // the bracket as fp32 values: the order key is monotone in the value
      // except that it puts -0 below +0, so against a nonzero bound a float
      // compare decides exactly what the key compare would
      lo_s[e] = __float_as_uint(key_to_float(p.lo[e]));
      hi_s[e] = __float_as_uint(key_to_float(p.hi[e]));
      above_s[e] = 0u;
      stage_n[e] = 0u;
    }
  }
  __syncthreads();

  uint32_t valid = 0u;  // this lane's slots that hold an expert
#pragma unroll
  for (int j = 0; j < V; ++j) valid |= (static_cast<int>(slot_expert(lane, j)) < E) ? (1u << j) : 0u;
  int gate_n = 0;
  // a lane whose brackets include a zero bound compares keys (the exact -0 < +0 order)
  bool zero_bound = false;
  if constexpr (kWindow) {
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (!kFull && !(valid & (1u << j))) continue;
      const uint32_t e = slot_expert(lane, j);
      zero_bound |= (__uint_as_float(hi_s[e]) == 0.f) || (__uint_as_float(lo_s[e]) == 0.f);
    }
  }

  const int64_t rows_per_block = static_cast<int64_t>(kWarps) * p.rows_per_warp;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * rows_per_block; base < p.N;
       base += static_cast<int64_t>(gridDim.x) * rows_per_block) {
    const int64_t r0 = base + static_cast<int64_t>(warp) * p.rows_per_warp;
    const int64_t r1 = (r0 + p.rows_per_warp < p.N) ? r0 + p.rows_per_warp : p.N;
    // per-lane counts of keys above the bracket, one byte per slot (<= 32 rows per batch)
    uint32_t above_b[kWindow ? Q : 1];
    if constexpr (kWindow) {
#pragma unroll
      for (int q = 0; q < Q; ++q) above_b[q] = 0u;
    }
    float znext[V];
    float anext = 0.f;
    if (r0 < r1) {
      load_row<Q, kFull>(p.z + r0 * E, E, lane, znext);
      if constexpr (kAlphaIn) anext = __ldg(p.alpha_in + r0);
    }
    for (int64_t row = r0; row < r1; ++row) {
      float z[V];
#pragma unroll
      for (int j = 0; j < V; ++j) z[j] = znext[j];
      const float acur = anext;
      if (row + 1 < r1) {
        load_row<Q, kFull>(p.z + (row + 1) * E, E, lane, znext);
        if constexpr (kAlphaIn) anext = __ldg(p.alpha_in + row + 1);
      }
      if constexpr (kWindow && kAlphaIn) {
        // the EQB pass streams Z once: the row after next goes to L2 now
        // (one prefetch per 128-byte line), so each warp has three rows in
        // flight while holding only two in registers
        if (row + kRowPrefetch < r1 && (lane & 7) == 0) {
          const float* pr = p.z + (row + kRowPrefetch) * E;
#pragma unroll
          for (int q = 0; q < Q; ++q)
            if (kFull || 128 * q + 4 * lane < E)
              asm volatile("prefetch.global.L2 [%0];" ::"l"(pr + 128 * q + 4 * lane));
        }
      }

      float alpha;
      if constexpr (!kAlphaIn) {
        int rank;
        uint32_t key, id;
        warp_select_row<Q, kFull, kBias>(z, beta_s, valid, K, lane, ws.sel, rank, key, id);
        const uint32_t kth = __ballot_sync(0xffffffffu, rank == K);
        alpha = -key_to_float(__shfl_sync(0xffffffffu, key, __ffs(kth) - 1));
        if constexpr (kRoute) {
          if (rank >= 0 && rank < K) {
            // id < E for finite inputs; clamp so no input can index outside
            const uint32_t e = id < static_cast<uint32_t>(E) ? id : 0u;
            p.ids[row * K + rank] = static_cast<int32_t>(id);
            ws.gz[gate_n + rank] = ws.sel.row[buffer_pos<Q>(e)];
            ws.gidx[gate_n + rank] = static_cast<uint32_t>(row * K + rank);
          }
          gate_n += K;
          if (gate_n + K > 32) {
            __syncwarp();
            flush_gates(p.gates, ws.gz, ws.gidx, gate_n, lane);
            gate_n = 0;
          }
        }
        if constexpr (kAlphaOut) {
          if (lane == 0) p.alpha_out[row] = alpha;
        }
        __syncwarp();
      } else {
        alpha = acur;
      }

      if constexpr (kWindow) {
        uint32_t wmask = 0u;
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          if (!kFull && !(valid & (1u << (4 * q)))) continue;
          const int e0 = 128 * q + 4 * lane;
          const float4 hq = *reinterpret_cast<const float4*>(&hi_s[e0]);
          const float4 lq = *reinterpret_cast<const float4*>(&lo_s[e0]);
          const float hv[4] = {hq.x, hq.y, hq.z, hq.w};
          const float lv[4] = {lq.x, lq.y, lq.z, lq.w};
          if (!zero_bound) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float f = __fadd_rn(z[4 * q + i], alpha);
              const bool ab = f > hv[i];
              above_b[q] += ab ? (1u << (8 * i)) : 0u;
              wmask |= (!ab && f >= lv[i]) ? (1u << (4 * q + i)) : 0u;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t k = order_key(__fadd_rn(z[4 * q + i], alpha));
              const bool ab = k > order_key(hv[i]);
              above_b[q] += ab ? (1u << (8 * i)) : 0u;
              wmask |= (!ab && k >= order_key(lv[i])) ? (1u << (4 * q + i)) : 0u;
            }
          }
        }
        while (wmask) {  // rare: keys inside the bracket
          const int j = __ffs(wmask) - 1;
          wmask &= wmask - 1u;
          const uint32_t e = slot_expert(lane, j);
          const uint32_t k = order_key(__fadd_rn(__ldg(p.z + row * E + e), alpha));
          stage_bracket_key(e, k, stage_n, stage, p.cand_cnt, p.cand, p.cap);
        }
      }
    }
    if constexpr (kWindow) {
#pragma unroll
      for (int q = 0; q < Q; ++q) {
        if (above_b[q] == 0u) continue;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t n = (above_b[q] >> (8 * i)) & 0xffu;
          if (n) atomicAdd(&above_s[128 * q + 4 * lane + i], n);
        }
      }
      __syncthreads();
      for (int e = threadIdx.x; e < E; e += kThreads) {
        uint32_t n = stage_n[e];
        if (n > kStageSlots) n = kStageSlots;
        if (n) {
          const uint32_t g = atomicAdd(p.cand_cnt + e, n);
          for (uint32_t i = 0; i < n; ++i)
            if (g + i < p.cap) p.cand[static_cast<int64_t>(e) * p.cap + g + i] = stage[e * kStageSlots + i];
        }
        stage_n[e] = 0u;
      }
      __syncthreads();
    }
  }
  if constexpr (kRoute) {
    __syncwarp();
    flush_gates(p.gates, ws.gz, ws.gidx, gate_n, lane);
  }
  if constexpr (kWindow) {
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads)
      if (above_s[e] != 0u) atomicAdd(p.above + e, above_s[e]);
  }
}

// Keys of Z + alpha at sampled rows t = s * stride, written expert-major:
// sample[e * S + s].  A block handles 32 consecutive samples and transposes
// them through shared memory so every expert row is written in 128-byte runs.
// zero_word (nullable) is cleared by block 0 for the kernels after this one.
constexpr int kSampleRows = 32;

template <int Q, bool kAlphaIn, bool kBias>
__global__ void __launch_bounds__(kThreads) sample_keys_kernel(
    const float* __restrict__ z, const float* __restrict__ alpha_in, const float* __restrict__ beta,
    int64_t N, int E, int K, int64_t S, int64_t stride, int64_t S_ld,
    uint32_t* __restrict__ sample, uint32_t* __restrict__ zero_word) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int V = 4 * Q;
  const int ld = E + 1;
  uint32_t* tile = reinterpret_cast<uint32_t*>(smem);  // [kSampleRows][E + 1]
  float* beta_s = reinterpret_cast<float*>(smem + ((4 * kSampleRows * ld + 15) & ~15));
  RowScratch<Q>* scr = reinterpret_cast<RowScratch<Q>*>(
      smem + ((4 * kSampleRows * ld + 15) & ~15) + ((4 * E + 15) & ~15));
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t s0 = static_cast<int64_t>(blockIdx.x) * kSampleRows;
  pdl_wait();       // Z and alpha come from the kernels before this one
  pdl_trigger();
  if (zero_word != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0u;
  if constexpr (kBias) {
    for (int e = threadIdx.x; e < E; e += kThreads) beta_s[e] = beta[e];
  }
  __syncthreads();
  uint32_t valid = 0u;
#pragma unroll
  for (int j = 0; j < V; ++j) valid |= (static_cast<int>(slot_expert(lane, j)) < E) ? (1u << j) : 0u;

  if constexpr (kAlphaIn) {
    // the warp's rows r = warp + kWarps i: every load issued before the first
    // use, one memory round trip
    constexpr int kPerWarp = kSampleRows / kWarps;
    float zv[kPerWarp][V];
    float al[kPerWarp];
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
      const int64_t s = s0 + warp + kWarps * i;
      al[i] = 0.f;
      if (s < S) {
        const int64_t row = s * stride;
        load_row<Q, false>(z + row * E, E, lane, zv[i]);
        al[i] = __ldg(alpha_in + row);
      }
    }
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
      const int r = warp + kWarps * i;
      if (s0 + r >= S) break;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int e = static_cast<int>(slot_expert(lane, j));
        if (e < E) tile[r * ld + e] = order_key(__fadd_rn(zv[i][j], al[i]));
      }
    }
  } else
  for (int r = warp; r < kSampleRows; r += kWarps) {
    const int64_t s = s0 + r;
    if (s >= S) break;
    const int64_t row = s * stride;
    float zv[V];
    load_row<Q, false>(z + row * E, E, lane, zv);
    float alpha;
    if constexpr (kAlphaIn) {
      alpha = __ldg(alpha_in + row);
    } else {
      int rank;
      uint32_t key, id;
      warp_select_row<Q, false, kBias>(zv, beta_s, valid, K, lane, scr[warp], rank, key, id);
      const uint32_t kth = __ballot_sync(0xffffffffu, rank == K);
      alpha = -key_to_float(__shfl_sync(0xffffffffu, key, __ffs(kth) - 1));
      __syncwarp();
    }
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int e = static_cast<int>(slot_expert(lane, j));
      if (e < E) tile[r * ld + e] = order_key(__fadd_rn(zv[j], alpha));
    }
  }
  __syncthreads();
  const int64_t rows_here = (S - s0) < kSampleRows ? (S - s0) : kSampleRows;
  for (int i = threadIdx.x; i < E * kSampleRows; i += kThreads) {
    const int e = i / kSampleRows, r = i % kSampleRows;
    if (r < rows_here) sample[static_cast<int64_t>(e) * S_ld + s0 + r] = tile[r * ld + e];
  }
}

// Rows left unfinished by the fused logits + selection kernel carry a NaN
// alpha (more candidates than its per-row buffer holds).  One warp checks 32
// rows at a time and runs the exact row selection on each marked row.
template <int Q, bool kFull, bool kBias>
__global__ void __launch_bounds__(kThreads) select_fixup_kernel(
    const float* __restrict__ z, const float* __restrict__ beta, int64_t N, int E, int K,
    int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ alpha) {
  __shared__ __align__(16) float beta_s[128 * Q];
  __shared__ RowScratch<Q> scratch[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < 128 * Q; e += kThreads) beta_s[e] = (kBias && e < E) ? beta[e] : 0.f;
  __syncthreads();
  uint32_t valid = 0u;
#pragma unroll
  for (int j = 0; j < 4 * Q; ++j) valid |= (static_cast<int>(slot_expert(lane, j)) < E) ? (1u << j) : 0u;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kWarps * 32;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * 32; base < N; base += step) {
    const int64_t t = base + lane;
    uint32_t m = __ballot_sync(0xffffffffu, t < N && isnan(alpha[t]));
    while (m) {
      const int i = __ffs(m) - 1;
      m &= m - 1u;
      const int64_t row = base + i;
      float zr[4 * Q];
      load_row<Q, kFull>(z + row * E, E, lane, zr);
      int rank;
      uint32_t key, id;
      warp_select_row<Q, kFull, kBias>(zr, beta_s, valid, K, lane, scratch[warp], rank, key, id);
      if (rank >= 0 && rank < K) {
        const uint32_t e = id < static_cast<uint32_t>(E) ? id : 0u;
        ids[row * K + rank] = static_cast<int32_t>(id);
        gates[row * K + rank] = gate_sigmoid(scratch[warp].row[buffer_pos<Q>(e)]);
      }
      if (rank == K) alpha[row] = -key_to_float(key);
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------
// Selection alone over large batches: eight lanes per row, four rows per warp.
//
// The same exact rule as warp_select_row (top K + 1 of B = Z + beta by order
// key, ties to the lower expert id), laid out so that the warp-wide steps
// serve four rows at once.  Lane s of a row's segment holds the C = E / 32
// chunks c = 8 i + s (columns 32 i + 4 s .. + 3), loaded as float4.
//  1. threshold: the lanes cut their chunks into GPL groups (24 or 32
//     groups per row); K + 1 rounds of a segment-wide maximum over the lanes'
//     sorted group maxima, each round removing the maximum from every lane
//     that holds it.  After the last round at least K + 1 distinct elements
//     (group maxima) are >= its value T, so T is at most the (K+1)-th
//     largest score, and only a few scores per row reach it;
//  2. candidates (scores >= T, a few per row) go to a 32-slot row buffer in
//     shared memory, in any order, as 64-bit composites (order key, then
//     511 - id) with their raw logit;
//  3. each candidate's rank is the number of the row's candidates with a
//     larger composite (a larger key, or the same key and a lower id); the
//     candidates of rank 0..K are the K selected experts and alpha.
// A row with more than 32 candidates (heavy ties), or fewer than K + 1
// (non-finite values), is finished by the whole warp with warp_select_row.
constexpr int kSegRows = 4;                   // rows per warp
constexpr int kSegSlots = 32;                 // candidates per row

template <int C>
struct SegScratch {
  float z[kSegRows][32 * C];                  // the rows' raw logits (lane-chunk order)
  uint64_t comp[kSegRows][kSegSlots + 1];     // (key, 511 - id); one pad word pair per row
  float zc[kSegRows][kSegSlots + 2];          // the candidates' raw logits
  uint32_t win[kSegRows][24];                 // slot of rank r (r <= K)
};

// Groups per lane: 3 of four chunks at C = 12, else 4 (8 GPL >= 24 >= K + 1).
template <int C>
struct SegGroups {
  static constexpr int kGPL = C == 12 ? 3 : 4;
  static constexpr int kGS = C / kGPL;             // chunks per group
  static_assert(C % kGPL == 0, "whole groups");
};

// kOverlap: instead of writing the selection, count how many of each row's
// K experts (selected on Z alone) are among the K ids given for the row, and
// add the count over all rows to *overlap (the intervention rate's
// numerator).
template <int C, bool kBias, bool kOverlap>
__global__ void __launch_bounds__(kThreads, C >= 16 ? 2 : 3) seg_select_kernel(
    const float* __restrict__ z, const float* __restrict__ beta, int64_t N, int E, int K,
    int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ alpha,
    unsigned long long* __restrict__ overlap) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int V = 4 * C;
  float* beta_s = reinterpret_cast<float*>(smem);
  SegScratch<C>& sc = reinterpret_cast<SegScratch<C>*>(smem + 4 * 32 * C)[threadIdx.x >> 5];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = lane >> 3, sl = lane & 7;
  pdl_wait();       // Z comes from the kernel before this one
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += kThreads) beta_s[e] = kBias ? beta[e] : 0.f;
  __syncthreads();
  // kOverlap: is expert e among row t's given ids
  auto routed = [&](int64_t t, uint32_t e) {
    bool hit = false;
    for (int k = 0; k < K; ++k) hit |= __ldg(ids + t * K + k) == static_cast<int32_t>(e);
    return hit;
  };
  uint32_t hits = 0u;
  const int64_t step = static_cast<int64_t>(gridDim.x) * kWarps * kSegRows;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * kSegRows; base < N; base += step) {
    const int64_t row = base + seg;
    const bool live = row < N;
    float zv[V];
#pragma unroll
    for (int i = 0; i < C; ++i) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (live) v = __ldg(reinterpret_cast<const float4*>(z + row * E + 32 * i + 4 * sl));
      zv[4 * i] = v.x;
      zv[4 * i + 1] = v.y;
      zv[4 * i + 2] = v.z;
      zv[4 * i + 3] = v.w;
    }
    {
      // the warp's next rows go to L2 while these are worked on: the row's
      // 128-byte lines split over the segment's lanes
      const int64_t nrow = row + step;
      if (nrow < N) {
        const char* pr = reinterpret_cast<const char*>(z + nrow * E);
        for (int ln = sl; ln < E / 32; ln += 8) asm volatile("prefetch.global.L2 [%0];" ::"l"(pr + 128 * ln));
      }
    }
    // scores, chunk maxima, group maxima
    constexpr int GS = SegGroups<C>::kGS;       // chunks per group
    float cmax[C];
    float g[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < C; ++i) {
      const float4 bq = *reinterpret_cast<const float4*>(&beta_s[32 * i + 4 * sl]);
      const float b0 = kBias ? __fadd_rn(zv[4 * i], bq.x) : zv[4 * i];
      const float b1 = kBias ? __fadd_rn(zv[4 * i + 1], bq.y) : zv[4 * i + 1];
      const float b2 = kBias ? __fadd_rn(zv[4 * i + 2], bq.z) : zv[4 * i + 2];
      const float b3 = kBias ? __fadd_rn(zv[4 * i + 3], bq.w) : zv[4 * i + 3];
      const float m = fmaxf(fmaxf(b0, b1), fmaxf(b2, b3));
      cmax[i] = m;
      g[i / GS] = fmaxf(g[i / GS], m);
    }
    // this lane's group maxima sorted descending (GPL = 3 leaves g[3] at -inf)
#define KOLIBRI_FCE(a, b)                    \
  {                                          \
    const float hi_ = fmaxf(g[a], g[b]);     \
    g[b] = fminf(g[a], g[b]);                \
    g[a] = hi_;                              \
  }
    KOLIBRI_FCE(0, 1) KOLIBRI_FCE(2, 3) KOLIBRI_FCE(0, 2) KOLIBRI_FCE(1, 3) KOLIBRI_FCE(1, 2)
#undef KOLIBRI_FCE
    float T = -INFINITY;
    for (int r = 0; r <= K; ++r) {
      float m = g[0];
#pragma unroll
      for (int d = 1; d < 8; d <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
      T = m;
      if (g[0] == m) {            // every lane holding the maximum drops it
        g[0] = g[1];
        g[1] = g[2];
        g[2] = g[3];
        g[3] = -INFINITY;
      }
    }
    // the row in shared memory (candidates are read back by chunk index)
    __syncwarp();
#pragma unroll
    for (int i = 0; i < C; ++i)
      *reinterpret_cast<float4*>(&sc.z[seg][32 * i + 4 * sl]) =
          make_float4(zv[4 * i], zv[4 * i + 1], zv[4 * i + 2], zv[4 * i + 3]);
    uint32_t cm = 0u;   // chunks holding a candidate
#pragma unroll
    for (int i = 0; i < C; ++i) cm |= (cmax[i] >= T) ? (1u << i) : 0u;
    // candidates per lane, then their positions in the row buffer
    uint32_t cnt = 0u;
    {
      uint32_t mm = cm;
      while (mm) {
        const int i = __ffs(mm) - 1;
        mm &= mm - 1u;
        const float4 zq = *reinterpret_cast<const float4*>(&sc.z[seg][32 * i + 4 * sl]);
        const float4 bq = *reinterpret_cast<const float4*>(&beta_s[32 * i + 4 * sl]);
        cnt += (kBias ? __fadd_rn(zq.x, bq.x) : zq.x) >= T;
        cnt += (kBias ? __fadd_rn(zq.y, bq.y) : zq.y) >= T;
        cnt += (kBias ? __fadd_rn(zq.z, bq.z) : zq.z) >= T;
        cnt += (kBias ? __fadd_rn(zq.w, bq.w) : zq.w) >= T;
      }
    }
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d, 8);
      if (sl >= d) incl += t;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 7, 8);
    // the candidates as 64-bit composites (order key, then 511 - id), with
    // their logits
    if (total <= kSegSlots) {
      uint32_t pos = incl - cnt;
      while (cm) {
        const int i = __ffs(cm) - 1;
        cm &= cm - 1u;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = 32 * i + 4 * sl + u;
          const float zz = sc.z[seg][e];
          const float bb = kBias ? __fadd_rn(zz, beta_s[e]) : zz;
          if (bb >= T) {
            sc.comp[seg][pos] = (static_cast<uint64_t>(order_key(bb)) << 32) | (511u - static_cast<uint32_t>(e));
            sc.zc[seg][pos] = zz;
            ++pos;
          }
        }
      }
    }
    __syncwarp();
    const bool fine = live && total >= static_cast<uint32_t>(K + 1) && total <= kSegSlots;
    // rank of each candidate: how many of the row's candidates come first
    // (larger key, or the same key and a lower id); ranks 0..K are the result
    if (fine) {
      uint64_t c[4];
      uint32_t rk[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t slot = static_cast<uint32_t>(sl + 8 * q);
        c[q] = slot < total ? sc.comp[seg][slot] : 0ull;
        rk[q] = 0u;
      }
      for (uint32_t t = 0; t < total; ++t) {
        const uint64_t o = sc.comp[seg][t];
#pragma unroll
        for (int q = 0; q < 4; ++q) rk[q] += (o > c[q]) ? 1u : 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t slot = static_cast<uint32_t>(sl + 8 * q);
        if (slot < total && rk[q] <= static_cast<uint32_t>(K)) sc.win[seg][rk[q]] = slot;
      }
    }
    __syncwarp();
    if (live && fine) {
      {
        // lane s writes ranks s, s + 8, s + 16
        for (int r = sl; r <= K; r += 8) {
          const uint32_t slot = sc.win[seg][r];
          const uint64_t w = sc.comp[seg][slot];
          const uint32_t id = 511u - static_cast<uint32_t>(w & 511u);
          if constexpr (kOverlap) {
            if (r < K) hits += routed(row, id) ? 1u : 0u;
          } else if (r < K) {
            ids[row * K + r] = static_cast<int32_t>(id);
            gates[row * K + r] = gate_sigmoid(sc.zc[seg][slot]);
          } else if (alpha != nullptr) {
            alpha[row] = -key_to_float(static_cast<uint32_t>(w >> 32));
          }
        }
      }
    }
    __syncwarp();
    // Rows left open (more than 32 candidates: heavy ties; or fewer than
    // K + 1: non-finite values) take the exact warp-per-row selection of
    // route.cuh, the whole warp on each, with the rows' buffer as scratch.
    constexpr int Q = C / 4;
    static_assert(sizeof(RowScratch<Q>) <= sizeof(sc.z), "the row scratch fits the rows' buffer");
    unsigned open = __ballot_sync(0xffffffffu, sl == 0 && live && !fine);
    while (open) {
      const int sg = (__ffs(open) - 1) >> 3;
      open &= open - 1u;
      const int64_t rr = base + sg;
      float zr[4 * Q];
      load_row<Q, true>(z + rr * E, E, lane, zr);
      RowScratch<Q>& rs = *reinterpret_cast<RowScratch<Q>*>(&sc.z[0][0]);
      int rank;
      uint32_t key, id;
      warp_select_row<Q, true, kBias>(zr, beta_s, 0xffffffffu, K, lane, rs, rank, key, id);
      if constexpr (kOverlap) {
        if (rank >= 0 && rank < K) hits += routed(rr, id) ? 1u : 0u;
      } else {
        if (rank >= 0 && rank < K) {
          const uint32_t e = id < static_cast<uint32_t>(E) ? id : 0u;
          ids[rr * K + rank] = static_cast<int32_t>(id);
          gates[rr * K + rank] = gate_sigmoid(rs.row[buffer_pos<Q>(e)]);
        }
        if (rank == K && alpha != nullptr) alpha[rr] = -key_to_float(key);
      }
      __syncwarp();
    }
  }
  if constexpr (kOverlap) {
    const uint32_t sum = __reduce_add_sync(0xffffffffu, hits);
    if (lane == 0 && sum != 0u) atomicAdd(overlap, static_cast<unsigned long long>(sum));
  }
}

template <int C>
cudaError_t launch_seg(const float* z, const float* bias, int64_t N, int E, int K, int32_t* ids,
                       float* gates, float* alpha, cudaStream_t s, unsigned long long* overlap = nullptr) {
  auto kern = overlap ? seg_select_kernel<C, false, true>
                      : (bias ? seg_select_kernel<C, true, false> : seg_select_kernel<C, false, false>);
  const size_t smem = 4 * 32 * C + sizeof(SegScratch<C>) * kWarps;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  const int64_t rows_per_block = static_cast<int64_t>(kWarps) * kSegRows;
  int64_t blocks = (N + rows_per_block - 1) / rows_per_block;
  const int64_t resident = static_cast<int64_t>(device_sm_count()) * per_sm;
  if (blocks > resident) blocks = resident;
  return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), smem, s, dim3(0, 0, 0), z, bias,
                    N, E, K, ids, gates, alpha, overlap);
}

// Batches at least this large take the segment kernel; decode-sized ones
// keep the warp-per-row kernel.
constexpr int64_t kSegMinRows = 4096;

bool seg_select_applies(int64_t N, int E, int K) {
  return N >= kSegMinRows && (E == 128 || E == 256 || E == 384 || E == 512) && K + 1 <= 24;
}

cudaError_t launch_seg_select(const float* z, const float* bias, int64_t N, int E, int K, int32_t* ids,
                              float* gates, float* alpha, cudaStream_t s) {
  switch (E / 32) {
    case 4: return launch_seg<4>(z, bias, N, E, K, ids, gates, alpha, s);
    case 8: return launch_seg<8>(z, bias, N, E, K, ids, gates, alpha, s);
    case 12: return launch_seg<12>(z, bias, N, E, K, ids, gates, alpha, s);
    case 16: return launch_seg<16>(z, bias, N, E, K, ids, gates, alpha, s);
    default: return cudaErrorNotSupported;
  }
}

template <int Q, bool kFull, bool kBias, bool kRoute, bool kAlphaOut, bool kAlphaIn, bool kWindow>
cudaError_t launch_rows(RouteParams p, cudaStream_t s) {
  auto kern = route_rows_kernel<Q, kFull, kBias, kRoute, kAlphaOut, kAlphaIn, kWindow>;
  const SmemLayout L = smem_layout<Q, kWindow>(p.E);
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, L.total);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  // each warp walks its rows one after another, so a batch that does not
  // fill the resident warps gets fewer rows per warp (one, for decode sizes)
  const int64_t resident = static_cast<int64_t>(device_sm_count()) * per_sm;
  const int64_t warps = resident * kWarps;
  int64_t rpw = (p.N + warps - 1) / warps;
  if (rpw < 1) rpw = 1;
  if (rpw > kRowsPerWarp) rpw = kRowsPerWarp;
  p.rows_per_warp = static_cast<int>(rpw);
  const int64_t rows_per_block = static_cast<int64_t>(kWarps) * rpw;
  int64_t blocks = (p.N + rows_per_block - 1) / rows_per_block;
  if (blocks > resident) blocks = resident;
  return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), L.total, s, dim3(0, 0, 0), p);
}

// route: write ids/gates; alpha_out: write alpha; alpha_in: read alpha
// instead of selecting; window: bracketed full pass.
template <int Q, bool kFull>
cudaError_t dispatch_q(const RouteParams& p, bool route, bool alpha_out, bool alpha_in, bool window,
                       cudaStream_t s) {
  const bool bias = p.beta != nullptr;
#define KOLIBRI_ROWS(B, R, AO, AI, W)                                                   \
  if (bias == B && route == R && alpha_out == AO && alpha_in == AI && window == W) \
    return launch_rows<Q, kFull, B, R, AO, AI, W>(p, s);
  KOLIBRI_ROWS(true, true, true, false, false)
  KOLIBRI_ROWS(true, true, false, false, false)
  KOLIBRI_ROWS(false, true, true, false, false)
  KOLIBRI_ROWS(false, true, false, false, false)
  KOLIBRI_ROWS(true, true, true, false, true)
  KOLIBRI_ROWS(false, true, true, false, true)
  KOLIBRI_ROWS(true, false, true, false, true)
  KOLIBRI_ROWS(false, false, true, false, true)
  KOLIBRI_ROWS(false, false, false, true, true)
#undef KOLIBRI_ROWS
  return cudaErrorInvalidValue;
}

cudaError_t dispatch(const RouteParams& p, bool route, bool alpha_out, bool alpha_in, bool window,
                     cudaStream_t s) {
  const bool full = (p.E % 128) == 0;
  switch ((p.E + 127) / 128) {
    case 1: return full ? dispatch_q<1, true>(p, route, alpha_out, alpha_in, window, s)
                        : dispatch_q<1, false>(p, route, alpha_out, alpha_in, window, s);
    case 2: return full ? dispatch_q<2, true>(p, route, alpha_out, alpha_in, window, s)
                        : dispatch_q<2, false>(p, route, alpha_out, alpha_in, window, s);
    case 3: return full ? dispatch_q<3, true>(p, route, alpha_out, alpha_in, window, s)
                        : dispatch_q<3, false>(p, route, alpha_out, alpha_in, window, s);
    case 4: return full ? dispatch_q<4, true>(p, route, alpha_out, alpha_in, window, s)
                        : dispatch_q<4, false>(p, route, alpha_out, alpha_in, window, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int Q>
cudaError_t launch_sample_q(const float* z, const float* alpha, const float* bias, int64_t N,
                            int E, int K, int64_t S, int64_t stride, int64_t S_ld,
                            uint32_t* sample, cudaStream_t s, uint32_t* zero_word) {
  static_assert(kSampleRows % kWarps == 0, "whole rows per warp");
  const size_t smem = ((4 * kSampleRows * (E + 1) + 15) & ~15) + ((4 * E + 15) & ~15) +
                      sizeof(RowScratch<Q>) * kWarps;
  dim3 grid(static_cast<unsigned>((S + kSampleRows - 1) / kSampleRows)), block(kThreads);
  auto k = alpha ? sample_keys_kernel<Q, true, false>
                 : (bias ? sample_keys_kernel<Q, false, true> : sample_keys_kernel<Q, false, false>);
  cudaError_t err =
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(k, grid, block, smem, s, dim3(0, 0, 0), z, alpha, bias, N, E, K, S, stride, S_ld, sample,
                    zero_word);
}

}  // namespace

bool seg_overlap_applies(int64_t N, int32_t E, int32_t K) { return seg_select_applies(N, E, K); }

cudaError_t launch_seg_overlap(const float* z, const int32_t* ids, int64_t N, int32_t E, int32_t K,
                               unsigned long long* total, cudaStream_t s) {
  int32_t* idv = const_cast<int32_t*>(ids);   // read only in this mode
  switch (E / 32) {
    case 4: return launch_seg<4>(z, nullptr, N, E, K, idv, nullptr, nullptr, s, total);
    case 8: return launch_seg<8>(z, nullptr, N, E, K, idv, nullptr, nullptr, s, total);
    case 12: return launch_seg<12>(z, nullptr, N, E, K, idv, nullptr, nullptr, s, total);
    case 16: return launch_seg<16>(z, nullptr, N, E, K, idv, nullptr, nullptr, s, total);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_topk(const float* z, const float* bias, int64_t N, int32_t E, int32_t K,
                        int32_t* ids, float* gates, float* alpha, cudaStream_t s) {
  if (seg_select_applies(N, E, K)) return launch_seg_select(z, bias, N, E, K, ids, gates, alpha, s);
  RouteParams p{};
  p.z = z;
  p.beta = bias;
  p.N = N;
  p.E = E;
  p.K = K;
  p.ids = ids;
  p.gates = gates;
  p.alpha_out = alpha;
  return dispatch(p, true, alpha != nullptr, false, false, s);
}

cudaError_t launch_select_fixup(const float* z, const float* bias, int64_t N, int32_t E, int32_t K,
                                int32_t* ids, float* gates, float* alpha, cudaStream_t s) {
  const int64_t rows_per_block = static_cast<int64_t>(kWarps) * 32;
  int64_t blocks = (N + rows_per_block - 1) / rows_per_block;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 4;
  if (blocks > cap) blocks = cap;
  const bool full = (E % 128) == 0, b = bias != nullptr;
  const dim3 grid(static_cast<unsigned>(blocks)), block(kThreads);
#define KOLIBRI_FIXUP(Q)                                                                       \
  if (full) {                                                                                  \
    if (b) select_fixup_kernel<Q, true, true><<<grid, block, 0, s>>>(z, bias, N, E, K, ids, gates, alpha); \
    else select_fixup_kernel<Q, true, false><<<grid, block, 0, s>>>(z, bias, N, E, K, ids, gates, alpha); \
  } else {                                                                                     \
    if (b) select_fixup_kernel<Q, false, true><<<grid, block, 0, s>>>(z, bias, N, E, K, ids, gates, alpha); \
    else select_fixup_kernel<Q, false, false><<<grid, block, 0, s>>>(z, bias, N, E, K, ids, gates, alpha); \
  }
  switch ((E + 127) / 128) {
    case 1: KOLIBRI_FIXUP(1) break;
    case 2: KOLIBRI_FIXUP(2) break;
    case 3: KOLIBRI_FIXUP(3) break;
    case 4: KOLIBRI_FIXUP(4) break;
    default: return cudaErrorInvalidValue;
  }
#undef KOLIBRI_FIXUP
  return cudaGetLastError();
}

cudaError_t launch_eqb_sample(const float* z, const float* alpha, const float* bias, int64_t N,
                              int32_t E, int32_t K, int64_t S, int64_t stride, int64_t S_ld,
                              uint32_t* sample, cudaStream_t s, uint32_t* zero_word) {
  switch ((E + 127) / 128) {
    case 1: return launch_sample_q<1>(z, alpha, bias, N, E, K, S, stride, S_ld, sample, s, zero_word);
    case 2: return launch_sample_q<2>(z, alpha, bias, N, E, K, S, stride, S_ld, sample, s, zero_word);
    case 3: return launch_sample_q<3>(z, alpha, bias, N, E, K, S, stride, S_ld, sample, s, zero_word);
    case 4: return launch_sample_q<4>(z, alpha, bias, N, E, K, S, stride, S_ld, sample, s, zero_word);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_route_window_pass(const float* z, const float* bias, const float* alpha_in,
                                     int64_t N, int32_t E, int32_t K, int32_t* ids, float* gates,
                                     float* alpha_out, const uint32_t* lo, const uint32_t* hi,
                                     uint32_t* above, uint32_t* cnt, uint32_t* cand, int64_t cap,
                                     cudaStream_t s) {
  RouteParams p{};
  p.z = z;
  p.beta = alpha_in ? nullptr : bias;
  p.N = N;
  p.E = E;
  p.K = K;
  p.ids = ids;
  p.gates = gates;
  p.alpha_out = alpha_out;
  p.alpha_in = alpha_in;
  p.lo = lo;
  p.hi = hi;
  p.above = above;
  p.cand_cnt = cnt;
  p.cand = cand;
  p.cap = cap;
  const bool route = ids != nullptr;
  return dispatch(p, route, alpha_out != nullptr, alpha_in != nullptr, true, s);
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_route)

}  // namespace kolibri
