// expert_ffn.cu -- the expert layer after the router: dispatch, the two
// grouped SwiGLU projections on the 5th-generation tensor cores, combine.
//
// "Kolibri Pre-Training from Scratch" 6.1: y_t = f_shared(x_t) +
// sum_{e in I_t} S_t,e f_e(x_t), the mixture weights the unbiased sigmoid
// scores (not renormalised).  "Kolibri 1 im Detail", experts: every routed
// or shared expert is a SwiGLU MLP, two projections 2560 -> 512 forming
// SiLU(gate) x up, then one projection 512 -> 2560.
//
// Data flow for N tokens, K slots each (slot j = t*K + k), E experts:
//   dispatch   x_perm[p] = x[perm[p] / K]           rows grouped by expert
//   gate_up    h[p] = bf16(SiLU(x_perm[p] Wg_e^T) * (x_perm[p] Wu_e^T))
//   down       y_perm[p] = h[p] Wd_e^T              fp32
//   combine    y[t] = y_shared[t] + sum_k S_t,k y_perm[inv[t*K+k]]  (fp32, k ascending)
// where e is the expert whose segment [offsets[e], offsets[e+1]) holds p.
// The shared expert runs the same two projections over x itself.
//
// The projections are one grouped GEMM kernel: a persistent kernel on SM
// pairs (tcgen05.mma.cta_group::2, bf16 in, fp32 accumulate in TMEM, two
// accumulator buffers so the epilogue of one tile runs under the MMAs of
// the next).  The weights are the MMA's M side (256 rows per pair) and the
// tokens its N side, so the last token block of an expert is an MMA of just
// its rows rounded up to 32 (with balanced loads of about 256 rows an
// expert, 256-row blocks of tokens on the M side would spend up to half of
// the tensor time on empty rows).  Tiles are (expert, token block, feature
// block); every CTA maps a tile index to them on the device from the
// offsets, so no host round trip is needed between the permutation and the
// GEMMs.  In the gate/up projection a CTA stages the gate rows and the up
// rows of the same 128 units and issues one MMA for each into its own
// columns, so a thread holds both sums of its unit and the epilogue forms
// SiLU(gate) * up in registers.  Stores are one token row segment per warp
// instruction.  No load uses cluster multicast.
#include <cuda_bf16.h>

#include "launch.h"
#include "gemm_pair.cuh"

namespace kolibri {

namespace {

using namespace gemm;

constexpr int kThreads = 192;            // warp 0 TMA, warp 1 TMEM + MMA, warps 2..5 epilogue
constexpr int kEpiWarps = 4;
constexpr int kFeat = 2 * kBM;           // weight rows per pair tile: the MMA's M
constexpr int kAccCols = 512;            // two accumulator buffers of 256 columns
constexpr int kMaxGroups = KOLIBRI_MAX_EXPERTS;
constexpr uint32_t kWBytes = kBM * kBK * 2;        // 128 weight rows x 64 (16 KB)

// Per projection: tokens per tile at most (the MMA's N), weight bytes and
// token bytes a CTA stages per k-block.  Gate/up: 128 gate rows and the same
// units' 128 up rows (two MMAs per k-step into two column ranges of one
// accumulator buffer), up to 128 tokens; down: 128 weight rows, up to 256
// tokens.
template <bool kGateUp>
struct Cfg {
  static constexpr int kTok = kGateUp ? 128 : 256;
  static constexpr uint32_t kW = kGateUp ? 2 * kWBytes : kWBytes;
  static constexpr uint32_t kX = static_cast<uint32_t>(kTok / 2) * kBK * 2;
  static constexpr uint32_t kStage = kW + kX;                    // 40 KB / 32 KB
};

struct GroupedParams {
  const int64_t* offsets;   // [G + 1] token segments, or null: one group [0, rows)
  int64_t rows;             // token rows (N*K routed, N shared)
  int G;                    // groups (experts)
  int kdim;                 // reduction length (d, or F)
  int n_tiles;              // feature blocks per token block
  int ncols;                // output row length (F for gate/up, d for down)
  int w_rows;               // weight rows per group: 2F (gate/up) or d (down)
  int stages;
  int w_stream;             // 1: weights read about once (routed), evict them first
  void* out;                // bf16 h [rows, F] or fp32 y [rows, d]
};

// Shared-memory map: the operand ring (1 KB aligned), then barriers.
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ __forceinline__ uint32_t empty(int s) const { return base + 8u * (kMaxStages + s); }
  __device__ __forceinline__ uint32_t tfull(int a) const { return base + 8u * (2 * kMaxStages + a); }
  __device__ __forceinline__ uint32_t tempty(int a) const { return base + 8u * (2 * kMaxStages + 2 + a); }
  __device__ __forceinline__ uint32_t holder() const { return base + 8u * (2 * kMaxStages + 4); }
};
constexpr int kBarBytes = 8 * (2 * kMaxStages + 5);

// Tokens in the tile (the MMA's N): the rows left in the group, rounded up
// to 32, at most tok.
__device__ __forceinline__ int tile_tokens(int64_t left, int tok) {
  const int64_t r = (left + 31) & ~static_cast<int64_t>(31);
  return static_cast<int>(r < tok ? r : tok);
}

// Token-block prefix over the groups, in shared memory: mt[g] = token blocks
// of the groups before g; mt[G] = all token blocks.
struct TileMap {
  const int32_t* mt;
  const int64_t* offsets;   // shared-memory copy of the group offsets [G + 1]
  int64_t rows;
  int G, n_tiles, tok;
  __device__ __forceinline__ int64_t total() const { return static_cast<int64_t>(mt[G]) * n_tiles; }
  // tile -> group, first token row of its block, rows left in the group from there, feature block
  __device__ __forceinline__ void map(int64_t tile, int& g, int64_t& row0, int64_t& left, int& n) const {
    const int mb = static_cast<int>(tile / n_tiles);
    n = static_cast<int>(tile - static_cast<int64_t>(mb) * n_tiles);
    int lo = 0, hi = G - 1;                   // last g with mt[g] <= mb
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (mt[mid] <= mb) lo = mid;
      else hi = mid - 1;
    }
    g = lo;
    const int64_t start = offsets[g];
    const int64_t end = offsets[g + 1];
    row0 = start + static_cast<int64_t>(mb - mt[g]) * tok;
    left = end - row0;
  }
};

// All threads: mt[0..G] from the offsets (a block-wide exclusive scan), and
// a shared-memory copy of the offsets (off[0..G]; without offsets: 0, rows).
// Offsets that do not start at 0, decrease, or pass the row count are
// flagged (device status) and give no tiles at all, so nothing is stored.
__device__ void build_tile_prefix(const GroupedParams& p, int tok, int32_t* mt, int64_t* off,
                                  int32_t* warp_tot) {
  __shared__ int bad_s;
  if (threadIdx.x == 0) bad_s = 0;
  __syncthreads();
  for (int g = threadIdx.x; g <= p.G; g += kThreads) {
    const int64_t o = p.offsets ? p.offsets[g] : (g == 0 ? 0 : p.rows);
    off[g] = o;
    const bool ok = (g == 0 ? o == 0 : true) && o <= p.rows &&
                    (g == 0 || !p.offsets || p.offsets[g - 1] <= o);
    if (!ok) bad_s = 1;
  }
  __syncthreads();
  const bool bad = bad_s != 0;
  if (bad && threadIdx.x == 0 && blockIdx.x == 0) raise_status(kStatusBadInput);
  constexpr int kPer = (kMaxGroups + kThreads - 1) / kThreads;   // 3
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t v[kPer];
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int g = tid * kPer + i;
    int32_t c = 0;
    if (g < p.G && !bad) {
      const int64_t len = off[g + 1] - off[g];
      c = static_cast<int32_t>((len + tok - 1) / tok);
    }
    v[i] = c;
    sum += c;
  }
  int32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int32_t base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  int32_t run = base + incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int g = tid * kPer + i;
    if (g <= p.G) mt[g] = run;      // g == G receives the total
    run += v[i];
  }
  __syncthreads();
}

// SiLU(g) = g / (1 + e^-g) with the fast exponential and division (errors of
// a few fp32 units, far below the bf16 step h is rounded to).  Large |g|:
// e^-g -> 0 gives g; e^-g -> inf gives -0.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }


// ---- the grouped projection ---------------------------------------------

// The weights are the MMA's A operand (M = 256 weight rows per pair, 128
// per CTA) and the tokens its B operand (N = the tile's tokens, a multiple
// of 32, half staged by each CTA), so a group's last token block costs only
// its own rows.  TMEM lane = weight row, column = token.
//
// kGateUp: tokens = x rows [rows, d]; weights = the experts' [gate; up]
// rows [G * 2F, d].  A feature block is 256 hidden units (128 per CTA): per
// k-step one MMA takes the CTA's 128 gate rows into columns [0, 128) of the
// accumulator buffer and one its 128 up rows into [128, 256), so a thread
// holds both sums of its unit for every token.  out = bf16 h [rows, F].
// Otherwise: tokens = h [rows, F]; weights = the down rows [G * d, F]; a
// feature block is 256 output columns; out = fp32 [rows, d].
template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_x, const GroupedParams p) {
  using C = Cfg<kGateUp>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int32_t mt_s[kMaxGroups + 1];
  __shared__ int64_t off_s[kMaxGroups + 1];
  __shared__ int32_t warp_tot[kThreads / 32];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t ring = (raw + 1023u) & ~1023u;
  Bars bars{ring + C::kStage * static_cast<uint32_t>(p.stages)};
  uint8_t* const holder_ptr = smem_raw + (bars.holder() - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t cid = cluster_id_x(), ncl = num_clusters_x();

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(bars.full(s), 1);
      mbar_init(bars.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bars.tfull(a), 1);
      mbar_init(bars.tempty(a), 2 * kEpiWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(bars.holder()),
                 "r"(kAccCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  build_tile_prefix(p, C::kTok, mt_s, off_s, warp_tot);
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(holder_ptr);
  const TileMap tmap{mt_s, off_s, p.rows, p.G, p.n_tiles, C::kTok};
  const int64_t tiles = tmap.total();
  const int k_blocks = p.kdim / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer of this CTA; both CTAs' copies land on the leader's full barrier.
      // Token rows are read by every feature block; routed weights about once.
      const uint64_t pol_x = policy_evict_last();
      const uint64_t pol_w = p.w_stream ? policy_evict_first() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t tile = cid; tile < tiles; tile += ncl) {
        int g, fb;
        int64_t row0, left;
        tmap.map(tile, g, row0, left, fb);
        const int nt = tile_tokens(left, C::kTok);
        const int x_row = static_cast<int>(row0) + static_cast<int>(rank) * (nt / 2);
        // first weight row of this CTA (gate/up: its first gate row; the up rows are F below)
        const int w_row = g * p.w_rows + fb * kFeat + static_cast<int>(rank) * kBM;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(bars.empty(stage), phase ^ 1u)) { ok = false; break; }
          const uint32_t fbar = map_to_rank(bars.full(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(bars.full(stage), 2u * C::kStage);
          const uint32_t w_dst = ring + C::kStage * stage;
          tma_load_2d_pair(w_dst, &tm_w, kb * kBK, w_row, fbar, pol_w);
          if constexpr (kGateUp)
            tma_load_2d_pair(w_dst + kWBytes, &tm_w, kb * kBK, w_row + p.w_rows / 2, fbar, pol_w);
          tma_load_2d_pair(w_dst + C::kW, &tm_x, kb * kBK, x_row, fbar, pol_x);
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      // the pair's single MMA thread: M = 256 weight rows, N = the tile's tokens
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int64_t tile = cid; tile < tiles; tile += ncl) {
        int g, fb;
        int64_t row0, left;
        tmap.map(tile, g, row0, left, fb);
        const uint32_t idesc = make_idesc(kFeat, tile_tokens(left, C::kTok));
        if (!mbar_wait(bars.tempty(acc), acc_phase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(bars.full(stage), phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w_addr = ring + C::kStage * stage;
          const uint64_t a_desc = sw128_desc(w_addr);
          const uint64_t b_desc = sw128_desc(w_addr + C::kW);
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks)
            tc_mma_pair(d_tmem, a_desc + 2u * ks, b_desc + 2u * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
          if constexpr (kGateUp) {
            const uint64_t u_desc = sw128_desc(w_addr + kWBytes);
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks)
              tc_mma_pair(d_tmem + 128u, u_desc + 2u * ks, b_desc + 2u * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
          }
          tc_commit_pair(bars.empty(stage));
          if (++stage == p.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(bars.tfull(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // epilogue warps 2..5: thread = weight row (TMEM lane); the lane quarter is warp % 4
    const int quarter = warp & 3;
    const int L = quarter * 32 + lane;                 // this CTA's weight row
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // The buffer of a tile is handed back at the start of the next tile's
    // epilogue, not right after its last TMEM read: the arrive is a release
    // and would otherwise wait for this warp's stores of the tile.  The MMA
    // of tile j + 2 still never waits for the epilogue of tile j + 1.
    int acc = 0, held = -1;
    uint32_t acc_phase = 0;
    for (int64_t tile = cid; tile < tiles; tile += ncl) {
      if (!mbar_wait(bars.tfull(acc), acc_phase)) break;
      if (held >= 0 && lane == 0) mbar_arrive_cluster(map_to_rank(bars.tempty(held), 0));
      held = -1;
      tc_fence_after();
      int g, fb;
      int64_t row0, left;
      tmap.map(tile, g, row0, left, fb);
      const int nt = tile_tokens(left, C::kTok);
      const int valid = static_cast<int>(left < nt ? left : nt);
      const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(acc * 256);
      const int64_t stride = p.ncols;
      if constexpr (kGateUp) {
        const int unit = fb * kFeat + static_cast<int>(rank) * kBM + L;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row0 * stride + unit;
#pragma unroll 1
        for (int c = 0; c < nt; c += 32) {
          uint32_t gr[32], ur[32];
          tmem_ld32(t0 + static_cast<uint32_t>(c), gr);
          tmem_ld32(t0 + 128u + static_cast<uint32_t>(c), ur);
          tmem_wait_ld();
          __nv_bfloat16* o = out + c * stride;
          const int n_ok = valid - c;                  // tokens of this chunk that are stored
          if (n_ok >= 32) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              o[i * stride] = __float2bfloat16_rn(silu_f32(__uint_as_float(gr[i])) * __uint_as_float(ur[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < n_ok)
                o[i * stride] = __float2bfloat16_rn(silu_f32(__uint_as_float(gr[i])) * __uint_as_float(ur[i]));
          }
        }
      } else {
        float* out = static_cast<float*>(p.out) + row0 * stride + fb * kFeat + static_cast<int>(rank) * kBM + L;
#pragma unroll 1
        for (int c = 0; c < nt; c += 32) {
          uint32_t r[32];
          tmem_ld32(t0 + static_cast<uint32_t>(c), r);
          tmem_wait_ld();
          float* o = out + c * stride;
          const int n_ok = valid - c;
          if (n_ok >= 32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i * stride] = __uint_as_float(r[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < n_ok) o[i * stride] = __uint_as_float(r[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      held = acc;
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (held >= 0 && lane == 0) mbar_arrive_cluster(map_to_rank(bars.tempty(held), 0));
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kAccCols)
                 : "memory");
  }
}

// ---- dispatch and combine -------------------------------------------------

// x_perm[p] = x[perm[p] / K]: a warp per row, 16-byte pieces; each lane
// issues all of its loads of the row (up to kDispatchPieces) before its
// stores, so a row is one memory round trip.
constexpr int kDispatchPieces = 16;      // 16-byte pieces per lane: rows up to 8192 bf16
__global__ void __launch_bounds__(256) dispatch_kernel(const uint4* __restrict__ x,
                                                       const int32_t* __restrict__ perm, int64_t NK,
                                                       int K, int64_t N, int row_pieces,
                                                       uint4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t p = blockIdx.x * 8 + (threadIdx.x >> 5); p < NK; p += warps) {
    const int32_t j = __ldg(perm + p);
    const int64_t t = j / K;
    if (j < 0 || t >= N) {
      if (lane == 0) raise_status(kStatusBadInput);
      continue;
    }
    const uint4* src = x + t * row_pieces;
    uint4* dst = x_perm + p * row_pieces;
    uint4 v[kDispatchPieces];
#pragma unroll
    for (int u = 0; u < kDispatchPieces; ++u) {
      const int i = lane + 32 * u;
      if (i < row_pieces) v[u] = __ldg(src + i);
    }
#pragma unroll
    for (int u = 0; u < kDispatchPieces; ++u) {
      const int i = lane + 32 * u;
      if (i < row_pieces) dst[i] = v[u];
    }
  }
}

// y[t] = y_shared[t] + sum_k S_t,k y_perm[inv[t*K+k]], fp32 multiply-adds in
// k order; a block per token, four columns per thread per step.
__global__ void __launch_bounds__(128) combine_kernel(const float4* __restrict__ y_perm,
                                                      const float4* __restrict__ y_shared,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gates, int64_t N,
                                                      int K, int64_t NK, int row4,
                                                      float4* __restrict__ y) {
  __shared__ int32_t slot[32];
  __shared__ float gate[32];
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < K) {
      const int32_t q = __ldg(inv + t * K + threadIdx.x);
      const bool ok = q >= 0 && q < NK;
      if (!ok) raise_status(kStatusBadInput);
      slot[threadIdx.x] = ok ? q : -1;
      gate[threadIdx.x] = __ldg(gates + t * K + threadIdx.x);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < row4; c += blockDim.x) {
      float4 a = y_shared ? __ldg(y_shared + t * row4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < K; ++k) {
        if (slot[k] < 0) continue;
        const float s = gate[k];
        const float4 v = __ldg(y_perm + static_cast<int64_t>(slot[k]) * row4 + c);
        a.x = __fmaf_rn(s, v.x, a.x);
        a.y = __fmaf_rn(s, v.y, a.y);
        a.z = __fmaf_rn(s, v.z, a.z);
        a.w = __fmaf_rn(s, v.w, a.w);
      }
      y[t * row4 + c] = a;
    }
  }
}

template <bool kGateUp>
cudaError_t launch_expert_gemm(const void* x, int64_t rows, const int64_t* offsets, int G,
                               const void* w, void* out, int kdim, int ncols, int w_rows,
                               cudaStream_t s) {
  GroupedParams p{};
  p.offsets = offsets;
  p.rows = rows;
  p.G = G;
  p.kdim = kdim;
  p.ncols = ncols;
  p.w_rows = w_rows;
  p.n_tiles = ncols / kFeat;
  p.w_stream = offsets != nullptr;
  p.out = out;
  using C = Cfg<kGateUp>;
  CUtensorMap tm_w, tm_x;
  if (!encode_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, static_cast<uint64_t>(kdim),
                 static_cast<uint64_t>(rows), kBK, C::kTok / 2) ||
      !encode_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, static_cast<uint64_t>(kdim),
                 static_cast<uint64_t>(G) * w_rows, kBK, kBM))
    return cudaErrorInvalidValue;
  auto kern = expert_gemm_kernel<kGateUp>;
  cudaFuncAttributes fa;
  cudaError_t err = cudaFuncGetAttributes(&fa, kern);
  if (err != cudaSuccess) return err;
  const size_t fixed = 1024 /*alignment slack*/ + kBarBytes;
  const size_t avail = static_cast<size_t>(kSmemLimit) - fa.sharedSizeBytes - fixed;
  int stages = static_cast<int>(avail / C::kStage);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  p.stages = stages;
  const size_t smem = fixed + static_cast<size_t>(C::kStage) * stages;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters[2] = {0, 0};
  int& mc = max_clusters[kGateUp ? 1 : 0];
  if (mc == 0) {
    cfg.gridDim = dim3(2 * static_cast<unsigned>(device_sm_count() / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = device_sm_count() / 2;
    mc = n;
  }
  // at most one pair per tile: token blocks <= rows / 256 + G (one partial block per group)
  const int64_t tiles_max = ((rows + C::kTok - 1) / C::kTok + G) * p.n_tiles;
  const int64_t clusters = tiles_max < mc ? tiles_max : mc;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  err = cudaLaunchKernelEx(&cfg, kern, tm_w, tm_x, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

bool expert_shape_supported(int32_t d, int32_t F, int32_t E) {
  return d >= kFeat && d % kFeat == 0 && d <= 8192 && F >= kFeat && F % kFeat == 0 && E >= 1 &&
         E <= kMaxGroups && static_cast<int64_t>(E) * 2 * F < (1LL << 31) &&
         static_cast<int64_t>(E) * d < (1LL << 31);
}

ExpertLayout expert_layout(int64_t N, int32_t d, int32_t F, int32_t K, bool shared) {
  ExpertLayout L{};
  const int64_t NK = N * K;
  size_t off = 0;
  L.off_x_perm = off;
  off += align256(sizeof(uint16_t) * static_cast<size_t>(NK) * d);
  L.off_h = off;
  off += align256(sizeof(uint16_t) * static_cast<size_t>(NK) * F);
  L.off_y_perm = off;
  off += align256(sizeof(float) * static_cast<size_t>(NK) * d);
  if (shared) {
    L.off_h_shared = off;
    off += align256(sizeof(uint16_t) * static_cast<size_t>(N) * F);
    L.off_y_shared = off;
    off += align256(sizeof(float) * static_cast<size_t>(N) * d);
  }
  L.total = off;
  return L;
}

cudaError_t launch_expert_dispatch(const void* x, const int32_t* perm, int64_t N, int32_t d,
                                   int32_t K, void* x_perm, cudaStream_t s) {
  const int64_t NK = N * K;
  const int row_pieces = d / 8;
  if (row_pieces > 32 * kDispatchPieces) return cudaErrorInvalidValue;
  int64_t blocks = (NK + 7) / 8;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  dispatch_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const uint4*>(x), perm, NK, K, N, row_pieces, static_cast<uint4*>(x_perm));
  return cudaGetLastError();
}

cudaError_t launch_expert_gate_up(const void* a, int64_t rows, const int64_t* offsets, int32_t G,
                                  const void* w_gate_up, void* h, int32_t d, int32_t F,
                                  cudaStream_t s) {
  return launch_expert_gemm<true>(a, rows, offsets, G, w_gate_up, h, d, F, 2 * F, s);
}

cudaError_t launch_expert_down(const void* h, int64_t rows, const int64_t* offsets, int32_t G,
                               const void* w_down, float* y, int32_t d, int32_t F, cudaStream_t s) {
  return launch_expert_gemm<false>(h, rows, offsets, G, w_down, y, F, d, d, s);
}

cudaError_t launch_expert_combine(const float* y_perm, const float* y_shared, const int32_t* inv,
                                  const float* gates, int64_t N, int32_t d, int32_t K, float* y,
                                  cudaStream_t s) {
  int64_t blocks = N;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 32;
  if (blocks > cap) blocks = cap;
  combine_kernel<<<static_cast<unsigned>(blocks), 128, 0, s>>>(
      reinterpret_cast<const float4*>(y_perm), reinterpret_cast<const float4*>(y_shared), inv,
      gates, N, K, N * K, d / 4, reinterpret_cast<float4*>(y));
  return cudaGetLastError();
}

cudaError_t launch_expert_ffn(const void* x, const int32_t* perm, const int64_t* offsets,
                              const int32_t* inv, const float* gates, const void* w_gate_up,
                              const void* w_down, const void* ws_gate_up, const void* ws_down,
                              float* y, int64_t N, int32_t d, int32_t F, int32_t E, int32_t K,
                              void* ws, cudaStream_t s) {
  const bool shared = ws_gate_up != nullptr;
  const ExpertLayout L = expert_layout(N, d, F, K, shared);
  char* base = static_cast<char*>(ws);
  void* x_perm = base + L.off_x_perm;
  void* h = base + L.off_h;
  float* y_perm = reinterpret_cast<float*>(base + L.off_y_perm);
  const int64_t NK = N * K;
  cudaError_t err = launch_expert_dispatch(x, perm, N, d, K, x_perm, s);
  if (err == cudaSuccess) err = launch_expert_gate_up(x_perm, NK, offsets, E, w_gate_up, h, d, F, s);
  if (err == cudaSuccess) err = launch_expert_down(h, NK, offsets, E, w_down, y_perm, d, F, s);
  float* y_shared = nullptr;
  if (shared && err == cudaSuccess) {
    void* h_s = base + L.off_h_shared;
    y_shared = reinterpret_cast<float*>(base + L.off_y_shared);
    err = launch_expert_gate_up(x, N, nullptr, 1, ws_gate_up, h_s, d, F, s);
    if (err == cudaSuccess) err = launch_expert_down(h_s, N, nullptr, 1, ws_down, y_shared, d, F, s);
  }
  if (err == cudaSuccess) err = launch_expert_combine(y_perm, y_shared, inv, gates, N, d, K, y, s);
  return err;
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_experts)

}  // namespace kolibri
