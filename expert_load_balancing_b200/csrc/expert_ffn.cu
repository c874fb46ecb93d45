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
// pairs (tcgen05.mma.cta_group::2, M = 256 rows, N = 256 columns, bf16 in,
// fp32 accumulate in TMEM, two accumulators so the epilogue of one tile
// runs under the MMAs of the next).  Tiles are (expert, 256-row block,
// column block); the kernel maps a tile index to them on the device from
// the offsets, so no host round trip is needed between the permutation and
// the GEMMs.  A row block may run past its expert's segment: those rows are
// loaded (or zero-filled past the end) but never stored.  In the gate/up
// projection the leader CTA loads 128 gate rows and its partner the 128 up
// rows of the same hidden units, so accumulator columns c and c + 128 of a
// row are the gate and up value of one unit and the epilogue forms the
// SwiGLU product in registers.  No load uses cluster multicast.
#include <cuda_bf16.h>

#include "launch.h"
#include "gemm_pair.cuh"

namespace kolibri {

namespace {

using namespace gemm;

constexpr int kThreads = 192;            // warp 0 TMA, warp 1 TMEM + MMA, warps 2..5 epilogue
constexpr int kEpiWarps = 4;
constexpr int kTileM = 2 * kBM;          // 256 rows per pair
constexpr int kTileN = 256;              // accumulator columns per tile
constexpr int kHalfN = kTileN / 2;       // B rows per CTA
constexpr int kAccCols = 2 * kTileN;     // two accumulators
constexpr int kMaxGroups = KOLIBRI_MAX_EXPERTS;
constexpr uint32_t kStageBytes = kBM * kBK * 2 + kHalfN * kBK * 2;   // 32 KB

struct GroupedParams {
  const int64_t* offsets;   // [G + 1] row segments, or null: one group [0, rows)
  int64_t rows;             // rows of A (N*K routed, N shared)
  int G;                    // groups (experts)
  int kdim;                 // reduction length (d, or F)
  int n_tiles;              // column blocks per row block
  int ncols;                // output row length (F for gate/up, d for down)
  int gate_up_rows;         // gate/up: 2F (B rows per expert); down: d
  int stages;
  int b_stream;             // 1: weights read about once (routed), evict them first
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

// Row-block prefix over the groups, in shared memory: mt[g] = row blocks of
// groups before g; mt[G] = all row blocks.
struct TileMap {
  const int32_t* mt;
  const int64_t* offsets;
  int64_t rows;
  int G, n_tiles;
  __device__ __forceinline__ int64_t total() const { return static_cast<int64_t>(mt[G]) * n_tiles; }
  // tile -> group, first row of its pair block, rows left in the group from there, column block
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
    const int64_t start = offsets ? offsets[g] : 0;
    const int64_t end = offsets ? offsets[g + 1] : rows;
    row0 = start + static_cast<int64_t>(mb - mt[g]) * kTileM;
    left = end - row0;
  }
};

// All threads: mt[0..G] from the offsets (a block-wide exclusive scan).
__device__ void build_tile_prefix(const GroupedParams& p, int32_t* mt, int32_t* warp_tot) {
  constexpr int kPer = (kMaxGroups + kThreads - 1) / kThreads;   // 3
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t v[kPer];
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int g = tid * kPer + i;
    int32_t c = 0;
    if (g < p.G) {
      const int64_t len = p.offsets ? (p.offsets[g + 1] - p.offsets[g]) : p.rows;
      c = static_cast<int32_t>((len + kTileM - 1) / kTileM);
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

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat16 a = __float2bfloat16_rn(lo), b = __float2bfloat16_rn(hi);
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

// ---- the grouped projection ---------------------------------------------

// kGateUp: A = x rows [rows, d], B = the experts' stacked [gate; up]
// weights [G * 2F, d], out = bf16 h [rows, F]; tile column block n covers
// hidden units [128 n, 128 n + 128).  Otherwise: A = h [rows, F], B = the
// down weights [G * d, F], out = fp32 [rows, d]; column block n covers
// output columns [256 n, 256 n + 256).
template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                       const __grid_constant__ CUtensorMap tm_b, const GroupedParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int32_t mt_s[kMaxGroups + 1];
  __shared__ int32_t warp_tot[kThreads / 32];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t ring = (raw + 1023u) & ~1023u;
  Bars bars{ring + kStageBytes * static_cast<uint32_t>(p.stages)};
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
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_a)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_b)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(bars.holder()),
                 "r"(kAccCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  build_tile_prefix(p, mt_s, warp_tot);
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(holder_ptr);
  const TileMap tmap{mt_s, p.offsets, p.rows, p.G, p.n_tiles};
  const int64_t tiles = tmap.total();
  const int k_blocks = p.kdim / kBK;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer of this CTA; both CTAs' copies land on the leader's full barrier
      // A row blocks are read by every column block; routed weights about once
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = p.b_stream ? policy_evict_first() : policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int64_t tile = cid; tile < tiles; tile += ncl) {
        int g, n;
        int64_t row0, left;
        tmap.map(tile, g, row0, left, n);
        const int a_row = static_cast<int>(row0 + rank * kBM);
        const int b_row = kGateUp
            ? g * p.gate_up_rows + static_cast<int>(rank) * (p.gate_up_rows / 2) + n * kHalfN
            : g * p.gate_up_rows + n * kTileN + static_cast<int>(rank) * kHalfN;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(bars.empty(stage), phase ^ 1u)) { ok = false; break; }
          const uint32_t fb = map_to_rank(bars.full(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(bars.full(stage), 2u * kStageBytes);
          const uint32_t a_dst = ring + kStageBytes * stage;
          tma_load_2d_pair(a_dst, &tm_a, kb * kBK, a_row, fb, pol_a);
          tma_load_2d_pair(a_dst + kBM * kBK * 2, &tm_b, kb * kBK, b_row, fb, pol_b);
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
      // the pair's single MMA thread: M = 256, N = 256, 4 MMAs of K = 16 per k-block
      const uint32_t idesc = make_idesc(kTileM, kTileN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int64_t tile = cid; tile < tiles; tile += ncl) {
        if (!mbar_wait(bars.tempty(acc), acc_phase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kTileN);
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(bars.full(stage), phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = ring + kStageBytes * stage;
          const uint64_t a_desc = sw128_desc(a_addr);
          const uint64_t b_desc = sw128_desc(a_addr + kBM * kBK * 2);
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks)
            tc_mma_pair(d_tmem, a_desc + 2u * ks, b_desc + 2u * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
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
    // epilogue warps 2..5: thread = row (TMEM lane); the lane quarter is warp % 4
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = cid; tile < tiles; tile += ncl) {
      if (!mbar_wait(bars.tfull(acc), acc_phase)) break;
      tc_fence_after();
      int g, n;
      int64_t row0, left;
      tmap.map(tile, g, row0, left, n);
      const int64_t local = static_cast<int64_t>(rank) * kBM + quarter * 32 + lane;
      const bool valid = local < left;
      const int64_t row = row0 + local;
      const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(acc * kTileN);
      if constexpr (kGateUp) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.ncols + n * kHalfN;
#pragma unroll 1
        for (int c = 0; c < kHalfN; c += 32) {
          uint32_t gr[32], ur[32];
          tmem_ld32(t0 + static_cast<uint32_t>(c), gr);
          tmem_ld32(t0 + static_cast<uint32_t>(kHalfN + c), ur);
          tmem_wait_ld();
          uint32_t hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = silu_f32(__uint_as_float(gr[2 * i])) * __uint_as_float(ur[2 * i]);
            const float h1 = silu_f32(__uint_as_float(gr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]);
            hv[i] = pack_bf16x2(h0, h1);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
          }
        }
      } else {
        float* out = static_cast<float*>(p.out) + row * p.ncols + n * kTileN;
#pragma unroll 1
        for (int c = 0; c < kTileN; c += 32) {
          uint32_t r[32];
          tmem_ld32(t0 + static_cast<uint32_t>(c), r);
          tmem_wait_ld();
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(bars.tempty(acc), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
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

// x_perm[p] = x[perm[p] / K]: a warp per row, 16-byte pieces.
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
    for (int i = lane; i < row_pieces; i += 32) dst[i] = __ldg(src + i);
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
cudaError_t launch_expert_gemm(const void* a, int64_t rows, const int64_t* offsets, int G,
                               const void* w, void* out, int kdim, int ncols, int w_rows_per_group,
                               cudaStream_t s) {
  GroupedParams p{};
  p.offsets = offsets;
  p.rows = rows;
  p.G = G;
  p.kdim = kdim;
  p.ncols = ncols;
  p.gate_up_rows = w_rows_per_group;
  p.n_tiles = kGateUp ? ncols / kHalfN : ncols / kTileN;
  p.b_stream = offsets != nullptr;
  p.out = out;
  CUtensorMap tm_a, tm_b;
  if (!encode_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a, static_cast<uint64_t>(kdim),
                 static_cast<uint64_t>(rows), kBK, kBM) ||
      !encode_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, static_cast<uint64_t>(kdim),
                 static_cast<uint64_t>(G) * w_rows_per_group, kBK, kHalfN))
    return cudaErrorInvalidValue;
  auto kern = expert_gemm_kernel<kGateUp>;
  cudaFuncAttributes fa;
  cudaError_t err = cudaFuncGetAttributes(&fa, kern);
  if (err != cudaSuccess) return err;
  const size_t fixed = 1024 /*alignment slack*/ + kBarBytes;
  const size_t avail = static_cast<size_t>(kSmemLimit) - fa.sharedSizeBytes - fixed;
  int stages = static_cast<int>(avail / kStageBytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  p.stages = stages;
  const size_t smem = fixed + static_cast<size_t>(kStageBytes) * stages;
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
  // at most one pair per tile: row blocks <= rows / 256 + G (one partial block per group)
  const int64_t tiles_max = ((rows + kTileM - 1) / kTileM + G) * p.n_tiles;
  const int64_t clusters = tiles_max < mc ? tiles_max : mc;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  err = cudaLaunchKernelEx(&cfg, kern, tm_a, tm_b, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

bool expert_shape_supported(int32_t d, int32_t F, int32_t E) {
  return d >= kTileN && d % kTileN == 0 && F >= kHalfN && F % kHalfN == 0 && E >= 1 &&
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
  int64_t blocks = (NK + 7) / 8;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
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
