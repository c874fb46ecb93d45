// router_logits.cu -- Z = x W^T on the 5th-generation tensor cores.
//
// "Kolibri Pre-Training from Scratch" 6.1 (router logits Z in R^{T x E});
// "Kolibri 1 im Detail", routing and FP8 sections: the router stays bf16 and
// its logits are fp32, tokens [N, 2560] -> logits [N, 384].
//
// The pair main loop (TMA producer, tcgen05 MMA issue) is in gemm_pair.cuh.
// Warp roles of this kernel:
//   warp 0      TMA producer (both CTAs; completions land on the leader's
//               full barrier)
//   warp 1      TMEM owner; in the leader, the single MMA-issuing thread
//   warps 2..5  epilogue: tcgen05.ld (thread = token row = TMEM lane),
//               registers -> 128B-swizzled shared staging -> TMA tensor store
#include "launch.h"
#include "gemm_pair.cuh"

namespace kolibri {

namespace {

using namespace gemm;

constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kStoreCols = 32;           // fp32 columns per TMA store box
constexpr int kStageBuf = kStoreCols * 32 * 4;  // 4 KB: 32 rows x 128 B
constexpr int kEpiBufs = 4;              // staging buffers per epilogue warp

// ---- kernel ---------------------------------------------------------------

__global__ void __launch_bounds__(kThreads, 1)
    router_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                            const __grid_constant__ CUtensorMap tm_w,
                            const __grid_constant__ CUtensorMap tm_z, const GemmShape sh) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  Ring rg = make_ring(sh, base, 0);
  const uint32_t staging = base + rg.stage_bytes * sh.stages;  // epilogue buffers (1 KB aligned)
  rg.bars = staging + kEpiWarps * kEpiBufs * kStageBuf;
  uint8_t* const holder_ptr = smem_raw + (rg.holder() - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t cid = cluster_id_x(), ncl = num_clusters_x();

  if (threadIdx.x == 0) {
    init_barriers(sh, rg, 2 * kEpiWarps);
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_z)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(rg.holder()),
                 "r"(sh.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(holder_ptr);

  if (warp == 0) {
    if (lane == 0) producer_loop(sh, rg, &tm_x, &tm_w, rank);
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) mma_loop(sh, rg, tmem_base);
  } else {
    // epilogue warps 2..5; TMEM lane quarter is fixed by warp % 4
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const uint32_t buf0 = staging + static_cast<uint32_t>(ew * kEpiBufs * kStageBuf);
    const uint32_t empty_leader = map_to_rank(rg.tmem_empty(), 0);
    uint32_t acc_phase = 0;
    int nbuf = 0;
    for (int64_t pt = cid; pt < sh.num_pairs; pt += ncl) {
      if (!mbar_wait(rg.tmem_full(), acc_phase)) break;
      tc_fence_after();
      const int row_base = static_cast<int>(pt * 2 * kBM + rank * kBM + quarter * 32);
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      for (int c0 = 0; c0 < sh.E; c0 += kStoreCols) {
        uint32_t r[32];
        tmem_ld32(lane_addr + static_cast<uint32_t>(c0), r);
        tmem_wait_ld();
        // staging buffer: 32 rows x 128 bytes, 16-byte chunks swizzled by row
        const uint32_t buf = buf0 + static_cast<uint32_t>(nbuf * kStageBuf);
        if (lane == 0) bulk_wait_read<kEpiBufs - 1>();  // the store that last used this buffer has read it
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t dst = buf + static_cast<uint32_t>(lane * 128 + ((q ^ (lane & 7)) * 16));
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(r[4 * q]),
                       "r"(r[4 * q + 1]), "r"(r[4 * q + 2]), "r"(r[4 * q + 3])
                       : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_z, c0, row_base, buf);
          bulk_commit();
        }
        nbuf = (nbuf + 1 == kEpiBufs) ? 0 : nbuf + 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(empty_leader);
      acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(sh.tmem_cols)
                 : "memory");
  }
}

}  // namespace

cudaError_t launch_router_logits(const void* x, const void* w, float* z, int64_t N, int32_t d,
                                 int32_t E, cudaStream_t s) {
  GemmShape sh;
  if (!plan_shape(N, d, E, sh)) return cudaErrorInvalidValue;
  const size_t stage_bytes = stage_bytes_of(sh);
  const size_t fixed = 1024 /*alignment slack*/ + kEpiWarps * kEpiBufs * kStageBuf + 8 * (2 * kMaxStages + 3);
  int stages = static_cast<int>((kSmemLimit - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  sh.stages = stages;

  CUtensorMap tm_x, tm_w, tm_z;
  if (!encode_operands(sh, x, w, &tm_x, &tm_w)) return cudaErrorInvalidValue;
  if (!encode_2d(&tm_z, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, z, static_cast<uint64_t>(E),
                 static_cast<uint64_t>(N), kStoreCols, 32))
    return cudaErrorInvalidValue;

  const size_t smem = fixed + stage_bytes * stages;
  cudaError_t err = cudaFuncSetAttribute(router_gemm_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
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
  // as many pairs as can be resident at once, at most one per tile
  static int max_clusters = 0;
  if (max_clusters == 0) {
    cfg.gridDim = dim3(2 * static_cast<unsigned>(device_sm_count() / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, router_gemm_pair_kernel, &cfg) != cudaSuccess || n < 1)
      n = device_sm_count() / 2;
    max_clusters = n;
  }
  int64_t clusters = sh.num_pairs < max_clusters ? sh.num_pairs : max_clusters;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  err = cudaLaunchKernelEx(&cfg, router_gemm_pair_kernel, tm_x, tm_w, tm_z, sh);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_logits)

}  // namespace kolibri
