// router_logits.cu -- Z = x W^T on the 5th-generation tensor cores.
//
// "Kolibri Pre-Training from Scratch" 6.1 (router logits Z in R^{T x E});
// "Kolibri 1 im Detail", routing and FP8 sections: the router stays bf16 and
// its logits are fp32, tokens [N, 2560] -> logits [N, 384].
//
// Design: persistent kernel, clusters of two CTAs on an SM pair.  A pair
// owns a 256-token tile; the leader issues tcgen05.mma.cta_group::2 (M = 256,
// bf16 x bf16 -> fp32, N = one or two expert chunks of at most 256), so each
// CTA stages its own 128 token rows but only HALF of the router weights: per
// 64-wide k-block a CTA loads 16 KB of x and E x 64 B of W instead of
// E x 128 B, which halves the L2 -> SM traffic per FLOP of a one-CTA tile.
//   warp 0      TMA producer (both CTAs; completions land on the leader's
//               full barrier)
//   warp 1      TMEM owner; in the leader, the single MMA-issuing thread
//   warps 2..5  epilogue: tcgen05.ld (thread = token row = TMEM lane),
//               registers -> 128B-swizzled shared staging -> TMA tensor store
// The E-wide accumulator of a tile lives in TMEM (E <= 512 columns), so every
// x tile is read from HBM once and W stays L2-resident.  No load uses cluster
// multicast; only tcgen05.commit multicasts its arrival to both CTAs.
#include <cuda.h>

#include "launch.h"
#include "common.cuh"

namespace kolibri {

namespace {

constexpr int kBM = 128;                 // token rows per CTA (256 per pair)
constexpr int kBK = 64;                  // one 128-byte swizzle atom of bf16
constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr int kEpiWarps = 4;
constexpr int kStoreCols = 32;           // fp32 columns per TMA store box
constexpr int kStageBuf = kStoreCols * 32 * 4;  // 4 KB: 32 rows x 128 B
constexpr int kEpiBufs = 4;              // staging buffers per epilogue warp
constexpr int kSmemLimit = 227 * 1024;

struct GemmShape {
  int64_t N;
  int d, E;
  int nchunks, chunk_n;   // expert chunks per MMA step (pair-wide width)
  int stages;
  uint32_t tmem_cols;
  int64_t num_pairs;      // 256-token tiles
};

// ---- PTX wrappers -------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// shared::cluster address of the same shared variable in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// TMA 2D load into this CTA's shared memory; completion bytes are counted on
// the mbarrier at `bar_cluster` (the pair leader's barrier).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0,
                                                 int c1, uint32_t bar_cluster, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int c0, int c1, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most kEpiBufs - 1 stores may still be reading their staging buffer
__device__ __forceinline__ void bulk_wait_read_ring() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kEpiBufs - 1) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on the barrier at the same offset in both CTAs of the pair
// when all previously issued MMAs of this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzle
// layout written by TMA: rows of 128 bytes, 8-row groups 1024 bytes apart
// (stride byte offset), version 1, swizzle mode 2 (128B).  The leading
// byte offset is unused for this layout.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3fffu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- kernel ---------------------------------------------------------------

__global__ void __launch_bounds__(kThreads, 1)
    router_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                            const __grid_constant__ CUtensorMap tm_w,
                            const __grid_constant__ CUtensorMap tm_z, const GemmShape sh) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const int half_n = sh.chunk_n / 2;                       // W rows per CTA per chunk
  const uint32_t a_bytes = kBM * kBK * 2;
  const uint32_t b_bytes = static_cast<uint32_t>(sh.nchunks * half_n) * kBK * 2;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const uint32_t staging = base + stage_bytes * sh.stages;  // epilogue buffers (1 KB aligned)
  const uint32_t bars = staging + kEpiWarps * kEpiBufs * kStageBuf;
  auto full_bar = [bars](int s) { return bars + 8u * s; };
  auto empty_bar = [bars](int s) { return bars + 8u * (kMaxStages + s); };
  const uint32_t tmem_full = bars + 8u * (2 * kMaxStages);
  const uint32_t tmem_empty = tmem_full + 8u;
  const uint32_t holder = tmem_empty + 8u;
  uint8_t* const holder_ptr = smem_raw + (holder - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int k_blocks = sh.d / kBK;
  const uint32_t cid = cluster_id_x(), ncl = num_clusters_x();

  if (threadIdx.x == 0) {
    for (int s = 0; s < sh.stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * kEpiWarps);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_z)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder),
                 "r"(sh.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(holder_ptr);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_first();
      const uint64_t pol_w = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t pt = cid; pt < sh.num_pairs && ok; pt += ncl) {
        const int row0 = static_cast<int>(pt * 2 * kBM + rank * kBM);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), 2u * stage_bytes);
          const uint32_t a_dst = base + stage_bytes * stage;
          const uint32_t b_dst = a_dst + a_bytes;
          tma_load_2d_pair(a_dst, &tm_x, kb * kBK, row0, fb, pol_x);
          for (int c = 0; c < sh.nchunks; ++c)
            tma_load_2d_pair(b_dst + static_cast<uint32_t>(c * half_n) * (kBK * 2), &tm_w, kb * kBK,
                             c * sh.chunk_n + static_cast<int>(rank) * half_n, fb, pol_w);
          if (++stage == sh.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = make_idesc(2 * kBM, sh.chunk_n);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t pt = cid; pt < sh.num_pairs && ok; pt += ncl) {
        if (!mbar_wait(tmem_empty, acc_phase ^ 1u)) break;
        tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(full_bar(stage), phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = base + stage_bytes * stage;
          const uint32_t b_addr = a_addr + a_bytes;
          const uint64_t a_desc = sw128_desc(a_addr);
          // one expert chunk at a time: back-to-back MMAs into the same
          // accumulator run faster than alternating accumulators
          for (int c = 0; c < sh.nchunks; ++c) {
            const uint64_t b_desc =
                sw128_desc(b_addr + static_cast<uint32_t>(c * half_n) * (kBK * 2));
#pragma unroll
            for (int ks = 0; ks < kBK / 16; ++ks) {
              // 16 bf16 along K = 32 bytes inside the swizzle atom
              tc_mma_pair(tmem_base + static_cast<uint32_t>(c * sh.chunk_n), a_desc + 2u * ks,
                          b_desc + 2u * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit_pair(empty_bar(stage));
          if (++stage == sh.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(tmem_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    // epilogue warps 2..5; TMEM lane quarter is fixed by warp % 4
    const int quarter = warp & 3;
    const int ew = warp - 2;
    const uint32_t buf0 = staging + static_cast<uint32_t>(ew * kEpiBufs * kStageBuf);
    const uint32_t empty_leader = map_to_rank(tmem_empty, 0);
    uint32_t acc_phase = 0;
    int nbuf = 0;
    for (int64_t pt = cid; pt < sh.num_pairs; pt += ncl) {
      if (!mbar_wait(tmem_full, acc_phase)) break;
      tc_fence_after();
      const int row_base = static_cast<int>(pt * 2 * kBM + rank * kBM + quarter * 32);
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      for (int c0 = 0; c0 < sh.E; c0 += kStoreCols) {
        uint32_t r[32];
        tmem_ld32(lane_addr + static_cast<uint32_t>(c0), r);
        tmem_wait_ld();
        // staging buffer: 32 rows x 128 bytes, 16-byte chunks swizzled by row
        const uint32_t buf = buf0 + static_cast<uint32_t>(nbuf * kStageBuf);
        if (lane == 0) bulk_wait_read_ring();  // the store that last used this buffer has read it
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

// ---- host -----------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, size_t elem, const void* ptr,
               uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_router_logits(const void* x, const void* w, float* z, int64_t N, int32_t d,
                                 int32_t E, cudaStream_t s) {
  GemmShape sh{};
  sh.N = N;
  sh.d = d;
  sh.E = E;
  sh.nchunks = (E + 255) / 256;
  const int cn = (E + sh.nchunks - 1) / sh.nchunks;
  sh.chunk_n = (cn + 15) / 16 * 16;
  if (sh.chunk_n < 32) sh.chunk_n = 32;  // M = 256 needs N >= 32 so each half is >= 16 rows
  const int cols = sh.nchunks * sh.chunk_n;
  uint32_t tc = 32;
  while (tc < static_cast<uint32_t>(cols)) tc <<= 1;
  sh.tmem_cols = tc;
  const size_t stage_bytes =
      static_cast<size_t>(kBM) * kBK * 2 + static_cast<size_t>(cols / 2) * kBK * 2;
  const size_t fixed = 1024 /*alignment slack*/ + kEpiWarps * kEpiBufs * kStageBuf + 8 * (2 * kMaxStages + 3);
  int stages = static_cast<int>((kSmemLimit - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  sh.stages = stages;
  sh.num_pairs = (N + 2 * kBM - 1) / (2 * kBM);

  CUtensorMap tm_x, tm_w, tm_z;
  if (!encode_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, static_cast<uint64_t>(d),
                 static_cast<uint64_t>(N), kBK, kBM))
    return cudaErrorInvalidValue;
  if (!encode_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, static_cast<uint64_t>(d),
                 static_cast<uint64_t>(E), kBK, static_cast<uint32_t>(sh.chunk_n / 2)))
    return cudaErrorInvalidValue;
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

}  // namespace kolibri
