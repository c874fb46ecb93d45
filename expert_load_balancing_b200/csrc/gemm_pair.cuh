// gemm_pair.cuh -- the main loop shared by the router GEMM kernels.
//
// "Kolibri Pre-Training from Scratch" 6.1 (router logits Z in R^{T x E});
// "Kolibri 1 im Detail", routing and FP8 sections: the router stays bf16 and
// its logits are fp32, tokens [N, 2560] -> logits [N, 384].
//
// A persistent kernel runs on clusters of two CTAs (an SM pair).  A pair owns
// a 256-token tile; the leader issues tcgen05.mma.cta_group::2 (M = 256,
// bf16 x bf16 -> fp32, N = one or two expert chunks of at most 256), so each
// CTA stages its own 128 token rows but only HALF of the router weights: per
// 64-wide k-block a CTA loads 16 KB of x and E x 64 B of W instead of
// E x 128 B, which halves the L2 -> SM traffic per FLOP of a one-CTA tile.
// The E-wide accumulator of a tile lives in TMEM (E <= 512 columns), so every
// x tile is read from HBM once and W stays L2-resident.  No load uses cluster
// multicast; only tcgen05.commit multicasts its arrival to both CTAs.
//
// This header holds the PTX wrappers, the TMA producer loop and the MMA loop;
// the kernels that include it differ only in their epilogues.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace kolibri {
namespace gemm {

constexpr int kBM = 128;                 // token rows per CTA (256 per pair)
constexpr int kBK = 64;                  // one 128-byte swizzle atom of bf16
constexpr int kMaxStages = 8;
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
// at most N bulk groups of this thread may still be reading shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
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

// ---- pipeline pieces ------------------------------------------------------

// Shared-memory map of the operand ring and its barriers.  `base` is the
// 1 KB aligned start of dynamic shared memory; `bars` holds
// 2 * kMaxStages + 3 eight-byte words after the epilogue's own region.
struct Ring {
  uint32_t base, a_bytes, b_bytes, stage_bytes, bars;
  int half_n;
  __device__ __forceinline__ uint32_t full_bar(int s) const { return bars + 8u * s; }
  __device__ __forceinline__ uint32_t empty_bar(int s) const { return bars + 8u * (kMaxStages + s); }
  __device__ __forceinline__ uint32_t tmem_full() const { return bars + 8u * (2 * kMaxStages); }
  __device__ __forceinline__ uint32_t tmem_empty() const { return tmem_full() + 8u; }
  __device__ __forceinline__ uint32_t holder() const { return tmem_empty() + 8u; }
};

__device__ __forceinline__ Ring make_ring(const GemmShape& sh, uint32_t base, uint32_t bars) {
  Ring r;
  r.base = base;
  r.half_n = sh.chunk_n / 2;                                  // W rows per CTA per chunk
  r.a_bytes = kBM * kBK * 2;
  r.b_bytes = static_cast<uint32_t>(sh.nchunks * r.half_n) * kBK * 2;
  r.stage_bytes = r.a_bytes + r.b_bytes;
  r.bars = bars;
  return r;
}

// Thread 0: barrier initialisation.  `epi_arrivals` = arrivals per tile on
// the leader's TMEM-empty barrier (epilogue warps of both CTAs).
__device__ __forceinline__ void init_barriers(const GemmShape& sh, const Ring& rg,
                                              uint32_t epi_arrivals) {
  for (int s = 0; s < sh.stages; ++s) {
    mbar_init(rg.full_bar(s), 1);
    mbar_init(rg.empty_bar(s), 1);
  }
  mbar_init(rg.tmem_full(), 1);
  mbar_init(rg.tmem_empty(), epi_arrivals);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One lane: the TMA producer of this CTA.  Both CTAs' copies complete on the
// leader's full barrier, which expects the pair's bytes.
__device__ __forceinline__ void producer_loop(const GemmShape& sh, const Ring& rg,
                                              const CUtensorMap* tm_x, const CUtensorMap* tm_w,
                                              uint32_t rank) {
  const bool leader = rank == 0;
  const int k_blocks = sh.d / kBK;
  const uint32_t cid = cluster_id_x(), ncl = num_clusters_x();
  const uint64_t pol_x = policy_evict_first();
  const uint64_t pol_w = policy_evict_last();
  int stage = 0;
  uint32_t phase = 0;
  for (int64_t pt = cid; pt < sh.num_pairs; pt += ncl) {
    const int row0 = static_cast<int>(pt * 2 * kBM + rank * kBM);
    for (int kb = 0; kb < k_blocks; ++kb) {
      if (!mbar_wait(rg.empty_bar(stage), phase ^ 1u)) return;
      const uint32_t fb = map_to_rank(rg.full_bar(stage), 0);
      if (leader) mbar_arrive_expect_tx(rg.full_bar(stage), 2u * rg.stage_bytes);
      const uint32_t a_dst = rg.base + rg.stage_bytes * stage;
      const uint32_t b_dst = a_dst + rg.a_bytes;
      tma_load_2d_pair(a_dst, tm_x, kb * kBK, row0, fb, pol_x);
      for (int c = 0; c < sh.nchunks; ++c)
        tma_load_2d_pair(b_dst + static_cast<uint32_t>(c * rg.half_n) * (kBK * 2), tm_w, kb * kBK,
                         c * sh.chunk_n + static_cast<int>(rank) * rg.half_n, fb, pol_w);
      if (++stage == sh.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
}

// The leader's single MMA thread.  Per k-block it issues one expert chunk at
// a time: back-to-back MMAs into the same accumulator run faster than
// alternating accumulators.
__device__ __forceinline__ void mma_loop(const GemmShape& sh, const Ring& rg, uint32_t tmem_base) {
  const int k_blocks = sh.d / kBK;
  const uint32_t cid = cluster_id_x(), ncl = num_clusters_x();
  const uint32_t idesc = make_idesc(2 * kBM, sh.chunk_n);
  int stage = 0;
  uint32_t phase = 0, acc_phase = 0;
  for (int64_t pt = cid; pt < sh.num_pairs; pt += ncl) {
    if (!mbar_wait(rg.tmem_empty(), acc_phase ^ 1u)) return;
    tc_fence_after();
    for (int kb = 0; kb < k_blocks; ++kb) {
      if (!mbar_wait(rg.full_bar(stage), phase)) return;
      tc_fence_after();
      const uint32_t a_addr = rg.base + rg.stage_bytes * stage;
      const uint32_t b_addr = a_addr + rg.a_bytes;
      const uint64_t a_desc = sw128_desc(a_addr);
      for (int c = 0; c < sh.nchunks; ++c) {
        const uint64_t b_desc = sw128_desc(b_addr + static_cast<uint32_t>(c * rg.half_n) * (kBK * 2));
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks) {
          // 16 bf16 along K = 32 bytes inside the swizzle atom
          tc_mma_pair(tmem_base + static_cast<uint32_t>(c * sh.chunk_n), a_desc + 2u * ks,
                      b_desc + 2u * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
        }
      }
      tc_commit_pair(rg.empty_bar(stage));
      if (++stage == sh.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    tc_commit_pair(rg.tmem_full());
    acc_phase ^= 1u;
  }
}

// ---- host -----------------------------------------------------------------

// Expert chunking and TMEM width for E experts.  Returns false when the
// shape cannot run (E too large for TMEM).
inline bool plan_shape(int64_t N, int32_t d, int32_t E, GemmShape& sh) {
  sh = GemmShape{};
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
  sh.num_pairs = (N + 2 * kBM - 1) / (2 * kBM);
  return tc <= 512;
}

inline size_t stage_bytes_of(const GemmShape& sh) {
  return static_cast<size_t>(kBM) * kBK * 2 +
         static_cast<size_t>(sh.nchunks * sh.chunk_n / 2) * kBK * 2;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

inline bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, size_t elem, const void* ptr,
                      uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Operand maps of x [N, d] and W [E, d] (bf16, K-major boxes of 64).
inline bool encode_operands(const GemmShape& sh, const void* x, const void* w, CUtensorMap* tm_x,
                            CUtensorMap* tm_w) {
  return encode_2d(tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, static_cast<uint64_t>(sh.d),
                   static_cast<uint64_t>(sh.N), kBK, kBM) &&
         encode_2d(tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, static_cast<uint64_t>(sh.d),
                   static_cast<uint64_t>(sh.E), kBK, static_cast<uint32_t>(sh.chunk_n / 2));
}

}  // namespace gemm
}  // namespace kolibri
