// router_logits.cu -- Z = x W^T on the 5th-generation tensor cores.
//
// "Kolibri Pre-Training from Scratch" 6.1 (router logits Z in R^{T x E});
// "Kolibri 1 im Detail", routing and FP8 sections: the router stays bf16 and
// its logits are fp32, tokens [N, 2560] -> logits [N, 384].
//
// Design (one CTA per SM, persistent over 128-token tiles):
//   warp 0      TMA producer: x tile [128 x 64] and W [E x 64] per k-block,
//               128-byte swizzle, into a ring of shared-memory stages;
//   warp 1      owns the TMEM allocation and issues tcgen05.mma (kind::f16,
//               bf16 x bf16 -> fp32, M = 128, N = one or two expert chunks of
//               at most 256) from a single thread, committing each stage
//               back to the producer and each finished tile to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (thread = token
//               row, TMEM lane) and 16-byte stores of Z.
// The whole E-wide row tile lives in TMEM (E <= 512 columns), so each x tile
// is read from HBM exactly once and W (<= 0.5 MB per k-block pass) stays in
// L2.  No cluster multicast is used.
#include <cuda.h>

#include "launch.h"
#include "common.cuh"

namespace kolibri {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;                  // one 128-byte swizzle atom of bf16
constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 227 * 1024;

struct GemmShape {
  int64_t N;
  int d, E;
  int nchunks, chunk_n;   // expert chunks per MMA step and their width
  int stages;
  uint32_t tmem_cols;
  int64_t num_tiles;
};

// ---- PTX wrappers -------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar), "l"(policy)
      : "memory");
}

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

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
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
    router_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_w, float* __restrict__ z,
                       const GemmShape sh) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t a_bytes = kBM * kBK * 2;
  const uint32_t b_bytes = static_cast<uint32_t>(sh.nchunks * sh.chunk_n) * kBK * 2;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const uint32_t bars = base + stage_bytes * sh.stages;
  // barrier block: full[kMaxStages], empty[kMaxStages], tmem_full, tmem_empty, holder
  auto full_bar = [bars](int s) { return bars + 8u * s; };
  auto empty_bar = [bars](int s) { return bars + 8u * (kMaxStages + s); };
  const uint32_t tmem_full = bars + 8u * (2 * kMaxStages);
  const uint32_t tmem_empty = tmem_full + 8u;
  const uint32_t holder = tmem_empty + 8u;
  uint8_t* const holder_ptr = smem_raw + (holder - raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k_blocks = sh.d / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < sh.stages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 128);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder),
                 "r"(sh.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(holder_ptr);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_first();
      const uint64_t pol_w = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < sh.num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), stage_bytes);
          const uint32_t a_dst = base + stage_bytes * stage;
          const uint32_t b_dst = a_dst + a_bytes;
          tma_load_2d(a_dst, &tm_x, kb * kBK, static_cast<int>(tile * kBM), full_bar(stage), pol_x);
          for (int c = 0; c < sh.nchunks; ++c)
            tma_load_2d(b_dst + static_cast<uint32_t>(c * sh.chunk_n) * (kBK * 2), &tm_w, kb * kBK,
                        c * sh.chunk_n, full_bar(stage), pol_w);
          if (++stage == sh.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kBM, sh.chunk_n);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < sh.num_tiles && ok; tile += gridDim.x) {
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
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks) {
            for (int c = 0; c < sh.nchunks; ++c) {
              const uint64_t b_desc =
                  sw128_desc(b_addr + static_cast<uint32_t>(c * sh.chunk_n) * (kBK * 2));
              // advancing 16 bf16 along K moves 32 bytes inside the swizzle atom
              tc_mma(tmem_base + static_cast<uint32_t>(c * sh.chunk_n), a_desc + 2u * ks,
                     b_desc + 2u * ks, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit(empty_bar(stage));
          if (++stage == sh.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tmem_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    // epilogue warps 2..5; TMEM lane quarter is fixed by warp % 4
    const int quarter = warp & 3;
    uint32_t acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < sh.num_tiles; tile += gridDim.x) {
      if (!mbar_wait(tmem_full, acc_phase)) break;
      tc_fence_after();
      const int64_t row = tile * kBM + quarter * 32 + lane;
      float* zrow = z + row * sh.E;
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      for (int c0 = 0; c0 < sh.E; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_addr + static_cast<uint32_t>(c0), r);
        tmem_wait_ld();
        if (row < sh.N) {
          const int ncols = (sh.E - c0) < 32 ? (sh.E - c0) : 32;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (4 * q < ncols) {
              float4 v = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                     __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
              *reinterpret_cast<float4*>(zrow + c0 + 4 * q) = v;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tmem_empty);
      acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
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

bool encode_bf16_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer,
                    uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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
  int cn = (E + sh.nchunks - 1) / sh.nchunks;
  sh.chunk_n = (cn + 15) / 16 * 16;
  const int cols = sh.nchunks * sh.chunk_n;
  uint32_t tc = 32;
  while (tc < static_cast<uint32_t>(cols)) tc <<= 1;
  sh.tmem_cols = tc;
  const size_t stage_bytes = static_cast<size_t>(kBM) * kBK * 2 + static_cast<size_t>(cols) * kBK * 2;
  const size_t fixed = 1024 /*alignment slack*/ + 8 * (2 * kMaxStages + 3);
  int stages = static_cast<int>((kSmemLimit - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  sh.stages = stages;
  sh.num_tiles = (N + kBM - 1) / kBM;

  CUtensorMap tm_x, tm_w;
  if (!encode_bf16_2d(&tm_x, x, static_cast<uint64_t>(d), static_cast<uint64_t>(N), kBK, kBM))
    return cudaErrorInvalidValue;
  if (!encode_bf16_2d(&tm_w, w, static_cast<uint64_t>(d), static_cast<uint64_t>(E), kBK,
                      static_cast<uint32_t>(sh.chunk_n)))
    return cudaErrorInvalidValue;

  const size_t smem = fixed + stage_bytes * stages;
  cudaError_t err = cudaFuncSetAttribute(router_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  int sms = device_sm_count();
  int64_t grid = sh.num_tiles < sms ? sh.num_tiles : sms;
  router_gemm_kernel<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(tm_x, tm_w, z, sh);
  return cudaGetLastError();
}

}  // namespace kolibri
