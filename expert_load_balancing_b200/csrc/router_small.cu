// router_small.cu -- router logits Z = x W^T for small token counts (decode
// batches: a few to a few thousand tokens per layer).
//
// "Kolibri Pre-Training from Scratch" 6.1 (router logits); "Kolibri 1 im
// Detail", routing: bf16 router, fp32 logits.
//
// At these sizes the work is reading W (E x d bf16, 1.97 MB at E = 384,
// d = 2560) once per layer, plus latency.  The pair GEMM gives the whole
// batch to one SM pair and walks d in 40 pipelined steps (about 30 us at
// any small N); here every CTA takes 8 to 64 experts x 16 to 64 tokens x
// an eighth (or a quarter) of d, issues all of its loads at once (one memory
// round trip), and the CTAs of a cluster add their partial tiles through
// distributed shared memory in a fixed order, so results repeat bit for bit
// and no workspace is needed.  The tiles are tensor-core mma.sync m16n8k16 (bf16
// in, fp32 accumulate): at these sizes the kernel waits on W and on
// latency, not on tensor throughput, and a tcgen05 tile would add TMEM
// allocation and completion round trips to every CTA without shortening
// either.
#include <cuda_bf16.h>

#include "launch.h"
#include "common.cuh"
#include "pdl.cuh"

namespace kolibri {

namespace {

constexpr int kTokPerWarp = 16;          // one m16 tile per warp

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  // pred false: 16 zero bytes (rows past N or experts past E)
  const int bytes = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t cluster_rank_small() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_small() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// grid: x = expert tiles of kX, y = token tiles of 16 * kWarps, z = the kS
// slices of d (one cluster of kS CTAs).  Each warp computes 16 tokens x kX
// experts over its CTA's slice.  Dynamic shared memory: the token rows and
// the kX W rows of the slice (rows padded by 16 bytes so the eight rows an
// ldmatrix reads fall on different banks), then the fp32 partial tile.
// After a cluster barrier every CTA adds up 1/kS of the tile, reading the
// kS partials in slice order 0 .. kS-1 wherever they are, so the sum of an
// element does not depend on which CTA forms it.
template <int kWarps, int kX, int kS>
__global__ void __launch_bounds__(32 * kWarps) small_logits_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w, float* __restrict__ z,
    int64_t N, int d, int E) {
  constexpr int kTok = kTokPerWarp * kWarps;
  constexpr int kNT = kX / 8;                        // n8 tiles per warp
  constexpr int kTile = kTok * kX;
  static_assert(kX % 16 == 0 || kX == 8, "B tiles come in pairs unless kX is 8");
  static_assert(kTile % kS == 0, "the tile splits evenly over the cluster");
  extern __shared__ __align__(16) uint8_t sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ks = d / kS;                             // this CTA's width of d (multiple of 16)
  const int ld = ks + 8;                             // padded row, in bf16
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sm);
  __nv_bfloat16* ws = xs + kTok * ld;
  float* part = reinterpret_cast<float*>(ws + kX * ld);   // [kTok][kX]
  const uint32_t rank = cluster_rank_small();
  const int k0 = static_cast<int>(rank) * ks;
  const int e0 = blockIdx.x * kX;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kTok;
  pdl_wait();       // x may come from the kernel before this one
  pdl_trigger();

  // every load at once: one round trip per CTA
  const int pieces = ks / 8;                         // 16-byte pieces per row
  for (int i = tid; i < kTok * pieces; i += 32 * kWarps) {
    const int r = i / pieces, pc = i - r * pieces;
    const int64_t t = t0 + r;
    const bool ok = t < N;
    cp_async16(smem_u32(xs + r * ld + pc * 8), x + (ok ? t : 0) * d + k0 + pc * 8, ok);
  }
  for (int i = tid; i < kX * pieces; i += 32 * kWarps) {
    const int r = i / pieces, pc = i - r * pieces;
    const bool ok = e0 + r < E;
    cp_async16(smem_u32(ws + r * ld + pc * 8), w + static_cast<int64_t>(ok ? e0 + r : 0) * d + k0 + pc * 8,
               ok);
  }
  cp_async_commit_wait_all();
  __syncthreads();

  float acc[kNT][4];
#pragma unroll
  for (int n = 0; n < kNT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int ar = warp * kTokPerWarp + (lane & 7) + ((lane >> 3) & 1) * 8;
  const uint32_t a_base = smem_u32(xs + ar * ld + (lane >> 4) * 8);
  // x4 over B: matrices (n tile 2p, k lo), (2p, k hi), (2p+1, k lo), (2p+1, k hi)
  const uint32_t b_base = (kX == 8)
      ? smem_u32(ws + (lane & 7) * ld + ((lane >> 3) & 1) * 8)
      : smem_u32(ws + ((lane & 7) + (lane >> 4) * 8) * ld + ((lane >> 3) & 1) * 8);
#pragma unroll 2
  for (int kk = 0; kk < ks; kk += 16) {
    uint32_t a0, a1, a2, a3;
    ldmatrix_x4(a_base + 2u * kk, a0, a1, a2, a3);
    if constexpr (kX == 8) {
      uint32_t b0, b1;
      ldmatrix_x2(b_base + 2u * kk, b0, b1);
      mma_bf16_16816(acc[0], a0, a1, a2, a3, b0, b1);
    } else {
#pragma unroll
      for (int pr = 0; pr < kNT / 2; ++pr) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(b_base + 2u * (pr * 16 * ld + kk), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * pr], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * pr + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }
  // accumulator of n tile n: rows lane/4 and lane/4 + 8, columns 8n + 2 (lane % 4) and + 1
  const int rr = warp * kTokPerWarp + (lane >> 2), cc = 2 * (lane & 3);
#pragma unroll
  for (int n = 0; n < kNT; ++n) {
    *reinterpret_cast<float2*>(part + rr * kX + 8 * n + cc) = make_float2(acc[n][0], acc[n][1]);
    *reinterpret_cast<float2*>(part + (rr + 8) * kX + 8 * n + cc) = make_float2(acc[n][2], acc[n][3]);
  }
  cluster_sync_small();
  {
    constexpr int kPer = kTile / kS;                 // elements this CTA adds up
    const int i0 = static_cast<int>(rank) * kPer;
    for (int i = i0 + tid; i < i0 + kPer; i += 32 * kWarps) {
      const int r = i / kX, c = i - r * kX;
      const int64_t t = t0 + r;
      const uint32_t addr = smem_u32(part + i);
      float v = ld_cluster_f32(addr, 0);
#pragma unroll
      for (int q = 1; q < kS; ++q) v = __fadd_rn(v, ld_cluster_f32(addr, static_cast<uint32_t>(q)));
      if (t < N && e0 + c < E) z[t * E + e0 + c] = v;
    }
  }
  cluster_sync_small();   // every CTA keeps its partials until all have been read
}

template <int kWarps, int kX, int kS>
cudaError_t launch_small(const __nv_bfloat16* x, const __nv_bfloat16* w, float* z, int64_t N, int d,
                         int E, cudaStream_t s) {
  constexpr int kTok = kTokPerWarp * kWarps;
  if (d % (16 * kS) != 0) return cudaErrorInvalidValue;
  const int64_t ty = (N + kTok - 1) / kTok;
  if (ty > 65535) return cudaErrorInvalidValue;
  const int ld = d / kS + 8;
  const size_t smem = static_cast<size_t>(kTok + kX) * ld * 2 + sizeof(float) * kTok * kX;
  auto kern = small_logits_kernel<kWarps, kX, kS>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(static_cast<unsigned>((E + kX - 1) / kX), static_cast<unsigned>(ty), kS),
                    dim3(32 * kWarps), smem, s, dim3(1, 1, kS), x, w, z, N, d, E);
}

}  // namespace

// Small batches go here when the pair GEMM would use few SMs.
bool router_small_preferred(int64_t N) { return N <= kSmallTokenLimit; }

cudaError_t launch_router_logits_small(const void* x, const void* w, float* z, int64_t N, int32_t d,
                                       int32_t E, cudaStream_t s) {
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* wb = static_cast<const __nv_bfloat16*>(w);
  // tiles by batch size, measured over 50 layers of d = 2560, E = 384 (x and W
  // of each layer distinct): 4.5 us at N <= 16, 5.7 at 64, 8.2 at 256, 15 at
  // 512, 25 at 1024.  d not a multiple of 128 takes the four-way split.
  if (d % 128 != 0) {
    if (N <= 16) return launch_small<1, 8, 4>(xb, wb, z, N, d, E, s);
    if (N <= 32) return launch_small<2, 8, 4>(xb, wb, z, N, d, E, s);
    return launch_small<4, 32, 4>(xb, wb, z, N, d, E, s);
  }
  if (N <= 16) return launch_small<1, 8, 8>(xb, wb, z, N, d, E, s);
  if (N <= 32) return launch_small<2, 16, 8>(xb, wb, z, N, d, E, s);
  if (N <= 512) return launch_small<4, 32, 8>(xb, wb, z, N, d, E, s);
  return launch_small<4, 64, 8>(xb, wb, z, N, d, E, s);
}

cudaError_t launch_router_logits_by_size(const void* x, const void* w, float* z, int64_t N,
                                         int32_t d, int32_t E, cudaStream_t s) {
  // the same kernel, and so the same sums, as router_forward_by_size picks
  if (router_decode_supported(N, d, E, 1)) {
    const cudaError_t err = launch_router_decode(x, w, nullptr, z, N, d, E, 1, nullptr, nullptr, nullptr, s);
    if (err != cudaErrorNotSupported) return err;
  }
  if (router_small_preferred(N)) return launch_router_logits_small(x, w, z, N, d, E, s);
  return launch_router_logits(x, w, z, N, d, E, s);
}

cudaError_t router_forward_by_size(const void* x, const void* w, const float* bias, float* z,
                                   int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                   float* gates, float* alpha, cudaStream_t s) {
  if (router_decode_supported(N, d, E, K)) {
    const cudaError_t err = launch_router_decode(x, w, bias, z, N, d, E, K, ids, gates, alpha, s);
    if (err != cudaErrorNotSupported) return err;
  }
  if (router_small_preferred(N)) {
    // decode batches: the clustered logits kernel, then one row per warp
    const cudaError_t err = launch_router_logits_small(x, w, z, N, d, E, s);
    if (err != cudaSuccess) return err;
    return launch_topk(z, bias, N, E, K, ids, gates, alpha, s);
  }
  return router_forward_any(x, w, bias, z, N, d, E, K, ids, gates, alpha, s);
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_small)

}  // namespace kolibri
