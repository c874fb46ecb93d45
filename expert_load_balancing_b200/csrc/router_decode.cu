// router_decode.cu -- the whole router forward of a decode batch in one
// launch: logits Z = x W^T, then per token the bias add, top-K, gates and
// token bias.
//
// "Kolibri Pre-Training from Scratch" 6.1 (routing equations) and 7.1
// (alpha_t = -Q_K(Z_t,: + beta)); "Kolibri 1 im Detail", routing: bf16
// router, fp32 logits, the two-step rule (select on Z + beta, weight with
// sigma(Z)).
//
// A cluster of 16 CTAs owns 16 tokens and all E experts: CTA c holds the
// full-width router rows of experts [c E/16, (c+1) E/16) and the 16 token
// rows in shared memory (bulk copies, one memory round trip), and its eight
// warps each form the 16 x E/16 logits over an eighth of d with mma.sync
// m16n8k16 (bf16 in, fp32 accumulate); the eighths are added in a fixed
// order.  After a cluster barrier CTA r takes token r: its warp 0 reads the
// token's E logits out of the 16 CTAs' shared memory (distributed shared
// memory) into the lane layout of the row selection (route.cuh) and writes
// ids, gates and alpha.  No workspace, no second launch, results repeat
// bit for bit.  Used for batches of at most a few dozen tokens, where the
// separate logits and selection launches are each mostly latency.
#include <cuda_bf16.h>

#include "launch.h"
#include "route.cuh"
#include "pdl.cuh"

namespace kolibri {

namespace {

constexpr int kDecTok = 16;              // tokens per cluster (one m16 tile)
constexpr int kDecCtas = 16;             // CTAs per cluster (non-portable size)
constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecParts = 8;             // d is summed in 8 parts, one per warp, added in order

struct DecLayout {
  int ld;                                // padded row length of x and W rows, in bf16
  int ec;                                // experts per CTA
  uint32_t off_x, off_w, off_zp, off_zc, off_beta, off_sc, off_pids, off_pcnt, off_poff, off_bar,
      total;
};

// The permutation outputs when the forward also groups the slots (counts
// null: it does not).
struct DecPerm {
  int32_t* counts;
  int64_t* offsets;
  int32_t* perm;
  int32_t* inv;
};

template <int Q>
__host__ __device__ inline DecLayout dec_layout(int d, int E) {
  DecLayout L;
  L.ld = d + 8;                          // 16 bytes of padding: ldmatrix rows on distinct banks
  L.ec = E / kDecCtas;
  uint32_t o = 0;
  L.off_x = o;
  o += static_cast<uint32_t>(kDecTok * L.ld * 2);
  L.off_w = o;
  o += static_cast<uint32_t>(L.ec * L.ld * 2);
  L.off_zp = o;
  o += static_cast<uint32_t>(kDecWarps * kDecTok * L.ec * 4);
  L.off_zc = o;
  o += static_cast<uint32_t>(kDecTok * L.ec * 4);
  L.off_beta = o;
  o += static_cast<uint32_t>(128 * Q * 4);
  L.off_sc = o;
  o += static_cast<uint32_t>((sizeof(RowScratch<Q>) + 15) & ~static_cast<size_t>(15));
  L.off_pids = o;                        // CTA 0: every slot's expert (16 tokens x K <= 16)
  o += 4 * kDecTok * 16;
  L.off_pcnt = o;                        // CTA 0: counts per expert
  o += 4 * 512;
  L.off_poff = o;                        // CTA 0: starts per expert, then one word per warp
  o += 4 * (512 + kDecWarps);
  L.off_bar = o;
  o += 16;
  L.total = o;
  return L;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t dec_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void dec_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void dsmem_st_u32(uint32_t local_addr, uint32_t rank, uint32_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}
__device__ __forceinline__ float dsmem_ld_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}
// One row of bytes from global memory into this CTA's shared memory,
// completing on the mbarrier at `bar`.
__device__ __forceinline__ void bulk_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Counts, offsets and the stable grouping of a decode batch's nk slots
// (experts ascending, slot index j = t K + k ascending inside an expert),
// exactly as kolibri_expert_permute.  pid: every slot's expert (shared),
// pre-filled with kNoId so that a slot the selection did not fill (a row
// with NaN scores) is counted under expert 0 and reported, never used as an
// index; cnt: E words, start: 512 words followed by one word per warp
// (shared).  Called by all kThreads threads of the block; E <= 512.
// The 16-wide k-steps of part w of d: [w S / 8, (w + 1) S / 8) of S = d / 16.
// Both decode kernels use this split and add the parts in order 0..7, so
// they form the same Z bit for bit.
__device__ __forceinline__ void part_steps(int d, int w, int& s0, int& s1) {
  const int S = d / 16;
  s0 = w * S / kDecParts;
  s1 = (w + 1) * S / kDecParts;
}
// ((p_0 + p_1) + p_2) + ... + p_7 of element i, part w at p + w n.
__device__ __forceinline__ float sum_parts(const float* p, int n, int i) {
  float v = p[i];
#pragma unroll
  for (int w = 1; w < kDecParts; ++w) v = __fadd_rn(v, p[w * n + i]);
  return v;
}

template <int kThreads>
__device__ void group_slots(const uint32_t* pid, int nk, int E, uint32_t* cnt, uint32_t* start,
                            const DecPerm& pm) {
  constexpr int kPer = 512 / kThreads;   // experts per thread in the scan
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* wsum = start + 512;
  for (int e = tid; e < E; e += kThreads) cnt[e] = 0u;
  __syncthreads();
  for (int j = tid; j < nk; j += kThreads) {
    uint32_t e = pid[j];
    if (e >= static_cast<uint32_t>(E)) {
      raise_status(kStatusBadInput);
      e = 0u;
    }
    atomicAdd(&cnt[e], 1u);
  }
  __syncthreads();
  uint32_t v[kPer], sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = kPer * tid + i;
    v[i] = e < E ? cnt[e] : 0u;
    sum += v[i];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint32_t run = incl - sum;
  for (int w2 = 0; w2 < warp; ++w2) run += wsum[w2];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = kPer * tid + i;
    if (e < E) {
      start[e] = run;
      pm.counts[e] = static_cast<int32_t>(v[i]);
      pm.offsets[e] = run;
    }
    run += v[i];
  }
  if (tid == 0) pm.offsets[E] = nk;
  __syncthreads();
  const auto expert_of = [&](int j) {
    const uint32_t e = pid[j];
    return e < static_cast<uint32_t>(E) ? e : 0u;
  };
  for (int j = tid; j < nk; j += kThreads) {
    const uint32_t e = expert_of(j);
    uint32_t before = 0;                 // earlier slots of the same expert
    for (int i = 0; i < j; ++i) before += (expert_of(i) == e) ? 1u : 0u;
    const uint32_t pos = start[e] + before;
    pm.perm[pos] = j;
    if (pm.inv) pm.inv[j] = static_cast<int32_t>(pos);
  }
}

template <int Q, bool kBias>
__global__ void __launch_bounds__(kDecThreads, 1) decode_forward_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
    const float* __restrict__ bias, float* __restrict__ z, int64_t N, int d, int E, int K,
    int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ alpha, const DecPerm pm) {
  extern __shared__ __align__(16) uint8_t sm[];
  const DecLayout L = dec_layout<Q>(d, E);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = dec_rank();
  const int ec = L.ec, e0 = static_cast<int>(rank) * ec;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kDecTok;
  const int nv = static_cast<int>(N - t0 < kDecTok ? N - t0 : kDecTok);   // tokens of this tile
  const uint32_t base = smem_u32(sm);
  const uint32_t bar = base + L.off_bar;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sm + L.off_x);
  float* zp = reinterpret_cast<float*>(sm + L.off_zp);
  float* zc = reinterpret_cast<float*>(sm + L.off_zc);
  float* beta_s = reinterpret_cast<float*>(sm + L.off_beta);
  RowScratch<Q>& sc = *reinterpret_cast<RowScratch<Q>*>(sm + L.off_sc);

  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (rank == 0)                         // the slot list of the grouping (CTA 0), see group_slots
    for (int j = tid; j < kDecTok * 16; j += kDecThreads) reinterpret_cast<uint32_t*>(sm + L.off_pids)[j] = kNoId;
  // token rows past the batch are zero (their logits are never stored)
  for (int i = tid; i < (kDecTok - nv) * (L.ld / 8); i += kDecThreads) {
    const int r = nv + i / (L.ld / 8), c = i % (L.ld / 8);
    *reinterpret_cast<uint4*>(xs + r * L.ld + c * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  pdl_wait();                            // x may come from the kernel before this one
  pdl_trigger();
  if constexpr (kBias) {
    for (int e = tid; e < 128 * Q; e += kDecThreads) beta_s[e] = e < E ? bias[e] : 0.f;
  }
  const uint32_t row_bytes = static_cast<uint32_t>(d) * 2;
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nv + ec) * row_bytes);
    __syncwarp();
    for (int r = lane; r < nv + ec; r += 32) {
      if (r < nv)
        bulk_row(base + L.off_x + static_cast<uint32_t>(r * L.ld * 2), x + (t0 + r) * d, row_bytes, bar);
      else
        bulk_row(base + L.off_w + static_cast<uint32_t>((r - nv) * L.ld * 2),
                 w + static_cast<int64_t>(e0 + r - nv) * d, row_bytes, bar);
    }
  }
  const bool loaded = mbar_wait(bar, 0);

  // ---- logits: warp w sums part w of d (part_steps)
  if (loaded) {
    float acc[Q][4];
#pragma unroll
    for (int j = 0; j < Q; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    int s0, s1;
    part_steps(d, warp, s0, s1);
    const uint32_t a_base =
        base + L.off_x + static_cast<uint32_t>((((lane & 7) + ((lane >> 3) & 1) * 8) * L.ld + (lane >> 4) * 8) * 2);
    const uint32_t b_base = base + L.off_w + static_cast<uint32_t>(((lane & 7) * L.ld + ((lane >> 3) & 1) * 8) * 2);
#pragma unroll 4
    for (int st = s0; st < s1; ++st) {
      const uint32_t kb = 32u * static_cast<uint32_t>(st);   // 16 bf16 per step
      uint32_t a0, a1, a2, a3;
      ldsm_x4(a_base + kb, a0, a1, a2, a3);
#pragma unroll
      for (int j = 0; j < Q; ++j) {
        uint32_t b0, b1;
        ldsm_x2(b_base + static_cast<uint32_t>(8 * j * L.ld * 2) + kb, b0, b1);
        mma16816(acc[j], a0, a1, a2, a3, b0, b1);
      }
    }
    // accumulator of n tile j: rows lane/4 and lane/4 + 8, columns 8j + 2 (lane % 4) and + 1
    float* mine = zp + warp * kDecTok * ec;
    const int rr = lane >> 2, cc = 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < Q; ++j) {
      mine[rr * ec + 8 * j + cc] = acc[j][0];
      mine[rr * ec + 8 * j + cc + 1] = acc[j][1];
      mine[(rr + 8) * ec + 8 * j + cc] = acc[j][2];
      mine[(rr + 8) * ec + 8 * j + cc + 1] = acc[j][3];
    }
  }
  __syncthreads();
  if (loaded) {
    // the eight parts in order; then Z out
    for (int i = tid; i < kDecTok * ec; i += kDecThreads) {
      const float v = sum_parts(zp, kDecTok * ec, i);
      zc[i] = v;
      const int r = i / ec, c = i - r * ec;
      if (r < nv) z[(t0 + r) * E + e0 + c] = v;
    }
  }
  dec_cluster_sync();                    // every CTA's logits are in its shared memory

  // ---- selection: CTA r takes token r of the tile (ids null: logits only)
  if (ids != nullptr && warp == 0 && static_cast<int>(rank) < nv && loaded) {
    const int64_t t = t0 + rank;
    float zr[4 * Q];
#pragma unroll
    for (int j = 0; j < 4 * Q; ++j) {
      const uint32_t e = slot_expert(lane, j);     // < 128 Q = E: E is a multiple of 128
      const uint32_t owner = e / static_cast<uint32_t>(ec);
      const uint32_t col = e - owner * static_cast<uint32_t>(ec);
      zr[j] = dsmem_ld_f32(base + L.off_zc + (rank * static_cast<uint32_t>(ec) + col) * 4u, owner);
    }
    int rk;
    uint32_t key, id;
    warp_select_row<Q, true, kBias>(zr, beta_s, 0xffffffffu, K, lane, sc, rk, key, id);
    if (rk >= 0 && rk < K) {
      const uint32_t e = id < static_cast<uint32_t>(E) ? id : 0u;
      ids[t * K + rk] = static_cast<int32_t>(id);
      gates[t * K + rk] = gate_sigmoid(sc.row[buffer_pos<Q>(e)]);
      // the slot's expert, into CTA 0's list when this launch also groups the slots
      if (pm.counts != nullptr && gridDim.y == 1)
        dsmem_st_u32(base + L.off_pids + 4u * (rank * static_cast<uint32_t>(K) + static_cast<uint32_t>(rk)),
                     0u, e);
    }
    if (rk == K && alpha) alpha[t] = -key_to_float(key);
  }
  dec_cluster_sync();                    // no CTA leaves while its logits may still be read; the
                                         // slots' experts are in CTA 0

  // ---- the permutation, when the batch is this one cluster: CTA 0 forms
  // counts, offsets and the stable grouping
  const bool permute = pm.counts != nullptr && ids != nullptr && gridDim.y == 1 && rank == 0;
  if (permute)
    group_slots<kDecThreads>(reinterpret_cast<const uint32_t*>(sm + L.off_pids), nv * K, E,
                             reinterpret_cast<uint32_t*>(sm + L.off_pcnt),
                             reinterpret_cast<uint32_t*>(sm + L.off_poff), pm);
}

template <int Q, bool kBias>
cudaError_t launch_dec(const void* x, const void* w, const float* bias, float* z, int64_t N, int d,
                       int E, int K, int32_t* ids, float* gates, float* alpha, const DecPerm& pm,
                       cudaStream_t s) {
  const DecLayout L = dec_layout<Q>(d, E);
  auto kern = decode_forward_kernel<Q, kBias>;
  static int checked = 0;                // 1: runs, -1: this device cannot place the cluster
  if (checked == 0) {
    checked = -1;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(L.total)) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = kDecCtas;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(kDecCtas, 1, 1);
      cfg.blockDim = dim3(kDecThreads, 1, 1);
      cfg.dynamicSmemBytes = L.total;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1) checked = 1;
    }
    (void)cudaGetLastError();
  }
  if (checked < 0) return cudaErrorNotSupported;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L.total));
  if (err != cudaSuccess) return err;
  const unsigned tiles = static_cast<unsigned>((N + kDecTok - 1) / kDecTok);
  return launch_pdl(kern, dim3(kDecCtas, tiles, 1), dim3(kDecThreads), L.total, s, dim3(kDecCtas, 1, 1),
                    static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w), bias, z, N,
                    d, E, K, ids, gates, alpha, pm);
}

// ---- the ticketed form of a batch of at most 16 tokens (no cluster).  The
// router rows are spread over E/8 CTAs, so each SM brings in 8 of them
// instead of E/16: CTA b forms the logits of experts [8b, 8b + 8) with the
// same eight partial sums as the clustered form (the same Z bit for bit) and
// writes them to z.  Each CTA then takes a ticket (an atomic counter in the
// caller's workspace, zero between calls); the last one to arrive reads the
// batch's full rows of Z back from L2 and forms the selection and the
// grouping, then sets the counter back to zero.  No CTA waits on another.
constexpr int kTkExperts = 8;            // experts per CTA: one n8 tile
constexpr int kTkWarps = 8;              // selection: one token per warp at a time
constexpr int kTkThreads = 32 * kTkWarps;
constexpr int kTkMmaWarps = kDecParts;   // d in eighths, as the clustered form

struct TkLayout {
  int ld;
  uint32_t off_x, off_w, off_zp, off_beta, off_sc, sc_bytes, off_pids, off_pcnt, off_poff, off_bar, total;
};

template <int Q>
__host__ __device__ inline TkLayout tk_layout(int d) {
  TkLayout L;
  L.ld = d + 8;
  uint32_t o = 0;
  L.off_x = o;
  o += static_cast<uint32_t>(kDecTok * L.ld * 2);
  L.off_w = o;
  o += static_cast<uint32_t>(kTkExperts * L.ld * 2);
  L.off_zp = o;
  o += static_cast<uint32_t>(kTkMmaWarps * kDecTok * kTkExperts * 4);
  L.off_beta = o;
  o += static_cast<uint32_t>(128 * Q * 4);
  L.sc_bytes = static_cast<uint32_t>((sizeof(RowScratch<Q>) + 15) & ~static_cast<size_t>(15));
  L.off_sc = o;
  o += kTkWarps * L.sc_bytes;
  L.off_pids = o;                        // every slot's expert (16 tokens x K <= 16)
  o += 4 * kDecTok * 16;
  L.off_pcnt = o;                        // counts per expert
  o += 4 * 512;
  L.off_poff = o;                        // starts per expert, then one word per warp
  o += 4 * (512 + kTkWarps);
  L.off_bar = o;                         // mbarrier (8 bytes), then the last-CTA flag
  o += 16;
  L.total = o;
  return L;
}

template <int Q, bool kBias>
__global__ void __launch_bounds__(kTkThreads, 1) decode_ticket_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w,
    const float* __restrict__ bias, float* __restrict__ z, int nv, int d, int E, int K,
    int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ alpha, const DecPerm pm,
    uint32_t* __restrict__ ticket) {
  extern __shared__ __align__(16) uint8_t sm[];
  const TkLayout L = tk_layout<Q>(d);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e0 = static_cast<int>(blockIdx.x) * kTkExperts;
  const uint32_t base = smem_u32(sm);
  const uint32_t bar = base + L.off_bar;
  volatile int* last_flag = reinterpret_cast<volatile int*>(sm + L.off_bar + 8);
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sm + L.off_x);
  float* zp = reinterpret_cast<float*>(sm + L.off_zp);

  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int j = tid; j < kDecTok * 16; j += kTkThreads)   // the slot list, see group_slots
    reinterpret_cast<uint32_t*>(sm + L.off_pids)[j] = kNoId;
  // token rows past the batch are zero (their logits are never stored)
  for (int i = tid; i < (kDecTok - nv) * (L.ld / 8); i += kTkThreads) {
    const int r = nv + i / (L.ld / 8), c = i % (L.ld / 8);
    *reinterpret_cast<uint4*>(xs + r * L.ld + c * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  pdl_wait();                            // x, the bias and the ticket follow the kernel before
  pdl_trigger();
  const uint32_t row_bytes = static_cast<uint32_t>(d) * 2;
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nv + kTkExperts) * row_bytes);
    __syncwarp();
    for (int r = lane; r < nv + kTkExperts; r += 32) {
      if (r < nv)
        bulk_row(base + L.off_x + static_cast<uint32_t>(r * L.ld * 2), x + static_cast<int64_t>(r) * d,
                 row_bytes, bar);
      else
        bulk_row(base + L.off_w + static_cast<uint32_t>((r - nv) * L.ld * 2),
                 w + static_cast<int64_t>(e0 + r - nv) * d, row_bytes, bar);
    }
  }
  const bool loaded = mbar_wait(bar, 0);

  // ---- logits: warp w sums part w of d (part_steps) for the CTA's 8 experts
  if (loaded && warp < kTkMmaWarps) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int s0, s1;
    part_steps(d, warp, s0, s1);
    const uint32_t a_base =
        base + L.off_x + static_cast<uint32_t>((((lane & 7) + ((lane >> 3) & 1) * 8) * L.ld + (lane >> 4) * 8) * 2);
    const uint32_t b_base = base + L.off_w + static_cast<uint32_t>(((lane & 7) * L.ld + ((lane >> 3) & 1) * 8) * 2);
#pragma unroll 4
    for (int st = s0; st < s1; ++st) {
      const uint32_t kb = 32u * static_cast<uint32_t>(st);   // 16 bf16 per step
      uint32_t a0, a1, a2, a3, b0, b1;
      ldsm_x4(a_base + kb, a0, a1, a2, a3);
      ldsm_x2(b_base + kb, b0, b1);
      mma16816(acc, a0, a1, a2, a3, b0, b1);
    }
    float* mine = zp + warp * kDecTok * kTkExperts;
    const int rr = lane >> 2, cc = 2 * (lane & 3);
    mine[rr * kTkExperts + cc] = acc[0];
    mine[rr * kTkExperts + cc + 1] = acc[1];
    mine[(rr + 8) * kTkExperts + cc] = acc[2];
    mine[(rr + 8) * kTkExperts + cc + 1] = acc[3];
  }
  __syncthreads();
  if (loaded) {
    constexpr int n = kDecTok * kTkExperts;
    for (int i = tid; i < nv * kTkExperts; i += kTkThreads) {
      const float v = sum_parts(zp, n, i);
      const int r = i / kTkExperts, c = i - r * kTkExperts;
      z[static_cast<int64_t>(r) * E + e0 + c] = v;
    }
  }
  __syncthreads();                       // this CTA's logits are stored
  if (tid == 0) {
    __threadfence();                     // ... and visible before its ticket
    const uint32_t C = gridDim.x;
    const uint32_t t = atomicAdd(ticket, 1u);
    if (t >= C) raise_status(kStatusBadInput);   // the counter was not zero at the start
    const int last = t == C - 1;
    if (last) {
      __threadfence();                   // every CTA's logits before this CTA's reads
      atomicExch(ticket, 0u);            // all C tickets are taken: zero for the next call
    }
    *last_flag = last;
  }
  __syncthreads();
  if (!*last_flag) return;

  // ---- the last CTA: selection of every token (warp per token), then the grouping
  float* beta_s = reinterpret_cast<float*>(sm + L.off_beta);
  uint32_t* pid = reinterpret_cast<uint32_t*>(sm + L.off_pids);
  if constexpr (kBias) {
    for (int e = tid; e < 128 * Q; e += kTkThreads) beta_s[e] = e < E ? bias[e] : 0.f;
  }
  __syncthreads();
  RowScratch<Q>& sc = *reinterpret_cast<RowScratch<Q>*>(sm + L.off_sc + static_cast<uint32_t>(warp) * L.sc_bytes);
  for (int r = warp; r < nv; r += kTkWarps) {
    float zr[4 * Q];
    const float* zrow = z + static_cast<int64_t>(r) * E;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(zrow + 128 * q + 4 * lane));
      zr[4 * q + 0] = v.x;
      zr[4 * q + 1] = v.y;
      zr[4 * q + 2] = v.z;
      zr[4 * q + 3] = v.w;
    }
    int rk;
    uint32_t key, id;
    warp_select_row<Q, true, kBias>(zr, beta_s, 0xffffffffu, K, lane, sc, rk, key, id);
    if (rk >= 0 && rk < K) {
      const uint32_t e = id < static_cast<uint32_t>(E) ? id : 0u;
      ids[r * K + rk] = static_cast<int32_t>(id);
      gates[r * K + rk] = gate_sigmoid(sc.row[buffer_pos<Q>(e)]);
      pid[r * K + rk] = e;
    }
    if (rk == K && alpha) alpha[r] = -key_to_float(key);
    __syncwarp();
  }
  __syncthreads();
  group_slots<kTkThreads>(pid, nv * K, E, reinterpret_cast<uint32_t*>(sm + L.off_pcnt),
                          reinterpret_cast<uint32_t*>(sm + L.off_poff), pm);
}

template <int Q, bool kBias>
cudaError_t launch_tk(const void* x, const void* w, const float* bias, float* z, int64_t N, int d, int E,
                      int K, int32_t* ids, float* gates, float* alpha, const DecPerm& pm, uint32_t* ticket,
                      cudaStream_t s) {
  const TkLayout L = tk_layout<Q>(d);
  auto kern = decode_ticket_kernel<Q, kBias>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L.total));
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(static_cast<unsigned>(E / kTkExperts)), dim3(kTkThreads), L.total, s,
                    dim3(0, 0, 0), static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w),
                    bias, z, static_cast<int>(N), d, E, K, ids, gates, alpha, pm, ticket);
}

}  // namespace

// ids, gates and alpha null: the logits alone (the same sums as the forward).
bool router_decode_supported(int64_t N, int32_t d, int32_t E, int32_t K) {
  if (N < 1 || N > kDecodeTokenLimit || E % 128 != 0 || E > 512 || d % 64 != 0 || K + 1 > 32) return false;
  const int Q = E / 128;
  const size_t total = Q == 1 ? dec_layout<1>(d, E).total
                     : Q == 2 ? dec_layout<2>(d, E).total
                     : Q == 3 ? dec_layout<3>(d, E).total
                              : dec_layout<4>(d, E).total;
  return total <= 227u * 1024u;
}

static cudaError_t decode_dispatch(const void* x, const void* w, const float* bias, float* z,
                                   int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                   float* gates, float* alpha, const DecPerm& pm, cudaStream_t s) {
  if (!router_decode_supported(N, d, E, K)) return cudaErrorNotSupported;
  const bool b = bias != nullptr;
  switch (E / 128) {
    case 1: return b ? launch_dec<1, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s)
                     : launch_dec<1, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s);
    case 2: return b ? launch_dec<2, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s)
                     : launch_dec<2, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s);
    case 3: return b ? launch_dec<3, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s)
                     : launch_dec<3, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s);
    default: return b ? launch_dec<4, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s)
                      : launch_dec<4, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, s);
  }
}

cudaError_t launch_router_decode(const void* x, const void* w, const float* bias, float* z,
                                 int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                 float* gates, float* alpha, cudaStream_t s) {
  return decode_dispatch(x, w, bias, z, N, d, E, K, ids, gates, alpha, DecPerm{}, s);
}

bool router_decode_permutes(int64_t N, int32_t d, int32_t E, int32_t K) {
  return N <= kDecTok && router_decode_supported(N, d, E, K);
}

cudaError_t launch_router_decode_permute(const void* x, const void* w, const float* bias, float* z,
                                         int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                         float* gates, float* alpha, int32_t* counts,
                                         int64_t* offsets, int32_t* perm, int32_t* inv,
                                         cudaStream_t s) {
  if (!router_decode_permutes(N, d, E, K)) return cudaErrorNotSupported;
  return decode_dispatch(x, w, bias, z, N, d, E, K, ids, gates, alpha,
                         DecPerm{counts, offsets, perm, inv}, s);
}

// Only where the forward itself takes the clustered kernel: the two forms
// share their sums, so Z is the forward's bit for bit.
bool router_decode_ticket_supported(int64_t N, int32_t d, int32_t E, int32_t K) {
  if (N < 1 || N > kDecTok || E % 128 != 0 || E > 512 || d % 64 != 0 || K < 1 || K > 16) return false;
  if (!router_decode_supported(N, d, E, K)) return false;
  const int Q = E / 128;
  const size_t total = Q == 1 ? tk_layout<1>(d).total
                     : Q == 2 ? tk_layout<2>(d).total
                     : Q == 3 ? tk_layout<3>(d).total
                              : tk_layout<4>(d).total;
  return total <= 227u * 1024u;
}

cudaError_t launch_router_decode_ticket(const void* x, const void* w, const float* bias, float* z,
                                        int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                        float* gates, float* alpha, int32_t* counts, int64_t* offsets,
                                        int32_t* perm, int32_t* inv, uint32_t* ticket, cudaStream_t s) {
  if (!router_decode_ticket_supported(N, d, E, K) || ticket == nullptr) return cudaErrorNotSupported;
  const DecPerm pm{counts, offsets, perm, inv};
  const bool b = bias != nullptr;
  switch (E / 128) {
    case 1: return b ? launch_tk<1, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s)
                     : launch_tk<1, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s);
    case 2: return b ? launch_tk<2, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s)
                     : launch_tk<2, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s);
    case 3: return b ? launch_tk<3, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s)
                     : launch_tk<3, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s);
    default: return b ? launch_tk<4, true>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s)
                      : launch_tk<4, false>(x, w, bias, z, N, d, E, K, ids, gates, alpha, pm, ticket, s);
  }
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_decode)

}  // namespace kolibri
