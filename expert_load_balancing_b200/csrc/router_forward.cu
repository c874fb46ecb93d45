// router_forward.cu -- router logits and token selection in one kernel.
//
// "Kolibri Pre-Training from Scratch" 6.1 (routing equations) and 7.1 (token
// bias); "Kolibri 1 im Detail", routing steps 1-2:
//   Z_t,e   = x_t . W_e                        (bf16 x bf16 -> fp32)
//   B_t,e   = Z_t,e + beta_e                   (fp32, round to nearest even)
//   I_t     = the K largest B_t,e              (ties: lower expert id first)
//   S_t,e   = sigmoid(Z_t,e) for e in I_t      (raw logits, no renormalising)
//   alpha_t = -(the (K+1)-th largest B_t,e)
//
// The main loop is the pair GEMM of gemm_pair.cuh.  The epilogue takes a
// whole 256 x E accumulator tile out of TMEM into registers at once (thread
// = token row, 128 fp32 columns per thread) and hands TMEM back to the MMA
// before doing anything else, so selection overlaps the next tile's MMAs.
// Z still goes to HBM (the EQB update reads it): each 32 x 16 block passes
// through shared memory so the global stores are coalesced.
//
// Warp roles (512 threads, setmaxnreg: warpgroup 0 at 32 registers, the
// three epilogue warpgroups at 160):
//   warp 0       TMA producer
//   warp 1       TMEM owner; in the leader, the MMA-issuing thread
//   warps 2, 3   idle
//   warps 4..15  epilogue: TMEM lane quarter q = warp % 4 (32 rows), column
//                third j = (warp - 4) / 4 (128 experts)
//
// Selection per row, exact for every finite input:
//  1. each epilogue warp takes the maxima of its column groups (kG columns)
//     and sorts them; group maxima are distinct elements of the row, so the
//     (K+1)-th largest of all the row's group maxima, T, is a lower bound of
//     the row's (K+1)-th largest score;
//  2. scores >= T are candidates (z and expert id to a per-row buffer);
//  3. one warp per quarter takes K+1 rounds over the row's candidates in the
//     order (key descending, expert id ascending), where key is the
//     order-preserving integer of the fp32 score.
// Rows with more than kCap candidates (heavy ties) are marked with a NaN
// alpha and finished by the row kernel (launch_select_fixup).
#include "launch.h"
#include "gemm_pair.cuh"

namespace kolibri {

namespace {

using namespace gemm;

constexpr int kThreads = 512;
constexpr int kCtrlWarps = 4;            // warpgroup 0
constexpr int kEpiWarps = 12;            // warpgroups 1..3
constexpr int kColsPerWarp = 128;
constexpr int kMaxE = 3 * kColsPerWarp;
constexpr int kRegsCtrl = 32;
constexpr int kRegsEpi = 160;
static_assert(kCtrlWarps * 32 * kRegsCtrl + kEpiWarps * 32 * kRegsEpi <= kThreads * 128,
              "register split exceeds what 512 threads are launched with");
constexpr int kZCols = 16;               // columns per block of the Z / candidate pass
constexpr int kZBuf = kZCols * 32 * 4;   // per-warp copy of one block (2 KB)
constexpr int kCap = 32;                 // candidate slots per row

struct FwdParams {
  float* z;            // [N, E] logits, written
  const float* beta;   // null: B = Z
  int32_t* ids;
  float* gates;
  float* alpha;
  int K;
};

// Shared memory after the operand ring (offsets from the 1 KB aligned base).
struct FwdLayout {
  uint32_t zstage, beta, gsort, cz, cc, rowcnt, alpha, qbar, bars, total;
};

__host__ __device__ inline FwdLayout fwd_layout(uint32_t ring_bytes, int groups_per_warp) {
  FwdLayout L;
  uint32_t o = ring_bytes;                 // multiple of 1 KB
  L.zstage = o;
  o += kEpiWarps * kZBuf;
  L.beta = o;
  o += kMaxE * 4;
  L.gsort = o;                             // f32 [3][groups][128]
  o += 3u * groups_per_warp * 128 * 4;
  L.cz = o;                                // f32 [kCap][128]
  o += kCap * 128 * 4;
  L.cc = o;                                // u16 [kCap][128]
  o += kCap * 128 * 2;
  L.rowcnt = o;                            // u32 [128]
  o += 128 * 4;
  L.alpha = o;                             // f32 [128] this tile's token biases
  o += 128 * 4;
  o = (o + 7u) & ~7u;
  L.qbar = o;                              // per quarter: three mbarriers
  o += 4 * 3 * 8;
  L.bars = o;
  o += 8 * (2 * kMaxStages + 3);
  L.total = o;
  return L;
}

// Byte offset of 16-byte chunk `c` of row `row` in a warp's 32 x 64 B block
// copy.  The XOR keeps both access patterns free of bank conflicts: a lane
// per row (writes, candidate reads) and four lanes per row (the copy-out).
__device__ __forceinline__ uint32_t zstage_off(int row, int c) {
  return static_cast<uint32_t>(row * 64 + ((c ^ ((row >> 1) & 3)) << 4));
}

// 32 columns of TMEM into r[OFF .. OFF+31] (compile-time offsets only, so
// the array stays in registers).
#define KOLIBRI_R8(o) "=r"(r[OFF + o]), "=r"(r[OFF + o + 1]), "=r"(r[OFF + o + 2]), \
    "=r"(r[OFF + o + 3]), "=r"(r[OFF + o + 4]), "=r"(r[OFF + o + 5]), "=r"(r[OFF + o + 6]), \
    "=r"(r[OFF + o + 7])
template <int OFF>
__device__ __forceinline__ void tmem_ld32_at(uint32_t taddr, uint32_t (&r)[kColsPerWarp]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : KOLIBRI_R8(0), KOLIBRI_R8(8), KOLIBRI_R8(16), KOLIBRI_R8(24)
      : "r"(taddr));
}
#undef KOLIBRI_R8

template <bool kBias>
__device__ __forceinline__ float score(uint32_t zbits, float beta) {
  const float z = __uint_as_float(zbits);
  return kBias ? __fadd_rn(z, beta) : z;
}

// Bitonic sort of n (power of two) values, descending.
template <int n>
__device__ __forceinline__ void sort_desc(float (&v)[n]) {
#pragma unroll
  for (int k = 2; k <= n; k <<= 1) {
#pragma unroll
    for (int s = k >> 1; s > 0; s >>= 1) {
#pragma unroll
      for (int i = 0; i < n; ++i) {
        const int l = i ^ s;
        if (l > i) {
          const float a = v[i], b = v[l];
          const bool desc = (i & k) == 0;
          v[i] = desc ? fmaxf(a, b) : fminf(a, b);
          v[l] = desc ? fminf(a, b) : fmaxf(a, b);
        }
      }
    }
  }
}

// Candidate (k, c) precedes the running best (bk, bc): key descending, then
// expert id ascending.
__device__ __forceinline__ bool precedes(uint32_t k, uint32_t c, uint32_t bk, uint32_t bc) {
  return k > bk || (k == bk && c < bc);
}

// Barrier of the three warps of one lane quarter (96 arrivals), bounded.
__device__ __forceinline__ bool quarter_sync(uint32_t bar, uint32_t parity) {
  mbar_arrive(bar);
  return mbar_wait(bar, parity);
}

// ---- epilogue ---------------------------------------------------------------

template <int kG, bool kBias>
__device__ __forceinline__ void forward_epilogue(const GemmShape& sh, const FwdParams& p,
                                                 const Ring& rg,
                                                 const FwdLayout& L, uint8_t* gbase,
                                                 uint32_t tmem_base, uint32_t rank, int warp,
                                                 int lane) {
  constexpr int kGPW = kColsPerWarp / kG;    // column groups per warp
  const uint32_t base = rg.base;
  const float* beta_s = reinterpret_cast<const float*>(gbase + L.beta);
  float* gsort = reinterpret_cast<float*>(gbase + L.gsort);
  float* cz = reinterpret_cast<float*>(gbase + L.cz);
  uint16_t* cc = reinterpret_cast<uint16_t*>(gbase + L.cc);
  uint32_t* rowcnt = reinterpret_cast<uint32_t*>(gbase + L.rowcnt);
  float* alpha_s = reinterpret_cast<float*>(gbase + L.alpha);

  const int q = warp & 3;                    // TMEM lane quarter
  const int j = (warp - 4) >> 2;             // column third
  const int col0 = j * kColsPerWarp;
  const int ncols = max(0, min(kColsPerWarp, sh.E - col0));  // multiple of 16
  const int rl = q * 32 + lane;              // row within the CTA's 128
  const uint32_t zbuf = base + L.zstage + static_cast<uint32_t>((warp - 4) * kZBuf);
  const uint32_t empty_leader = map_to_rank(rg.tmem_empty(), 0);
  const uint32_t bar_a = base + L.qbar + 24u * q, bar_b = bar_a + 8u, bar_c = bar_a + 16u;
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
  uint32_t cl[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    cl[i] = static_cast<uint32_t>(min(col0 + 32 * i, static_cast<int>(sh.tmem_cols) - 32));
  const uint32_t cid = cluster_id_x(), ncl = num_clusters_x();
  const int K = p.K;
  uint32_t acc_phase = 0, qphase = 0;

  for (int64_t pt = cid; pt < sh.num_pairs; pt += ncl) {
    if (!mbar_wait(rg.tmem_full(), acc_phase)) return;
    tc_fence_after();
    // all four loads run unconditionally (the values past E are never used);
    // columns are clamped into the allocation, which is >= 32 wide
    uint32_t r[kColsPerWarp];
    tmem_ld32_at<0>(lane_addr + cl[0], r);
    tmem_ld32_at<32>(lane_addr + cl[1], r);
    tmem_ld32_at<64>(lane_addr + cl[2], r);
    tmem_ld32_at<96>(lane_addr + cl[3], r);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(empty_leader);  // TMEM is free for the next tile
    acc_phase ^= 1u;

    const int row_base = static_cast<int>(pt * 2 * kBM + rank * kBM + q * 32);
    const int64_t row = row_base + lane;

    // 1. sorted group maxima of this warp's columns
    {
      float gm[kGPW];
#pragma unroll
      for (int g = 0; g < kGPW; ++g) {
        float m = -INFINITY;
        if (g * kG < ncols) {
#pragma unroll
          for (int i = 0; i < kG; i += 4) {
            const float4 bq = *reinterpret_cast<const float4*>(&beta_s[col0 + g * kG + i]);
            m = fmaxf(m, score<kBias>(r[g * kG + i], bq.x));
            m = fmaxf(m, score<kBias>(r[g * kG + i + 1], bq.y));
            m = fmaxf(m, score<kBias>(r[g * kG + i + 2], bq.z));
            m = fmaxf(m, score<kBias>(r[g * kG + i + 3], bq.w));
          }
        }
        gm[g] = m;
      }
      sort_desc<kGPW>(gm);
#pragma unroll
      for (int g = 0; g < kGPW; ++g) gsort[(j * kGPW + g) * 128 + rl] = gm[g];
    }
    if (!quarter_sync(bar_a, qphase)) return;

    // threshold T: the (K+1)-th largest of the three sorted lists
    float T = -INFINITY;
    {
      const float* l0 = gsort + rl;
      const float* l1 = gsort + kGPW * 128 + rl;
      const float* l2 = gsort + 2 * kGPW * 128 + rl;
      int i0 = 0, i1 = 0, i2 = 0;
      float h0 = l0[0], h1 = l1[0], h2 = l2[0];
      for (int t = 0; t <= K; ++t) {
        if (h0 >= h1 && h0 >= h2) {
          T = h0;
          h0 = (++i0 < kGPW) ? l0[i0 * 128] : -INFINITY;
        } else if (h1 >= h2) {
          T = h1;
          h1 = (++i1 < kGPW) ? l1[i1 * 128] : -INFINITY;
        } else {
          T = h2;
          h2 = (++i2 < kGPW) ? l2[i2 * 128] : -INFINITY;
        }
      }
    }

    // 2. Z and the candidates, kZCols columns at a time.  The block goes to
    // this warp's shared copy (a lane per row), then out to HBM with four
    // lanes per row, so each store instruction writes eight whole 64-byte
    // row segments; the candidates (scores >= T) are read from the copy.
#pragma unroll
    for (int b = 0; b < kColsPerWarp / kZCols; ++b) {
      if (b * kZCols < ncols) {
#pragma unroll
        for (int c = 0; c < kZCols / 4; ++c) {
          const int o = b * kZCols + 4 * c;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(zbuf + zstage_off(lane, c)),
                       "r"(r[o]), "r"(r[o + 1]), "r"(r[o + 2]), "r"(r[o + 3])
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rr = 8 * k + (lane >> 2), ch = lane & 3;
          uint32_t v0, v1, v2, v3;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                       : "r"(zbuf + zstage_off(rr, ch))
                       : "memory");
          const int64_t grow = static_cast<int64_t>(row_base) + rr;
          if (grow < sh.N)
            *reinterpret_cast<uint4*>(p.z + grow * sh.E + col0 + b * kZCols + 4 * ch) =
                make_uint4(v0, v1, v2, v3);
        }
        uint32_t m = 0u;
#pragma unroll
        for (int i = 0; i < kZCols; i += 4) {
          const float4 bq = *reinterpret_cast<const float4*>(&beta_s[col0 + b * kZCols + i]);
          const int o = b * kZCols + i;
          m |= (score<kBias>(r[o], bq.x) >= T) ? (1u << i) : 0u;
          m |= (score<kBias>(r[o + 1], bq.y) >= T) ? (2u << i) : 0u;
          m |= (score<kBias>(r[o + 2], bq.z) >= T) ? (4u << i) : 0u;
          m |= (score<kBias>(r[o + 3], bq.w) >= T) ? (8u << i) : 0u;
        }
        while (m) {
          const int i = __ffs(m) - 1;
          m &= m - 1u;
          float zv;
          asm volatile("ld.shared.f32 %0, [%1];"
                       : "=f"(zv)
                       : "r"(zbuf + zstage_off(lane, i >> 2) + 4u * static_cast<uint32_t>(i & 3)));
          const uint32_t slot = atomicAdd(&rowcnt[rl], 1u);
          if (slot < kCap) {
            cz[slot * 128 + rl] = zv;
            cc[slot * 128 + rl] = static_cast<uint16_t>(col0 + b * kZCols + i);
          }
        }
        __syncwarp();   // every lane is done with the copy before the next block
      }
    }
    if (!quarter_sync(bar_b, qphase)) return;

    // 3. one warp per quarter ranks the row's candidates: their keys and
    // ids go to registers once, then K+1 rounds pick the best not yet taken
    if (j == 0) {
      uint32_t n = rowcnt[rl];
      rowcnt[rl] = 0u;
      if (row >= sh.N) n = 0u;
      const bool overflow = n > static_cast<uint32_t>(kCap);
      if (overflow) n = 0u;
      // candidates in chunks of 8, as many chunks as the fullest row needs
      const uint32_t nmax = __reduce_max_sync(0xffffffffu, n);
      uint32_t ck[kCap], ci[kCap];
#pragma unroll
      for (int c8 = 0; c8 < kCap / 8; ++c8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = 8 * c8 + u;
          ck[i] = 0u;
          ci[i] = 0xffffu;
          if (static_cast<uint32_t>(8 * c8) < nmax && static_cast<uint32_t>(i) < n) {
            const uint32_t c = cc[i * 128 + rl];
            ck[i] = order_key(score<kBias>(__float_as_uint(cz[i * 128 + rl]), beta_s[c]));
            ci[i] = c;
          }
        }
      }
      // K+1 rounds, each a scan of the candidates in four independent
      // chains; the winners' ids go out at once, their slots to the (now
      // read) id buffer for the gate step below
      uint32_t taken = 0u, akey = 0u;
#pragma unroll 1
      for (int t = 0; t <= K; ++t) {
        uint32_t bk[4] = {0u, 0u, 0u, 0u}, bc[4] = {0xffffu, 0xffffu, 0xffffu, 0xffffu};
        uint32_t bi[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int c8 = 0; c8 < kCap / 8; ++c8) {
          if (static_cast<uint32_t>(8 * c8) < nmax) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = 8 * c8 + u, ch = u & 3;
              const bool better = !((taken >> i) & 1u) && precedes(ck[i], ci[i], bk[ch], bc[ch]);
              bk[ch] = better ? ck[i] : bk[ch];
              bc[ch] = better ? ci[i] : bc[ch];
              bi[ch] = better ? static_cast<uint32_t>(i) : bi[ch];
            }
          }
        }
#pragma unroll
        for (int ch = 1; ch < 4; ++ch) {
          const bool better = precedes(bk[ch], bc[ch], bk[0], bc[0]);
          bk[0] = better ? bk[ch] : bk[0];
          bc[0] = better ? bc[ch] : bc[0];
          bi[0] = better ? bi[ch] : bi[0];
        }
        taken |= 1u << bi[0];
        if (t < K) {
          if (n > 0u) p.ids[row * K + t] = static_cast<int32_t>(bc[0]);
          cc[t * 128 + rl] = static_cast<uint16_t>(bi[0]);
        } else {
          akey = bk[0];
        }
      }
      if (n > 0u) p.alpha[row] = -key_to_float(akey);
      if (overflow && row < sh.N) p.alpha[row] = __uint_as_float(0x7fc00000u);  // finished by the row kernel
      alpha_s[rl] = (n > 0u) ? -key_to_float(akey) : __uint_as_float(0x7fc00000u);
    }

    // the three warps share the fp64 gates: warp j takes ranks t = j mod 3
    if (!quarter_sync(bar_c, qphase)) return;
    if (!isnan(alpha_s[rl])) {
      for (int t = j; t < K; t += 3)
        p.gates[row * K + t] = gate_sigmoid(cz[cc[t * 128 + rl] * 128 + rl]);
    }

    qphase ^= 1u;
  }
}

// ---- kernel ---------------------------------------------------------------

template <int kG, bool kBias>
__global__ void __launch_bounds__(kThreads, 1)
    router_forward_kernel(const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_w,
                          const GemmShape sh,
                          const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);
  Ring rg = make_ring(sh, base, 0);
  const FwdLayout L = fwd_layout(rg.stage_bytes * sh.stages, kColsPerWarp / kG);
  rg.bars = base + L.bars;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();

  if (threadIdx.x == 0) {
    for (int qq = 0; qq < 12; ++qq) mbar_init(base + L.qbar + 8u * qq, 96);
    init_barriers(sh, rg, 2 * kEpiWarps);
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
  }
  {
    float* beta_s = reinterpret_cast<float*>(gbase + L.beta);
    for (int i = threadIdx.x; i < kMaxE; i += kThreads)
      beta_s[i] = (kBias && i < sh.E) ? p.beta[i] : 0.f;
    uint32_t* rowcnt = reinterpret_cast<uint32_t*>(gbase + L.rowcnt);
    for (int i = threadIdx.x; i < 128; i += kThreads) rowcnt[i] = 0u;

  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(rg.holder()),
                 "r"(sh.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();          // barriers, beta and counters ready in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(gbase + (rg.holder() - base));

  if (warp < kCtrlWarps) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtrl));
    if (warp == 0) {
      if (lane == 0) producer_loop(sh, rg, &tm_x, &tm_w, rank);
    } else if (warp == 1) {
      if (rank == 0 && lane == 0) mma_loop(sh, rg, tmem_base);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    forward_epilogue<kG, kBias>(sh, p, rg, L, gbase, tmem_base, rank, warp, lane);
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

template <int kG, bool kBias>
cudaError_t launch_fwd(const CUtensorMap& tm_x, const CUtensorMap& tm_w,
                       const GemmShape& sh, const FwdParams& p, size_t smem, cudaStream_t s) {
  auto kern = router_forward_kernel<kG, kBias>;
  // setmaxnreg hands registers between warpgroups inside the block's launch
  // allocation; refuse to launch if the build gave the kernel fewer than the
  // split needs (an increase could then never be satisfied).
  static int regs_ok = 0;
  if (regs_ok == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return cudaErrorNotSupported;
    const long need = static_cast<long>(kCtrlWarps) * 32 * kRegsCtrl +
                      static_cast<long>(kEpiWarps) * 32 * kRegsEpi;
    regs_ok = (static_cast<long>(fa.numRegs) * kThreads >= need && fa.maxThreadsPerBlock >= kThreads)
                  ? 1 : -1;
  }
  if (regs_ok < 0) return cudaErrorNotSupported;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
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
  static int max_clusters = 0;
  if (max_clusters == 0) {
    cfg.gridDim = dim3(2 * static_cast<unsigned>(device_sm_count() / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1)
      n = device_sm_count() / 2;
    max_clusters = n;
  }
  const int64_t clusters = sh.num_pairs < max_clusters ? sh.num_pairs : max_clusters;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  err = cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w, sh, p);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

bool router_forward_supported(int32_t E, int32_t K) {
  if (E > kMaxE || E % 16 != 0) return false;
  return (E / 8) >= K + 1;
}

cudaError_t launch_router_forward(const void* x, const void* w, const float* bias, float* z,
                                  int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                  float* gates, float* alpha, cudaStream_t s) {
  if (!router_forward_supported(E, K)) return cudaErrorNotSupported;
  // column groups of 16 when there are enough of them for a (K+1)-th maximum
  const int kg = (E / 16 >= K + 1) ? 16 : 8;
  GemmShape sh;
  if (!plan_shape(N, d, E, sh)) return cudaErrorNotSupported;
  const size_t stage_bytes = stage_bytes_of(sh);
  const FwdLayout L0 = fwd_layout(0, kColsPerWarp / kg);
  const size_t fixed = 1024 /*alignment slack*/ + L0.total;
  int stages = static_cast<int>((kSmemLimit - fixed) / stage_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorNotSupported;
  sh.stages = stages;
  const size_t smem = fixed + stage_bytes * stages;

  CUtensorMap tm_x, tm_w;
  if (!encode_operands(sh, x, w, &tm_x, &tm_w)) return cudaErrorInvalidValue;

  const FwdParams p{z, bias, ids, gates, alpha, K};
  const bool b = bias != nullptr;
  if (kg == 16)
    return b ? launch_fwd<16, true>(tm_x, tm_w, sh, p, smem, s)
             : launch_fwd<16, false>(tm_x, tm_w, sh, p, smem, s);
  return b ? launch_fwd<8, true>(tm_x, tm_w, sh, p, smem, s)
           : launch_fwd<8, false>(tm_x, tm_w, sh, p, smem, s);
}

cudaError_t router_forward_any(const void* x, const void* w, const float* bias, float* z,
                               int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                               float* gates, float* alpha, cudaStream_t s) {
  if (router_forward_supported(E, K)) {
    const cudaError_t err = launch_router_forward(x, w, bias, z, N, d, E, K, ids, gates, alpha, s);
    if (err == cudaSuccess) return launch_select_fixup(z, bias, N, E, K, ids, gates, alpha, s);
    if (err != cudaErrorNotSupported) return err;
  }
  // shapes outside the fused kernel: the two kernels one after the other
  const cudaError_t err = launch_router_logits(x, w, z, N, d, E, s);
  if (err != cudaSuccess) return err;
  return launch_topk(z, bias, N, E, K, ids, gates, alpha, s);
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_forward)

}  // namespace kolibri
