// permute.cu -- expert loads and the stable grouping of routed slots.
//
// Loads c_e are the per-expert counts of "Kolibri Pre-Training from
// Scratch" 6.1/6.2.  The grouping is a stable counting sort of the slot
// index j = t*K + k by expert: offsets = exclusive prefix sum of counts,
// perm[p] = j in (expert, j) order, inv[j] = p.
//
// Large inputs, three launches over tiles of 8192 slots:
//   A  each block counts its tile into a shared histogram and writes it to
//      tile_counts[tile][E] (coalesced);
//   B  one block per expert turns its column of tile counts into an
//      exclusive prefix; the last block to finish (ticket) scans the totals
//      into offsets/counts;
//   C  each block re-sorts its tile in shared memory with a stable counting
//      sort (one ballot per bit of the expert id groups a warp's lanes by
//      expert, per-warp running counters keep slot order), writes inv in
//      slot order and perm as one contiguous run per expert.
// Small inputs (decode) run the same steps inside one block.
#include "launch.h"
#include "common.cuh"
#include "pdl.cuh"

namespace kolibri {

namespace {

constexpr int kPermThreads = 256;
constexpr int kPermWarps = kPermThreads / kWarp;
constexpr int kSlotsPerThread = 32;
constexpr int64_t kTile = static_cast<int64_t>(kPermThreads) * kSlotsPerThread;  // 8192 slots
constexpr int64_t kSingleMax = 4096;    // N*K handled by one block

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Bits that index the experts and a spare value for "no expert": E < 2^bits.
__host__ __device__ inline int expert_bits(int E) {
  int b = 1;
  while ((1 << b) <= E) ++b;
  return b;
}

// The lanes of this warp holding the same value v < 2^NB: the AND, over v's
// bits, of the ballot of the lanes that agree with it on that bit.  The same
// mask as __match_any_sync, from vote instructions only.  NB is a
// compile-time count so that the NB ballots are independent and issue back
// to back.
template <int NB>
__device__ __forceinline__ unsigned lanes_with_value(uint32_t v) {
  unsigned ones[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) ones[b] = __ballot_sync(0xffffffffu, (v >> b) & 1u);
  unsigned peers = 0xffffffffu;
#pragma unroll
  for (int b = 0; b < NB; ++b) peers &= ((v >> b) & 1u) ? ones[b] : ~ones[b];
  return peers;
}

__global__ void __launch_bounds__(kPermThreads) tile_count_kernel(
    const int32_t* __restrict__ ids, int64_t NK, int E, uint32_t* __restrict__ tile_counts,
    uint32_t* __restrict__ ticket) {
  __shared__ uint32_t hist[KOLIBRI_MAX_EXPERTS];
  for (int e = threadIdx.x; e < E; e += kPermThreads) hist[e] = 0u;
  // ids come from the kernel before this one; once it is complete the next
  // two kernels of the chain may be scheduled (the scatter reads ids before
  // its own wait)
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;   // read by the scan after this grid
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTile;
  // every load is issued before the first shared-memory add, so the tile
  // costs one memory round trip rather than one per slot
  int32_t x[kSlotsPerThread];
#pragma unroll
  for (int u = 0; u < kSlotsPerThread; ++u) {
    const int64_t j = t0 + u * kPermThreads + threadIdx.x;
    x[u] = j < NK ? __ldg(ids + j) : 0;
  }
  bool bad = false;
#pragma unroll
  for (int u = 0; u < kSlotsPerThread; ++u) {
    const int64_t j = t0 + u * kPermThreads + threadIdx.x;
    if (j < NK) {
      if (x[u] >= 0 && x[u] < E) atomicAdd(&hist[x[u]], 1u);
      else bad = true;
    }
  }
  if (bad) raise_status(kStatusBadInput);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kPermThreads)
    tile_counts[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

// One block per expert: exclusive prefix over chunks, then the last block
// scans the E totals.
__global__ void __launch_bounds__(kPermThreads) chunk_scan_kernel(
    uint32_t* __restrict__ chunk_counts, int64_t nchunks, int E, uint32_t* __restrict__ totals,
    uint32_t* __restrict__ ticket, int32_t* __restrict__ counts, int64_t* __restrict__ offsets) {
  __shared__ uint32_t warp_sums[kPermWarps];
  __shared__ uint32_t carry_s;
  __shared__ bool last_s;
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();       // the tile counts and the ticket
  pdl_trigger();    // the scatter may start ranking its tile meanwhile
  if (threadIdx.x == 0) carry_s = 0u;
  __syncthreads();
  for (int64_t c0 = 0; c0 < nchunks; c0 += kPermThreads) {
    int64_t c = c0 + threadIdx.x;
    uint32_t x = c < nchunks ? chunk_counts[c * E + e] : 0u;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    uint32_t wbase = 0, tile_total = 0;
    for (int w = 0; w < kPermWarps; ++w) {
      uint32_t s = warp_sums[w];
      if (w < warp) wbase += s;
      tile_total += s;
    }
    uint32_t carry = carry_s;
    if (c < nchunks) chunk_counts[c * E + e] = carry + wbase + incl - x;
    __syncthreads();
    if (threadIdx.x == 0) carry_s = carry + tile_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    totals[e] = carry_s;
    __threadfence();
    unsigned t = atomicAdd(ticket, 1u);
    last_s = (t == static_cast<unsigned>(gridDim.x) - 1u);
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();
  // exclusive scan of the E totals by the whole block (E <= 512: two per thread)
  __shared__ uint32_t tot_s[KOLIBRI_MAX_EXPERTS];
  for (int x = threadIdx.x; x < E; x += kPermThreads)
    tot_s[x] = *reinterpret_cast<volatile uint32_t*>(totals + x);
  __syncthreads();
  const int x0 = 2 * threadIdx.x;
  const uint32_t a0 = x0 < E ? tot_s[x0] : 0u, a1 = x0 + 1 < E ? tot_s[x0 + 1] : 0u;
  const uint32_t pair = a0 + a1;
  uint32_t incl = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += warp_sums[w];
  const uint32_t excl = wbase + incl - pair;
  if (x0 < E) {
    offsets[x0] = excl;
    counts[x0] = static_cast<int32_t>(a0);
  }
  if (x0 + 1 < E) {
    offsets[x0 + 1] = excl + a0;
    counts[x0 + 1] = static_cast<int32_t>(a1);
  }
  if (x0 + 1 == E || x0 + 2 == E) offsets[E] = excl + pair;  // the thread holding the last expert
  if (threadIdx.x == 0) *ticket = 0u;  // ready for the next call
}

// Exclusive prefix of n <= 2 * kPermThreads values held two per thread
// (thread t owns v0 = element 2t, v1 = element 2t+1); returns the prefix of
// element 2t and writes the grand total to *total.
__device__ __forceinline__ uint32_t block_scan_pairs(uint32_t v0, uint32_t v1, uint32_t* warp_sums,
                                                     uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t pair = v0 + v1;
  uint32_t incl = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0, all = 0;
  for (int w = 0; w < kPermWarps; ++w) {
    const uint32_t x = warp_sums[w];
    if (w < warp) wbase += x;
    all += x;
  }
  *total = all;
  return wbase + incl - pair;
}

// Stable counting sort of one tile in shared memory, then coalesced output.
// NB: bits of an expert id, with the value E meaning "no expert" (E < 2^NB).
// Each slot lives in one register from load to store: its expert in the low
// 10 bits, its rank inside the warp's run of that expert above them.
template <int NB>
__global__ void __launch_bounds__(kPermThreads, 2) tile_scatter_kernel(
    const int32_t* __restrict__ ids, int64_t NK, int E, const uint32_t* __restrict__ tile_prefix,
    const int64_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* cnt_w = sm;                                   // [kPermWarps][E]
  uint32_t* delta_e = cnt_w + kPermWarps * E;             // [E] global minus tile-local start of e's run
  uint32_t* sorted = delta_e + E;                         // [kTile] (tile slot << 10) | expert
  __shared__ uint32_t warp_sums[kPermWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTile;
  uint32_t* my_cnt = cnt_w + warp * E;
  for (int e = lane; e < E; e += 32) my_cnt[e] = 0u;
  __syncwarp();
  // ---- phase 1: per-warp stable ranks, 32 consecutive slots per round
  uint32_t xr[kSlotsPerThread];
  const int64_t w0 = t0 + static_cast<int64_t>(warp) * (kSlotsPerThread * 32);
  const uint32_t none = static_cast<uint32_t>(E);
#pragma unroll
  for (int r = 0; r < kSlotsPerThread; ++r) {
    // ids are complete before the scan this kernel follows was scheduled;
    // they are read through L2 (.cg), the point of coherence
    const int64_t j = w0 + r * 32 + lane;
    const int32_t x = j < NK ? __ldcg(ids + j) : -1;
    xr[r] = (x >= 0 && x < E) ? static_cast<uint32_t>(x) : none;
  }
#pragma unroll
  for (int r = 0; r < kSlotsPerThread; ++r) {
    const uint32_t e = xr[r];
    const unsigned peers = lanes_with_value<NB>(e);
    const uint32_t below = __popc(peers & lt);
    const uint32_t rk = (e != none) ? my_cnt[e] + below : 0u;
    __syncwarp();
    if (e != none && below == 0u) my_cnt[e] += __popc(peers);
    __syncwarp();
    xr[r] = e | (rk << 10);
  }
  // the scan's tile prefixes and offsets; perm and inv are written only
  // after this wait, so every earlier user of them has finished
  pdl_wait();
  __syncthreads();
  // ---- phase 2: per expert, the warps' runs one after another; the
  // expert's run in the tile after the lower experts' runs
  const int e0 = 2 * threadIdx.x, e1 = e0 + 1;
  uint32_t tot0 = 0u, tot1 = 0u;
  for (int w = 0; w < kPermWarps; ++w) {
    if (e0 < E) {
      const uint32_t c = cnt_w[w * E + e0];
      cnt_w[w * E + e0] = tot0;
      tot0 += c;
    }
    if (e1 < E) {
      const uint32_t c = cnt_w[w * E + e1];
      cnt_w[w * E + e1] = tot1;
      tot1 += c;
    }
  }
  uint32_t tile_total;
  const uint32_t start0 = block_scan_pairs(tot0, tot1, warp_sums, &tile_total);
  const uint32_t start1 = start0 + tot0;
  // warp starts become tile-local positions
  for (int w = 0; w < kPermWarps; ++w) {
    if (e0 < E) cnt_w[w * E + e0] += start0;
    if (e1 < E) cnt_w[w * E + e1] += start1;
  }
  if (e0 < E)
    delta_e[e0] = static_cast<uint32_t>(offsets[e0]) +
                  tile_prefix[static_cast<int64_t>(blockIdx.x) * E + e0] - start0;
  if (e1 < E)
    delta_e[e1] = static_cast<uint32_t>(offsets[e1]) +
                  tile_prefix[static_cast<int64_t>(blockIdx.x) * E + e1] - start1;
  __syncthreads();
  // ---- phase 3: tile-local positions; inv in slot order
#pragma unroll
  for (int r = 0; r < kSlotsPerThread; ++r) {
    const uint32_t e = xr[r] & 1023u;
    if (e != none) {
      const uint32_t lpos = my_cnt[e] + (xr[r] >> 10);
      const uint32_t jl = static_cast<uint32_t>(warp * (kSlotsPerThread * 32) + r * 32 + lane);
      sorted[lpos] = (jl << 10) | e;
      if (inv) inv[t0 + jl] = static_cast<int32_t>(delta_e[e] + lpos);
    }
  }
  __syncthreads();
  // ---- phase 4: perm as one contiguous run per expert
  for (uint32_t pidx = threadIdx.x; pidx < tile_total; pidx += kPermThreads) {
    const uint32_t v = sorted[pidx];
    perm[delta_e[v & 1023u] + pidx] = static_cast<int32_t>(t0 + (v >> 10));
  }
}

// All three steps in one block (small N*K, decode batches).  Each of the 16
// warps ranks a contiguous segment of slots (stable inside the segment: the
// lanes of a round are grouped by expert with __match_any_sync and a per-warp
// counter per expert carries the rounds); one thread per expert turns the
// per-warp counts into starts; a block scan gives the offsets.  Slot order is
// segment order, then round order, then lane order, which is j order.
constexpr int kSingleThreads = 512;
constexpr int kSingleWarps = kSingleThreads / kWarp;
constexpr int kSingleRounds = static_cast<int>(kSingleMax / (kSingleWarps * 32));   // 8
static_assert(kSingleMax % (kSingleWarps * 32) == 0, "segments of whole rounds");
static_assert(KOLIBRI_MAX_EXPERTS <= kSingleThreads, "one thread per expert");

__global__ void __launch_bounds__(kSingleThreads) permute_single_kernel(
    const int32_t* __restrict__ ids, int64_t NK, int E, int32_t* __restrict__ counts,
    int64_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  __shared__ uint32_t cnt_w[kSingleWarps][KOLIBRI_MAX_EXPERTS];   // per-warp counts, then starts
  __shared__ uint32_t start_e[KOLIBRI_MAX_EXPERTS];
  __shared__ uint32_t warp_sums[kSingleWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t* my_cnt = cnt_w[warp];
  for (int e = lane; e < E; e += 32) my_cnt[e] = 0u;
  __syncwarp();
  pdl_wait();       // ids come from the kernel before this one
  pdl_trigger();
  // ---- segment ranks: this warp's slots [w0, w0 + 32 * rounds)
  const int64_t seg = ((NK + kSingleWarps * 32 - 1) / (kSingleWarps * 32)) * 32;
  const int64_t w0 = static_cast<int64_t>(warp) * seg;
  int32_t ex[kSingleRounds];
  uint32_t rk[kSingleRounds];
  bool bad = false;
#pragma unroll
  for (int r = 0; r < kSingleRounds; ++r) {
    const int64_t j = w0 + r * 32 + lane;
    const bool in = r * 32 < seg && j < NK;
    int32_t x = in ? __ldg(ids + j) : -1;
    if (in && !(x >= 0 && x < E)) bad = true;
    x = (x >= 0 && x < E) ? x : -1;
    ex[r] = x;
    // one block, latency-bound: a single match instruction beats the chain of
    // per-bit ballots that the tiled scatter uses for throughput
    const unsigned peers = __match_any_sync(0xffffffffu, x);
    const uint32_t below = __popc(peers & lt);
    rk[r] = (x >= 0) ? my_cnt[x] + below : 0u;
    __syncwarp();
    if (x >= 0 && below == 0u) my_cnt[x] += __popc(peers);
    __syncwarp();
  }
  if (bad) raise_status(kStatusBadInput);
  __syncthreads();
  // ---- per expert: warp starts inside the expert's run, and its total
  uint32_t tot = 0u;
  if (tid < E) {
    for (int w = 0; w < kSingleWarps; ++w) {
      const uint32_t c = cnt_w[w][tid];
      cnt_w[w][tid] = tot;
      tot += c;
    }
  }
  // ---- exclusive scan of the totals over experts (E <= kSingleThreads)
  uint32_t incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  uint32_t wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += warp_sums[w];
  const uint32_t excl = wbase + incl - tot;
  if (tid < E) {
    start_e[tid] = excl;
    offsets[tid] = excl;
    counts[tid] = static_cast<int32_t>(tot);
    if (tid == E - 1) offsets[E] = excl + tot;
  }
  __syncthreads();
  // ---- positions
#pragma unroll
  for (int r = 0; r < kSingleRounds; ++r) {
    const int32_t e = ex[r];
    if (e >= 0) {
      const int64_t j = w0 + r * 32 + lane;
      const uint32_t pos = start_e[e] + my_cnt[e] + rk[r];
      perm[pos] = static_cast<int32_t>(j);
      if (inv) inv[j] = static_cast<int32_t>(pos);
    }
  }
}

}  // namespace

size_t tile_scatter_smem(int E) {
  return sizeof(uint32_t) * (static_cast<size_t>(kPermWarps) * E + static_cast<size_t>(E) +
                             static_cast<size_t>(kTile));
}

PermuteLayout permute_layout(int64_t N, int32_t E, int32_t K) {
  PermuteLayout L;
  const int64_t NK = N * K;
  L.chunk = kTile;
  L.nchunks = (NK + kTile - 1) / kTile;
  L.single_cta = NK <= kSingleMax;
  size_t off = 0;
  L.off_chunk_counts = off;
  off += align256(sizeof(uint32_t) * static_cast<size_t>(L.nchunks) * static_cast<size_t>(E));
  L.off_counts = off;
  off += align256(sizeof(uint32_t) * static_cast<size_t>(E));
  L.off_ticket = off;
  off += align256(sizeof(uint32_t));
  L.off_dec_ticket = off;
  off += align256(sizeof(uint32_t));
  L.total = off;
  return L;
}

cudaError_t launch_permute(const int32_t* ids, int64_t N, int32_t E, int32_t K, int32_t* counts,
                           int64_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                           cudaStream_t s) {
  const int64_t NK = N * K;
  const PermuteLayout L = permute_layout(N, E, K);
  if (L.single_cta) {
    return launch_pdl(permute_single_kernel, dim3(1), dim3(kSingleThreads), 0, s, dim3(0, 0, 0), ids,
                      NK, E, counts, offsets, perm, inv);
  }
  char* base = static_cast<char*>(ws);
  uint32_t* tile_counts = reinterpret_cast<uint32_t*>(base + L.off_chunk_counts);
  uint32_t* totals = reinterpret_cast<uint32_t*>(base + L.off_counts);
  uint32_t* ticket = reinterpret_cast<uint32_t*>(base + L.off_ticket);
  const unsigned tiles = static_cast<unsigned>(L.nchunks);
  const size_t smem = tile_scatter_smem(E);
  const int nb = expert_bits(E);   // E itself stands for "no expert"
  auto kern = nb <= 8 ? tile_scatter_kernel<8> : nb <= 9 ? tile_scatter_kernel<9> : tile_scatter_kernel<10>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  // a chain of programmatic dependent launches: see each kernel's waits
  err = launch_pdl(tile_count_kernel, dim3(tiles), dim3(kPermThreads), 0, s, dim3(0, 0, 0), ids, NK, E,
                   tile_counts, ticket);
  if (err != cudaSuccess) return err;
  err = launch_pdl(chunk_scan_kernel, dim3(static_cast<unsigned>(E)), dim3(kPermThreads), 0, s,
                   dim3(0, 0, 0), tile_counts, L.nchunks, E, totals, ticket, counts, offsets);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(tiles), dim3(kPermThreads), smem, s, dim3(0, 0, 0), ids, NK, E,
                    static_cast<const uint32_t*>(tile_counts), static_cast<const int64_t*>(offsets), perm, inv);
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_permute)

}  // namespace kolibri
