// permute.cu -- expert loads and the stable grouping of routed slots.
//
// Loads c_e are the per-expert counts of "Kolibri Pre-Training from
// Scratch" 6.1/6.2.  The grouping is a stable counting sort of the slot
// index j = t*K + k by expert: offsets = exclusive prefix sum of counts,
// perm[p] = j in (expert, j) order, inv[j] = p.
//
// Large inputs, three launches:
//   A  each warp counts its chunk of slots into a shared histogram and
//      writes it to chunk_counts[chunk][E] (coalesced);
//   B  one block per expert turns its column of chunk counts into an
//      exclusive prefix; the last block to finish (ticket) scans the totals
//      into offsets/counts;
//   C  each warp replays its chunk 32 slots at a time; __match_any_sync
//      groups lanes by expert, the rank inside the group is the popcount of
//      lower lanes, and a per-warp running cursor keeps the order stable.
// Small inputs (decode) run the same three steps inside one block.
#include "launch.h"
#include "common.cuh"

namespace kolibri {

namespace {

constexpr int kPermThreads = 256;
constexpr int kPermWarps = kPermThreads / kWarp;
constexpr int64_t kChunk = 1024;        // slots per warp chunk
constexpr int64_t kSingleMax = 4096;    // N*K handled by one block
constexpr int kUnroll = 8;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

__global__ void __launch_bounds__(kPermThreads) chunk_count_kernel(
    const int32_t* __restrict__ ids, int64_t NK, int E, int64_t nchunks,
    uint32_t* __restrict__ chunk_counts) {
  extern __shared__ uint32_t hist_all[];  // [kPermWarps][E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* hist = hist_all + warp * E;
  for (int e = lane; e < E; e += 32) hist[e] = 0u;
  __syncwarp();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kPermWarps + warp;
  if (c >= nchunks) return;
  const int64_t j0 = c * kChunk;
  const int64_t j1 = (j0 + kChunk < NK) ? j0 + kChunk : NK;
  bool bad = false;
  for (int64_t base = j0; base < j1; base += 32 * kUnroll) {
    int32_t v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t j = base + u * 32 + lane;
      v[u] = j < j1 ? __ldg(ids + j) : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t j = base + u * 32 + lane;
      if (j < j1) {
        if (v[u] >= 0 && v[u] < E) atomicAdd(&hist[v[u]], 1u);
        else bad = true;
      }
    }
  }
  if (bad) raise_status(kStatusBadInput);
  __syncwarp();
  for (int e = lane; e < E; e += 32) chunk_counts[c * E + e] = hist[e];
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

__device__ __forceinline__ void scatter_round(int32_t e, int64_t j, int lane, uint32_t* cursor,
                                              int32_t* __restrict__ perm,
                                              int32_t* __restrict__ inv) {
  const unsigned lt = (1u << lane) - 1u;
  unsigned peers = __match_any_sync(0xffffffffu, e);
  if (e >= 0) {
    unsigned rank = __popc(peers & lt);
    uint32_t pos = cursor[e] + rank;
    perm[pos] = static_cast<int32_t>(j);
    if (inv) inv[j] = static_cast<int32_t>(pos);
  }
  __syncwarp();
  if (e >= 0 && (peers & lt) == 0u) cursor[e] += __popc(peers);
  __syncwarp();
}

__global__ void __launch_bounds__(kPermThreads) chunk_scatter_kernel(
    const int32_t* __restrict__ ids, int64_t NK, int E, int64_t nchunks,
    const uint32_t* __restrict__ chunk_prefix, const int64_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ uint32_t cur_all[];  // [kPermWarps][E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* cursor = cur_all + warp * E;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kPermWarps + warp;
  if (c >= nchunks) return;
  for (int e = lane; e < E; e += 32)
    cursor[e] = static_cast<uint32_t>(offsets[e]) + chunk_prefix[c * E + e];
  __syncwarp();
  const int64_t j0 = c * kChunk;
  const int64_t j1 = (j0 + kChunk < NK) ? j0 + kChunk : NK;
  for (int64_t base = j0; base < j1; base += 32 * kUnroll) {
    int32_t v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t j = base + u * 32 + lane;
      int32_t x = j < j1 ? __ldg(ids + j) : -1;
      v[u] = (x >= 0 && x < E) ? x : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) scatter_round(v[u], base + u * 32 + lane, lane, cursor, perm, inv);
  }
}

// All three steps in one block (small N*K).
__global__ void __launch_bounds__(1024) permute_single_kernel(
    const int32_t* __restrict__ ids, int64_t NK, int E, int32_t* __restrict__ counts,
    int64_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  __shared__ uint32_t hist[KOLIBRI_MAX_EXPERTS];
  __shared__ uint32_t cursor[KOLIBRI_MAX_EXPERTS];
  const int tid = threadIdx.x, lane = tid & 31;
  for (int e = tid; e < E; e += blockDim.x) hist[e] = 0u;
  __syncthreads();
  bool bad = false;
  for (int64_t j = tid; j < NK; j += blockDim.x) {
    int32_t x = __ldg(ids + j);
    if (x >= 0 && x < E) atomicAdd(&hist[x], 1u);
    else bad = true;
  }
  if (bad) raise_status(kStatusBadInput);
  __syncthreads();
  if (tid == 0) {
    int64_t run = 0;
    for (int e = 0; e < E; ++e) {
      offsets[e] = run;
      counts[e] = static_cast<int32_t>(hist[e]);
      cursor[e] = static_cast<uint32_t>(run);
      run += hist[e];
    }
    offsets[E] = run;
  }
  __syncthreads();
  if (tid < 32) {
    for (int64_t base = 0; base < NK; base += 32) {
      int64_t j = base + lane;
      int32_t x = j < NK ? __ldg(ids + j) : -1;
      x = (x >= 0 && x < E) ? x : -1;
      scatter_round(x, j, lane, cursor, perm, inv);
    }
  }
}

}  // namespace

PermuteLayout permute_layout(int64_t N, int32_t E, int32_t K) {
  PermuteLayout L;
  const int64_t NK = N * K;
  L.chunk = kChunk;
  L.nchunks = (NK + kChunk - 1) / kChunk;
  L.single_cta = NK <= kSingleMax;
  size_t off = 0;
  L.off_chunk_counts = off;
  off += align256(sizeof(uint32_t) * static_cast<size_t>(L.nchunks) * static_cast<size_t>(E));
  L.off_counts = off;
  off += align256(sizeof(uint32_t) * static_cast<size_t>(E));
  L.off_ticket = off;
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
    permute_single_kernel<<<1, 1024, 0, s>>>(ids, NK, E, counts, offsets, perm, inv);
    return cudaGetLastError();
  }
  char* base = static_cast<char*>(ws);
  uint32_t* chunk_counts = reinterpret_cast<uint32_t*>(base + L.off_chunk_counts);
  uint32_t* totals = reinterpret_cast<uint32_t*>(base + L.off_counts);
  uint32_t* ticket = reinterpret_cast<uint32_t*>(base + L.off_ticket);
  cudaError_t err = cudaMemsetAsync(ticket, 0, sizeof(uint32_t), s);
  if (err != cudaSuccess) return err;
  const unsigned blocks = static_cast<unsigned>((L.nchunks + kPermWarps - 1) / kPermWarps);
  const size_t smem = sizeof(uint32_t) * kPermWarps * static_cast<size_t>(E);
  chunk_count_kernel<<<blocks, kPermThreads, smem, s>>>(ids, NK, E, L.nchunks, chunk_counts);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  chunk_scan_kernel<<<E, kPermThreads, 0, s>>>(chunk_counts, L.nchunks, E, totals, ticket, counts,
                                               offsets);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  chunk_scatter_kernel<<<blocks, kPermThreads, smem, s>>>(ids, NK, E, L.nchunks, chunk_counts,
                                                          offsets, perm, inv);
  return cudaGetLastError();
}

}  // namespace kolibri
