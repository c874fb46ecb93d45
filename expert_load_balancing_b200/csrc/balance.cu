// balance.cu -- the balancing pieces beside the routing path:
//   * EQB with bfloat16 keys, as the pages run it ("Kolibri Pre-Training
//     from Scratch" 7.3): every value of the column Z_:,e + alpha is rounded
//     to bf16 and encoded as an order-preserving 16-bit key; pass one builds
//     a 256-bin histogram of the high byte, the bins are scanned from the top
//     to the bin holding the target rank; pass two histograms the low byte of
//     the keys in that bin and reads off the exact key.  The histograms are
//     the only thing that crosses ranks in a distributed batch (one
//     all-reduce of 256 E counts per pass), so each pass is its own call.
//   * The same two-pass-per-byte scheme on the fp32 keys of the main update
//     (four passes), so that update too can run over a batch split across
//     ranks with only histograms crossing.
//   * Load-Error Injection (section 8): per-expert load error rho from the
//     microbatch counts, xi = |rho|_inf / tau, and G += lambda tanh(xi)/xi rho
//     on every token's score gradient; and the chain rule to the logits,
//     dZ = dS sigma(Z)(1 - sigma(Z)).
//   * The intervention rate (section 9): the share of the router's own top-K
//     that the bias moved out of the routed set.
#include <cuda_bf16.h>

#include "launch.h"
#include "route.cuh"

namespace kolibri {

namespace {

constexpr int kBins = 256;
constexpr int kColsPerCta = 64;          // a lane owns two columns of the group
// A column's bins sit kBinLd words apart in shared memory: with 256 every
// lane's column would start in the same bank, and the lanes of a warp (all
// on different columns, mostly on the same bin) would serialise their
// atomics 32-fold.
constexpr int kBinLd = kBins + 1;
constexpr int kRowBatch = 8;             // rows a warp loads before counting them
constexpr int kHistThreads = 256;

__device__ __forceinline__ uint32_t bf16_key_of(float z, float a) {
  const float c = __fadd_rn(z, a);
  const uint32_t b = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(c)));
  return (b & 0x8000u) ? (~b & 0xffffu) : (b | 0x8000u);
}

// One pass of the bf16 radix selection over rows of Z + alpha.  Pass one
// (prefix == nullptr): bin = high byte of the key.  Pass two: only keys whose
// high byte is prefix[e], bin = low byte.  hist [E][256] is accumulated
// (several launches, e.g. row blocks, may add into one histogram).
// Grid: x over row blocks, y over 128-column groups.
__global__ void __launch_bounds__(kHistThreads) bf16_hist_kernel(
    const float* __restrict__ z, const float* __restrict__ alpha, int64_t N, int E,
    const uint32_t* __restrict__ prefix, uint32_t* __restrict__ hist) {
  extern __shared__ uint32_t hist_smem[];
  uint32_t* h = hist_smem;                               // [64][kBinLd], 64 KB
  uint32_t* pre_s = hist_smem + kColsPerCta * kBinLd;    // [64]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col0 = blockIdx.y * kColsPerCta;
  for (int i = threadIdx.x; i < kColsPerCta * kBinLd; i += kHistThreads) h[i] = 0u;
  for (int i = threadIdx.x; i < kColsPerCta; i += kHistThreads)
    pre_s[i] = (prefix && col0 + i < E) ? prefix[col0 + i] : 0u;
  __syncthreads();
  const int c4 = 2 * lane;                               // this lane's columns in the group
  const bool active = col0 + c4 < E;                     // E % 4 == 0: two or none
  uint32_t pre[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) pre[i] = pre_s[(c4 + i) & (kColsPerCta - 1)];
  // a warp takes kRowBatch rows at a time and issues all their loads first
  const int64_t rows_per_block = static_cast<int64_t>(kHistThreads / 32) * kRowBatch;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * rows_per_block + warp * kRowBatch; t0 < N;
       t0 += static_cast<int64_t>(gridDim.x) * rows_per_block) {
    if (!active) continue;
    float2 v[kRowBatch];
    float a[kRowBatch];
#pragma unroll
    for (int r = 0; r < kRowBatch; ++r) {
      const int64_t t = t0 + r < N ? t0 + r : N - 1;
      a[r] = alpha ? __ldg(alpha + t) : 0.f;
      v[r] = __ldcs(reinterpret_cast<const float2*>(z + t * E + col0 + c4));
    }
#pragma unroll
    for (int r = 0; r < kRowBatch; ++r) {
      if (t0 + r >= N) break;
      const float vv[2] = {v[r].x, v[r].y};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t k = bf16_key_of(vv[i], a[r]);
        if (prefix == nullptr) {
          atomicAdd(&h[(c4 + i) * kBinLd + (k >> 8)], 1u);
        } else if ((k >> 8) == pre[i]) {
          atomicAdd(&h[(c4 + i) * kBinLd + (k & 0xffu)], 1u);
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kColsPerCta * kBins; i += kHistThreads) {
    const int c = i / kBins, b = i % kBins;
    const uint32_t n = h[c * kBinLd + b];
    if (col0 + c < E && n) atomicAdd(hist + static_cast<int64_t>(col0 + c) * kBins + b, n);
  }
}

// Per expert (one warp each): scan the bins from the top; the bin holding
// the rank-th largest key (0-based) becomes this pass's digit, and rank is
// reduced by the keys in the bins above it.
__global__ void bf16_digit_kernel(const uint32_t* __restrict__ hist, int E,
                                  int64_t* __restrict__ rank, uint32_t* __restrict__ digit) {
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  // lane l holds bins 255 - 8l ... 248 - 8l (the top bins in the low lanes)
  const uint32_t* he = hist + static_cast<int64_t>(e) * kBins;
  uint32_t c[8];
  uint64_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = he[255 - (8 * lane + i)];
    sum += c[i];
  }
  uint64_t incl = sum;                                   // inclusive scan over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  uint64_t above = incl - sum;                           // keys in higher bins
  const int64_t r = rank[e];
  const bool mine = static_cast<int64_t>(above) <= r && r < static_cast<int64_t>(incl);
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  if (mine) {
    int i = 0;
    while (i < 7 && static_cast<int64_t>(above + c[i]) <= r) {
      above += c[i];
      ++i;
    }
    digit[e] = static_cast<uint32_t>(255 - (8 * lane + i));
    rank[e] = r - static_cast<int64_t>(above);
  }
  if (who == 0u && lane == 0) digit[e] = 0xffffffffu;   // rank past the column: no such key
}

// v_e from the two digits (the bf16 key), then beta = -v, centred.
__global__ void bf16_value_kernel(const uint32_t* __restrict__ d_hi, const uint32_t* __restrict__ d_lo,
                                  int E, float* __restrict__ v) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const uint32_t k = ((d_hi[e] & 0xffu) << 8) | (d_lo[e] & 0xffu);
  const uint32_t b = (k & 0x8000u) ? (k & 0x7fffu) : (~k & 0xffffu);
  v[e] = __uint_as_float(b << 16);
}

// The same radix selection on the fp32 keys of the main update (the order
// key of Z + alpha), four passes of 8-bit digits from the top: pass p bins
// byte 3 - p of the keys whose top 8p bits equal prefix[e] (the digits of the
// earlier passes).  As above, only the histograms cross ranks.
__global__ void __launch_bounds__(kHistThreads) key_hist_kernel(
    const float* __restrict__ z, const float* __restrict__ alpha, int64_t N, int E, int pass,
    const uint32_t* __restrict__ prefix, uint32_t* __restrict__ hist) {
  extern __shared__ uint32_t hist_smem[];
  uint32_t* h = hist_smem;                               // [64][kBinLd], 64 KB
  uint32_t* pre_s = hist_smem + kColsPerCta * kBinLd;    // [64]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col0 = blockIdx.y * kColsPerCta;
  const int shift = 24 - 8 * pass;                       // this pass's byte
  for (int i = threadIdx.x; i < kColsPerCta * kBinLd; i += kHistThreads) h[i] = 0u;
  for (int i = threadIdx.x; i < kColsPerCta; i += kHistThreads)
    pre_s[i] = (pass > 0 && col0 + i < E) ? prefix[col0 + i] : 0u;
  __syncthreads();
  const int c4 = 2 * lane;
  const bool active = col0 + c4 < E;
  // keys match when their bits above this pass's byte equal the prefix's
  const uint32_t hi_mask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
  uint32_t pre[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) pre[i] = pre_s[(c4 + i) & (kColsPerCta - 1)] & hi_mask;
  const int64_t rows_per_block = static_cast<int64_t>(kHistThreads / 32) * kRowBatch;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * rows_per_block + warp * kRowBatch; t0 < N;
       t0 += static_cast<int64_t>(gridDim.x) * rows_per_block) {
    if (!active) continue;
    float2 v[kRowBatch];
    float a[kRowBatch];
#pragma unroll
    for (int r = 0; r < kRowBatch; ++r) {
      const int64_t t = t0 + r < N ? t0 + r : N - 1;
      a[r] = alpha ? __ldg(alpha + t) : 0.f;
      v[r] = __ldcs(reinterpret_cast<const float2*>(z + t * E + col0 + c4));
    }
#pragma unroll
    for (int r = 0; r < kRowBatch; ++r) {
      if (t0 + r >= N) break;
      const float vv[2] = {v[r].x, v[r].y};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t k = order_key(__fadd_rn(vv[i], a[r]));
        if ((k & hi_mask) == pre[i]) atomicAdd(&h[(c4 + i) * kBinLd + ((k >> shift) & 0xffu)], 1u);
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kColsPerCta * kBins; i += kHistThreads) {
    const int c = i / kBins, b = i % kBins;
    const uint32_t n = h[c * kBinLd + b];
    if (col0 + c < E && n) atomicAdd(hist + static_cast<int64_t>(col0 + c) * kBins + b, n);
  }
}

// Per expert: this pass's digit (as bf16_digit_kernel), then the prefix
// gains it as byte 3 - pass (pass 0 starts the prefix).
__global__ void key_digit_kernel(const uint32_t* __restrict__ hist, int E, int pass,
                                 int64_t* __restrict__ rank, uint32_t* __restrict__ prefix) {
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= E) return;
  const uint32_t* he = hist + static_cast<int64_t>(e) * kBins;
  uint32_t c[8];
  uint64_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = he[255 - (8 * lane + i)];
    sum += c[i];
  }
  uint64_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  uint64_t above = incl - sum;
  const int64_t r = rank[e];
  const bool mine = static_cast<int64_t>(above) <= r && r < static_cast<int64_t>(incl);
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  const int shift = 24 - 8 * pass;
  if (mine) {
    int i = 0;
    while (i < 7 && static_cast<int64_t>(above + c[i]) <= r) {
      above += c[i];
      ++i;
    }
    const uint32_t dgt = static_cast<uint32_t>(255 - (8 * lane + i));
    const uint32_t keep = pass == 0 ? 0u : (prefix[e] & (0xffffffffu << (shift + 8)));
    prefix[e] = keep | (dgt << shift);
    rank[e] = r - static_cast<int64_t>(above);
  }
  if (who == 0u && lane == 0) raise_status(kStatusBadInput);   // rank past the column
}

__global__ void key_value_kernel(const uint32_t* __restrict__ key, int E, float* __restrict__ v) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) v[e] = key_to_float(key[e]);
}

// The sampled-bracket update over a split batch.  After this rank's full
// pass, counts = [above | inside | overflow] per expert: overflow marks an
// expert whose bracketed keys did not all fit this rank's gather buffer.
__global__ void dist_count_finish_kernel(uint32_t* __restrict__ counts, int E, int64_t cap) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) counts[2 * E + e] = static_cast<int64_t>(counts[E + e]) > cap ? 1u : 0u;
}

// The ranks' gathered samples, rank-major [R][E][S], laid out expert-major
// [E][ld] (rank r's keys of expert e at e ld + r S) for the sample selection.
__global__ void dist_sample_transpose_kernel(const uint32_t* __restrict__ in, int R, int64_t S,
                                             int E, int64_t ld, uint32_t* __restrict__ out) {
  const int64_t total = static_cast<int64_t>(R) * E * S;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t s = i % S, re = i / S;
    const int64_t e = re % E, r = re / E;
    out[e * ld + r * S + s] = in[i];
  }
}

// From the counts summed over ranks: the target's rank among the bracketed
// keys, rank[e] = m - above[e], and flag[e] = 1 unless the target lies in
// the bracket (above <= m < above + inside) and no rank overflowed.
__global__ void dist_rank_kernel(const uint32_t* __restrict__ counts, int E, int64_t m,
                                 int64_t* __restrict__ rank, uint32_t* __restrict__ flag) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int64_t above = counts[e], inside = counts[E + e];
  const bool ok = counts[2 * E + e] == 0u && above <= m && m < above + inside;
  rank[e] = ok ? m - above : 0;
  flag[e] = ok ? 0u : 1u;
}

// One radix pass over this rank's bracketed keys of expert e (one block per
// expert): adds to hist[e] the count per byte 3 - pass among the keys whose
// top 8 pass bits equal prefix[e], as key_hist_kernel does over Z.
constexpr int kCandHistThreads = 256;
__global__ void __launch_bounds__(kCandHistThreads) dist_cand_hist_kernel(
    const uint32_t* __restrict__ cand, const uint32_t* __restrict__ counts, int64_t cap, int E,
    int pass, const uint32_t* __restrict__ prefix, uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[kBins];
  const int e = blockIdx.x;
  for (int b = threadIdx.x; b < kBins; b += kCandHistThreads) h[b] = 0u;
  __syncthreads();
  const int shift = 24 - 8 * pass;
  const uint32_t hi_mask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
  const uint32_t pre = pass == 0 ? 0u : (prefix[e] & hi_mask);
  int64_t n = counts[E + e];
  if (n > cap) n = cap;   // flagged: the result is discarded
  const uint32_t* keys = cand + static_cast<int64_t>(e) * cap;
  for (int64_t i = threadIdx.x; i < n; i += kCandHistThreads) {
    const uint32_t k = __ldg(keys + i);
    if ((k & hi_mask) == pre) atomicAdd(&h[(k >> shift) & 0xffu], 1u);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += kCandHistThreads)
    if (h[b]) hist[static_cast<int64_t>(e) * kBins + b] += h[b];
}

// rho_e = c_e / (K N / E) - 1, xi = max |rho| / tau, delta_e = lambda *
// (tanh(xi)/xi) * rho_e in fp64 (the factor is 1 at xi = 0), rounded once
// to fp32.  tanh(x) = (1 - e^(-2x)) / (1 + e^(-2x)) with the gate's exp.
__device__ __forceinline__ void lei_deltas(const int32_t* __restrict__ counts, int64_t N, int E,
                                           int K, double lambda, double tau, float* delta_s,
                                           double* red) {
  const double target =
      __ddiv_rn(__dmul_rn(static_cast<double>(K), static_cast<double>(N)), static_cast<double>(E));
  double mx = 0.0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const double rho = __dsub_rn(__ddiv_rn(static_cast<double>(counts[e]), target), 1.0);
    mx = fmax(mx, fabs(rho));
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    double m = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = fmax(m, red[w]);
    const double xi = __ddiv_rn(m, tau);
    double factor = 1.0;
    if (xi != 0.0) {
      double th = 1.0;
      if (!(xi > 350.0)) {
        const double t = gate_exp(__dmul_rn(-2.0, xi));
        th = __ddiv_rn(__dsub_rn(1.0, t), __dadd_rn(1.0, t));
      }
      factor = __ddiv_rn(th, xi);
    }
    red[0] = factor;
  }
  __syncthreads();
  const double factor = red[0];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const double rho = __dsub_rn(__ddiv_rn(static_cast<double>(counts[e]), target), 1.0);
    delta_s[e] = __double2float_rn(__dmul_rn(__dmul_rn(lambda, factor), rho));
  }
  __syncthreads();
}

constexpr int kLeiThreads = 256;

// G[t][e] += delta_e for every token of the microbatch; G [N, E] fp32.
__global__ void __launch_bounds__(kLeiThreads) lei_inject_kernel(
    const int32_t* __restrict__ counts, int64_t N, int E, int K, double lambda, double tau,
    float* __restrict__ g) {
  __shared__ float delta_s[KOLIBRI_MAX_EXPERTS];
  __shared__ double red[kLeiThreads / 32];
  lei_deltas(counts, N, E, K, lambda, tau, delta_s, red);
  const int64_t n4 = N * static_cast<int64_t>(E) / 4;   // E % 4 == 0
  float4* g4 = reinterpret_cast<float4*>(g);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kLeiThreads + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * kLeiThreads) {
    const int e = static_cast<int>((4 * i) % E);
    float4 v = g4[i];
    v.x = __fadd_rn(v.x, delta_s[e]);
    v.y = __fadd_rn(v.y, delta_s[e + 1]);
    v.z = __fadd_rn(v.z, delta_s[e + 2]);
    v.w = __fadd_rn(v.w, delta_s[e + 3]);
    g4[i] = v;
  }
}

// dZ = dS * sigma(Z) (1 - sigma(Z)): sigma in fp64 from the gate's exp
// (saturating outside |z| <= 700 as the gate does), the product in fp64,
// rounded once to fp32.
__device__ __forceinline__ float score_grad_one(float zi, float gi) {
  double s;
  if (zi > 700.0f) {
    s = 1.0;
  } else if (zi < -700.0f) {
    s = 0.0;
  } else {
    s = __ddiv_rn(1.0, __dadd_rn(1.0, gate_exp(-static_cast<double>(zi))));
  }
  return __double2float_rn(__dmul_rn(static_cast<double>(gi), __dmul_rn(s, __dsub_rn(1.0, s))));
}

__global__ void __launch_bounds__(kLeiThreads) score_grad_kernel(
    const float* __restrict__ z, const float* __restrict__ gs, int64_t n, float* __restrict__ gz) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kLeiThreads + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * kLeiThreads)
    gz[i] = score_grad_one(z[i], gs[i]);
}

// Four consecutive elements per thread (16-byte aligned arrays): the same
// arithmetic per element, four independent fp64 chains to interleave.
__global__ void __launch_bounds__(kLeiThreads) score_grad_vec_kernel(
    const float4* __restrict__ z, const float4* __restrict__ gs, int64_t n4, float4* __restrict__ gz,
    const float* __restrict__ z_tail, const float* __restrict__ gs_tail, int tail, float* __restrict__ gz_tail) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kLeiThreads + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * kLeiThreads) {
    const float4 zq = __ldg(z + i), gq = __ldg(gs + i);
    gz[i] = make_float4(score_grad_one(zq.x, gq.x), score_grad_one(zq.y, gq.y), score_grad_one(zq.z, gq.z),
                        score_grad_one(zq.w, gq.w));
  }
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < tail)
    gz_tail[threadIdx.x] = score_grad_one(z_tail[threadIdx.x], gs_tail[threadIdx.x]);
}

// Overlap of the router's own top-K (no bias) with the routed ids, summed
// over tokens into total[0].  One warp per token.
template <int Q, bool kFull>
__global__ void __launch_bounds__(256) overlap_kernel(const float* __restrict__ z,
                                                      const int32_t* __restrict__ ids, int64_t N,
                                                      int E, int K,
                                                      unsigned long long* __restrict__ total) {
  __shared__ RowScratch<Q> scratch[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t valid = 0u;
#pragma unroll
  for (int j = 0; j < 4 * Q; ++j) valid |= (static_cast<int>(slot_expert(lane, j)) < E) ? (1u << j) : 0u;
  unsigned long long mine = 0ull;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < N;
       row += static_cast<int64_t>(gridDim.x) * 8) {
    float zr[4 * Q];
    load_row<Q, kFull>(z + row * E, E, lane, zr);
    int rank;
    uint32_t key, id;
    warp_select_row<Q, kFull, false>(zr, nullptr, valid, K, lane, scratch[warp], rank, key, id);
    bool hit = false;
    if (rank >= 0 && rank < K)
      for (int k = 0; k < K; ++k) hit |= (ids[row * K + k] == static_cast<int32_t>(id));
    mine += __popc(__ballot_sync(0xffffffffu, hit));
    __syncwarp();
  }
  if (lane == 0 && mine) atomicAdd(total, mine);
}

__global__ void intervention_finish_kernel(const unsigned long long* total, int64_t N, int K,
                                           double* rate) {
  *rate = __dsub_rn(1.0, __ddiv_rn(static_cast<double>(*total),
                                   __dmul_rn(static_cast<double>(N), static_cast<double>(K))));
}

int grid_for(int64_t work, int per_block) {
  int64_t b = (work + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_bf16_hist(const float* z, const float* alpha, int64_t N, int32_t E,
                             const uint32_t* prefix, uint32_t* hist, cudaStream_t s) {
  const int groups = (E + kColsPerCta - 1) / kColsPerCta;
  int per_group = 3 * device_sm_count() / groups;        // three 64 KB CTAs per SM
  if (per_group < 1) per_group = 1;
  const int64_t rows_per_block = (kHistThreads / 32) * kRowBatch;
  int64_t gx = (N + rows_per_block - 1) / rows_per_block;
  if (gx > per_group) gx = per_group;
  const int smem = static_cast<int>(sizeof(uint32_t) * (kColsPerCta * kBinLd + kColsPerCta));
  cudaError_t err =
      cudaFuncSetAttribute(bf16_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  bf16_hist_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(groups)), kHistThreads,
                     smem, s>>>(z, alpha, N, E, prefix, hist);
  return cudaGetLastError();
}

cudaError_t launch_bf16_digit(const uint32_t* hist, int32_t E, int64_t* rank, uint32_t* digit,
                              cudaStream_t s) {
  const int warps = 8;
  bf16_digit_kernel<<<(E + warps - 1) / warps, 32 * warps, 0, s>>>(hist, E, rank, digit);
  return cudaGetLastError();
}

cudaError_t launch_bf16_value(const uint32_t* d_hi, const uint32_t* d_lo, int32_t E, float* v,
                              cudaStream_t s) {
  bf16_value_kernel<<<(E + 255) / 256, 256, 0, s>>>(d_hi, d_lo, E, v);
  return cudaGetLastError();
}

cudaError_t launch_key_hist(const float* z, const float* alpha, int64_t N, int32_t E, int32_t pass,
                            const uint32_t* prefix, uint32_t* hist, cudaStream_t s) {
  const int groups = (E + kColsPerCta - 1) / kColsPerCta;
  int per_group = 3 * device_sm_count() / groups;
  if (per_group < 1) per_group = 1;
  const int64_t rows_per_block = (kHistThreads / 32) * kRowBatch;
  int64_t gx = (N + rows_per_block - 1) / rows_per_block;
  if (gx > per_group) gx = per_group;
  const int smem = static_cast<int>(sizeof(uint32_t) * (kColsPerCta * kBinLd + kColsPerCta));
  cudaError_t err =
      cudaFuncSetAttribute(key_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  key_hist_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(groups)), kHistThreads, smem,
                    s>>>(z, alpha, N, E, pass, prefix, hist);
  return cudaGetLastError();
}

cudaError_t launch_key_digit(const uint32_t* hist, int32_t E, int32_t pass, int64_t* rank,
                             uint32_t* prefix, cudaStream_t s) {
  const int warps = 8;
  key_digit_kernel<<<(E + warps - 1) / warps, 32 * warps, 0, s>>>(hist, E, pass, rank, prefix);
  return cudaGetLastError();
}

cudaError_t launch_key_value(const uint32_t* key, int32_t E, float* v, cudaStream_t s) {
  key_value_kernel<<<(E + 255) / 256, 256, 0, s>>>(key, E, v);
  return cudaGetLastError();
}

cudaError_t launch_dist_count(const float* z, const float* alpha, int64_t N, int32_t E, int32_t K,
                              const uint32_t* lo, const uint32_t* hi, uint32_t* counts,
                              uint32_t* cand, int64_t cap, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(uint32_t) * 3 * static_cast<size_t>(E), s);
  if (err != cudaSuccess) return err;
  err = launch_route_window_pass(z, nullptr, alpha, N, E, K, nullptr, nullptr, nullptr, lo, hi,
                                 counts, counts + E, cand, cap, s);
  if (err != cudaSuccess) return err;
  dist_count_finish_kernel<<<(E + 255) / 256, 256, 0, s>>>(counts, E, cap);
  return cudaGetLastError();
}

cudaError_t launch_dist_sample_transpose(const uint32_t* gathered, int32_t R, int64_t S, int32_t E,
                                         int64_t ld, uint32_t* sample_em, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(R) * E * S;
  dist_sample_transpose_kernel<<<grid_for(total, 256), 256, 0, s>>>(gathered, R, S, E, ld, sample_em);
  return cudaGetLastError();
}

cudaError_t launch_dist_rank(const uint32_t* counts, int32_t E, int64_t m, int64_t* rank,
                             uint32_t* flag, cudaStream_t s) {
  dist_rank_kernel<<<(E + 255) / 256, 256, 0, s>>>(counts, E, m, rank, flag);
  return cudaGetLastError();
}

cudaError_t launch_dist_cand_hist(const uint32_t* cand, const uint32_t* counts, int64_t cap,
                                  int32_t E, int32_t pass, const uint32_t* prefix, uint32_t* hist,
                                  cudaStream_t s) {
  dist_cand_hist_kernel<<<E, kCandHistThreads, 0, s>>>(cand, counts, cap, E, pass, prefix, hist);
  return cudaGetLastError();
}

namespace {
// Rounding to bf16 (to nearest, ties to even) is monotone, so the (m+1)-th
// largest of the rounded column is the rounding of the (m+1)-th largest fp32
// value: v16 = bf16(v32), exactly.
__global__ void round_bf16_kernel(const float* __restrict__ v32, int E, float* __restrict__ v16) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) v16[e] = __bfloat162float(__float2bfloat16_rn(v32[e]));
}
}  // namespace

size_t eqb_bf16_ws_bytes(int64_t N, int32_t E, int32_t K) {
  return eqb_layout(N, E, K).total + ((sizeof(float) * 2 * static_cast<size_t>(E) + 255) & ~static_cast<size_t>(255));
}

// One GPU: the exact fp32 quantile (one bracketed read of Z), rounded to
// bf16, then the bias update.  Across ranks, the pages' two-pass histogram
// exchange above is the form that works (kolibri_eqb_bf16_*).
cudaError_t launch_eqb_bf16(const float* z, const float* alpha, float* bias, int64_t N, int32_t E,
                            int32_t K, float* quantiles, void* ws, cudaStream_t s) {
  char* p = static_cast<char*>(ws);
  float* v32 = reinterpret_cast<float*>(p + eqb_layout(N, E, K).total);
  float* v16 = v32 + E;
  // the fp32 update writes its quantiles to v32; its bias output is discarded
  // (bias is overwritten below), so pass a scratch copy target: v16 serves
  cudaError_t err = cudaMemcpyAsync(v16, bias, sizeof(float) * E, cudaMemcpyDeviceToDevice, s);
  if (err != cudaSuccess) return err;
  if ((err = launch_eqb(z, alpha, v16, N, E, K, v32, ws, s)) != cudaSuccess) return err;
  round_bf16_kernel<<<(E + 255) / 256, 256, 0, s>>>(v32, E, v16);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  return launch_bias_update(v16, E, bias, quantiles, s);
}

cudaError_t launch_lei_inject(const int32_t* counts, int64_t N, int32_t E, int32_t K, double lambda,
                              double tau, float* g, cudaStream_t s) {
  const int grid = grid_for(N * static_cast<int64_t>(E) / 4, kLeiThreads);
  lei_inject_kernel<<<grid, kLeiThreads, 0, s>>>(counts, N, E, K, lambda, tau, g);
  return cudaGetLastError();
}

cudaError_t launch_score_grad(const float* z, const float* gs, int64_t n, float* gz, cudaStream_t s) {
  const bool vec = ((reinterpret_cast<uintptr_t>(z) | reinterpret_cast<uintptr_t>(gs) |
                     reinterpret_cast<uintptr_t>(gz)) & 15u) == 0u;
  if (vec && n >= 4) {
    const int64_t n4 = n / 4;
    const int tail = static_cast<int>(n - 4 * n4);
    score_grad_vec_kernel<<<grid_for(n4, kLeiThreads), kLeiThreads, 0, s>>>(
        reinterpret_cast<const float4*>(z), reinterpret_cast<const float4*>(gs), n4, reinterpret_cast<float4*>(gz),
        z + 4 * n4, gs + 4 * n4, tail, gz + 4 * n4);
    return cudaGetLastError();
  }
  score_grad_kernel<<<grid_for(n, kLeiThreads), kLeiThreads, 0, s>>>(z, gs, n, gz);
  return cudaGetLastError();
}

cudaError_t launch_intervention(const float* z, const int32_t* ids, int64_t N, int32_t E, int32_t K,
                                unsigned long long* total, double* rate, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(total, 0, sizeof(unsigned long long), s);
  if (err != cudaSuccess) return err;
  if (seg_overlap_applies(N, E, K)) {
    if ((err = launch_seg_overlap(z, ids, N, E, K, total, s)) != cudaSuccess) return err;
    intervention_finish_kernel<<<1, 1, 0, s>>>(total, N, K, rate);
    return cudaGetLastError();
  }
  const bool full = (E % 128) == 0;
  const unsigned grid = static_cast<unsigned>(grid_for((N + 7) / 8, 1));
#define KOLIBRI_OVL(Q)                                                              \
  if (full) overlap_kernel<Q, true><<<grid, 256, 0, s>>>(z, ids, N, E, K, total);  \
  else overlap_kernel<Q, false><<<grid, 256, 0, s>>>(z, ids, N, E, K, total);
  switch ((E + 127) / 128) {
    case 1: KOLIBRI_OVL(1) break;
    case 2: KOLIBRI_OVL(2) break;
    case 3: KOLIBRI_OVL(3) break;
    case 4: KOLIBRI_OVL(4) break;
    default: return cudaErrorInvalidValue;
  }
#undef KOLIBRI_OVL
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  intervention_finish_kernel<<<1, 1, 0, s>>>(total, N, K, rate);
  return cudaGetLastError();
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_balance)

}  // namespace kolibri
