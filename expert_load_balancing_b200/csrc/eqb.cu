// eqb.cu -- Exact Quantile Balancing update on one GPU.
//
// Method ("Kolibri Pre-Training from Scratch", 7.1 update rule, 7.2 order
// of operations, 7.3 exact quantile by radix selection):
//   v_e    = Q_m(Z_:,e + alpha)        (m+1)-th largest, m = floor(N K / E)
//   beta_e = -v_e - mean_e'(-v_e')      (centred)
//
// The pages select the exact order statistic with radix passes whose digit
// histograms are summed over ranks.  On one B200 the column lives in one HBM,
// so the design reads Z once instead of once per digit:
//   1. keys of Z + alpha at S strided sample rows (S = N for N <= 16384:
//      then the sample IS the column and step 3 selects v directly);
//   2. per expert, two sample order statistics bracket the target rank with
//      a margin of six binomial standard deviations;
//   3. one full pass counts the keys above the bracket and gathers the keys
//      inside it;
//   4. per expert, the target is inside the bracket iff
//      above <= m < above + inside; then v is the (m - above)-th largest
//      gathered key, found by radix selection (11-bit digits, shared-memory
//      histograms, scanned from the top bin as on the pages);
//   5. any expert whose bracket missed (or overflowed the gather buffer)
//      falls back to radix selection over its whole column.
// Every path returns the exact order statistic; the bracket only decides
// how much of the column the radix passes must look at.
#include <cmath>

#include "launch.h"
#include "common.cuh"
#include "pdl.cuh"

namespace kolibri {

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kMaxRanks = 2;
constexpr int kHistWords = 2048;   // one 11-bit histogram, or two 10-bit ones

// Digit width of a selection of R ranks: the R histograms share kHistWords.
template <int R>
struct Digits {
  static constexpr int kBits = R == 1 ? 11 : 10;
  static constexpr int kBins = 1 << kBits;
  static_assert(R * kBins <= kHistWords, "histograms exceed their shared region");
  static_assert(kBins % kSelThreads == 0, "whole bins per thread");
};

struct SelectSmem {
  uint32_t hist[kHistWords];
  uint32_t wsum[kMaxRanks][kSelWarps];
  uint32_t red_min[kSelWarps];
  uint32_t red_max[kSelWarps];
  uint32_t bcast[2 + 2 * kMaxRanks];
};

// Block-wide minimum and maximum of the per-thread values (all threads).
__device__ __forceinline__ void block_minmax(uint32_t& mn, uint32_t& mx, SelectSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) {
    sm.red_min[warp] = mn;
    sm.red_max[warp] = mx;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = lane < kSelWarps ? sm.red_min[lane] : 0xffffffffu;
    uint32_t b = lane < kSelWarps ? sm.red_max[lane] : 0u;
    a = __reduce_min_sync(0xffffffffu, a);
    b = __reduce_max_sync(0xffffffffu, b);
    if (lane == 0) {
      sm.bcast[0] = a;
      sm.bcast[1] = b;
    }
  }
  __syncthreads();
  mn = sm.bcast[0];
  mx = sm.bcast[1];
  __syncthreads();
}

// Exact (rank[i]+1)-th largest keys of {key_at(j) : j < n}, rank[i] < n, for
// R ranks at once, given the block-wide minimum and maximum key.  Bits
// common to the minimum and maximum are skipped; the rest are resolved most
// significant first, one digit per pass over the keys.  Each rank follows
// its own prefix: ranks whose prefixes still agree share one histogram, so
// the passes serve all ranks.  Per pass: a shared-memory histogram of the
// digit of the keys that match the prefix, then a block-wide scan of the
// bins from the top (largest keys first) finds the bin holding the rank.
// Every thread of the block (kSelThreads) must call it; out[] is returned
// to all of them.  With max_passes, it stops after that many digits: out[i]
// then holds the resolved high bits with zeros below, and *unresolved the
// number of low bits left open (the rank's key lies in [out, out | 2^u - 1]).
template <int R, class KeyAt>
__device__ void block_select_ranks(KeyAt key_at, int64_t n, const int64_t (&rank)[R],
                                   uint32_t mn, uint32_t mx, uint32_t (&out)[R], SelectSmem& sm,
                                   int max_passes = 1 << 30, int* unresolved = nullptr) {
  using D = Digits<R>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (unresolved != nullptr) *unresolved = 0;
  if (mn == mx) {
#pragma unroll
    for (int i = 0; i < R; ++i) out[i] = mn;
    return;
  }
  int bits_left = 32 - __clz(static_cast<int>(mn ^ mx));  // lowest bits that still differ
  uint32_t prefix[R];
  int64_t r[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    prefix[i] = (bits_left == 32) ? 0u : (mx & ~((1u << bits_left) - 1u));
    r[i] = rank[i];
  }
  for (int pass = 0; bits_left > 0 && pass < max_passes; ++pass) {
    const int nb = bits_left < D::kBits ? bits_left : D::kBits;
    const int shift = bits_left - nb;
    const int nbins = 1 << nb;
    const uint32_t hi_mask = (shift + nb >= 32) ? 0u : (0xffffffffu << (shift + nb));
    // histogram h serves rank h; rank 1 reuses histogram 0 while the
    // prefixes agree
    const bool split = R > 1 && (prefix[R - 1] & hi_mask) != (prefix[0] & hi_mask);
    const int nh = split ? R : 1;
    for (int b = tid; b < nh * D::kBins; b += kSelThreads) sm.hist[b] = 0u;
    __syncthreads();
    const uint32_t p0 = prefix[0] & hi_mask, p1 = prefix[R - 1] & hi_mask;
    for (int64_t j = tid; j < n; j += kSelThreads) {
      const uint32_t k = key_at(j);
      const uint32_t kh = k & hi_mask, bin = (k >> shift) & static_cast<uint32_t>(nbins - 1);
      if (kh == p0) atomicAdd(&sm.hist[bin], 1u);
      else if (split && kh == p1) atomicAdd(&sm.hist[D::kBins + bin], 1u);
    }
    __syncthreads();
    // scan from the top: thread t owns bins top - t*per - q, q < per
    const int per = nbins >= kSelThreads ? nbins / kSelThreads : 1;
    const int top = nbins - 1 - tid * per;
    uint32_t part[R], incl[R];
#pragma unroll
    for (int h = 0; h < R; ++h) {
      part[h] = 0u;
      if (h < nh) {
        for (int q = 0; q < per; ++q)
          if (top - q >= 0) part[h] += sm.hist[h * D::kBins + top - q];
      }
      incl[h] = part[h];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
      for (int h = 0; h < R; ++h) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl[h], o);
        if (lane >= o) incl[h] += t;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int h = 0; h < R; ++h) sm.wsum[h][warp] = incl[h];
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < R; ++h) {
      uint32_t wb = 0u;
      for (int w = 0; w < warp; ++w) wb += sm.wsum[h][w];
      const uint32_t ex = wb + incl[h] - part[h];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int hi = split ? i : 0;
        if (hi != h) continue;
        if (part[h] != 0u && static_cast<int64_t>(ex) <= r[i] &&
            r[i] < static_cast<int64_t>(ex) + part[h]) {
          int64_t rr = r[i] - ex;
          int b = top;
          for (int q = 0; q < per; ++q, --b) {
            const uint32_t c = sm.hist[h * D::kBins + b];
            if (rr < static_cast<int64_t>(c)) break;
            rr -= c;
          }
          sm.bcast[2 + 2 * i] = static_cast<uint32_t>(b);
          sm.bcast[3 + 2 * i] = static_cast<uint32_t>(rr);
        }
      }
    }
    __syncthreads();
    // (unsplit prefixes are equal: both hold only bits above this digit)
#pragma unroll
    for (int i = 0; i < R; ++i) {
      prefix[i] |= sm.bcast[2 + 2 * i] << shift;
      r[i] = sm.bcast[3 + 2 * i];
    }
    bits_left = shift;
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < R; ++i) out[i] = prefix[i];
  if (unresolved != nullptr) *unresolved = bits_left;
}

// Keys of one expert staged in shared memory when they fit (kSmemKeys),
// otherwise read from global memory (L2) on every pass.  Either way the
// block-wide minimum and maximum key come back in mn / mx.
constexpr int kSmemKeys = 16384;

__device__ __forceinline__ void stage_keys(const uint32_t* __restrict__ keys, int64_t n,
                                           uint32_t* keys_s, uint32_t& mn, uint32_t& mx,
                                           SelectSmem& sm) {
  mn = 0xffffffffu;
  mx = 0u;
  const bool to_smem = n <= kSmemKeys;
  // 16-byte vector loads only from a 16-byte aligned source
  const bool vec = (reinterpret_cast<uintptr_t>(keys) & 15u) == 0u;
  const int64_t n4 = vec ? (n & ~static_cast<int64_t>(3)) : 0;
  for (int64_t i = 4 * threadIdx.x; i < n4; i += 4 * kSelThreads) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(keys + i));
    if (to_smem) *reinterpret_cast<uint4*>(keys_s + i) = v;
    mn = min(min(mn, v.x), min(v.y, min(v.z, v.w)));
    mx = max(max(mx, v.x), max(v.y, max(v.z, v.w)));
  }
  for (int64_t i = n4 + threadIdx.x; i < n; i += kSelThreads) {
    const uint32_t v = __ldg(keys + i);
    if (to_smem) keys_s[i] = v;
    mn = min(mn, v);
    mx = max(mx, v);
  }
  block_minmax(mn, mx, sm);   // its barriers also publish keys_s
}

// a5 by the last block of an update's final grid: beta = -v, centred, with
// the arithmetic of bias_update_kernel (fp64 sum in ascending expert order by
// one thread, mean rounded once to fp32, subtraction in fp32).  Every block
// calls it after thread 0 wrote its v[e]; each makes that write visible
// (fence) and takes a ticket; the block drawing the last ticket reads all E
// values and updates the bias, then puts the ticket back to zero.  No block
// waits for another.  The ticket must be zero when the grid starts.
__device__ void bias_by_last_block(const float* v, int E, uint32_t* ticket, float* bias,
                                   float* quantiles, SelectSmem& sm) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    sm.bcast[0] = (atomicAdd(ticket, 1u) == gridDim.x - 1u) ? 1u : 0u;
  }
  __syncthreads();
  if (sm.bcast[0] == 0u) return;
  __threadfence();
  float* v_s = reinterpret_cast<float*>(sm.hist);       // E <= 512 < kHistWords
  for (int e = threadIdx.x; e < E; e += kSelThreads) v_s[e] = __ldcg(v + e);
  __syncthreads();
  if (threadIdx.x == 0) {
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum = __dadd_rn(sum, static_cast<double>(-v_s[e]));
    sm.red_min[0] = __float_as_uint(__double2float_rn(__ddiv_rn(sum, static_cast<double>(E))));
    *ticket = 0u;
  }
  __syncthreads();
  const float mean = __uint_as_float(sm.red_min[0]);
  for (int e = threadIdx.x; e < E; e += kSelThreads) {
    const float ve = v_s[e];
    bias[e] = __fsub_rn(-ve, mean);
    if (quantiles) quantiles[e] = ve;
  }
}

// Step 2 (or the whole selection when the sample is the column).
// The bracket path also clears this expert's counters of the full pass
// (clear non-null: above, cnt, flag).
__global__ void __launch_bounds__(kSelThreads) sample_select_kernel(
    const uint32_t* __restrict__ sample, int64_t S, int64_t m_exact, int64_t r_hi, int64_t r_lo,
    int64_t S_ld, bool exact, float* __restrict__ v, uint32_t* __restrict__ lo,
    uint32_t* __restrict__ hi, uint32_t* __restrict__ clear_above, uint32_t* __restrict__ clear_cnt,
    uint32_t* __restrict__ clear_flag, uint32_t* __restrict__ ticket, float* __restrict__ bias,
    float* __restrict__ quantiles) {
  __shared__ SelectSmem sm;
  extern __shared__ __align__(16) uint32_t keys_s[];
  const int e = blockIdx.x;
  pdl_wait();       // the sample comes from the kernel before this one
  pdl_trigger();
  if (clear_above != nullptr && threadIdx.x == 0) {
    clear_above[e] = 0u;
    clear_cnt[e] = 0u;
    clear_flag[e] = 0u;
  }
  const uint32_t* keys = sample + static_cast<int64_t>(e) * S_ld;
  uint32_t mn, mx;
  stage_keys(keys, S, keys_s, mn, mx, sm);
  const bool in_smem = S <= kSmemKeys;
  auto at = [keys, in_smem](int64_t i) {
    extern __shared__ __align__(16) uint32_t ks[];
    return in_smem ? ks[i] : __ldg(keys + i);
  };
  if (exact) {
    const int64_t rk[1] = {m_exact};
    uint32_t k[1];
    block_select_ranks<1>(at, S, rk, mn, mx, k, sm);
    if (threadIdx.x == 0) v[e] = key_to_float(k[0]);
    // ticket given: this grid also ends the update (bias from all v)
    if (ticket != nullptr) bias_by_last_block(v, static_cast<int>(gridDim.x), ticket, bias, quantiles, sm);
  } else {
    // both bracket ranks in the same passes (r_hi <= r_lo), two digits deep:
    // the bracket only has to contain the two sample keys, so it takes the
    // outer edges of their bins (at 20 resolved bits a bin holds a few keys
    // of the column near the target; the counts decide exactness)
    const int64_t rk[2] = {r_hi, r_lo};
    uint32_t k[2];
    int open_bits = 0;
    block_select_ranks<2>(at, S, rk, mn, mx, k, sm, 2, &open_bits);
    if (threadIdx.x == 0) {
      // widened bounds stay within [key(-inf), key(+inf)] when the keys were,
      // so the pass may compare them as floats
      constexpr uint32_t kKeyNegInf = 0x007fffffu, kKeyPosInf = 0xff800000u;
      const uint32_t low = open_bits >= 32 ? 0xffffffffu : ((1u << open_bits) - 1u);
      uint32_t h = k[0] | low, l = k[1];
      if (k[0] <= kKeyPosInf && h > kKeyPosInf) h = kKeyPosInf;
      if (l < kKeyNegInf && (k[1] | low) >= kKeyNegInf) l = kKeyNegInf;
      hi[e] = h;
      lo[e] = l;
    }
  }
}

// Steps 4-5 and a5 in one grid, one block per expert.  If the target lies
// inside the expert's bracket (above <= m < above + inside, and the gather
// did not overflow), v is the (m - above)-th largest gathered key; otherwise
// the block selects over the whole column of Z + alpha.  The block drawing
// the last ticket then updates the bias.
__global__ void __launch_bounds__(kSelThreads) bracket_finish_kernel(
    const uint32_t* __restrict__ cand, const uint32_t* __restrict__ cnt,
    const uint32_t* __restrict__ above, int64_t cap, int64_t m, const float* __restrict__ z,
    const float* __restrict__ alpha, int64_t N, float* __restrict__ v, uint32_t* __restrict__ ticket,
    float* __restrict__ bias, float* __restrict__ quantiles) {
  __shared__ SelectSmem sm;
  extern __shared__ __align__(16) uint32_t keys_s[];
  const int e = blockIdx.x;
  const int E = static_cast<int>(gridDim.x);
  pdl_wait();       // counts and gathered keys come from the full pass
  pdl_trigger();
  const int64_t c = cnt[e], ab = above[e];
  const bool ok = c <= cap && ab <= m && m < ab + c;
  uint32_t k[1];
  if (ok) {
    const uint32_t* keys = cand + static_cast<int64_t>(e) * cap;
    uint32_t mn, mx;
    stage_keys(keys, c, keys_s, mn, mx, sm);
    const bool in_smem = c <= kSmemKeys;
    auto at = [keys, in_smem](int64_t i) {
      extern __shared__ __align__(16) uint32_t ks[];
      return in_smem ? ks[i] : __ldg(keys + i);
    };
    const int64_t rk[1] = {m - ab};
    block_select_ranks<1>(at, c, rk, mn, mx, k, sm);
  } else {
    // the bracket missed (or its gather overflowed): the whole column
    auto at = [z, alpha, E, e](int64_t t) {
      return order_key(__fadd_rn(__ldg(z + t * E + e), __ldg(alpha + t)));
    };
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (int64_t t = threadIdx.x; t < N; t += kSelThreads) {
      const uint32_t kk = at(t);
      mn = min(mn, kk);
      mx = max(mx, kk);
    }
    block_minmax(mn, mx, sm);
    const int64_t rk[1] = {m};
    block_select_ranks<1>(at, N, rk, mn, mx, k, sm);
  }
  if (threadIdx.x == 0) v[e] = key_to_float(k[0]);
  bias_by_last_block(v, E, ticket, bias, quantiles, sm);
}

// a5: beta = -v, centred.  fp64 sum in ascending expert order (one thread),
// mean rounded once to fp32, subtraction in fp32.
__global__ void bias_update_kernel(const float* __restrict__ v, int E, float* __restrict__ bias,
                                   float* __restrict__ quantiles) {
  __shared__ float mean_s;
  __shared__ float v_s[KOLIBRI_MAX_EXPERTS];
  pdl_wait();       // v comes from the kernels before this one
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) v_s[e] = v[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum = __dadd_rn(sum, static_cast<double>(-v_s[e]));
    mean_s = __double2float_rn(__ddiv_rn(sum, static_cast<double>(E)));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float ve = v[e];
    bias[e] = __fsub_rn(-ve, mean_s);
    if (quantiles) quantiles[e] = ve;
  }
}

}  // namespace

EqbLayout eqb_layout(int64_t N, int32_t E, int32_t K) {
  (void)K;
  EqbLayout L;
  L.exact_small = N <= kSampleMax;
  L.S = L.exact_small ? N : kSampleMax;
  L.stride = L.exact_small ? 1 : N / L.S;
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.S_ld = (L.S + 3) & ~static_cast<int64_t>(3);  // 16-byte aligned expert rows
  L.off_sample = take(sizeof(uint32_t) * static_cast<size_t>(E) * static_cast<size_t>(L.S_ld));
  L.off_lo = take(sizeof(uint32_t) * E);
  L.off_hi = take(sizeof(uint32_t) * E);
  L.off_above = take(sizeof(uint32_t) * E);
  L.off_cnt = take(sizeof(uint32_t) * E);
  L.off_flag = take(sizeof(uint32_t) * E);
  L.off_v = take(sizeof(float) * E);
  L.off_alpha = take(sizeof(float) * static_cast<size_t>(N));
  if (!L.exact_small)
    L.off_cand = take(sizeof(uint32_t) * static_cast<size_t>(E) * static_cast<size_t>(kCandCap));
  L.total = off;
  return L;
}

namespace {

size_t select_smem(int64_t n) {
  return sizeof(uint32_t) * static_cast<size_t>(n < kSmemKeys ? n : kSmemKeys);
}

cudaError_t set_select_smem() {
  const int bytes = static_cast<int>(sizeof(uint32_t) * kSmemKeys);
  cudaError_t err = cudaFuncSetAttribute(sample_select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) return err;
  return cudaFuncSetAttribute(bracket_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              bytes);
}

struct EqbBuffers {
  EqbLayout L;
  uint32_t *sample, *lo, *hi, *above, *cnt, *flag, *cand;
  float *v, *alpha_ws;
  char* base;
};

EqbBuffers eqb_buffers(int64_t N, int32_t E, int32_t K, void* ws) {
  EqbBuffers b;
  b.L = eqb_layout(N, E, K);
  b.base = static_cast<char*>(ws);
  auto u32 = [&b](size_t off) { return reinterpret_cast<uint32_t*>(b.base + off); };
  b.sample = u32(b.L.off_sample);
  b.lo = u32(b.L.off_lo);
  b.hi = u32(b.L.off_hi);
  b.above = u32(b.L.off_above);
  b.cnt = u32(b.L.off_cnt);
  b.flag = u32(b.L.off_flag);
  b.cand = b.L.exact_small ? nullptr : u32(b.L.off_cand);
  b.v = reinterpret_cast<float*>(b.base + b.L.off_v);
  b.alpha_ws = reinterpret_cast<float*>(b.base + b.L.off_alpha);
  return b;
}

// Step 2 from the sample keys: either the exact quantile and the bias update
// (small N: the sample is the column), or the per-expert bracket, with the
// full-pass counters cleared.
cudaError_t eqb_brackets(int64_t N, int32_t E, int32_t K, const EqbBuffers& b, float* bias,
                         float* quantiles, cudaStream_t s) {
  const EqbLayout& L = b.L;
  const int64_t m = (N * static_cast<int64_t>(K)) / E;
  cudaError_t err;
  if (L.exact_small) {
    err = set_select_smem();
    if (err != cudaSuccess) return err;
    return launch_pdl(sample_select_kernel, dim3(E), dim3(kSelThreads), select_smem(L.S), s, dim3(0, 0, 0),
                      b.sample, L.S, m, static_cast<int64_t>(0), static_cast<int64_t>(0), L.S_ld, true, b.v,
                      b.lo, b.hi, static_cast<uint32_t*>(nullptr), static_cast<uint32_t*>(nullptr),
                      static_cast<uint32_t*>(nullptr), b.flag, bias, quantiles);
  }
  // bracket ranks in the sample, descending order: the target sits at
  // about q*S with q = (m+1)/N; margin 6 binomial standard deviations
  const double q = static_cast<double>(m + 1) / static_cast<double>(N);
  const double center = q * static_cast<double>(L.S);
  const double sd = std::sqrt(center * (1.0 - q));
  const int64_t margin = static_cast<int64_t>(std::ceil(6.0 * sd)) + 8;
  int64_t r_hi = static_cast<int64_t>(std::floor(center)) - margin;
  int64_t r_lo = static_cast<int64_t>(std::ceil(center)) + margin;
  if (r_hi < 0) r_hi = 0;
  if (r_lo > L.S - 1) r_lo = L.S - 1;
  err = set_select_smem();
  if (err != cudaSuccess) return err;
  // the select also clears the full pass's counters (above, cnt, flag)
  return launch_pdl(sample_select_kernel, dim3(E), dim3(kSelThreads), select_smem(L.S), s, dim3(0, 0, 0),
                    b.sample, L.S, static_cast<int64_t>(0), r_hi, r_lo, L.S_ld, false, b.v, b.lo, b.hi,
                    b.above, b.cnt, b.flag, static_cast<uint32_t*>(nullptr), static_cast<float*>(nullptr),
                    static_cast<float*>(nullptr));
}

// Steps 1-2: sample keys (token bias given, or computed from the bias), then
// the brackets, or for small N the exact quantile and the bias update.  The
// word b.flag[0] is the ticket of the grid that ends the update: cleared
// by the sample kernel (small N) or by the sample select (the bracket path).
cudaError_t eqb_begin(const float* z, const float* alpha, float* bias, int64_t N, int32_t E,
                      int32_t K, float* quantiles, const EqbBuffers& b, cudaStream_t s) {
  const EqbLayout& L = b.L;
  cudaError_t err = launch_eqb_sample(z, alpha, alpha ? nullptr : bias, N, E, K, L.S, L.stride,
                                      L.S_ld, b.sample, s, L.exact_small ? b.flag : nullptr);
  if (err != cudaSuccess) return err;
  return eqb_brackets(N, E, K, b, bias, quantiles, s);
}

// Steps 4-5 and the bias update, in one grid (the bracket path; for small N
// eqb_begin already finished the update).
cudaError_t eqb_end(const float* z, const float* alpha_used, float* bias, int64_t N, int32_t E,
                    int32_t K, float* quantiles, const EqbBuffers& b, cudaStream_t s) {
  if (b.L.exact_small) return cudaSuccess;
  const int64_t m = (N * static_cast<int64_t>(K)) / E;
  const cudaError_t err = set_select_smem();
  if (err != cudaSuccess) return err;
  return launch_pdl(bracket_finish_kernel, dim3(E), dim3(kSelThreads), select_smem(kSmemKeys), s,
                    dim3(0, 0, 0), b.cand, b.cnt, b.above, static_cast<int64_t>(kCandCap), m, z, alpha_used, N,
                    b.v, b.flag, bias, quantiles);
}

}  // namespace

cudaError_t launch_bias_update(const float* v, int32_t E, float* bias, float* quantiles,
                               cudaStream_t s) {
  return launch_pdl(bias_update_kernel, dim3(1), dim3(512), 0, s, dim3(0, 0, 0), v, E, bias, quantiles);
}

cudaError_t launch_eqb(const float* z, const float* alpha, float* bias, int64_t N, int32_t E,
                       int32_t K, float* quantiles, void* ws, cudaStream_t s) {
  const EqbBuffers b = eqb_buffers(N, E, K, ws);
  cudaError_t err = eqb_begin(z, alpha, bias, N, E, K, quantiles, b, s);
  if (err != cudaSuccess) return err;
  const float* alpha_used = alpha;
  if (!b.L.exact_small) {
    // the full pass; it also derives alpha from bias_in when none is given
    err = launch_route_window_pass(z, bias, alpha, N, E, K, nullptr, nullptr,
                                   alpha ? nullptr : b.alpha_ws, b.lo, b.hi, b.above, b.cnt,
                                   b.cand, kCandCap, s);
    if (err != cudaSuccess) return err;
    if (!alpha) alpha_used = b.alpha_ws;
  }
  return eqb_end(z, alpha_used, bias, N, E, K, quantiles, b, s);
}

// Logits, routing and the EQB update from the tokens: the fused GEMM +
// selection, then the update from the alpha it wrote.  (Running the
// bracketed full pass inside the GEMM epilogue as well, from brackets taken
// first on a sampled-row GEMM, measured slower on B200: the epilogue is
// latency-bound and the separate pass streams Z near HBM speed.)
cudaError_t launch_forward_eqb(const void* x, const void* w, float* bias, float* z, int64_t N,
                               int32_t d, int32_t E, int32_t K, int32_t* ids, float* gates,
                               float* alpha, float* quantiles, void* ws, cudaStream_t s) {
  const EqbBuffers b = eqb_buffers(N, E, K, ws);
  float* alpha_out = alpha ? alpha : b.alpha_ws;
  const cudaError_t err = router_forward_by_size(x, w, bias, z, N, d, E, K, ids, gates, alpha_out, s);
  if (err != cudaSuccess) return err;
  return launch_eqb(z, alpha_out, bias, N, E, K, quantiles, ws, s);
}

cudaError_t launch_route_balance(const float* z, float* bias, int64_t N, int32_t E, int32_t K,
                                 int32_t* ids, float* gates, float* alpha, float* quantiles,
                                 void* ws, cudaStream_t s) {
  const EqbBuffers b = eqb_buffers(N, E, K, ws);
  float* alpha_out = alpha ? alpha : b.alpha_ws;
  cudaError_t err;
  if (b.L.exact_small) {
    // the sample is the whole column: route first, then select from its alpha
    err = launch_topk(z, bias, N, E, K, ids, gates, alpha_out, s);
    if (err != cudaSuccess) return err;
    err = eqb_begin(z, alpha_out, bias, N, E, K, quantiles, b, s);
    if (err != cudaSuccess) return err;
  } else {
    // Routing first (writes alpha), then the bracketed pass with alpha given.
    // Two streams over Z; a single fused pass measured slower on B200 (its
    // per-row dependency chain is longer than 24 warps per SM can hide).
    err = launch_topk(z, bias, N, E, K, ids, gates, alpha_out, s);
    if (err != cudaSuccess) return err;
    err = eqb_begin(z, alpha_out, bias, N, E, K, quantiles, b, s);
    if (err != cudaSuccess) return err;
    err = launch_route_window_pass(z, bias, alpha_out, N, E, K, nullptr, nullptr, nullptr, b.lo,
                                   b.hi, b.above, b.cnt, b.cand, kCandCap, s);
    if (err != cudaSuccess) return err;
  }
  return eqb_end(z, alpha_out, bias, N, E, K, quantiles, b, s);
}

KOLIBRI_DEFINE_STATUS_TAKE(status_take_eqb)

}  // namespace kolibri

namespace kolibri {

// Brackets of the EQB update over a batch split across ranks: the same
// sample selection as the one-GPU update, over the ranks' gathered samples
// laid out expert-major ([E][ld], n keys per expert, ld a multiple of 4).
cudaError_t launch_dist_brackets(const uint32_t* sample_em, int64_t n, int64_t ld, int32_t E,
                                 int64_t m, int64_t N_total, uint32_t* lo, uint32_t* hi,
                                 cudaStream_t s) {
  // sample ranks about q n with q = (m+1)/N_total, six binomial standard
  // deviations (plus a few keys) either side, as for one GPU
  const double q = static_cast<double>(m + 1) / static_cast<double>(N_total);
  const double center = q * static_cast<double>(n);
  const double sd = std::sqrt(center * (1.0 - q));
  const int64_t margin = static_cast<int64_t>(std::ceil(6.0 * sd)) + 8;
  int64_t r_hi = static_cast<int64_t>(std::floor(center)) - margin;
  int64_t r_lo = static_cast<int64_t>(std::ceil(center)) + margin;
  if (r_hi < 0) r_hi = 0;
  if (r_lo > n - 1) r_lo = n - 1;
  if (r_hi > r_lo) r_hi = r_lo;
  cudaError_t err = set_select_smem();
  if (err != cudaSuccess) return err;
  return launch_pdl(sample_select_kernel, dim3(E), dim3(kSelThreads), select_smem(n), s,
                    dim3(0, 0, 0), sample_em, n, static_cast<int64_t>(0), r_hi, r_lo, ld, false,
                    static_cast<float*>(nullptr), lo, hi, static_cast<uint32_t*>(nullptr),
                    static_cast<uint32_t*>(nullptr), static_cast<uint32_t*>(nullptr),
                    static_cast<uint32_t*>(nullptr), static_cast<float*>(nullptr), static_cast<float*>(nullptr));
}

}  // namespace kolibri
