// route.cu -- row-wise kernels over the logits Z [N, E] fp32:
//   * selection: bias add, top-K ids, sigmoid gates, token bias alpha
//     ("Kolibri Pre-Training from Scratch" 6.1 and 7.1; "Kolibri 1 im
//     Detail", routing steps 1-2);
//   * the two row passes of the exact EQB quantile (7.1, 7.3): the keys of
//     Z + alpha at sampled rows, and the full pass that counts keys above a
//     per-expert bracket and gathers the keys inside it.
//
// One warp per row; rows are HBM-streamed once with 512-byte warp loads.
#include "launch.h"
#include "route.cuh"

namespace kolibri {

namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / kWarp;

struct RouteArgs {
  const float* z;
  const float* beta;  // may be null
  int64_t N;
  int E, K;
  int32_t* ids;
  float* gates;
  float* alpha_out;
  const float* alpha_in;
  // bracketed full pass
  const uint32_t* lo;
  const uint32_t* hi;
  uint32_t* above;
  uint32_t* cand_cnt;
  uint32_t* cand;
  int64_t cap;
};

template <int Q>
__device__ __forceinline__ void load_lane_vec(const float* __restrict__ p, int E, int lane,
                                              float (&v)[4 * Q]) {
  load_row<Q>(p, E, lane, v);
}

template <int Q>
__device__ __forceinline__ void load_lane_u32(const uint32_t* __restrict__ p, int E, int lane,
                                              uint32_t (&v)[4 * Q]) {
#pragma unroll
  for (int q = 0; q < Q; ++q) {
    int e0 = 128 * q + 4 * lane;
    uint4 t = make_uint4(0u, 0u, 0u, 0u);
    if (e0 < E) t = __ldg(reinterpret_cast<const uint4*>(p + e0));
    v[4 * q + 0] = t.x;
    v[4 * q + 1] = t.y;
    v[4 * q + 2] = t.z;
    v[4 * q + 3] = t.w;
  }
}

// kRoute: write ids/gates.  kAlphaOut: write alpha.  kAlphaIn: read alpha
// instead of selecting (only without kRoute).  kWindow: bracketed pass.
template <int Q, bool kRoute, bool kAlphaOut, bool kAlphaIn, bool kWindow>
__global__ void __launch_bounds__(kRouteThreads) route_rows_kernel(const RouteArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * kRouteWarps + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kRouteWarps;
  const int E = a.E, K = a.K;

  float beta_l[4 * Q];
  const bool has_bias = a.beta != nullptr;
  if (has_bias) load_lane_vec<Q>(a.beta, E, lane, beta_l);
  else {
#pragma unroll
    for (int j = 0; j < 4 * Q; ++j) beta_l[j] = 0.f;
  }
  uint32_t lo_l[4 * Q], hi_l[4 * Q], above_l[4 * Q];
  if constexpr (kWindow) {
    load_lane_u32<Q>(a.lo, E, lane, lo_l);
    load_lane_u32<Q>(a.hi, E, lane, hi_l);
#pragma unroll
    for (int j = 0; j < 4 * Q; ++j) above_l[j] = 0u;
  }

  for (int64_t row = warp0; row < a.N; row += nwarps) {
    const float* zrow = a.z + row * E;
    float z[4 * Q];
    load_row<Q>(zrow, E, lane, z);
    float alpha = 0.f;
    if constexpr (!kAlphaIn) {
      uint32_t key[4 * Q];
      row_keys<Q>(z, beta_l, has_bias, E, lane, key);
      uint32_t out_key, out_id;
      warp_topk<Q>(key, K, lane, out_key, out_id);
      if constexpr (kRoute) {
        if (lane < K) {
          float zs = __ldg(zrow + out_id);
          a.ids[row * K + lane] = static_cast<int32_t>(out_id);
          a.gates[row * K + lane] = gate_sigmoid(zs);
        }
      }
      uint32_t kk = __shfl_sync(0xffffffffu, out_key, K);
      alpha = -key_to_float(kk);
      if constexpr (kAlphaOut) {
        if (lane == 0) a.alpha_out[row] = alpha;
      }
    } else {
      alpha = __ldg(a.alpha_in + row);
    }
    if constexpr (kWindow) {
#pragma unroll
      for (int j = 0; j < 4 * Q; ++j) {
        int e = static_cast<int>(slot_expert(lane, j));
        if (e < E) {
          uint32_t k = order_key(__fadd_rn(z[j], alpha));
          if (k > hi_l[j]) {
            above_l[j] += 1u;
          } else if (k >= lo_l[j]) {
            uint32_t pos = atomicAdd(a.cand_cnt + e, 1u);
            if (pos < a.cap) a.cand[static_cast<int64_t>(e) * a.cap + pos] = k;
          }
        }
      }
    }
  }
  if constexpr (kWindow) {
#pragma unroll
    for (int j = 0; j < 4 * Q; ++j) {
      int e = static_cast<int>(slot_expert(lane, j));
      if (e < E && above_l[j] != 0u) atomicAdd(a.above + e, above_l[j]);
    }
  }
}

// Keys of Z + alpha at sampled rows t = s * stride, written expert-major:
// sample[e * S + s].  A block handles 32 consecutive samples and transposes
// them through shared memory so every expert row is written in 128-byte runs.
constexpr int kSampleRows = 32;

template <int Q, bool kAlphaIn>
__global__ void __launch_bounds__(kRouteThreads) sample_keys_kernel(
    const float* __restrict__ z, const float* __restrict__ alpha_in, const float* __restrict__ beta,
    int64_t N, int E, int K, int64_t S, int64_t stride, uint32_t* __restrict__ sample) {
  extern __shared__ uint32_t tile[];  // [kSampleRows][E + 1]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t s0 = static_cast<int64_t>(blockIdx.x) * kSampleRows;
  const int ld = E + 1;

  float beta_l[4 * Q];
  const bool has_bias = beta != nullptr;
  if (has_bias) load_row<Q>(beta, E, lane, beta_l);
  else {
#pragma unroll
    for (int j = 0; j < 4 * Q; ++j) beta_l[j] = 0.f;
  }

  for (int r = warp; r < kSampleRows; r += kRouteWarps) {
    int64_t s = s0 + r;
    if (s >= S) break;
    int64_t row = s * stride;
    const float* zrow = z + row * E;
    float zv[4 * Q];
    load_row<Q>(zrow, E, lane, zv);
    float alpha;
    if constexpr (kAlphaIn) {
      alpha = __ldg(alpha_in + row);
    } else {
      uint32_t key[4 * Q];
      row_keys<Q>(zv, beta_l, has_bias, E, lane, key);
      uint32_t out_key, out_id;
      warp_topk<Q>(key, K, lane, out_key, out_id);
      alpha = -key_to_float(__shfl_sync(0xffffffffu, out_key, K));
    }
#pragma unroll
    for (int j = 0; j < 4 * Q; ++j) {
      int e = static_cast<int>(slot_expert(lane, j));
      if (e < E) tile[r * ld + e] = order_key(__fadd_rn(zv[j], alpha));
    }
  }
  __syncthreads();
  const int64_t rows_here = (S - s0) < kSampleRows ? (S - s0) : kSampleRows;
  for (int i = threadIdx.x; i < E * kSampleRows; i += blockDim.x) {
    int e = i / kSampleRows, r = i % kSampleRows;
    if (r < rows_here) sample[static_cast<int64_t>(e) * S + s0 + r] = tile[r * ld + e];
  }
}

template <int Q>
cudaError_t launch_route_q(const RouteArgs& a, bool route, bool alpha_out, bool alpha_in,
                           bool window, cudaStream_t s) {
  int64_t warps_needed = a.N;
  int sms = device_sm_count();
  int64_t blocks = (warps_needed + kRouteWarps - 1) / kRouteWarps;
  int64_t cap_blocks = static_cast<int64_t>(sms) * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  if (blocks < 1) blocks = 1;
  dim3 grid(static_cast<unsigned>(blocks)), block(kRouteThreads);
  if (route && alpha_out && !window)
    route_rows_kernel<Q, true, true, false, false><<<grid, block, 0, s>>>(a);
  else if (route && !alpha_out && !window)
    route_rows_kernel<Q, true, false, false, false><<<grid, block, 0, s>>>(a);
  else if (route && alpha_out && window)
    route_rows_kernel<Q, true, true, false, true><<<grid, block, 0, s>>>(a);
  else if (!route && alpha_in && window)
    route_rows_kernel<Q, false, false, true, true><<<grid, block, 0, s>>>(a);
  else if (!route && !alpha_in && window && alpha_out)
    route_rows_kernel<Q, false, true, false, true><<<grid, block, 0, s>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& a, bool route, bool alpha_out, bool alpha_in,
                         bool window, cudaStream_t s) {
  int Q = (a.E + 127) / 128;
  switch (Q) {
    case 1: return launch_route_q<1>(a, route, alpha_out, alpha_in, window, s);
    case 2: return launch_route_q<2>(a, route, alpha_out, alpha_in, window, s);
    case 3: return launch_route_q<3>(a, route, alpha_out, alpha_in, window, s);
    case 4: return launch_route_q<4>(a, route, alpha_out, alpha_in, window, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int Q>
cudaError_t launch_sample_q(const float* z, const float* alpha, const float* bias, int64_t N,
                            int E, int K, int64_t S, int64_t stride, uint32_t* sample,
                            cudaStream_t s) {
  size_t smem = sizeof(uint32_t) * kSampleRows * (E + 1);
  dim3 grid(static_cast<unsigned>((S + kSampleRows - 1) / kSampleRows)), block(kRouteThreads);
  if (alpha) {
    auto k = sample_keys_kernel<Q, true>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k<<<grid, block, smem, s>>>(z, alpha, bias, N, E, K, S, stride, sample);
  } else {
    auto k = sample_keys_kernel<Q, false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k<<<grid, block, smem, s>>>(z, alpha, bias, N, E, K, S, stride, sample);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk(const float* z, const float* bias, int64_t N, int32_t E, int32_t K,
                        int32_t* ids, float* gates, float* alpha, cudaStream_t s) {
  RouteArgs a{};
  a.z = z;
  a.beta = bias;
  a.N = N;
  a.E = E;
  a.K = K;
  a.ids = ids;
  a.gates = gates;
  a.alpha_out = alpha;
  return launch_route(a, true, alpha != nullptr, false, false, s);
}

cudaError_t launch_eqb_sample(const float* z, const float* alpha, const float* bias, int64_t N,
                              int32_t E, int32_t K, int64_t S, int64_t stride, uint32_t* sample,
                              cudaStream_t s) {
  int Q = (E + 127) / 128;
  switch (Q) {
    case 1: return launch_sample_q<1>(z, alpha, bias, N, E, K, S, stride, sample, s);
    case 2: return launch_sample_q<2>(z, alpha, bias, N, E, K, S, stride, sample, s);
    case 3: return launch_sample_q<3>(z, alpha, bias, N, E, K, S, stride, sample, s);
    case 4: return launch_sample_q<4>(z, alpha, bias, N, E, K, S, stride, sample, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_eqb_window_pass(const float* z, const float* alpha_in, const float* bias,
                                   float* alpha_out, int64_t N, int32_t E, int32_t K,
                                   const uint32_t* lo, const uint32_t* hi, uint32_t* above,
                                   uint32_t* cnt, uint32_t* cand, int64_t cap, cudaStream_t s) {
  RouteArgs a{};
  a.z = z;
  a.beta = bias;
  a.N = N;
  a.E = E;
  a.K = K;
  a.alpha_in = alpha_in;
  a.alpha_out = alpha_out;
  a.lo = lo;
  a.hi = hi;
  a.above = above;
  a.cand_cnt = cnt;
  a.cand = cand;
  a.cap = cap;
  if (alpha_in) return launch_route(a, false, false, true, true, s);
  return launch_route(a, false, true, false, true, s);
}

}  // namespace kolibri
