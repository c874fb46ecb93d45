// api.cu -- the extern "C" boundary declared in include/kolibri_router.h:
// argument validation, workspace sizing and the device status word.
#include <cstdint>

#include "launch.h"
#include "common.cuh"

namespace kolibri {

KOLIBRI_DEFINE_STATUS_TAKE(status_take_api)

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0u; }

kolibri_status check_ek(int64_t N, int32_t E, int32_t K) {
  if (N < 1 || E < 1 || K < 1) return KOLIBRI_ERR_INVALID_ARG;
  if (K >= E) return KOLIBRI_ERR_INVALID_ARG;
  if (E > KOLIBRI_MAX_EXPERTS || K > KOLIBRI_MAX_TOPK || (E % 4) != 0)
    return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (N * static_cast<int64_t>(K) >= (static_cast<int64_t>(1) << 31))
    return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return KOLIBRI_OK;
}

kolibri_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KOLIBRI_OK : KOLIBRI_ERR_CUDA; }

// One warp waits, through the kernels' bounded wait, on a shared-memory
// barrier that nothing arrives at: the wait gives up after about limit_ns,
// records the timeout in the status word and the kernel returns.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) mbar_init(b, 1);
  __syncthreads();
  mbar_wait(b, 0u, limit_ns);
}

}  // namespace
}  // namespace kolibri

using namespace kolibri;

extern "C" {

const char* kolibri_status_string(kolibri_status s) {
  switch (s) {
    case KOLIBRI_OK: return "KOLIBRI_OK";
    case KOLIBRI_ERR_INVALID_ARG: return "KOLIBRI_ERR_INVALID_ARG";
    case KOLIBRI_ERR_UNSUPPORTED_SHAPE: return "KOLIBRI_ERR_UNSUPPORTED_SHAPE";
    case KOLIBRI_ERR_WORKSPACE_TOO_SMALL: return "KOLIBRI_ERR_WORKSPACE_TOO_SMALL";
    case KOLIBRI_ERR_CUDA: return "KOLIBRI_ERR_CUDA";
    case KOLIBRI_ERR_TIMEOUT: return "KOLIBRI_ERR_TIMEOUT";
    case KOLIBRI_ERR_DEVICE: return "KOLIBRI_ERR_DEVICE";
  }
  return "KOLIBRI_ERR_UNKNOWN";
}

size_t kolibri_workspace_bytes(int op, int64_t N, int32_t E, int32_t K) {
  if (check_ek(N, E, K) != KOLIBRI_OK) return 0;
  if (op == KOLIBRI_OP_PERMUTE) return permute_layout(N, E, K).total;
  if (op == KOLIBRI_OP_EQB) return eqb_layout(N, E, K).total;
  if (op == KOLIBRI_OP_EQB_BF16) return eqb_bf16_ws_bytes(N, E, K);
  return 0;
}

kolibri_status kolibri_router_logits(const void* x, const void* w, float* z, int64_t N, int32_t d,
                                     int32_t E, void* stream) {
  if (!x || !w || !z) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(z)) return KOLIBRI_ERR_INVALID_ARG;
  if (N < 1 || d < 1 || E < 1) return KOLIBRI_ERR_INVALID_ARG;
  if (d % 64 != 0 || E % 16 != 0 || E > KOLIBRI_MAX_EXPERTS) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (N >= (static_cast<int64_t>(1) << 31)) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_router_logits_by_size(x, w, z, N, d, E, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_router_forward(const void* x, const void* w, const float* bias, float* z,
                                      int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                      float* gates, float* alpha, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!x || !w || !z || !ids || !gates || !alpha) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(z) || (bias && !aligned16(bias)))
    return KOLIBRI_ERR_INVALID_ARG;
  if (d < 1) return KOLIBRI_ERR_INVALID_ARG;
  if (d % 64 != 0 || E % 16 != 0) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(router_forward_by_size(x, w, bias, z, N, d, E, K, ids, gates, alpha,
                                      static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_router_forward_permute(const void* x, const void* w, const float* bias,
                                              float* z, int64_t N, int32_t d, int32_t E, int32_t K,
                                              int32_t* ids, float* gates, float* alpha,
                                              int32_t* counts, int64_t* offsets, int32_t* perm,
                                              int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!x || !w || !z || !ids || !gates || !alpha || !counts || !offsets || !perm)
    return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(z) || (bias && !aligned16(bias)))
    return KOLIBRI_ERR_INVALID_ARG;
  if (d < 1) return KOLIBRI_ERR_INVALID_ARG;
  if (d % 64 != 0 || E % 16 != 0) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  const PermuteLayout L = permute_layout(N, E, K);
  if (!L.single_cta) {
    if (!ws) return KOLIBRI_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ws && aligned16(ws) && ws_bytes >= L.total && router_decode_ticket_supported(N, d, E, K)) {
    uint32_t* ticket = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + L.off_dec_ticket);
    const cudaError_t err = launch_router_decode_ticket(x, w, bias, z, N, d, E, K, ids, gates, alpha, counts,
                                                        offsets, perm, inv, ticket, s);
    if (err != cudaErrorNotSupported) return from_cuda(err);
  }
  if (router_decode_permutes(N, d, E, K)) {
    const cudaError_t err = launch_router_decode_permute(x, w, bias, z, N, d, E, K, ids, gates, alpha,
                                                         counts, offsets, perm, inv, s);
    if (err != cudaErrorNotSupported) return from_cuda(err);
  }
  cudaError_t err = router_forward_by_size(x, w, bias, z, N, d, E, K, ids, gates, alpha, s);
  if (err == cudaSuccess) err = launch_permute(ids, N, E, K, counts, offsets, perm, inv, ws, s);
  return from_cuda(err);
}

kolibri_status kolibri_router_forward_eqb(const void* x, const void* w, float* bias, float* z,
                                          int64_t N, int32_t d, int32_t E, int32_t K,
                                          int32_t* ids, float* gates, float* alpha,
                                          float* quantiles, void* ws, size_t ws_bytes,
                                          void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!x || !w || !bias || !z || !ids || !gates || !ws) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(z) || !aligned16(bias) || !aligned16(ws))
    return KOLIBRI_ERR_INVALID_ARG;
  if (d < 1) return KOLIBRI_ERR_INVALID_ARG;
  if (d % 64 != 0 || E % 16 != 0) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < eqb_layout(N, E, K).total) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_forward_eqb(x, w, bias, z, N, d, E, K, ids, gates, alpha, quantiles, ws,
                                      static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_router_topk(const float* z, const float* bias, int64_t N, int32_t E,
                                   int32_t K, int32_t* ids, float* gates, float* alpha,
                                   void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!z || !ids || !gates) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(z) || (bias && !aligned16(bias))) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(
      launch_topk(z, bias, N, E, K, ids, gates, alpha, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_expert_permute(const int32_t* ids, int64_t N, int32_t E, int32_t K,
                                      int32_t* counts, int64_t* offsets, int32_t* perm,
                                      int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!ids || !counts || !offsets || !perm) return KOLIBRI_ERR_INVALID_ARG;
  const PermuteLayout L = permute_layout(N, E, K);
  if (!L.single_cta) {
    if (!ws) return KOLIBRI_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  }
  return from_cuda(launch_permute(ids, N, E, K, counts, offsets, perm, inv, ws,
                                  static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_update(const float* z, const float* alpha, float* bias, int64_t N,
                                  int32_t E, int32_t K, float* quantiles, void* ws,
                                  size_t ws_bytes, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!z || !bias || !ws) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(bias) || !aligned16(ws)) return KOLIBRI_ERR_INVALID_ARG;
  if (ws_bytes < eqb_layout(N, E, K).total) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(
      launch_eqb(z, alpha, bias, N, E, K, quantiles, ws, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_route_and_balance(const float* z, float* bias, int64_t N, int32_t E,
                                         int32_t K, int32_t* ids, float* gates, float* alpha,
                                         float* quantiles, void* ws, size_t ws_bytes,
                                         void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!z || !bias || !ids || !gates || !ws) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(bias) || !aligned16(ws)) return KOLIBRI_ERR_INVALID_ARG;
  if (ws_bytes < eqb_layout(N, E, K).total) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_route_balance(z, bias, N, E, K, ids, gates, alpha, quantiles, ws,
                                        static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_update_bf16(const float* z, const float* alpha, float* bias, int64_t N,
                                       int32_t E, int32_t K, float* quantiles, void* ws,
                                       size_t ws_bytes, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!z || !bias || !ws) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(ws) || !aligned16(bias)) return KOLIBRI_ERR_INVALID_ARG;
  if (ws_bytes < eqb_bf16_ws_bytes(N, E, K)) return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_eqb_bf16(z, alpha, bias, N, E, K, quantiles, ws,
                                   static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_bf16_histogram(const float* z, const float* alpha, int64_t N, int32_t E,
                                          const uint32_t* prefix, uint32_t* hist, void* stream) {
  if (N < 1 || E < 4 || E > KOLIBRI_MAX_EXPERTS || (E % 4) != 0)
    return N < 1 ? KOLIBRI_ERR_INVALID_ARG : KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!z || !hist || !aligned16(z)) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_bf16_hist(z, alpha, N, E, prefix, hist, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_bf16_digit(const uint32_t* hist, int32_t E, int64_t* rank,
                                      uint32_t* digit, void* stream) {
  if (E < 1 || E > KOLIBRI_MAX_EXPERTS) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!hist || !rank || !digit) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_bf16_digit(hist, E, rank, digit, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_bf16_bias(const uint32_t* digit_hi, const uint32_t* digit_lo, int32_t E,
                                     float* bias, float* quantiles, void* stream) {
  if (E < 1 || E > KOLIBRI_MAX_EXPERTS) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!digit_hi || !digit_lo || !bias || !quantiles) return KOLIBRI_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t err = launch_bf16_value(digit_hi, digit_lo, E, quantiles, s);
  if (err != cudaSuccess) return KOLIBRI_ERR_CUDA;
  return from_cuda(launch_bias_update(quantiles, E, bias, quantiles, s));
}

kolibri_status kolibri_eqb_key_histogram(const float* z, const float* alpha, int64_t N, int32_t E,
                                         int32_t pass, const uint32_t* prefix, uint32_t* hist,
                                         void* stream) {
  if (N < 1 || pass < 0 || pass > 3) return KOLIBRI_ERR_INVALID_ARG;
  if (E < 4 || E > KOLIBRI_MAX_EXPERTS || (E % 4) != 0) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!z || !hist || !aligned16(z) || (pass > 0 && !prefix)) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_key_hist(z, alpha, N, E, pass, prefix, hist, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_key_digit(const uint32_t* hist, int32_t E, int32_t pass, int64_t* rank,
                                     uint32_t* prefix, void* stream) {
  if (E < 1 || E > KOLIBRI_MAX_EXPERTS) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!hist || !rank || !prefix || pass < 0 || pass > 3) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_key_digit(hist, E, pass, rank, prefix, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_key_bias(const uint32_t* key, int32_t E, float* bias, float* quantiles,
                                    void* stream) {
  if (E < 1 || E > KOLIBRI_MAX_EXPERTS) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (!key || !bias || !quantiles) return KOLIBRI_ERR_INVALID_ARG;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t err = launch_key_value(key, E, quantiles, s);
  if (err != cudaSuccess) return KOLIBRI_ERR_CUDA;
  return from_cuda(launch_bias_update(quantiles, E, bias, quantiles, s));
}

kolibri_status kolibri_eqb_split_sample(const float* z, const float* alpha, int64_t N, int32_t E,
                                       int32_t K, int64_t S, uint32_t* sample, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (S < 1 || S > N) return KOLIBRI_ERR_INVALID_ARG;
  if (!z || !alpha || !sample || !aligned16(z)) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_eqb_sample(z, alpha, nullptr, N, E, K, S, N / S, S, sample,
                                     static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_split_brackets(const uint32_t* sample, int32_t R, int64_t S, int32_t E,
                                          int64_t N_total, int32_t K, uint32_t* scratch,
                                          uint32_t* lo, uint32_t* hi, void* stream) {
  kolibri_status st = check_ek(N_total, E, K);
  if (st != KOLIBRI_OK) return st;
  if (R < 1 || S < 1 || static_cast<int64_t>(R) * S > N_total) return KOLIBRI_ERR_INVALID_ARG;
  if (!sample || !scratch || !lo || !hi || !aligned16(scratch)) return KOLIBRI_ERR_INVALID_ARG;
  const int64_t m = (N_total * static_cast<int64_t>(K)) / E;
  const int64_t n = static_cast<int64_t>(R) * S;
  const int64_t ld = (n + 3) & ~static_cast<int64_t>(3);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t err = launch_dist_sample_transpose(sample, R, S, E, ld, scratch, s);
  if (err != cudaSuccess) return KOLIBRI_ERR_CUDA;
  return from_cuda(launch_dist_brackets(scratch, n, ld, E, m, N_total, lo, hi, s));
}

kolibri_status kolibri_eqb_split_count(const float* z, const float* alpha, int64_t N, int32_t E,
                                       int32_t K, const uint32_t* lo, const uint32_t* hi,
                                       uint32_t* counts, uint32_t* cand, int64_t cap,
                                       void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (cap < 1 || !z || !alpha || !lo || !hi || !counts || !cand || !aligned16(z))
    return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_dist_count(z, alpha, N, E, K, lo, hi, counts, cand, cap,
                                     static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_split_rank(const uint32_t* counts, int32_t E, int64_t N_total, int32_t K,
                                      int64_t* rank, uint32_t* flag, void* stream) {
  kolibri_status st = check_ek(N_total, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!counts || !rank || !flag) return KOLIBRI_ERR_INVALID_ARG;
  const int64_t m = (N_total * static_cast<int64_t>(K)) / E;
  return from_cuda(launch_dist_rank(counts, E, m, rank, flag, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_eqb_split_histogram(const uint32_t* cand, const uint32_t* counts,
                                           int64_t cap, int32_t E, int32_t pass,
                                           const uint32_t* prefix, uint32_t* hist, void* stream) {
  if (E < 1 || E > KOLIBRI_MAX_EXPERTS) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (cap < 1 || pass < 0 || pass > 3 || !cand || !counts || !hist || (pass > 0 && !prefix))
    return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_dist_cand_hist(cand, counts, cap, E, pass, prefix, hist,
                                         static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_lei_inject(const int32_t* counts, int64_t N, int32_t E, int32_t K,
                                  double lambda, double tau, float* g, void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!counts || !g || !aligned16(g) || !(tau > 0.0)) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_lei_inject(counts, N, E, K, lambda, tau, g,
                                     static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_score_grad_to_logits(const float* z, const float* gs, int64_t n, float* gz,
                                            void* stream) {
  if (n < 1 || !z || !gs || !gz) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_score_grad(z, gs, n, gz, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_intervention_rate(const float* z, const int32_t* ids, int64_t N, int32_t E,
                                         int32_t K, double* rate, unsigned long long* overlaps,
                                         void* stream) {
  kolibri_status st = check_ek(N, E, K);
  if (st != KOLIBRI_OK) return st;
  if (!z || !ids || !rate || !overlaps || !aligned16(z)) return KOLIBRI_ERR_INVALID_ARG;
  return from_cuda(launch_intervention(z, ids, N, E, K, overlaps, rate,
                                       static_cast<cudaStream_t>(stream)));
}

namespace {
constexpr int64_t kExpertRowLimit = (static_cast<int64_t>(1) << 31) - 512;
}

size_t kolibri_expert_ffn_workspace_size(int64_t N, int32_t d, int32_t F, int32_t K,
                                         int32_t shared) {
  if (N < 1 || K < 1 || d < 1 || F < 1) return 0;
  return expert_layout(N, d, F, K, shared != 0).total;
}

kolibri_status kolibri_expert_ffn(const void* x, const int32_t* perm, const int64_t* offsets,
                                  const int32_t* inv, const float* gates, const void* w_gate_up,
                                  const void* w_down, const void* ws_gate_up, const void* ws_down,
                                  float* y, int64_t N, int32_t d, int32_t F, int32_t E, int32_t K,
                                  void* ws, size_t ws_bytes, void* stream) {
  if (!x || !perm || !offsets || !inv || !gates || !w_gate_up || !w_down || !y || !ws)
    return KOLIBRI_ERR_INVALID_ARG;
  if ((ws_gate_up == nullptr) != (ws_down == nullptr)) return KOLIBRI_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(y) ||
      !aligned16(ws) || (ws_gate_up && (!aligned16(ws_gate_up) || !aligned16(ws_down))))
    return KOLIBRI_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || K > 32 || K > E) return KOLIBRI_ERR_INVALID_ARG;
  if (!expert_shape_supported(d, F, E) || N * K >= kExpertRowLimit) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < expert_layout(N, d, F, K, ws_gate_up != nullptr).total)
    return KOLIBRI_ERR_WORKSPACE_TOO_SMALL;
  return from_cuda(launch_expert_ffn(x, perm, offsets, inv, gates, w_gate_up, w_down, ws_gate_up,
                                     ws_down, y, N, d, F, E, K, ws, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_expert_dispatch(const void* x, const int32_t* perm, int64_t N, int32_t d,
                                       int32_t K, void* x_perm, void* stream) {
  if (!x || !perm || !x_perm || !aligned16(x) || !aligned16(x_perm)) return KOLIBRI_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || d < 1) return KOLIBRI_ERR_INVALID_ARG;
  if (d % 8 != 0 || d > 8192 || N * K >= kExpertRowLimit) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_expert_dispatch(x, perm, N, d, K, x_perm, static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_expert_gate_up(const void* a, int64_t rows, const int64_t* offsets, int32_t G,
                                      const void* w_gate_up, void* h, int32_t d, int32_t F,
                                      void* stream) {
  if (!a || !w_gate_up || !h || !aligned16(a) || !aligned16(w_gate_up) || !aligned16(h))
    return KOLIBRI_ERR_INVALID_ARG;
  if (rows < 1 || (offsets == nullptr && G != 1)) return KOLIBRI_ERR_INVALID_ARG;
  if (!expert_shape_supported(d, F, G) || rows >= kExpertRowLimit) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_expert_gate_up(a, rows, offsets, G, w_gate_up, h, d, F,
                                         static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_expert_down(const void* h, int64_t rows, const int64_t* offsets, int32_t G,
                                   const void* w_down, float* y, int32_t d, int32_t F, void* stream) {
  if (!h || !w_down || !y || !aligned16(h) || !aligned16(w_down) || !aligned16(y))
    return KOLIBRI_ERR_INVALID_ARG;
  if (rows < 1 || (offsets == nullptr && G != 1)) return KOLIBRI_ERR_INVALID_ARG;
  if (!expert_shape_supported(d, F, G) || rows >= kExpertRowLimit) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_expert_down(h, rows, offsets, G, w_down, y, d, F,
                                      static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_expert_combine(const float* y_perm, const float* y_shared, const int32_t* inv,
                                      const float* gates, int64_t N, int32_t d, int32_t K, float* y,
                                      void* stream) {
  if (!y_perm || !inv || !gates || !y || !aligned16(y_perm) || !aligned16(y) ||
      (y_shared && !aligned16(y_shared)))
    return KOLIBRI_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || K > 32 || d < 4) return KOLIBRI_ERR_INVALID_ARG;
  if (d % 4 != 0 || N * K >= kExpertRowLimit) return KOLIBRI_ERR_UNSUPPORTED_SHAPE;
  return from_cuda(launch_expert_combine(y_perm, y_shared, inv, gates, N, d, K, y,
                                         static_cast<cudaStream_t>(stream)));
}

kolibri_status kolibri_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return KOLIBRI_ERR_INVALID_ARG;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return from_cuda(cudaGetLastError());
}

kolibri_status kolibri_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KOLIBRI_ERR_CUDA;
  const unsigned v = status_take_api() | status_take_eqb() | status_take_noalloc() |
                     status_take_permute() | status_take_route() | status_take_logits() |
                     status_take_forward() | status_take_balance() | status_take_small() |
                     status_take_experts() | status_take_decode();
  if (v & kStatusReadFailed) return KOLIBRI_ERR_CUDA;
  if (v & kStatusTimeout) return KOLIBRI_ERR_TIMEOUT;
  if (v & kStatusBadInput) return KOLIBRI_ERR_DEVICE;
  return KOLIBRI_OK;
}

}  // extern "C"
