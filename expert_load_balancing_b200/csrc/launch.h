// launch.h -- host launchers of the router kernels (internal to the library).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace kolibri {

// Row sample used by the EQB bracket: S rows t = s * stride, s < S.
constexpr int64_t kSampleMax = 16384;
// Candidate capacity per expert in the bracketed full pass.
constexpr int64_t kCandCap = 65536;

struct EqbLayout {
  int64_t S = 0, stride = 1;
  int64_t S_ld = 0;           // row stride of the sample buffer (multiple of 4)
  bool exact_small = false;   // S == N: the sample is the whole column
  size_t off_sample = 0;      // u32 [E][S]   keys of Z + alpha at sampled rows
  size_t off_lo = 0;          // u32 [E]      lower bracket key
  size_t off_hi = 0;          // u32 [E]      upper bracket key
  size_t off_above = 0;       // u32 [E]      keys above the bracket
  size_t off_cnt = 0;         // u32 [E]      keys inside the bracket
  size_t off_flag = 0;        // u32 [E]      1 = bracket missed, radix fallback
  size_t off_v = 0;           // f32 [E]      the quantiles v_e
  size_t off_cand = 0;        // u32 [E][cap] keys inside the bracket
  size_t off_alpha = 0;       // f32 [N]      token bias when none is given
  size_t total = 0;
};
EqbLayout eqb_layout(int64_t N, int32_t E, int32_t K);

struct PermuteLayout {
  int64_t chunk = 0;          // slots per chunk
  int64_t nchunks = 0;
  bool single_cta = false;
  size_t off_chunk_counts = 0;  // u32 [E][nchunks]
  size_t off_counts = 0;        // u32 [E]
  size_t off_ticket = 0;        // u32 [1]
  size_t off_dec_ticket = 0;    // u32 [1]: the decode forward's counter, zero between calls
  size_t total = 0;
};
PermuteLayout permute_layout(int64_t N, int32_t E, int32_t K);

cudaError_t launch_router_logits(const void* x, const void* w, float* z, int64_t N, int32_t d,
                                 int32_t E, cudaStream_t s);

// Small batches (decode): logits by router_small.cu instead of the pair GEMM.
constexpr int64_t kSmallTokenLimit = 1024;
bool router_small_preferred(int64_t N);
cudaError_t launch_router_logits_small(const void* x, const void* w, float* z, int64_t N, int32_t d,
                                       int32_t E, cudaStream_t s);

// The expert layer (expert_ffn.cu): workspace regions and the stages.
struct ExpertLayout {
  size_t off_x_perm, off_h, off_y_perm, off_h_shared, off_y_shared, total;
};
bool expert_shape_supported(int32_t d, int32_t F, int32_t E);
ExpertLayout expert_layout(int64_t N, int32_t d, int32_t F, int32_t K, bool shared);
cudaError_t launch_expert_dispatch(const void* x, const int32_t* perm, int64_t N, int32_t d,
                                   int32_t K, void* x_perm, cudaStream_t s);
cudaError_t launch_expert_gate_up(const void* a, int64_t rows, const int64_t* offsets, int32_t G,
                                  const void* w_gate_up, void* h, int32_t d, int32_t F,
                                  cudaStream_t s);
cudaError_t launch_expert_down(const void* h, int64_t rows, const int64_t* offsets, int32_t G,
                               const void* w_down, float* y, int32_t d, int32_t F, cudaStream_t s);
cudaError_t launch_expert_combine(const float* y_perm, const float* y_shared, const int32_t* inv,
                                  const float* gates, int64_t N, int32_t d, int32_t K, float* y,
                                  cudaStream_t s);
cudaError_t launch_expert_ffn(const void* x, const int32_t* perm, const int64_t* offsets,
                              const int32_t* inv, const float* gates, const void* w_gate_up,
                              const void* w_down, const void* ws_gate_up, const void* ws_down,
                              float* y, int64_t N, int32_t d, int32_t F, int32_t E, int32_t K,
                              void* ws, cudaStream_t s);

// Fused logits + selection (router_forward.cu).  Returns cudaErrorNotSupported
// for shapes it does not cover; the caller then runs logits and top-K apart.
// Rows it could not finish carry a NaN alpha; launch_select_fixup completes them.
bool router_forward_supported(int32_t E, int32_t K);
cudaError_t launch_router_forward(const void* x, const void* w, const float* bias, float* z,
                                  int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                  float* gates, float* alpha, cudaStream_t s);
cudaError_t launch_select_fixup(const float* z, const float* bias, int64_t N, int32_t E, int32_t K,
                                int32_t* ids, float* gates, float* alpha, cudaStream_t s);

// The intervention rate's overlap count in the selection's eight-lanes-per-
// row layout (from 4096 rows, E in 128, 256, 384, 512): adds to *total the
// number of (row, k) whose own top-K expert on Z alone is among ids[row].
bool seg_overlap_applies(int64_t N, int32_t E, int32_t K);
cudaError_t launch_seg_overlap(const float* z, const int32_t* ids, int64_t N, int32_t E, int32_t K,
                               unsigned long long* total, cudaStream_t s);
cudaError_t launch_topk(const float* z, const float* bias, int64_t N, int32_t E, int32_t K,
                        int32_t* ids, float* gates, float* alpha, cudaStream_t s);

cudaError_t launch_permute(const int32_t* ids, int64_t N, int32_t E, int32_t K, int32_t* counts,
                           int64_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                           cudaStream_t s);

cudaError_t launch_eqb(const float* z, const float* alpha, float* bias, int64_t N, int32_t E,
                       int32_t K, float* quantiles, void* ws, cudaStream_t s);

// Logits + selection by whichever path covers the shape (fused kernel and
// its row check, or the GEMM then the row kernel).
cudaError_t router_forward_any(const void* x, const void* w, const float* bias, float* z,
                               int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                               float* gates, float* alpha, cudaStream_t s);

// Decode batches (router_decode.cu): logits and selection in one clustered
// launch.  Returns cudaErrorNotSupported where it does not apply.
constexpr int64_t kDecodeTokenLimit = 96;
bool router_decode_supported(int64_t N, int32_t d, int32_t E, int32_t K);
cudaError_t launch_router_decode(const void* x, const void* w, const float* bias, float* z,
                                 int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                 float* gates, float* alpha, cudaStream_t s);
// Batches of one cluster (at most 16 tokens): the same launch also forms
// counts, offsets, perm and inv (inv may be null).
bool router_decode_permutes(int64_t N, int32_t d, int32_t E, int32_t K);
cudaError_t launch_router_decode_permute(const void* x, const void* w, const float* bias, float* z,
                                         int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                         float* gates, float* alpha, int32_t* counts,
                                         int64_t* offsets, int32_t* perm, int32_t* inv,
                                         cudaStream_t s);
// The same outputs from E/8 CTAs without a cluster, the last of which (by the
// counter `ticket`, zero on entry and left zero) selects and groups.
bool router_decode_ticket_supported(int64_t N, int32_t d, int32_t E, int32_t K);
cudaError_t launch_router_decode_ticket(const void* x, const void* w, const float* bias, float* z,
                                        int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                        float* gates, float* alpha, int32_t* counts, int64_t* offsets,
                                        int32_t* perm, int32_t* inv, uint32_t* ticket, cudaStream_t s);

// The logits by batch size, with the same choice of kernel as the forward.
cudaError_t launch_router_logits_by_size(const void* x, const void* w, float* z, int64_t N,
                                         int32_t d, int32_t E, cudaStream_t s);

// The forward by batch size: decode batches take router_decode.cu, small
// ones (router_small_preferred) the small logits kernel and the row kernel,
// the rest router_forward_any.
cudaError_t router_forward_by_size(const void* x, const void* w, const float* bias, float* z,
                                   int64_t N, int32_t d, int32_t E, int32_t K, int32_t* ids,
                                   float* gates, float* alpha, cudaStream_t s);

cudaError_t launch_forward_eqb(const void* x, const void* w, float* bias, float* z, int64_t N,
                               int32_t d, int32_t E, int32_t K, int32_t* ids, float* gates,
                               float* alpha, float* quantiles, void* ws, cudaStream_t s);

cudaError_t launch_route_balance(const float* z, float* bias, int64_t N, int32_t E, int32_t K,
                                 int32_t* ids, float* gates, float* alpha, float* quantiles,
                                 void* ws, cudaStream_t s);

// pieces of the EQB update living in route.cu (they walk rows of Z)
// zero_word (nullable): a word the sampling kernel sets to zero for the
// kernels after it.
cudaError_t launch_eqb_sample(const float* z, const float* alpha, const float* bias, int64_t N,
                              int32_t E, int32_t K, int64_t S, int64_t stride, int64_t S_ld,
                              uint32_t* sample, cudaStream_t s, uint32_t* zero_word = nullptr);
// Bracketed full pass.  alpha_in given: use it.  Otherwise alpha is derived
// from bias (and written to alpha_out); with ids/gates non-null the same
// pass also writes the routing.
cudaError_t launch_route_window_pass(const float* z, const float* bias, const float* alpha_in,
                                     int64_t N, int32_t E, int32_t K, int32_t* ids, float* gates,
                                     float* alpha_out, const uint32_t* lo, const uint32_t* hi,
                                     uint32_t* above, uint32_t* cnt, uint32_t* cand, int64_t cap,
                                     cudaStream_t s);

// beta = -v, centred (fp64 sum in ascending e, one rounding); quantiles (nullable) = v.
cudaError_t launch_bias_update(const float* v, int32_t E, float* bias, float* quantiles,
                               cudaStream_t s);

// balance.cu: bf16-key EQB passes, Load-Error Injection, intervention rate.
cudaError_t launch_bf16_hist(const float* z, const float* alpha, int64_t N, int32_t E,
                             const uint32_t* prefix, uint32_t* hist, cudaStream_t s);
cudaError_t launch_bf16_digit(const uint32_t* hist, int32_t E, int64_t* rank, uint32_t* digit,
                              cudaStream_t s);
cudaError_t launch_bf16_value(const uint32_t* d_hi, const uint32_t* d_lo, int32_t E, float* v,
                              cudaStream_t s);
size_t eqb_bf16_ws_bytes(int64_t N, int32_t E, int32_t K);
cudaError_t launch_eqb_bf16(const float* z, const float* alpha, float* bias, int64_t N, int32_t E,
                            int32_t K, float* quantiles, void* ws, cudaStream_t s);
cudaError_t launch_lei_inject(const int32_t* counts, int64_t N, int32_t E, int32_t K, double lambda,
                              double tau, float* g, cudaStream_t s);
cudaError_t launch_score_grad(const float* z, const float* gs, int64_t n, float* gz, cudaStream_t s);
cudaError_t launch_intervention(const float* z, const int32_t* ids, int64_t N, int32_t E, int32_t K,
                                unsigned long long* total, double* rate, cudaStream_t s);

int device_sm_count();

// Read and clear the status word of one translation unit (see common.cuh).
// fp32-key radix passes of the EQB quantile over a split batch (balance.cu).
cudaError_t launch_key_hist(const float* z, const float* alpha, int64_t N, int32_t E, int32_t pass,
                            const uint32_t* prefix, uint32_t* hist, cudaStream_t s);
cudaError_t launch_key_digit(const uint32_t* hist, int32_t E, int32_t pass, int64_t* rank,
                             uint32_t* prefix, cudaStream_t s);
cudaError_t launch_key_value(const uint32_t* key, int32_t E, float* v, cudaStream_t s);

// The sampled-bracket EQB update over a split batch (eqb.cu, balance.cu).
cudaError_t launch_dist_brackets(const uint32_t* sample_em, int64_t n, int64_t ld, int32_t E,
                                 int64_t m, int64_t N_total, uint32_t* lo, uint32_t* hi,
                                 cudaStream_t s);
cudaError_t launch_dist_sample_transpose(const uint32_t* gathered, int32_t R, int64_t S, int32_t E,
                                         int64_t ld, uint32_t* sample_em, cudaStream_t s);
cudaError_t launch_dist_count(const float* z, const float* alpha, int64_t N, int32_t E, int32_t K,
                              const uint32_t* lo, const uint32_t* hi, uint32_t* counts,
                              uint32_t* cand, int64_t cap, cudaStream_t s);
cudaError_t launch_dist_rank(const uint32_t* counts, int32_t E, int64_t m, int64_t* rank,
                             uint32_t* flag, cudaStream_t s);
cudaError_t launch_dist_cand_hist(const uint32_t* cand, const uint32_t* counts, int64_t cap,
                                  int32_t E, int32_t pass, const uint32_t* prefix, uint32_t* hist,
                                  cudaStream_t s);

unsigned status_take_api();
unsigned status_take_eqb();
unsigned status_take_noalloc();
unsigned status_take_permute();
unsigned status_take_route();
unsigned status_take_logits();
unsigned status_take_forward();
unsigned status_take_balance();
unsigned status_take_small();
unsigned status_take_experts();
unsigned status_take_decode();

}  // namespace kolibri
