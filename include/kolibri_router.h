/*
 * kolibri_router.h -- C ABI of the B200 (sm_100a) sigmoid MoE router with
 * Exact Quantile Balancing (EQB).
 *
 * The method (page "Kolibri Pre-Training from Scratch: UniBPE, Hybrid
 * Attention and Exact Quantile Balancing", sections 6.1 and 7; page
 * "Kolibri 1 im Detail: hybride RNoPE-Attention, Sparse MoE und FP8-Serving",
 * section "Routing: Auswahl-Bias und Mischgewichte sind getrennt"):
 *
 *   Z = x W^T                         router logits, bf16 in, fp32 out
 *   B = Z + 1 beta^T                  selection bias, used for selection only
 *   I_t = Top-K(B_t,:)                the K experts of token t
 *   S_t,e = sigma(Z_t,e), e in I_t    mixing weights from the RAW logits,
 *                                     not renormalised
 *   alpha_t = -Q_K(B_t,:)             token bias
 *   beta_e  = -Q_r(Z_:,e + alpha),    expert bias, r = N K / E, then centred
 *
 * Q_m(list) is the (m+1)-th largest entry (section 1).  EQB computes the
 * column quantile exactly, not by a histogram approximation (section 7.3).
 *
 * Conventions shared by every call
 *   - All data pointers are DEVICE pointers owned by the caller.  No call
 *     allocates or frees device memory, and none synchronises the host,
 *     except kolibri_device_status().  Work is enqueued on `stream`, a
 *     cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Arrays are dense and row-major with the shapes given below.  Pointers
 *     must be 16-byte aligned.
 *   - Order of fp32 scores: the total order of the order-preserving key of
 *     the bit pattern (so -0.0 ranks below +0.0).  Equal scores rank the
 *     lower expert id first.  Inputs must be finite (not checked).
 *   - Arguments are validated on the host before anything is enqueued; on
 *     an argument error nothing is written.
 *   - Each call returns KOLIBRI_OK once its work is enqueued.  A launch
 *     failure returns KOLIBRI_ERR_CUDA.  Errors found later on the device
 *     (a bounded wait that expired, an expert id out of range) are recorded
 *     in a per-device status word read by kolibri_device_status().
 *   - Calls on different streams may run concurrently if they use separate
 *     workspaces; one workspace must not be shared by calls that can
 *     overlap on the GPU.
 *   - The first call of an entry point in a process looks up launch limits
 *     (occupancy, kernel attributes) and keeps them in process-wide
 *     variables.  Make the first call of each entry point before calling it
 *     from several host threads at once.
 */
#ifndef KOLIBRI_ROUTER_H
#define KOLIBRI_ROUTER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KOLIBRI_API __attribute__((visibility("default")))
#else
#define KOLIBRI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kolibri_status {
    KOLIBRI_OK = 0,
    KOLIBRI_ERR_INVALID_ARG = 1,        /* null pointer, misalignment, K >= E ... */
    KOLIBRI_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside the supported range      */
    KOLIBRI_ERR_WORKSPACE_TOO_SMALL = 3,/* ws_bytes < kolibri_workspace_bytes()   */
    KOLIBRI_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed   */
    KOLIBRI_ERR_TIMEOUT = 5,            /* a bounded device-side wait expired     */
    KOLIBRI_ERR_DEVICE = 6              /* a device-side check failed (bad id)    */
} kolibri_status;

/* Operation selector for kolibri_workspace_bytes(). */
enum {
    KOLIBRI_OP_PERMUTE = 1,
    KOLIBRI_OP_EQB = 2,
    KOLIBRI_OP_EQB_BF16 = 3
};

/* Limits.  E (experts) and K (top-K) must satisfy 1 <= K < E <= 512,
 * K <= 16, E % 4 == 0.  N (tokens) must satisfy 1 <= N and N*K < 2^31.
 * d (width) must satisfy 64 <= d, d % 64 == 0. */
#define KOLIBRI_MAX_EXPERTS 512
#define KOLIBRI_MAX_TOPK 16

/* Human-readable name of a status code (static string, never NULL). */
KOLIBRI_API const char *kolibri_status_string(kolibri_status status);

/* Bytes of caller-provided device workspace that `op` needs for these sizes
 * (0 if the sizes are invalid).  The workspace need not be initialised, with
 * one exception: a KOLIBRI_OP_PERMUTE workspace given to
 * kolibri_router_forward_permute holds a counter that must be zero when the
 * workspace is first used (zero-fill it once after allocating it); every call
 * leaves the counter zero. */
KOLIBRI_API size_t kolibri_workspace_bytes(int op, int64_t N, int32_t E, int32_t K);

/*
 * Router logits Z = x W^T ("Kolibri Pre-Training from Scratch" 6.1; "Kolibri
 * 1 im Detail", routing: bf16 router, tokens [N, d] -> fp32 logits [N, E]).
 *   x  [N, d] bf16 (raw 16-bit patterns), row-major
 *   w  [E, d] bf16, row-major (one row per expert)
 *   z  [N, E] fp32, row-major, written
 * Products are exact, accumulation is fp32 on the tensor cores (tcgen05).
 * Shapes: d % 64 == 0, E % 16 == 0, 16 <= E <= 512.
 */
KOLIBRI_API kolibri_status kolibri_router_logits(const void *x, const void *w, float *z,
                                     int64_t N, int32_t d, int32_t E, void *stream);

/*
 * Router logits and selection in one call: kolibri_router_logits followed by
 * kolibri_router_topk, with identical results ("Kolibri Pre-Training from
 * Scratch" 6.1 and 7.1; "Kolibri 1 im Detail", routing steps 1 and 2).
 *   x, w, z        as in kolibri_router_logits (z is still written in full)
 *   bias           [E] fp32 selection bias beta, or NULL (B = Z exactly)
 *   ids, gates     [N, K], written as by kolibri_router_topk
 *   alpha          [N] fp32, written; required here (not NULL)
 * For 16 <= E <= 384 with E >= 8 (K + 1) the selection runs inside the GEMM
 * epilogue while the tensor cores compute the next tile, so Z is not read
 * back for routing; rows with many tied scores are finished by a second
 * kernel on the same stream.  Other shapes run the two kernels one after the
 * other.  Shapes: d % 64 == 0, E % 16 == 0, plus the limits above.  Errors:
 * KOLIBRI_ERR_INVALID_ARG for NULL or misaligned pointers (all 16-byte
 * aligned), KOLIBRI_ERR_UNSUPPORTED_SHAPE otherwise; nothing is enqueued.
 */
KOLIBRI_API kolibri_status kolibri_router_forward(const void *x, const void *w, const float *bias,
                                                  float *z, int64_t N, int32_t d, int32_t E,
                                                  int32_t K, int32_t *ids, float *gates,
                                                  float *alpha, void *stream);

/*
 * kolibri_router_forward followed by kolibri_expert_permute on its ids, in
 * one call: the arguments and outputs of both ("Kolibri Pre-Training from
 * Scratch" 6.1 and 7.1; loads and grouping 6.1/6.2).  A decode batch of at
 * most 16 tokens with E a multiple of 128, whose E/16 router rows of d and 16
 * token rows fit in one CTA's shared memory (as for kolibri_router_forward's
 * one-launch form), takes a single launch:
 *   - with ws (not NULL, 16-byte aligned, ws_bytes at least
 *     kolibri_workspace_bytes(KOLIBRI_OP_PERMUTE, N, E, K)): E/8 blocks, each
 *     forming the logits of 8 experts; the last block to finish (by a counter
 *     in ws, which must be zero on the workspace's first use and is left
 *     zero) forms the selection and the grouping.  A counter found nonzero
 *     sets KOLIBRI_ERR_DEVICE in the device status word and leaves the
 *     outputs unspecified.  The same ws must not be used by two calls that
 *     may run at the same time.
 *   - without ws: one 16-CTA cluster (E/16 router rows per CTA) forms the
 *     logits, the selection and the grouping.
 * Z equals kolibri_router_forward's bit for bit in both forms.  Other batches
 * run the forward and then the permutation.  ws / ws_bytes otherwise as for
 * kolibri_expert_permute (may be NULL when N*K <= 4096).  inv may be NULL.
 */
KOLIBRI_API kolibri_status kolibri_router_forward_permute(const void *x, const void *w,
                                                          const float *bias, float *z, int64_t N,
                                                          int32_t d, int32_t E, int32_t K,
                                                          int32_t *ids, float *gates, float *alpha,
                                                          int32_t *counts, int64_t *offsets,
                                                          int32_t *perm, int32_t *inv, void *ws,
                                                          size_t ws_bytes, void *stream);

/*
 * One training step's routing from the tokens: logits, selection with bias
 * beta_in, and the EQB update of bias to beta_out ("Kolibri Pre-Training
 * from Scratch" 6.1, 7.1 update rule, 7.2 order of operations, 7.3 exact
 * quantile): kolibri_router_forward followed by kolibri_eqb_update with the
 * alpha it produced, in one call on one stream.
 *   x, w, z, ids, gates   as in kolibri_router_forward
 *   bias                  [E] fp32, in: beta_in (routes), out: beta_out
 *   alpha                 [N] fp32, written if not NULL (else kept in ws)
 *   quantiles             [E] fp32, written if not NULL: v_e
 *   ws, ws_bytes          kolibri_workspace_bytes(KOLIBRI_OP_EQB, N, E, K)
 * Errors: as kolibri_router_forward and kolibri_eqb_update.
 */
KOLIBRI_API kolibri_status kolibri_router_forward_eqb(const void *x, const void *w, float *bias,
                                                      float *z, int64_t N, int32_t d, int32_t E,
                                                      int32_t K, int32_t *ids, float *gates,
                                                      float *alpha, float *quantiles, void *ws,
                                                      size_t ws_bytes, void *stream);

/*
 * Bias add, top-K selection and sigmoid gates ("Kolibri Pre-Training from
 * Scratch" 6.1 and 7.1; "Kolibri 1 im Detail", routing steps 1 and 2).
 *   z      [N, E] fp32 logits
 *   bias   [E] fp32 selection bias beta, or NULL for no bias (B = Z exactly)
 *   ids    [N, K] int32, written: the K experts of each token, biased score
 *          descending, ties to the lower id
 *   gates  [N, K] fp32, written: sigma(z[t, ids[t,k]]) from the raw logits,
 *          computed in fp64 and rounded once; not renormalised
 *   alpha  [N] fp32, written if not NULL: -(the (K+1)-th largest biased
 *          score), the token bias of section 7.1
 */
KOLIBRI_API kolibri_status kolibri_router_topk(const float *z, const float *bias, int64_t N, int32_t E,
                                   int32_t K, int32_t *ids, float *gates, float *alpha,
                                   void *stream);

/*
 * Expert loads and the grouping of routed slots by expert (loads c_e of
 * "Kolibri Pre-Training from Scratch" 6.1/6.2).  Slot j = t*K + k.
 *   ids      [N, K] int32 expert ids in [0, E)
 *   counts   [E] int32, written: c_e
 *   offsets  [E+1] int64, written: exclusive prefix sum of counts
 *   perm     [N*K] int32, written: perm[p] = slot at grouped position p;
 *            experts ascending, slots ascending inside an expert (stable)
 *   inv      [N*K] int32, written if not NULL: inv[perm[p]] = p
 *   ws       device workspace of kolibri_workspace_bytes(KOLIBRI_OP_PERMUTE)
 * An id outside [0, E) sets KOLIBRI_ERR_DEVICE in the device status word;
 * the outputs are then unspecified.
 */
KOLIBRI_API kolibri_status kolibri_expert_permute(const int32_t *ids, int64_t N, int32_t E, int32_t K,
                                      int32_t *counts, int64_t *offsets, int32_t *perm,
                                      int32_t *inv, void *ws, size_t ws_bytes, void *stream);

/*
 * kolibri_expert_permute for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment convenience.  Some
 * callers may not call cudaMalloc at all: inference servers that reserve all
 * of device memory for their own pool up front, plugins that run inside
 * another runtime's memory budget, and code paths that must not risk the
 * implicit synchronisation an allocation can cause.  This variant takes no
 * workspace: its scratch is a fixed array of KOLIBRI_NOALLOC_SCRATCH_BYTES
 * inside the library, which every GPU that loads the library holds until
 * the process exits.
 *   Arguments and results are those of kolibri_expert_permute, without ws.
 *   Sizes whose scratch (kolibri_workspace_bytes(KOLIBRI_OP_PERMUTE, N, E,
 *   K)) exceeds the array return KOLIBRI_ERR_WORKSPACE_TOO_SMALL and
 *   enqueue nothing (at E = 384, up to 11,173,888 routed slots N*K fit).
 *   The first call on each device looks up the array's device address with
 *   that device current; make that first call before any stream capture.
 *   Every call shares the one array: calls that can overlap on the GPU (on
 *   different streams, or from different threads) race and must not be
 *   issued.  The array keeps the previous call's contents; what must start
 *   at zero is cleared on the stream by each call.
 */
#define KOLIBRI_NOALLOC_SCRATCH_BYTES (2u << 20)
KOLIBRI_API kolibri_status kolibri_expert_permute_noalloc(const int32_t *ids, int64_t N,
                                                          int32_t E, int32_t K, int32_t *counts,
                                                          int64_t *offsets, int32_t *perm,
                                                          int32_t *inv, void *stream);

/*
 * Exact Quantile Balancing update ("Kolibri Pre-Training from Scratch" 7.1
 * update rule, 7.2 order of operations, 7.3 exactness):
 *   v_e  = Q_m(Z_:,e + alpha), the (m+1)-th largest entry of the fp32 sums,
 *          m = floor(N*K/E), computed exactly (radix selection on keys)
 *   beta = -v, then centred: mean = fp32(fp64 sum over e ascending / E),
 *          beta_e = -v_e - mean in fp32
 *   z          [N, E] fp32 logits
 *   alpha      [N] fp32 token bias (from kolibri_router_topk), or NULL: then
 *              alpha_t = -Q_K(Z_t,: + bias_in) is computed here
 *   bias       [E] fp32: read as beta_in when alpha is NULL; always
 *              overwritten with the new centred beta
 *   quantiles  [E] fp32, written if not NULL: v_e
 *   ws         device workspace of kolibri_workspace_bytes(KOLIBRI_OP_EQB)
 * The result is exact for every input; large batches are first bracketed
 * from a strided row sample and fall back to full radix passes for any
 * expert whose bracket misses.
 */
KOLIBRI_API kolibri_status kolibri_eqb_update(const float *z, const float *alpha, float *bias,
                                  int64_t N, int32_t E, int32_t K, float *quantiles,
                                  void *ws, size_t ws_bytes, void *stream);

/*
 * Routing and the EQB update in one call: the outputs of
 * kolibri_router_topk(z, bias, ...) followed by kolibri_eqb_update(z, alpha,
 * bias, ...) on the token biases that routing produced ("Kolibri
 * Pre-Training from Scratch" 7.1: each step performs one token update, then
 * one expert update; routing uses the current beta).  Large batches stream Z
 * from HBM once for both: the bracket of step 2 of the update comes from
 * sampled rows routed with the same bias, and the routing pass gathers the
 * bracketed keys.
 *   z          [N, E] fp32 logits
 *   bias       [E] fp32: beta used for routing, then overwritten with the
 *              new centred beta
 *   ids, gates [N, K], written as by kolibri_router_topk
 *   alpha      [N] fp32, written if not NULL
 *   quantiles  [E] fp32, written if not NULL
 *   ws         device workspace of kolibri_workspace_bytes(KOLIBRI_OP_EQB)
 */
KOLIBRI_API kolibri_status kolibri_route_and_balance(const float *z, float *bias, int64_t N,
                                                     int32_t E, int32_t K, int32_t *ids,
                                                     float *gates, float *alpha, float *quantiles,
                                                     void *ws, size_t ws_bytes, void *stream);

/*
 * EQB with bfloat16 keys, as the pages run it ("Kolibri Pre-Training from
 * Scratch" 7.3): per expert, C = bf16(Z_:,e + alpha) (the fp32 sum rounded
 * once to bf16, ties to even), each value encoded as an order-preserving
 * 16-bit key; v_e = the (m+1)-th largest C, m = floor(N K / E); then
 * beta = -v, centred as in kolibri_eqb_update.  Rounding to bf16 is
 * monotone, so v_e is exactly the bf16 rounding of kolibri_eqb_update's fp32
 * quantile, and on one GPU that is how it is computed (one bracketed read of
 * Z).  Across ranks the pages' two histogram passes below apply.
 *   z [N, E] fp32, alpha [N] fp32 (NULL: alpha from bias, as
 *   kolibri_eqb_update), bias [E] in/out, quantiles [E] out if not NULL,
 *   ws: kolibri_workspace_bytes(KOLIBRI_OP_EQB_BF16, N, E, K) bytes.
 * Errors as kolibri_eqb_update.
 */
KOLIBRI_API kolibri_status kolibri_eqb_update_bf16(const float *z, const float *alpha, float *bias,
                                                   int64_t N, int32_t E, int32_t K,
                                                   float *quantiles, void *ws, size_t ws_bytes,
                                                   void *stream);

/*
 * The bf16-key EQB in pieces, for batches split over ranks (section 7.3:
 * "the histograms are summed with one all-reduce"): each rank adds its
 * histogram, the caller sums the histograms over ranks (an all-reduce of
 * 256 E 32-bit counts, e.g. NCCL), and every rank then picks the same digit.
 *   kolibri_eqb_bf16_histogram: ADDS this rank's counts into hist [E][256]
 *     (uint32; zero it before each pass) for the keys of bf16(z + alpha)
 *     (alpha NULL: of bf16(z)).  prefix NULL: pass one (bins of
 *     the high byte of every key); else pass two (bins of the low byte of the
 *     keys whose high byte is prefix[e]).  E % 4 == 0.
 *   kolibri_eqb_bf16_digit: per expert, scans the summed hist from the top
 *     bin to the one holding the rank[e]-th largest key (0-based; start with
 *     rank[e] = m = floor(N_total K / E)); writes that bin to digit[e] and
 *     subtracts the keys of the bins above it from rank[e].
 *   kolibri_eqb_bf16_bias: v_e from the two digits (the key), written to
 *     quantiles [E] (required), then bias = -v, centred.
 * Sequence per update: zero h; histogram(NULL); all-reduce h; digit(h, rank,
 * d_hi); zero h; histogram(d_hi); all-reduce h; digit(h, rank, d_lo);
 * bias(d_hi, d_lo).  On one rank the all-reduces are skipped.
 */
KOLIBRI_API kolibri_status kolibri_eqb_bf16_histogram(const float *z, const float *alpha,
                                                      int64_t N, int32_t E,
                                                      const uint32_t *prefix, uint32_t *hist,
                                                      void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_bf16_digit(const uint32_t *hist, int32_t E, int64_t *rank,
                                                  uint32_t *digit, void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_bf16_bias(const uint32_t *digit_hi,
                                                 const uint32_t *digit_lo, int32_t E,
                                                 float *bias, float *quantiles, void *stream);

/*
 * The EQB quantile of kolibri_eqb_update (fp32 keys) over a batch split
 * across ranks: the same radix selection in four passes of 8-bit digits
 * (the design of the pages' section 7.3 applied to the 32-bit order key of
 * Z + alpha, so the result is the exact fp32 quantile of the union, equal to
 * kolibri_eqb_update's on one rank).
 *   kolibri_eqb_key_histogram: pass p (0..3) adds to hist [E][256] (uint32,
 *     zeroed by the caller before each pass) the count of keys, per expert
 *     and byte 3 - p, among the keys whose top 8p bits equal prefix[e] (the
 *     digits so far; prefix is not read at pass 0).  alpha may be NULL (0).
 *   kolibri_eqb_key_digit: per expert, the bin holding the rank[e]-th
 *     largest key (0-based; start with rank[e] = m = floor(N_total K / E));
 *     writes it into prefix[e] as byte 3 - p (pass 0 overwrites prefix) and
 *     subtracts the keys of the bins above it from rank[e].  A rank past the
 *     column sets KOLIBRI_ERR_DEVICE.
 *   kolibri_eqb_key_bias: v_e from the finished key, written to quantiles
 *     [E] (required), then bias = -v, centred.
 * Sequence per update: for p = 0..3 { zero hist; histogram(p); all-reduce
 * hist; digit(p) }; bias.  On one rank the all-reduces are skipped.
 */
KOLIBRI_API kolibri_status kolibri_eqb_key_histogram(const float *z, const float *alpha, int64_t N,
                                                     int32_t E, int32_t pass,
                                                     const uint32_t *prefix, uint32_t *hist,
                                                     void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_key_digit(const uint32_t *hist, int32_t E, int32_t pass,
                                                 int64_t *rank, uint32_t *prefix, void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_key_bias(const uint32_t *key, int32_t E, float *bias,
                                                float *quantiles, void *stream);

/*
 * kolibri_eqb_update's sampled-bracket design over a batch split across R
 * ranks ("Kolibri Pre-Training from Scratch" 7.3: each rank holds its own
 * tokens, only counts cross ranks, every rank ends with the same exact
 * quantile of the union and the same bias).  Z is read once per rank; the
 * exchange is one all-gather of the samples, one all-reduce of 3 E counts
 * and four all-reduces of 256 E counts.  The result equals the four-pass
 * form above and, on one rank, kolibri_eqb_update, bit for bit.
 *   kolibri_eqb_split_sample: keys of z + alpha at the S rows t = s (N / S),
 *     s < S, of this rank's N tokens, written expert-major to sample [E][S]
 *     (uint32 order keys; 1 <= S <= N).  The caller gathers every rank's
 *     sample rank-major into [R][E][S] (all-gather; the same S everywhere).
 *   kolibri_eqb_split_brackets: per expert, two order statistics of the R S
 *     gathered keys bracket the target (m+1)-th largest of the union, m =
 *     floor(N_total K / E) (sample ranks about (m+1) R S / N_total, six
 *     binomial standard deviations apart): keys lo[E] <= hi[E].  The same on
 *     every rank.  scratch: caller-owned [E][ld] uint32, ld = R S rounded up
 *     to a multiple of 4, 16-byte aligned (the samples laid out expert-major).
 *   kolibri_eqb_split_count: one pass over this rank's z + alpha: counts
 *     [3][E] uint32 = keys above hi, keys in [lo, hi], and 1 where the latter
 *     exceeded cap; the keys in [lo, hi] go to cand [E][cap].  The caller
 *     keeps these counts and sums a copy over ranks (all-reduce).
 *   kolibri_eqb_split_rank: from the summed counts, rank[e] = m - above[e]
 *     (int64, the target's rank among the bracketed keys of the union) and
 *     flag[e] = 1 where the target lies outside [lo, hi] or a rank's gather
 *     overflowed.  If any flag is set (the caller reads flag), the update is
 *     finished with the four-pass form (kolibri_eqb_key_histogram over z)
 *     instead; this happens only when the sample misleads.
 *   kolibri_eqb_split_histogram: pass p (0..3) adds to hist [E][256] the
 *     counts per byte 3 - p of this rank's bracketed keys (cand, with this
 *     rank's own counts) whose top 8p bits equal prefix[e]: the gathered keys'
 *     form of kolibri_eqb_key_histogram.  Then kolibri_eqb_key_digit with
 *     rank, and after four passes kolibri_eqb_key_bias, as in that form.
 * Sequence per update: sample; all-gather; brackets; count; all-reduce a
 * copy of counts; rank; read flag; for p = 0..3 { zero hist; histogram(p);
 * all-reduce hist; key_digit(p) }; key_bias.  On one rank the exchange
 * steps are skipped (R = 1).  alpha is required: the token bias of the
 * routing, as kolibri_router_topk writes it.
 */
KOLIBRI_API kolibri_status kolibri_eqb_split_sample(const float *z, const float *alpha, int64_t N,
                                                    int32_t E, int32_t K, int64_t S,
                                                    uint32_t *sample, void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_split_brackets(const uint32_t *sample, int32_t R, int64_t S,
                                                      int32_t E, int64_t N_total, int32_t K,
                                                      uint32_t *scratch, uint32_t *lo, uint32_t *hi,
                                                      void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_split_count(const float *z, const float *alpha, int64_t N,
                                                   int32_t E, int32_t K, const uint32_t *lo,
                                                   const uint32_t *hi, uint32_t *counts,
                                                   uint32_t *cand, int64_t cap, void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_split_rank(const uint32_t *counts, int32_t E,
                                                  int64_t N_total, int32_t K, int64_t *rank,
                                                  uint32_t *flag, void *stream);
KOLIBRI_API kolibri_status kolibri_eqb_split_histogram(const uint32_t *cand,
                                                       const uint32_t *counts, int64_t cap,
                                                       int32_t E, int32_t pass,
                                                       const uint32_t *prefix, uint32_t *hist,
                                                       void *stream);

/*
 * Load-Error Injection ("Kolibri Pre-Training from Scratch" 8) on the score
 * gradient of one microbatch of N tokens:
 *   f_e = counts[e] / (K N / E), rho_e = f_e - 1, xi = max_e |rho_e| / tau,
 *   delta_e = lambda (tanh(xi) / xi) rho_e (the factor is 1 at xi = 0), in
 *   fp64, rounded once to fp32 (tanh from the gate's exp);
 *   g[t][e] += delta_e for every token t and expert e (fp32).
 * The pages use lambda = 1e-5 and tau = 1.  counts [E] int32 (e.g. from
 * kolibri_expert_permute), g [N, E] fp32 in/out, 16-byte aligned.
 */
KOLIBRI_API kolibri_status kolibri_lei_inject(const int32_t *counts, int64_t N, int32_t E,
                                              int32_t K, double lambda, double tau, float *g,
                                              void *stream);

/*
 * The chain rule from the score gradient to the router logits (section 8,
 * numerical check): gz[i] = gs[i] * sigma(z[i]) (1 - sigma(z[i])), sigma in
 * fp64 from the gate's exp (saturating where the gate does), the product in
 * fp64, rounded once to fp32.  n elements of each array.
 */
KOLIBRI_API kolibri_status kolibri_score_grad_to_logits(const float *z, const float *gs,
                                                        int64_t n, float *gz, void *stream);

/*
 * Intervention rate ("Kolibri Pre-Training from Scratch" 9): the router's
 * own choice I^u_t = TopK(Z_t,:) (no bias; ties to the lower id) against the
 * routed ids; rate = 1 - (sum over tokens of |I^u_t and I_t|) / (N K).
 * Random routing gives 1 - K/E.  rate [1] double and overlaps [1] (the
 * summed overlap count) are device memory, written.
 */
KOLIBRI_API kolibri_status kolibri_intervention_rate(const float *z, const int32_t *ids, int64_t N,
                                                     int32_t E, int32_t K, double *rate,
                                                     unsigned long long *overlaps, void *stream);

/*
 * The expert layer ("Kolibri Pre-Training from Scratch" 6.1, with the
 * experts of "Kolibri 1 im Detail": every routed or shared expert a SwiGLU
 * MLP, two d -> F projections forming SiLU(gate) x up, then F -> d):
 *   y_t = f_shared(x_t) + sum_k S_t,k f_{e_t,k}(x_t),  f(x) = (SiLU(x Wg^T) * (x Wu^T)) Wd^T
 * with the gates S of kolibri_router_forward (unbiased sigmoid scores, not
 * renormalised) and the grouping of kolibri_expert_permute.
 *
 * Arithmetic: bf16 operands, fp32 accumulation on the tensor cores; the
 * activation h = SiLU(g) u is formed in fp32 and rounded once to bf16 (the
 * operand of the down projection); the routed outputs are kept in fp32 and
 * combined in fp32 multiply-adds in the order shared, k = 0 .. K-1.
 *
 * Layouts (row-major, bf16 unless noted, all 16-byte aligned):
 *   x [N, d]; perm [N*K] int32, offsets [E+1] int64, inv [N*K] int32 from
 *   kolibri_expert_permute; gates [N, K] fp32;
 *   w_gate_up [E, 2F, d]: per expert the F gate rows, then the F up rows;
 *   w_down [E, d, F]; shared expert ws_gate_up [2F, d], ws_down [d, F], or
 *   both NULL for a layer without one; y [N, d] fp32, written.
 * Shapes: d and F multiples of 256, 1 <= E <= 512,
 * N*K < 2^31 - 512.  Otherwise KOLIBRI_ERR_UNSUPPORTED_SHAPE.
 * ws: kolibri_expert_ffn_workspace_size(N, d, F, K, shared) bytes of device
 * memory (the gathered rows, h and the routed outputs; about
 * N K (6 d + 2 F) bytes), owned by the caller.  Out-of-range entries of perm
 * or inv are skipped and set KOLIBRI_ERR_DEVICE in kolibri_device_status;
 * offsets that do not start at 0, decrease, or pass N*K make the projections
 * store nothing and set the same status.
 */
KOLIBRI_API size_t kolibri_expert_ffn_workspace_size(int64_t N, int32_t d, int32_t F, int32_t K,
                                                     int32_t shared);
KOLIBRI_API kolibri_status kolibri_expert_ffn(const void *x, const int32_t *perm,
                                              const int64_t *offsets, const int32_t *inv,
                                              const float *gates, const void *w_gate_up,
                                              const void *w_down, const void *ws_gate_up,
                                              const void *ws_down, float *y, int64_t N, int32_t d,
                                              int32_t F, int32_t E, int32_t K, void *ws,
                                              size_t ws_bytes, void *stream);

/*
 * The four stages of kolibri_expert_ffn, each callable on its own:
 *   kolibri_expert_dispatch: x_perm [N*K, d] with x_perm[p] = x[perm[p] / K]
 *     (d a multiple of 8, at most 8192).
 *   kolibri_expert_gate_up: h [rows, F] bf16 = bf16(SiLU(a Wg^T) * (a Wu^T))
 *     where rows [offsets[g], offsets[g+1]) of a [rows, d] use expert g of
 *     w_gate_up [G, 2F, d]; offsets NULL: one group of all rows (G = 1).
 *   kolibri_expert_down: y [rows, d] fp32 = h Wd_g^T per group, w_down [G, d, F].
 *   kolibri_expert_combine: y [N, d] = y_shared (or 0 when NULL) + sum_k
 *     gates[t,k] y_perm[inv[t*K+k]] in fp32 multiply-adds, k ascending.
 */
KOLIBRI_API kolibri_status kolibri_expert_dispatch(const void *x, const int32_t *perm, int64_t N,
                                                   int32_t d, int32_t K, void *x_perm,
                                                   void *stream);
KOLIBRI_API kolibri_status kolibri_expert_gate_up(const void *a, int64_t rows,
                                                  const int64_t *offsets, int32_t G,
                                                  const void *w_gate_up, void *h, int32_t d,
                                                  int32_t F, void *stream);
KOLIBRI_API kolibri_status kolibri_expert_down(const void *h, int64_t rows, const int64_t *offsets,
                                               int32_t G, const void *w_down, float *y, int32_t d,
                                               int32_t F, void *stream);
KOLIBRI_API kolibri_status kolibri_expert_combine(const float *y_perm, const float *y_shared,
                                                  const int32_t *inv, const float *gates,
                                                  int64_t N, int32_t d, int32_t K, float *y,
                                                  void *stream);

/*
 * Diagnostic of the device-side failure path: launches one warp that waits,
 * through the same bounded wait the kernels use, on a shared-memory barrier
 * that nothing arrives at.  After about limit_ns nanoseconds (1e3 to 1e9,
 * else KOLIBRI_ERR_INVALID_ARG) the wait gives up, records
 * KOLIBRI_ERR_TIMEOUT in the device status word and the kernel returns, so
 * kolibri_device_status(stream) then reports the timeout and the context
 * stays usable.  Touches no caller memory.
 */
KOLIBRI_API kolibri_status kolibri_selftest_bounded_wait(uint64_t limit_ns, void *stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: KOLIBRI_OK, KOLIBRI_ERR_TIMEOUT or KOLIBRI_ERR_DEVICE
 * (the first recorded), or KOLIBRI_ERR_CUDA if the synchronisation failed.
 */
KOLIBRI_API kolibri_status kolibri_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KOLIBRI_ROUTER_H */
