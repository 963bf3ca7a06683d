/*
 * moe_zc.h -- C ABI of the B200 (sm_100a) MoE layer with zero-computation
 * experts.
 *
 * The layer (LongCat-Flash write-up "Meituan's large model goes viral for its
 * speed", itouyu.top, section "Zero-computation experts"): the expert pool
 * holds N SwiGLU FFN experts and Z zero-computation experts that return their
 * input unchanged.  A softmax router R scores all E = N + Z experts of each
 * token x_t; the expert bias b_i is added to those scores to pick the top K
 * experts, and the gate of each pick is its unbiased softmax probability.  So
 *
 *   p_t   = softmax(x_t W_r^T)                 over all E experts
 *   S_t   = top-K indices of p_t + b           (equal scores: lower index)
 *   out_t = sum_{i in S_t, i >= N} p_{t,i} x_t
 *         + sum_{i in S_t, i <  N} p_{t,i} W_down,i (SiLU(W_gate,i x_t) * W_up,i x_t)
 *
 * The page prints only the symbol glossary of this formula (the formula
 * itself is lost); the readings above -- softmax over all E experts, bias
 * added after the softmax and used for selection only, no renormalisation of
 * the gates, SwiGLU without biases -- are the plainest ones it supports.
 * The number of FFN experts a token runs varies from 0 to K.
 *
 * Data layout (all row-major, like nn.Linear.weight):
 *   x       [T, d]     bf16     tokens
 *   W_r     [E, d]     bf16     router; rows 0..N-1 FFN experts, N..E-1 zero experts
 *   b       [E]        fp32     expert bias (selection only)
 *   W_gate  [N, I, d]  bf16
 *   W_up    [N, I, d]  bf16
 *   W_down  [N, d, I]  bf16
 *   out     [T, d]     bf16
 *
 * Ownership and concurrency: every pointer argument of moe_zc_forward* is
 * device memory owned by the caller, 16-byte aligned, not freed or kept by the
 * library past the call's stream work.  The library owns one workspace per
 * device (grown on demand by moe_zc_forward*, or sized up front by
 * moe_zc_reserve) and the routing of the last forward.  It is not re-entrant:
 * one forward in flight per process; callers serialise.  Forward calls are
 * asynchronous on `stream` (a cudaStream_t, NULL = legacy default stream).
 *
 * Errors: every call returns a moe_zc_status; nothing aborts or traps.
 * Device-side waits are bounded; a wait that runs out sets a device flag that
 * moe_zc_synchronize / moe_zc_expert_load report as MOE_ZC_ERR_TIMEOUT.
 */
#ifndef MOE_ZC_H
#define MOE_ZC_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_zc_status {
  MOE_ZC_OK = 0,
  MOE_ZC_ERR_INVALID_ARG = -1,  /* null pointer, K < 1, K > E, T < 0, N < 0, Z < 0, E < 1 */
  MOE_ZC_ERR_UNSUPPORTED = -2,  /* d % 64, I % 128, K > 32, E > 1024, misaligned pointer */
  MOE_ZC_ERR_CUDA = -3,         /* a CUDA runtime or driver call failed */
  MOE_ZC_ERR_OOM = -4,          /* workspace allocation failed */
  MOE_ZC_ERR_TIMEOUT = -5,      /* a bounded device-side wait ran out */
  MOE_ZC_ERR_NO_RESULT = -6     /* no forward has run yet on this device */
} moe_zc_status;

/* Largest supported sizes. */
#define MOE_ZC_MAX_K 32
#define MOE_ZC_MAX_E 1024

/*
 * Forward pass of the layer defined above ("Zero-computation experts").
 * T may be 0 (no work, returns MOE_ZC_OK; x and out may then be NULL, and
 * the expert-load histogram of the call is all zero).  N may be 0 (every pick is a zero
 * expert) and Z may be 0 (plain softmax top-K MoE).  Requires d % 64 == 0,
 * I % 128 == 0, 1 <= K <= min(E, 32), E <= 1024, 16-byte aligned pointers.
 * W_gate/W_up/W_down may be NULL only when N == 0.
 * Asynchronous on `stream`; the expert-load histogram and routing of this
 * call stay available through moe_zc_expert_load / moe_zc_last_routing.
 * The call may be captured into a CUDA graph (stream capture on `stream`,
 * after moe_zc_reserve has sized the workspace, so that the captured call
 * allocates nothing): each replay recomputes the layer from the buffers the
 * call was given, and the result queries then wait for the whole device.
 * Batches of 1024 tokens or more leave a copy of their expert-load histogram
 * in pinned host memory (asynchronously); a later forward on the device uses
 * it to choose how the expert GEMMs are launched.  That choice changes speed
 * only: every launch gives the same bits.  A batch of at most 64 tokens is
 * two kernels: the router GEMM, then one grid of at most one block per
 * multiprocessor that routes the tokens, assigns their slots and copies
 * them, runs both expert GEMMs (down-projection tiles wait, bounded like
 * every device wait, for other blocks' gate/up results) and combines, with
 * bounded grid-wide barriers between those phases.  That grid is launched as
 * a cooperative launch, so the driver either makes all its blocks resident
 * at once or refuses it, and a refused launch (e.g. too few multiprocessors
 * free to this process) falls back to separate launches with the same bits
 * (moe_zc_plan shows the choice).
 */
int moe_zc_forward(const void* x, const void* W_r, const float* b,
                   const void* W_gate, const void* W_up, const void* W_down,
                   int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I,
                   void* out, void* stream);

/*
 * moe_zc_forward with an optional per-expert router-logit offset
 * (logit_offset [E] fp32 device memory, or NULL), added to x_t W_r^T before
 * the softmax, so it moves gates as well as picks.  It exists to skew expert
 * load in synthetic workloads; the write-up's layer has no such term.
 */
int moe_zc_forward_ex(const void* x, const void* W_r, const float* b,
                      const void* W_gate, const void* W_up, const void* W_down,
                      int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I,
                      const float* logit_offset, void* out, void* stream);

/*
 * moe_zc_forward_ex on HOST buffers: x_host [T, d] bf16 in, out_host [T, d]
 * bf16 out (page-locked memory for overlap; pageable memory works but its
 * copies do not overlap).  The weights, b and logit_offset stay device
 * memory.  The tokens go in chunks of chunk_tokens (<= 0: about T/4,
 * rounded up to 256 and at least 1024, with the first and the last chunk
 * half as long -- or all T at once when earlier forwards on the device hit
 * at least half of the FFN experts, as each chunk would then stream nearly
 * all expert weights again): while the kernels of one chunk run on
 * `stream`, the next chunk is copied in and the previous one out on two
 * streams of the library's own, so copies overlap compute.  Tokens are
 * independent, so each chunk's rows equal those of moe_zc_forward_ex on the
 * same chunk bit for bit (and those of one call on all T tokens wherever
 * the router GEMM slices K the same way for both batch sizes; where it does
 * not, logits differ in rounding only).  Asynchronous: out_host is
 * complete when `stream` is.  Afterwards moe_zc_expert_load reports the
 * histogram of all T tokens; moe_zc_last_routing and moe_zc_last_expert
 * describe the last chunk only.  Uses device staging for two chunks in and
 * two out (4 * chunk_tokens * d * 2 bytes) in the workspace.
 */
int moe_zc_forward_host(const void* x_host, const void* W_r, const float* b,
                        const void* W_gate, const void* W_up, const void* W_down,
                        int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I,
                        const float* logit_offset, void* out_host, int64_t chunk_tokens,
                        void* stream);

/*
 * Expert-load histogram of the last forward on the current device: the number
 * of tokens that picked each of the E experts, zero experts included.  This is
 * the "recent expert usage" that the write-up's bias controller (section
 * "Zero-computation experts") steers b_i by.  out_counts: host int32[E].
 * Waits for the last forward to finish; returns MOE_ZC_ERR_TIMEOUT if one of
 * its device waits ran out, MOE_ZC_ERR_NO_RESULT before the first forward.
 */
int moe_zc_expert_load(int32_t* out_counts);

/*
 * Routing of the last forward (for tests and debugging): idx host int32[T*K],
 * gate host float[T*K], row t holding token t's picks in descending biased
 * score (ties: lower index first).  Either pointer may be NULL.  Waits like
 * moe_zc_expert_load.
 */
int moe_zc_last_routing(int32_t* idx, float* gate);

/*
 * Intermediate activations of FFN expert e in the last forward (for tests):
 * the tokens routed to e in slot order (tokens, host int32[n]), their SwiGLU
 * hidden rows H (host bf16 [n, I]) and their expert outputs Y (host bf16
 * [n, d]) before gating.  *n_rows receives the count n; at most max_rows rows
 * are copied.  Any output pointer except n_rows may be NULL.
 */
int moe_zc_last_expert(int32_t e, int32_t max_rows, int32_t* n_rows,
                       int32_t* tokens, void* H, void* Y);

/*
 * Host-side PID controller of the expert biases (write-up, section
 * "Zero-computation experts": the biases follow recent expert usage through
 * a PID controller; no gains, set-point or window are given).  Plain host
 * code: it reads a histogram (e.g. from moe_zc_expert_load, summed over
 * ranks and steps as the caller sees fit) and writes new biases, which the
 * caller hands to the next forward.
 *
 *   set-point  zero experts together get target_zero_frac = rho of the
 *              tokens*K picks, FFN experts share the rest evenly:
 *              L*_i = (1-rho) tokens K / N (i < N), rho tokens K / Z (i >= N)
 *   error      e_i = (L*_i - counts_i) / (tokens K / E)
 *   update     b_i = base_i + clip(kp e_i + ki sum e_i + kd (e_i - e_prev,i))
 *
 * state: host float[3E] = [base | integral | previous error], set up by
 * moe_zc_bias_controller_init from the starting biases b (host float[E]).
 * moe_zc_bias_controller_step updates state and writes b (host float[E]).
 * max_shift <= 0 disables the clip.  rho must be 1 when N == 0 and 0 when
 * Z == 0.  Not thread-safe on a shared state.
 */
typedef struct moe_zc_pid {
  float target_zero_frac;
  float kp, ki, kd;
  float max_shift;
} moe_zc_pid;
int moe_zc_bias_controller_init(const float* b, int32_t E, float* state);
int moe_zc_bias_controller_step(const int32_t* counts, int32_t N, int32_t Z, int64_t tokens,
                                int32_t K, const moe_zc_pid* pid, float* state, float* b);

/*
 * FP8 (E4M3) block quantisation of one weight matrix, on the host (write-up,
 * section "System-level optimisation": fine-grained block quantisation as in
 * DeepSeek-V3).  Host reference of the FP8 formats; moe_zc_forward_fp8 takes
 * weights quantised on the device by moe_zc_fp8_quantize_weights.
 *   W       host bf16 [rows, cols], row-major (e.g. W_gate[e], [I, d])
 *   mode    MOE_ZC_FP8_BLOCK128: 128 x 128 blocks, scale = amax / 448 in fp32;
 *           MOE_ZC_FP8_MX32: 1 x 32 blocks along a row, scale = the smallest
 *           power of two with amax / scale <= 448
 *   codes   host uint8 [rows, cols]: E4M3 codes of W / scale (division in
 *           fp32), nearest value, ties to the even code, saturating at 448;
 *           E4M3 = sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 *           infinities, 0x7F / 0xFF NaN
 *   scales  host float [ceil(rows/br), ceil(cols/bc)] for br x bc blocks
 * A block of zeros, or holding a NaN or an infinity, gets scale 1.  Element (r, c)
 * stands for decode(codes[r, c]) * scales[r / br, c / bc].
 * Returns MOE_ZC_ERR_INVALID_ARG for null pointers, rows or cols < 1, or an
 * unknown mode.
 */
enum { MOE_ZC_FP8_BLOCK128 = 0, MOE_ZC_FP8_MX32 = 1 };
int moe_zc_fp8_quantize(const void* W, int64_t rows, int64_t cols, int32_t mode,
                        uint8_t* codes, float* scales);

/*
 * How moe_zc_forward would launch a batch of these sizes on a device with
 * `sms` multiprocessors, of which the one-grid expert GEMMs could hold
 * `resident_blocks` blocks at once (the forward passes its device's
 * occupancy).  Plain host code (no CUDA call); the forward takes its
 * decisions from the same function.
 *   kernels                 kernels one forward launches (0 for T = 0)
 *   router_grid             blocks of the router GEMM
 *   router_token_tile       tokens per router tile
 *   router_k_slices         contraction slices of the router GEMM (1: none)
 *   expert_gemms_one_grid   1: gate/up and down GEMMs in one persistent grid
 *                           (batches of at most 64 tokens whose grid can be
 *                           resident at once), 0: two launches
 *   expert_grid             blocks of that one grid, or of the gate/up GEMM
 *   one_grid_step           1: that grid also routes the tokens, assigns their
 *                           slots, copies them into the GEMM's token buffer
 *                           and combines the outputs (phases separated by grid
 *                           barriers), so the forward is two kernels: the
 *                           router GEMM and that grid
 * Returns the forward's argument-check status (nothing is written unless
 * MOE_ZC_OK), or MOE_ZC_ERR_INVALID_ARG for a NULL plan or sms < 1.
 */
typedef struct moe_zc_launch_plan {
  int32_t kernels;
  int32_t router_grid;
  int32_t router_token_tile;
  int32_t router_k_slices;
  int32_t expert_gemms_one_grid;
  int32_t expert_grid;
  int32_t one_grid_step;
} moe_zc_launch_plan;
int moe_zc_plan(int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I,
                int32_t sms, int32_t resident_blocks, moe_zc_launch_plan* plan);

/*
 * FP8 (E4M3) quantisation of one weight matrix ON THE DEVICE, in the
 * block-scaled form moe_zc_forward_fp8 takes (write-up, section
 * "System-level optimisation": fine-grained block quantisation; the form is
 * MOE_ZC_FP8_MX32's: 1 x 32 blocks along a row, scale = the smallest power of
 * two with amax / scale <= 448, codes of W / scale rounded to nearest, ties to
 * even; an all-zero or non-finite block gets scale 1).
 *   W       device bf16 [rows, cols], row-major (e.g. all of W_gate as
 *           [N * I, d]); rows % 128 == 0, cols % 128 == 0
 *   codes   device uint8 [rows, cols]: the E4M3 codes
 *   scales  device uint8 [rows * cols / 32]: each block's scale as a UE8M0
 *           byte (2^(byte - 127); blocks with amax < 448 * 2^-127 take
 *           byte 0), laid out in 512-byte atoms of 128 rows x 128 columns:
 *           the byte of row r and 32-column block k sits at
 *           ((r / 128) * (cols / 128) + k / 4) * 512 + (r % 32) * 16
 *             + ((r % 128) / 32) * 4 + k % 4
 *           (the order in which the tensor cores take scale factors)
 * Asynchronous on `stream`; allocates nothing.  Codes and scales equal
 * moe_zc_fp8_quantize(..., MOE_ZC_FP8_MX32, ...) of the same matrix (scales
 * there as floats in row-major order).  Returns MOE_ZC_ERR_INVALID_ARG for
 * null pointers or sizes < 1, MOE_ZC_ERR_UNSUPPORTED for sizes that are not
 * multiples of 128 or pointers not 16-byte aligned.
 */
int moe_zc_fp8_quantize_weights(const void* W, int64_t rows, int32_t cols, void* codes,
                                void* scales, void* stream);

/*
 * moe_zc_forward_ex with the gate and up projections in block-scaled FP8
 * (write-up, section "System-level optimisation", quantisation paragraph:
 * fine-grained block FP8, with the down projection -- whose input
 * activations reach extreme magnitudes -- kept in higher precision).
 * W_gate8 / W_up8 (device uint8 [N, I, d]) and W_gate_sf / W_up_sf are
 * moe_zc_fp8_quantize_weights of W_gate / W_up taken as [N * I, d]; W_down
 * stays bf16.  Each token's row is quantised the same way (1 x 32 blocks
 * along d) by the forward itself; the gate/up GEMM runs the tensor cores'
 * block-scaled FP8 MMA with fp32 accumulation; H, the down GEMM, the
 * router and the combine are those of moe_zc_forward.  Requires d % 128 == 0
 * besides moe_zc_forward's conditions.  The first FP8 forward on a device
 * grows the workspace by the quantised tokens (their count, rounded as for
 * the bf16 buffers, times d bytes) and their scales.
 */
int moe_zc_forward_fp8(const void* x, const void* W_r, const float* b, const void* W_gate8,
                       const void* W_gate_sf, const void* W_up8, const void* W_up_sf,
                       const void* W_down, int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K,
                       int32_t I, const float* logit_offset, void* out, void* stream);

/*
 * The forward's steps as separate calls, for expert parallelism across GPUs
 * (write-up, section "Shortcut-connected MoE": the expert computation sits
 * between a dispatch and a combine communication step; "System-level
 * optimisation": expert parallelism over many GPUs).  With the FFN experts
 * split into contiguous ranges, one per rank, a rank runs
 *   moe_zc_route     its tokens' picks, gates, zero-gate sums, histogram
 *   moe_zc_dispatch  its FFN picks' rows packed by expert, so the rows for
 *                    each rank's expert range are contiguous
 *   (the caller exchanges rows, their expert ids and counts between ranks)
 *   moe_zc_experts   the SwiGLU experts of its range on the rows it received
 *   (the caller sends the result rows back, in the order received)
 *   moe_zc_combine   out_t = zsum_t x_t + sum_k gate_{t,k} Y[slot_{t,k}]
 * Zero-expert picks never leave the rank: they are folded into zsum by
 * moe_zc_route.  All pointers are device memory (bf16 rows, int32 / fp32
 * arrays, 16-byte aligned row buffers); every call is asynchronous on
 * `stream`; device-side wait timeouts are reported by moe_zc_synchronize.
 * On one rank, route -> dispatch -> experts -> combine gives moe_zc_forward's
 * output bit for bit (the experts' rows are computed by the same GEMMs in the
 * same reduction order).
 *
 * moe_zc_route: x [T, d], W_r [E, d], b [E], logit_offset [E] or NULL as for
 *   moe_zc_forward_ex; writes idx [T*K], gate [T*K] (the unbiased softmax
 *   probabilities), zsum [T] (sum of the gates on zero experts) and counts
 *   [E] (histogram of all picks).  Uses the device workspace for logits.
 * moe_zc_dispatch: x [T, d], idx [T*K] and counts [>= N] from moe_zc_route;
 *   writes slot [T*K] (row of pick (t, k) in `send`, or -1 for a zero-expert
 *   pick), send [sum(counts[0..N-1]), d] (x rows grouped by expert, expert 0
 *   first, no padding; the order inside an expert is not fixed) and
 *   send_expert [same rows] (each row's expert).  N >= 1, d % 8 == 0.
 * moe_zc_experts: x_rows [R, d] and expert [R]: row i goes to FFN expert
 *   expert[i] - expert_base of the N given (W_gate [N, I, d], W_up, W_down
 *   [N, d, I]); y [R, d] receives E_e(x_i) in bf16 (rows whose expert lies
 *   outside [expert_base, expert_base + N) get zeros).  Conditions on d and
 *   I as for moe_zc_forward.  Runs the forward's dispatch, GEMMs and
 *   combine with gate 1, so moe_zc_last_routing, moe_zc_last_expert and
 *   moe_zc_expert_load describe this call afterwards.
 * moe_zc_combine: x [T, d], y_rows (the rows slot indexes), slot, gate
 *   [T*K], zsum [T] -> out [T, d] bf16: fp32 accumulation in k order, one
 *   rounding.  d % 8 == 0.
 */
int moe_zc_route(const void* x, const void* W_r, const float* b, const float* logit_offset,
                 int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t* idx,
                 float* gate, float* zsum, int32_t* counts, void* stream);
int moe_zc_dispatch(const void* x, const int32_t* idx, const int32_t* counts, int64_t T,
                    int32_t d, int32_t N, int32_t K, int32_t* slot, void* send,
                    int32_t* send_expert, void* stream);
int moe_zc_experts(const void* x_rows, const int32_t* expert, int32_t expert_base, int64_t R,
                   int32_t d, int32_t N, int32_t I, const void* W_gate, const void* W_up,
                   const void* W_down, void* y, void* stream);
int moe_zc_combine(const void* x, const void* y_rows, const int32_t* slot, const float* gate,
                   const float* zsum, int64_t T, int32_t d, int32_t K, void* out, void* stream);

/*
 * moe_zc_forward_fp8 on HOST buffers: x_host and out_host as for
 * moe_zc_forward_host (chunks whose copies overlap the kernels of their
 * neighbours), the weights as for moe_zc_forward_fp8.  Each chunk's rows
 * equal those of moe_zc_forward_fp8 on the same chunk bit for bit.
 */
int moe_zc_forward_host_fp8(const void* x_host, const void* W_r, const float* b,
                            const void* W_gate8, const void* W_gate_sf, const void* W_up8,
                            const void* W_up_sf, const void* W_down, int64_t T, int32_t d,
                            int32_t N, int32_t Z, int32_t K, int32_t I,
                            const float* logit_offset, void* out_host, int64_t chunk_tokens,
                            void* stream);

/* Wait for the last forward; report (and clear) a device-side timeout. */
int moe_zc_synchronize(void);

/*
 * Size the current device's workspace for forwards up to these sizes, so
 * later forwards allocate nothing.  Optional.
 */
int moe_zc_reserve(int64_t T, int32_t d, int32_t N, int32_t Z, int32_t K, int32_t I);

/* Free every device's workspace and cached state. */
void moe_zc_release(void);

/* Text for a status code. */
const char* moe_zc_status_string(int status);

/*
 * Per-stage timing of forwards with CUDA events recorded on the forward's own
 * stream between its kernels.  moe_zc_profile(1) starts (or restarts)
 * recording on the current device -- at most 256 forwards are kept --
 * moe_zc_profile(0) stops.  moe_zc_profile_read waits for the last recorded
 * forward and writes, for each stage i < max_stages, the milliseconds summed
 * over the recorded forwards (stage_ms: host float[max_stages]; 7 stages,
 * named by moe_zc_stage_name: router_gemm, route, assign_slots, permute,
 * gateup_gemm, down_gemm, combine) and their count to *n_forwards.  A batch
 * of at most 64 tokens runs both expert GEMMs as one kernel: its time is
 * under gateup_gemm, and down_gemm covers no kernel.
 */
int moe_zc_profile(int32_t enable);
int moe_zc_profile_read(float* stage_ms, int32_t max_stages, int32_t* n_forwards);
const char* moe_zc_stage_name(int32_t i);

/*
 * Routing without any device allocation.  The write-up has no counterpart to
 * this entry point: it exists for callers that cannot let a library call
 * cudaMalloc while they run -- e.g. a server that hands all device memory to
 * its own pool at start-up, or a process under a hard device-memory cap --
 * because a late allocation can fail, take memory promised elsewhere, or
 * synchronise the device mid-step.
 *
 * It computes exactly the routing part of moe_zc_forward_ex (same kernels):
 * idx (device int32 [T*K], picks in descending biased score), gate (device
 * float [T*K], unbiased softmax probabilities) and counts (device int32 [E],
 * expert-load histogram, cleared by the call).  x, W_r, b, logit_offset
 * (may be NULL) as for moe_zc_forward_ex.  dev_status (required, device
 * int32): the call clears it and the kernels set it non-zero if a bounded
 * wait (2 s) runs out; that is the only place such a timeout is reported,
 * so read it once the stream's work is done (NULL: MOE_ZC_ERR_INVALID_ARG).
 * Asynchronous on `stream`.
 *
 * Its scratch (fp32 logits and zero-gate sums) is one fixed array of
 * MOE_ZC_NOALLOC_SCRATCH_BYTES in the library image, held by every GPU that
 * loads the library until the process exits; sizes need
 * 256*ceil(T*E*4/256) + 256*ceil(T*4/256) <= that, else the call
 * returns MOE_ZC_ERR_UNSUPPORTED and launches nothing (e.g. E = 768 allows
 * T <= 1363).  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  All calls share the array and it keeps the
 * last call's contents, so calls whose GPU work overlaps (two streams or two
 * threads) race: serialise them.
 */
#define MOE_ZC_NOALLOC_SCRATCH_BYTES (4u << 20)
int moe_zc_route_noalloc(const void* x, const void* W_r, const float* b,
                         const float* logit_offset, int64_t T, int32_t d, int32_t N,
                         int32_t Z, int32_t K, int32_t* idx, float* gate, int32_t* counts,
                         int32_t* dev_status, void* stream);

/*
 * Test hook for the error paths: make the next n workspace allocations fail
 * (MOE_ZC_ERR_OOM), and/or make every bounded device wait of the next forward
 * give up after `wait_limit` nanoseconds (0 = the normal 2 s), so that the
 * timeout path runs without a fault.  (Device waits count SM clock cycles at
 * 2 per nanosecond: at clocks up to 2 GHz a wait lasts at least its limit.)
 * Not for production use.
 */
void moe_zc_test_inject(int32_t fail_allocs, int64_t wait_limit);

/*
 * Test hook for the launch paths of batches of at most 64 tokens (all give
 * the same bits): mode 1 never runs the two expert GEMMs in one grid (the
 * fallback path); mode 2 runs them in one grid but routes, dispatches and
 * combines in kernels of their own; 0 (or any other value) restores the
 * default, where the one grid does all but the router GEMM.  Not for
 * production use.
 */
void moe_zc_test_one_grid(int32_t mode);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ZC_H */
