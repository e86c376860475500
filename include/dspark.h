/*
 * dspark.h -- C ABI of libdspark.so: the data-parallel hot path of one DSpark
 * speculative-decoding round (Markov-head draft, rejection-sampling verify,
 * TV confidence labels, prefix survival, hardware-aware prefix scheduler) as
 * CUDA kernels for one NVIDIA B200 (sm_100a).
 *
 * Sources (three public web pages on DSpark):
 *   [P1] "大模型推理加速的系统级工程：DeepSeek V4-Pro DSpark 推测解码方案深度解析与开源工具链 DeepSpec"
 *        (austery.github.io)
 *   [P3] "DSpark Speculative Decoding" (lukebest.github.io concept note)
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the library
 *     never allocates, frees or keeps device memory between calls (the one fixed
 *     scratch array of dspark_verify_noalloc is part of the library image).
 *   - All tensors are dense and row-major (C order), with the shapes given.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL means the legacy default stream).  Outputs are valid once the stream
 *     has reached the call.
 *   - The return value is a dspark_status.  Argument errors are found on the
 *     host before anything is launched (DSPARK_EINVAL, nothing written).  A
 *     failed launch returns DSPARK_ECUDA.
 *   - Problems found in the DATA on the device never stop a call: they set bits
 *     in the per-request word flags[b] (bits below), which the caller zeroes
 *     before the round; calls OR their bits in.  Device-side waits are bounded;
 *     a wait that gives up sets DSPARK_FLAG_DEVICE_TIMEOUT in every flags word
 *     the kernel could reach and, where a workspace is passed, DSPARK_ETIMEOUT
 *     in its status word (dspark_workspace_status).
 *   - Scaled logits z = l * (1/T) are formed as the fp32 product of the fp32
 *     logit and the fp32 reciprocal of T; T == 0 selects greedy decoding
 *     (argmax, lowest index on ties).
 *   - Random numbers are inputs: uniforms in [0, 1) passed as fp32 tensors.
 */
#ifndef DSPARK_H_
#define DSPARK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSPARK_OK = 0,
  DSPARK_EINVAL = 1,    /* bad argument (null, size <= 0, gamma > 64, T < 0, bad dtype, workspace too small) */
  DSPARK_ECUDA = 2,     /* a CUDA launch or driver call failed */
  DSPARK_ENOTIMPL = 3,  /* shape outside what the kernels support (message in dspark_last_error) */
  DSPARK_ETIMEOUT = 4   /* a bounded device wait gave up (read through dspark_workspace_status) */
} dspark_status;

/* weight dtypes */
enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 };

/* layouts of the draft logits U and l_d (rows of V fp32 values):
 *   DSPARK_POSITION_MAJOR  [gamma, B, V]: step k of the draft reads and writes one contiguous
 *                          block of B rows (the fast layout: see dspark_markov_draft)
 *   DSPARK_REQUEST_MAJOR   [B, gamma, V]: as a backbone that emits all positions of a request
 *                          together writes them */
enum { DSPARK_POSITION_MAJOR = 0, DSPARK_REQUEST_MAJOR = 1 };

/* scheduler modes */
enum { DSPARK_SCHED_ARGMAX = 0, DSPARK_SCHED_EARLY_STOP = 1 };

/* workspace kinds for dspark_workspace_size */
enum { DSPARK_WS_DRAFT = 0, DSPARK_WS_VERIFY = 1, DSPARK_WS_SCHEDULE = 2, DSPARK_WS_RNN_DRAFT = 3 };

/* bits of flags[b] */
#define DSPARK_FLAG_DRAFT_NEAR_TIE    (1u << 0) /* |u - F| < 1e-6 at the drafted token, or greedy top-2 gap <= 1e-6*max(1,|z|) */
#define DSPARK_FLAG_ACCEPT_NEAR_TIE   (1u << 1) /* |u - p_t/p_d| < 1e-6 at a verified position */
#define DSPARK_FLAG_SAMPLE_NEAR_TIE   (1u << 2) /* |u - F| < 1e-6 at the residual or bonus token */
#define DSPARK_FLAG_SMALL_RESIDUAL    (1u << 3) /* residual mass < 1e-3 at the first rejection */
#define DSPARK_FLAG_NONFINITE         (1u << 4) /* NaN or +Inf among the logits (-Inf is a masked token) */
#define DSPARK_FLAG_TOKEN_RANGE       (1u << 5) /* a token id outside [0, V) */
#define DSPARK_FLAG_CONF_RANGE        (1u << 6) /* a confidence outside [0, 1] */
#define DSPARK_FLAG_SCHED_NEAR_TIE    (1u << 7) /* the chosen D is within 1e-12 (relative) of another */
#define DSPARK_FLAG_RAGGED_OFFSETS    (1u << 8) /* flattened l_t: lt_off[b+1] - lt_off[b] != L[b] + 1, or outside [0, lt_nrows] */
#define DSPARK_FLAG_DEVICE_TIMEOUT    (1u << 31)

/* Human-readable name of a status code. */
const char* dspark_status_string(int status);

/* Text of the last host-side error of this thread ("" if none). */
const char* dspark_last_error(void);

/* Tuning knobs (process-wide, host side; no effect on results beyond the choice of kernel and,
 * within the stated tolerances, the order of floating-point sums):
 *   "draft_tc_min_b"  bf16 drafts with B >= value use the tensor-core main pass (default 1: at
 *                     gamma = 16, V = 151936 it was measured faster at every B, 0.38 against
 *                     0.41 ms at B = 1 and 0.40 against 1.36 ms at B = 8)
 *   "draft_path"      0 automatic, 1 always the CUDA-core GEMV pass, 2 always tensor cores
 *   "draft_pdl"       1 (default) chain draft kernels with programmatic dependent launch
 *   "draft_fused"     1 (default) tensor-core draft: all gamma positions in one cooperative
 *                     launch with grid barriers (falls back to one launch pair per position
 *                     when the grid cannot be co-resident); 0 always one pair per position
 *   "verify_impl"     verification with a workspace (V % 4 == 0, 16-byte aligned rows):
 *                     0 (default) the streaming kernels; 1 the column-sliced kernels (every row
 *                     read from HBM once, rows exchanged through L2; slower at the sizes measured);
 *                     2 the per-row cluster kernels.  Calls the chosen kernels cannot take fall
 *                     back to the next ones and finally to the per-row kernels.
 *   "verify_stream_cluster"  CTAs per cluster of the streaming verify, 1..16; 0 (default) picks 3,
 *                     or 6 when B*(gamma+1) is below 4/3 of the SM count (few rows per cluster)
 *   "verify_stream_l2hint"   1 (default) first-pass copies evict-last, second-pass evict-first
 *   "verify_groups"   column-sliced verify: CTA groups (0: slices of about 16 KB per row)
 *   "verify_cluster"  0 automatic, else the cluster size of the per-row verify kernels (1..16,
 *                     power of 2)
 *   "verify_persistent" 1 (default) per-row sampled verification and labels run on persistent
 *                     clusters with double-buffered rows; 0 one cluster per row
 *   "sm_count"        0 query the device, else the SM count used to size persistent grids
 *   "debug_wait_limit", "debug_unreachable_barrier"  test-only: the first shortens the bounded
 *                     device waits (draft: polls per wait; streaming verify: nanoseconds; 0: the
 *                     defaults of about a second and 2 s); the second makes one wait unsatisfiable
 *                     (1: the fused draft's first grid barrier, 2: the streaming verify's cluster
 *                     exchange), so that a test can check that the kernel returns with
 *                     DSPARK_ETIMEOUT in the workspace status and DEVICE_TIMEOUT in the flags
 * The environment variables DSPARK_DRAFT_TC_MIN_B, DSPARK_DRAFT_PATH, DSPARK_DRAFT_PDL,
 * DSPARK_DRAFT_FUSED, DSPARK_VERIFY_CLUSTER, DSPARK_VERIFY_PERSISTENT, DSPARK_VERIFY_IMPL,
 * DSPARK_VERIFY_GROUPS and DSPARK_VERIFY_STREAM_CLUSTER set the initial values of the keys of the
 * same names.
 * Returns DSPARK_EINVAL for an unknown key. */
int dspark_set_option(const char* key, long value);

/* Device workspace bytes an entry point needs for the given sizes (r is used by
 * DSPARK_WS_DRAFT only).  Returns 0 for an unknown kind.  The workspace holds
 * per-call scratch only: its contents need not be preserved between calls. */
size_t dspark_workspace_size(int which, int B, int gamma, int V, int r);

/* Read the status word of a workspace after the stream has reached the call
 * that used it (synchronous copy).  Returns DSPARK_OK or DSPARK_ETIMEOUT. */
int dspark_workspace_status(const void* ws, void* stream);

/* --------------------------------------------------------------------------
 * dspark_markov_draft -- the Markov-head sequential draft stage.
 *
 * [P3 §Semi-Autoregressive Generation] p_k(v) ∝ exp(U_k(v) + B_k(v)) with the
 * low-rank Markov bias B_k = W1[x_{k-1}] · W2 (rank r); [P1 §"DSpark 架构设计：
 * 半自回归生成与马尔可夫修正"] the head only looks at the previous sampled token and
 * fills the block left to right.  For each request b and k = 1..gamma:
 *     l_d[k,b,:] = U[k,b,:] + W1[x_{k-1}, :] · W2        (x_0 = x0[b])
 *     x_k        = min{ v : sum_{w<=v} exp(z_w - max z) > u_draft[b,k] * sum_w exp(z_w - max z) },
 *                  z = l_d[k,b,:] * (1/T)              (T > 0)
 *     x_k        = argmax_v l_d[k,b,v], lowest index    (T == 0)
 *
 * U        fp32 base logits of the parallel stage, [gamma, B, V] (layout DSPARK_POSITION_MAJOR)
 *          or [B, gamma, V] (DSPARK_REQUEST_MAJOR).  Step k reads and writes one position of
 *          every request; position-major keeps those B rows in one contiguous block.
 * layout   DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR, for U and ld_out alike.
 * W1       [V, r]  and  W2 [r, V]   Markov-head factors, dtype w_dtype
 *          (DSPARK_BF16 or DSPARK_F32), fp32 accumulation.
 * x0       [B] int32    last committed token of each request (must be in [0, V)).
 * u_draft  [B, gamma] fp32 uniforms in [0, 1) (ignored when T == 0).
 * x_out    [B, gamma] int32   drafted tokens.
 * ld_out   raw draft logits l_d (U + bias) in the layout of U, kept for verify.
 * flags    [B] uint32   OR'ed with DRAFT_NEAR_TIE / NONFINITE / TOKEN_RANGE.
 * ws       workspace of at least dspark_workspace_size(DSPARK_WS_DRAFT, B, gamma, V, r) bytes.
 * Limits: 1 <= gamma <= 64, B >= 1, V >= 2, r >= 1, T >= 0.
 * -------------------------------------------------------------------------- */
int dspark_markov_draft(const float* U, const void* W1, const void* W2, int w_dtype,
                        const int32_t* x0, const float* u_draft,
                        int B, int gamma, int V, int r, float T, int layout,
                        int32_t* x_out, float* ld_out, uint32_t* flags,
                        void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * dspark_rnn_draft -- the draft stage with the recurrent (RNN) head instead of the Markov head.
 *
 * [P1 §"DSpark 架构设计：半自回归生成与马尔可夫修正"] the optional RNN head keeps and updates a
 * hidden state that accumulates the whole drafted prefix (the pages find its small accuracy gain
 * not worth the cost and keep the Markov head in production); [P3 §Semi-Autoregressive
 * Generation] p_k(v) ∝ exp(U_k(v) + B_k(x_<k, v)) with a recurrent state inside the block.
 * The pages give no functional form.  Reading taken (rank r, as the Markov head):
 *     h_{-1} = 0,  x_{-1} = x0,  h_k = tanh(W1[x_{k-1}] + h_{k-1} W_h),  l_d[k] = U_k + h_k W2
 * so that W_h = 0 is the Markov head on tanh(W1).  The state is fp32 and the whole stage runs
 * on the CUDA-core pass (one state kernel, one main pass and one combine per position); the
 * fused tensor-core launch is not used (it would round the state to bf16).
 * Wh      [r, r] in w_dtype, row i multiplies h[i].
 * h_out   [B, gamma, r] fp32 device or NULL: the states h_k.
 * ws      dspark_workspace_size(DSPARK_WS_RNN_DRAFT, B, gamma, V, r) bytes.
 * Other arguments, outputs, flags and limits as dspark_markov_draft; r <= 1024.
 * -------------------------------------------------------------------------- */
int dspark_rnn_draft(const float* U, const void* W1, const void* W2, const void* Wh, int w_dtype,
                     const int32_t* x0, const float* u_draft, int B, int gamma, int V, int r, float T, int layout,
                     int32_t* x_out, float* ld_out, float* h_out, uint32_t* flags,
                     void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * dspark_verify -- lossless rejection-sampling verification of the drafted block.
 *
 * [P1 §"大模型推理的显存瓶颈与推测解码的演进逻辑"] the target checks the drafted tokens
 * left to right, keeps the longest prefix that passes the rejection-sampling
 * test, resamples one token at the first failure and drops the rest;
 * [P3, opening paragraph] longest consistent prefix plus a bonus token.
 * For each request b with L = L[b] (gamma when L is NULL):
 *     p_d,k = softmax(l_d[k,b] / T),  p_t,k = softmax(l_t[b,k] / T)
 *     accept position k (k = 0..L-1, in order) iff u_acc[b,k] * p_d,k(x_k) < p_t,k(x_k)
 *     n = number of leading accepted positions
 *     n < L : y_n ~ max(0, p_t,n - p_d,n) / Z   (inverse CDF with u_res[b];
 *             Z == 0 falls back to p_t,n)
 *     n == L: y_L ~ p_t,L (the bonus row)       (inverse CDF with u_res[b])
 *     T == 0: accept iff x_k == argmax l_t,k; the resampled/bonus token is argmax l_t,n.
 *
 * ld     fp32 draft logits, [gamma, B, V] or [B, gamma, V] as ld_layout says (dspark_markov_draft's
 *        ld_out).
 * ld_layout  DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR.
 * lt     [B, gamma+1, V] fp32 target logits (row gamma = bonus position).
 * x      [B, gamma] int32 drafted tokens.
 * L      [B] int32 verify lengths in [0, gamma] (e.g. from dspark_prefix_schedule), or NULL.
 * u_acc  [B, gamma] fp32, u_res [B] fp32 uniforms in [0, 1).
 * n_acc  [B] int32 accepted count n.
 * y_out  [B, gamma+1] int32: y[0..n-1] = x[0..n-1], y[n] = resampled/bonus token, rest -1.
 * c_star [B, gamma] fp32 TV labels of every position (as dspark_tv_labels), or NULL.
 * flags  [B] uint32 OR'ed with ACCEPT_NEAR_TIE / SAMPLE_NEAR_TIE / SMALL_RESIDUAL /
 *        NONFINITE / TOKEN_RANGE.
 * ws     workspace of at least dspark_workspace_size(DSPARK_WS_VERIFY, B, gamma, V, 0) bytes.
 * Rows of l_t beyond L[b] (and rows of l_d at or beyond L[b]) are not read
 * unless c_star is requested.
 * -------------------------------------------------------------------------- */
int dspark_verify(const float* ld, const float* lt, const int32_t* x, const int32_t* L,
                  const float* u_acc, const float* u_res,
                  int B, int gamma, int V, float T, int ld_layout,
                  int32_t* n_acc, int32_t* y_out, float* c_star, uint32_t* flags,
                  void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * dspark_ragged_layout -- row offsets and token tags of a flattened verify block.
 *
 * [P1 §"极致的工程实现与内核优化", inference paragraph] all tokens a batch verifies are
 * flattened into one contiguous 1-D array without padding, and a light token-tag tensor
 * tells which sequence, and where in it, each token belongs; [P3 §Confidence-Scheduled
 * Verification, production notes] variable-length verify over flattened tokens with a
 * marker tensor.  Request b (verify length L_b, clamped to [0, gamma]) owns the L_b + 1 rows
 *     lt_off[b] .. lt_off[b] + L_b,  lt_off[0] = 0,  lt_off[b+1] = lt_off[b] + L_b + 1,
 * its L_b verified positions and the resample/bonus position; lt_off[B] is the row count.
 * L       [B] int32 device (e.g. dspark_prefix_schedule's L_out).
 * lt_off  [B+1] int64 device, written.
 * tags    [B*(gamma+1)] int32 device or NULL: row lt_off[b] + k gets b*(gamma+1) + k; the
 *         entries past lt_off[B] get -1.
 * One CTA; no workspace.
 * -------------------------------------------------------------------------- */
int dspark_ragged_layout(const int32_t* L, int B, int gamma, int64_t* lt_off, int32_t* tags, void* stream);

/* --------------------------------------------------------------------------
 * dspark_verify_ragged -- dspark_verify over a flattened target block.
 *
 * The same verification as dspark_verify with L given, reading request b's target row k
 * (k = 0..L_b) from row lt_off[b] + k of the flattened lt instead of row k of a padded
 * [B, gamma+1, V] block: the target forward then computes and stores only the
 * sum over b of (L_b + 1) rows that verification uses (dspark_ragged_layout gives
 * lt_off).  Results equal dspark_verify's on the padded block holding the same rows.
 * lt        [lt_nrows, V] fp32 device, the flattened target logits.
 * lt_off    [B+1] int64 device row offsets.  Offsets that do not give request b exactly
 *           L_b + 1 rows inside [0, lt_nrows] set RAGGED_OFFSETS in flags[b]; every row
 *           index is clamped into [0, lt_nrows - 1], so the call never reads outside lt
 *           (that request's results are then meaningless).
 * L         [B] int32 verify lengths, required.
 * c_star    [B, gamma] fp32 or NULL: TV labels at the positions k <= min(L_b, gamma-1) whose
 *           target row the block holds; NaN at the others.
 * Other arguments, flags and the workspace as dspark_verify.  The streaming kernels run
 * (verify_impl 0); with verify_impl 1 or 2 the per-row kernels do.
 * -------------------------------------------------------------------------- */
int dspark_verify_ragged(const float* ld, const float* lt, const int64_t* lt_off, int64_t lt_nrows,
                         const int32_t* x, const int32_t* L, const float* u_acc, const float* u_res,
                         int B, int gamma, int V, float T, int ld_layout,
                         int32_t* n_acc, int32_t* y_out, float* c_star, uint32_t* flags,
                         void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * dspark_verify_noalloc -- dspark_verify without a caller workspace.
 *
 * The pages have no counterpart to this entry point: it exists for callers that
 * cannot provide device scratch when they verify -- a serving engine that has
 * reserved nearly all of HBM for its KV cache and allows no further allocation
 * while decoding, or plugin code that gets raw device pointers from a host
 * framework but no access to its allocator.  Arguments, results and flags are
 * those of dspark_verify; the scratch is a fixed array inside libdspark.so
 * (213,248 bytes per GPU, held from load until the process exits), so the call
 * allocates and frees nothing.  It always runs the per-row cluster kernels, whose
 * scratch does not grow with V (results equal dspark_verify's within the stated
 * tolerances; tokens and lengths agree except at flagged near-ties).
 * Limits: B <= 4096 and B*(gamma+1) <= 16384, else DSPARK_EINVAL with a message;
 * V <= 409600 (one 16-CTA cluster per row), else DSPARK_ENOTIMPL.
 * The first call on a device (and the first after its context was destroyed and
 * recreated) looks up the array's device address; make that first call before any
 * stream capture.  All calls share the array and each clears the parts that must
 * start at zero: calls whose kernels overlap on the GPU race.
 * -------------------------------------------------------------------------- */
int dspark_verify_noalloc(const float* ld, const float* lt, const int32_t* x, const int32_t* L,
                          const float* u_acc, const float* u_res,
                          int B, int gamma, int V, float T, int ld_layout,
                          int32_t* n_acc, int32_t* y_out, float* c_star, uint32_t* flags, void* stream);

/* --------------------------------------------------------------------------
 * dspark_tv_labels -- confidence-head supervision labels.
 *
 * [P3 §Confidence-Scheduled Verification] c*_k = 1 - ½ ‖p_d,k - p_t,k‖₁;
 * [P1 §"硬件感知与置信度自适应调度机制"] the label is the analytic acceptance rate
 * obtained from the total-variation distance.  For every b and k = 0..gamma-1.
 * T == 0: c* = 1 if the argmaxes agree, else 0.
 *
 * ld      fp32 draft logits in the layout ld_layout names, as in dspark_verify.
 * lt      [B, lt_rows, V] fp32, lt_rows = gamma or gamma+1 (row stride of lt);
 *         only the first gamma rows of each request are read.
 * c_star  [B, gamma] fp32.
 * No workspace.
 * -------------------------------------------------------------------------- */
int dspark_tv_labels(const float* ld, const float* lt, int B, int gamma, int V, int lt_rows,
                     float T, int ld_layout, float* c_star, void* stream);

/* --------------------------------------------------------------------------
 * dspark_sts_fit -- sequential temperature scaling of the confidences, fitted on a validation set.
 *
 * [P1 §"硬件感知与置信度自适应调度机制"] the raw confidence head is over-confident; on a
 * validation set a 1-D grid search per candidate position finds the temperature that
 * calibrates it (expected calibration error from 3-8 % to about 1 %); temperature scaling
 * keeps the order of the confidences.  [P3 §Confidence-Scheduled Verification] STS
 * calibrates the cumulative product position by position.  Reading taken:
 *     scaled(c, tau) = sigma(logit(c) / tau)      (fp64; c clamped to [0, 1], NaN as 0)
 *     for k = 0 .. gamma-1, in order:
 *       s_i      = 1 if n_acc[i] >= k + 1 (sample i's positions 0..k all accepted), else 0
 *       a'_i(t)  = prod_{j<k} scaled(c[i,j], tau[j]) * scaled(c[i,k], t)
 *       ECE(t)   = sum over M equal-width bins of |sum_{i in bin} (s_i - a'_i(t))| / N
 *                  (bin of p: min(floor(p M), M - 1))
 *       tau[k]   = grid[j] for the first j minimising ECE(grid[j])
 *     ece_raw[k] is the ECE of the raw products prod_{j<=k} c[i,j].
 * c          [N, gamma] fp32 raw confidences.    n_acc  [N] int32 accepted counts.
 * grid       [n_grid] fp64 candidate temperatures (> 0).
 * tau_out    [gamma] fp64 (required);  index_out [gamma] int32, ece_raw / ece_cal [gamma] fp64,
 *            curve_out [gamma, n_grid] fp64 (ECE of every candidate) -- each may be NULL.
 * ws         dspark_sts_workspace_size(N, gamma, n_grid, n_bins) bytes, 256-byte aligned.
 * Limits: gamma <= 64, (n_grid + 1) * n_bins <= 25600.  2 * gamma launches on `stream`.
 * fp64 sums in atomic order: ECE values agree with a serial sum to about 1e-15.
 * -------------------------------------------------------------------------- */
size_t dspark_sts_workspace_size(int64_t N, int gamma, int n_grid, int n_bins);
int dspark_sts_fit(const float* c, const int32_t* n_acc, int64_t N, int gamma, const double* grid, int n_grid,
                   int n_bins, double* tau_out, int32_t* index_out, double* ece_raw, double* ece_cal,
                   double* curve_out, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * dspark_sts_apply -- calibrated confidences of a round: c_out[b,k] = fp32(scaled(c[b,k], tau[k]))
 * (the scaling of dspark_sts_fit, rounded once to fp32), ready for dspark_prefix_schedule.
 * c, c_out [B, gamma] fp32 (may be the same array);  tau [gamma] fp64.  No workspace.
 * -------------------------------------------------------------------------- */
int dspark_sts_apply(const float* c, const double* tau, int B, int gamma, float* c_out, void* stream);

/* --------------------------------------------------------------------------
 * dspark_prefix_schedule -- prefix survival + greedy hardware-aware prefix scheduler.
 *
 * [P3 §Confidence-Scheduled Verification] a_{b,j} = ∏_{i<=j} c_{b,i} and
 * Algorithm 1, maximise Θ = τ · SPS(B); [P1 §"硬件感知与置信度自适应调度机制"] all
 * candidate tokens are sorted by survival and added one at a time while the
 * expected throughput rises; the global search runs on the GPU.
 *     a     = running product of c along each request, fp32, left to right
 *     order = all B*gamma items by (a descending, b ascending, j ascending)
 *     S(D)  = sum of the first D survivals in that order (fp64)
 *     Θ(D)  = (B + S(D)) * sps[D],  D = 0..D_max
 *     D*    = ARGMAX: the smallest D attaining max Θ;
 *             EARLY_STOP: the first D with Θ(D+1) <= Θ(D), else D_max
 *     L[b]  = number of request b's items among the first D*.
 *
 * c          [B, gamma] fp32 confidences (conditional pass probabilities).
 * sps        [D_max+1] fp64 steps/s of the verify forward with D scheduled drafts.
 * D_max      token budget, 0 <= D_max <= B*gamma.
 * L_out      [B] int32.   a_out [B, gamma] fp32 or NULL.   theta_out [1] fp64 (Θ(D*)).
 * flags      [B] uint32 or NULL: CONF_RANGE for requests with c outside [0, 1];
 *            SCHED_NEAR_TIE in every word when the decision is within 1e-12.
 * Limits: B*gamma <= 16384.  No workspace (ws may be NULL, ws_bytes 0).
 * -------------------------------------------------------------------------- */
int dspark_prefix_schedule(const float* c, const double* sps, int B, int gamma, int D_max, int mode,
                           int32_t* L_out, float* a_out, double* theta_out, uint32_t* flags,
                           void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * dspark_prefix_schedule_t2 -- asynchronous scheduling: step t's capacity from step t-2.
 *
 * [P1 §"硬件感知与置信度自适应调度机制", last paragraph] the truncation of step t is
 * decided from the confidence history of step t-2, so the global search runs inside the
 * GPU pipeline, needs no host handshake and is compatible with CUDA-graph replay and
 * zero-overhead scheduling; [P3 §Confidence-Scheduled Verification, production notes,
 * "asynchronous"] confidences from two steps earlier predict the batch capacity K.
 * Reading taken: only the capacity comes from step t-2.  For the step t held in the ring,
 *     K_t   = D*_{t-2} (the search result of dspark_prefix_schedule on step t-2's c), or
 *             K_init for t < 2 (K_init < 0: D_max); clamped to [0, D_max]
 *     L[b]  = number of request b's items among the first K_t of THIS step's survival order
 *     Θ     = (B + S_t(K_t)) * sps[K_t]  -> theta_out
 * and the launch also runs the full search on this step's c (mode ARGMAX or EARLY_STOP),
 * stores D*_t in the ring for step t+2 and advances the ring's step counter.  With c, sps
 * and the ring in device memory, one captured graph replays the round step after step.
 *
 * ring   DSPARK_T2_RING_BYTES of device memory, 8-byte aligned, owned by the caller, zeroed
 *        (e.g. cudaMemsetAsync) before the first step of a sequence; one ring per sequence,
 *        calls on it ordered on one stream.  Layout (read it after a step to steer the host):
 *          offset  0  int64   t          steps taken
 *          offset  8  int32   D[4]       D*_s of step s at D[s % 4]
 *          offset 24  uint32  tie[4]     1 if that decision was within 1e-12 of another D
 *          offset 40  fp64    theta[4]   Θ_s(D*_s)
 *          offset 72  int32   K[4]       capacity applied at step s
 *        B may change from step to step (a capacity is clamped to the new D_max).
 * K_out  [1] int32 or NULL: K_t.   flags: CONF_RANGE as above; SCHED_NEAR_TIE in every
 *        word when the decision that produced K_t was a near-tie.
 * Other arguments and limits as dspark_prefix_schedule.  No workspace.
 * -------------------------------------------------------------------------- */
#define DSPARK_T2_RING_BYTES 128
int dspark_prefix_schedule_t2(const float* c, const double* sps, int B, int gamma, int D_max, int mode,
                              int K_init, void* ring, int32_t* L_out, float* a_out, double* theta_out,
                              int32_t* K_out, uint32_t* flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H_ */
