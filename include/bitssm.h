/*
 * bitssm.h - C ABI of the BitSSM forward library for NVIDIA B200 (sm_100a).
 *
 * BitSSM is the selective state-space sequence mixer of TriSSM whose
 * projections are BitNet b1.58 BitLinear layers: ternary {-1, 0, +1} weights
 * and int8 activations ("Associative Recall Under Ternary Quantization: A
 * Controlled Comparison of State Space Models and Transformers at 5M
 * Parameters", TriSSM repository README: opening paragraph, the caption "The
 * BitSSM sequence mixer", the Overview table and "Repository structure").
 * The W1.58A16 variant (16-bit activations, grouped weight scales) follows
 * "Ternary Mamba: Grouped Quantization-Aware Training of W1.58A16 State
 * Space Models" (abstract).
 *
 * Conventions shared by every entry point:
 *  - Tensor arguments are DEVICE pointers owned by the caller, row-major and
 *    densely packed unless a leading dimension is stated.  Structs
 *    (bitssm_tw, bitssm_layer) are HOST memory; their pointer fields are
 *    device pointers.  The library keeps no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work on that stream and return without
 *    synchronising; results are ready when the stream reaches them.
 *  - The forward entry points allocate no device memory: scratch comes from
 *    the caller's workspace `ws` of `ws_bytes` bytes (256-byte aligned),
 *    sized by the matching *_workspace_size query.
 *  - Return value: BITSSM_OK, or an error status.  Argument errors are
 *    detected on the host before anything is enqueued.  BITSSM_ERR_CUDA
 *    reports a launch error.  Device-side conditions (a bounded wait that ran
 *    out) are recorded in a device error word read by bitssm_device_error().
 *  - Element types: BITSSM_F32 (float), BITSSM_BF16 (bfloat16 bits),
 *    BITSSM_I32 (int32, only as a raw-accumulator output).
 *  - The library computes on the current CUDA device; pointers must belong
 *    to it.
 */
#ifndef BITSSM_H
#define BITSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BITSSM_ABI_VERSION 2

enum bitssm_status_code {
  BITSSM_OK = 0,
  BITSSM_ERR_INVALID_ARG = 1,      /* null pointer, negative size, bad enum */
  BITSSM_ERR_UNSUPPORTED_SHAPE = 2,/* a size the library does not support */
  BITSSM_ERR_WORKSPACE = 3,        /* workspace missing, misaligned or too small */
  BITSSM_ERR_CUDA = 4,             /* a CUDA launch or runtime call failed */
  BITSSM_ERR_TIMEOUT = 5,          /* a bounded device wait ran out (device error word) */
  BITSSM_ERR_DEVICE_FLAG = 6       /* another device-side check failed */
};

enum bitssm_dtype { BITSSM_F32 = 0, BITSSM_BF16 = 1, BITSSM_I32 = 2, BITSSM_I16 = 3 };

/* Activation modes.  A8: per-token absmax int8 activation codes (BitNet
 * b1.58; TriSSM README opening paragraph).  A16: bf16 activations without
 * activation quantisation, weights with per-group scales (W1.58A16; Ternary
 * Mamba abstract). */
enum bitssm_act_mode { BITSSM_A8 = 0, BITSSM_A16 = 1 };

/* Ternary weight matrix W_q [n_out, k_in] in the 2-bit encoding:
 *   packed: uint8 [n_out, ceil(k_in/4)]; element (n, k) is the code
 *           c = w + 1 in {0, 1, 2} at bits 2*(k mod 4) of byte k/4 of row n;
 *           code 3 is invalid; padding elements hold c = 1 (w = 0).
 *   scales: float absmean scales; group == 0: one float (per matrix);
 *           group == 128: float [n_out, ceil(k_in/128)], scale of each run
 *           of 128 consecutive k of one row.
 * A8 layers use group 0; A16 layers use group 128. */
typedef struct bitssm_tw {
  const uint8_t* packed;
  const float* scales;
  int n_out;
  int k_in;
  int group;
} bitssm_tw;

/* Weights of one BitSSM mixer.  Shapes (d = d_model, E = d_inner,
 * N = d_state, R = dt_rank):
 *   in_proj  [E, d]    dt_down [R, E]   b_proj [N, E]   c_proj [N, E]
 *   dt_up    [E, R]    out_proj [d, E]
 *   A [E, N] float (the negative decay rates), D [E] float (skip),
 *   dt_bias [E] float (added before the softplus).
 * `prepared` may point to a device buffer filled by bitssm_prepare_weights()
 * for this layer and act mode (the weights expanded to tensor-core operand
 * form), or be NULL: the forward then expands them into its workspace on
 * every call.  `flags`: 0, or BITSSM_KEEP_CODES to have the forward also
 * store the int8 activation codes of x, u and y in its workspace (see
 * bitssm_workspace_layout; for stage-by-stage checks). */
#define BITSSM_KEEP_CODES 1
/* Mamba-1 block form (d_conv != 0; A8 only, from a zero state): the layer
 * additionally has a gate branch and a depthwise causal conv on u,
 *   u_pre = BitLinear(x; in_proj),  z = BitLinear(x; z_proj)  (one set of
 *           int8 codes of x feeds both; z_proj [E, d], its own scale),
 *   u     = SiLU(conv_b[e] + sum_k conv_w[e, k] * u_pre[t - (d_conv-1) + k, e])
 *           (left zero padding: tap d_conv-1 is the current step),
 *   x_proj, Delta, scan as in the mixer, on u (its codes from its float
 *   value), then y_g = y * SiLU(z) and out = BitLinear(y_g; out_proj).
 * None of the pages names these pieces; they are the parts of the Mamba-1
 * block around the same selective scan.  conv_w: float [E, d_conv] (device),
 * conv_b: float [E] (device) or NULL for zero bias, 1 <= d_conv <= 4.  With
 * d_conv == 0 the fields z_proj, conv_w and conv_b are ignored. */
typedef struct bitssm_layer {
  bitssm_tw in_proj, dt_down, b_proj, c_proj, dt_up, out_proj;
  const float* A;
  const float* D;
  const float* dt_bias;
  int d_model;
  int d_inner;
  int d_state;
  int dt_rank;
  const void* prepared;
  int flags;
  bitssm_tw z_proj;
  const float* conv_w;
  const float* conv_b;
  int d_conv;
} bitssm_layer;

/* Version of this ABI (BITSSM_ABI_VERSION). */
int bitssm_version(void);

/* Static, NUL-terminated description of a status code (never NULL). */
const char* bitssm_status_string(int status);

/* Name and description of the last CUDA error a call of this library saw on
 * the calling thread (behind a BITSSM_ERR_CUDA status); "no error" before
 * any.  The string stays valid until the thread's next failing call. */
const char* bitssm_last_error(void);

/* Reads the device error word of the current device into *flags (bit 0: a
 * TMA wait ran out, bit 1: an MMA-completion wait ran out, bit 2: an
 * epilogue wait ran out, bit 3: the wait of bitssm_selftest_wait) after
 * synchronising the device; clears it when `clear` is non-zero.  Returns
 * BITSSM_OK, or BITSSM_ERR_TIMEOUT when any bit was set, or BITSSM_ERR_CUDA. */
int bitssm_device_error(unsigned int* flags, int clear);

/* Diagnostic of the failure-detection path: one kernel waits, through the
 * same bounded mbarrier wait every kernel of the library uses, on a barrier
 * that nothing completes, with a limit of limit_us microseconds (1 ..
 * 1,000,000) instead of the library's 2 s; it gives up, sets bit 3 of the
 * device error word and returns, leaving the context usable.  Asynchronous on
 * `stream`.  BITSSM_ERR_INVALID_ARG for a limit out of range.  The pages have
 * no counterpart; it exists so the error path can be exercised without a
 * fault. */
int bitssm_selftest_wait(unsigned int limit_us, void* stream);

/* ---------------------------------------------------------------------
 * Weight packing (offline).  Absmean ternarisation of the BitNet b1.58
 * BitLinear (TriSSM README opening paragraph; grouped scales: Ternary Mamba
 * abstract):
 *   s = mean |W| over the matrix (group 0) or over each run of `group`
 *       consecutive k of a row (group 128), summed in float64, stored as
 *       float;
 *   W_q = clip(rint(W / (s + 1e-5)), -1, 1), the division in float32,
 *       rint = round half to even.
 * W: float [n_out, k_in] device.  packed: uint8 [n_out, ceil(k_in/4)]
 * (every byte written).  scales: 1 float (group 0) or
 * [n_out, ceil(k_in/group)] floats.  ws: bitssm_pack_workspace_size bytes.
 * --------------------------------------------------------------------- */
int bitssm_pack_workspace_size(int n_out, int k_in, int group, size_t* bytes);
int bitssm_pack_ternary(const float* W, int n_out, int k_in, int group, uint8_t* packed,
                        float* scales, void* ws, size_t ws_bytes, void* stream);

/* Host-side check of a packed ternary matrix held in HOST memory (for
 * weights that come from a file rather than from bitssm_pack_ternary):
 * packed uint8 [n_out, ceil(k_in/4)] in the 2-bit encoding above.  Counts
 * the elements of the matrix that hold the invalid code 3 into *bad (the
 * padding elements past k_in must hold code 1 and are counted too when they
 * do not).  Returns BITSSM_OK when *bad == 0, BITSSM_ERR_INVALID_ARG when
 * any code is invalid or an argument is.  No device work.  The pages give no
 * interface for this; the encoding is the one packing defines. */
int bitssm_check_packed(const uint8_t* packed_host, int n_out, int k_in, long* bad);

/* ---------------------------------------------------------------------
 * BitLinear forward on M input rows (TriSSM README: opening paragraph and
 * the caption "an RMSNorm precedes each ternary projection"; multiply-free
 * ternary GEMM: "Ternary State-Space Models" abstract).
 *
 * A8: for each row v of x [M, k_in]: m = max|v|; codes
 *     q = clamp(rint(v * (127/m)), -128, 127) decided in float32 (all-zero
 *     codes when m = 0); acc = q W_q^T accumulated exactly in int32 on the
 *     tensor cores; r = 1/sqrt(mean(v^2) + 1e-5) (unit-gain RMSNorm folded
 *     into the quantiser); y = acc * s * m * r / 127.
 *     x_dtype: BITSSM_F32 or BITSSM_BF16.  y_dtype: F32, BF16, or I32 to
 *     receive the raw int32 accumulators acc.
 * A16: x bf16 [M, k_in] (k_in a multiple of 8), no activation codes:
 *     y = r * sum_j s[n, j] * sum_{k in group j} W_q[n, k] * x[k]; the group
 *     scale enters the bf16 tensor-core operand as bf16(s), so y carries a
 *     relative error of at most 2^-9 per group from that rounding.
 *     y_dtype: F32 or BF16.
 * y: [M, n_out].  ws: bitlinear_workspace_size bytes.
 * --------------------------------------------------------------------- */
int bitlinear_workspace_size(const bitssm_tw* w, int M, int act_mode, size_t* bytes);
int bitlinear_forward(const bitssm_tw* w, const void* x, int M, int x_dtype, void* y, int y_dtype,
                      int act_mode, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------
 * bitlinear_forward without a caller workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves, for example an operator running inside a host
 * framework whose allocator must own every device byte, code held to a
 * memory budget fixed at start-up, or a latency-critical path where an
 * allocation and its implicit synchronisation are not acceptable.
 *
 * Same arguments, results and errors as bitlinear_forward, minus ws and
 * ws_bytes: the scratch is a fixed array of BITSSM_NOALLOC_SCRATCH_BYTES
 * (16 MiB) inside the library, present on every GPU that loads the library
 * until the process exits.  A shape whose bitlinear_workspace_size exceeds
 * that returns BITSSM_ERR_WORKSPACE, with the sizes in bitssm_last_error().
 * The call allocates nothing (no cudaMalloc, no library allocator).
 *  - The first call on a device looks up the array's device address on the
 *    current device; make that first call before any stream capture.
 *  - Every call shares the one array: calls whose work overlaps on the GPU
 *    (different streams, or concurrent host threads) race and corrupt each
 *    other; serialise them, e.g. on one stream.  Nothing in the array needs
 *    to start at zero; each call rewrites what it reads.
 * --------------------------------------------------------------------- */
#define BITSSM_NOALLOC_SCRATCH_BYTES (16u << 20)
int bitlinear_forward_noalloc(const bitssm_tw* w, const void* x, int M, int x_dtype, void* y,
                              int y_dtype, int act_mode, void* stream);

/* ---------------------------------------------------------------------
 * Selective scan (the BitSSM recurrence; TriSSM README caption and
 * "Repository structure": the recurrence is evaluated with a parallel
 * associative scan).  For every batch b, channel e, state n, step t:
 *   delta = softplus(delta_raw[b,t,e] + delta_bias[e])
 *   h[b,e,n] = exp(delta * A[e,n]) * h[b,e,n] + delta * Bm[b,t,n] * u[b,t,e]
 *   y[b,t,e] = sum_n Cm[b,t,n] * h[b,e,n] + D[e] * u[b,t,e]
 * with h = h0 (or 0 when h0 is NULL) before step 0; h_last (nullable)
 * receives h after step L-1.  Arithmetic in float32.
 * u, delta_raw, y: [B, L, E] of `dtype` (F32 or BF16); Bm, Cm: float
 * [B, L, N]; A: float [E, N]; D, delta_bias: float [E]; h0, h_last: float
 * [B, E, N].  Supported: N = 16, E a multiple of 8, L >= 1.
 * --------------------------------------------------------------------- */
int selective_scan_forward(const void* u, const void* delta_raw, const float* delta_bias,
                           const float* A, const float* Bm, const float* Cm, const float* D,
                           const float* h0, void* y, float* h_last, int B, int L, int E, int N,
                           int dtype, void* stream);

/* ---------------------------------------------------------------------
 * BitSSM mixer forward (one layer): x [B, L, d_model] of `dtype` (F32 or
 * BF16) -> out [B, L, d_model] of the same dtype; with `residual`
 * (nullable, same shape and dtype) out = residual + mixer(x).
 *
 * A8 (TriSSM form):
 *   u      = BitLinear_in(x)                              [B,L,E]
 *   dt_low = BitLinear_dt_down(u), Bm = BitLinear_B(u), Cm = BitLinear_C(u),
 *            sharing one RMSNorm + quantisation of u, each with its own s
 *   delta  = softplus(BitLinear_dt_up(dt_low) + dt_bias)
 *   y      = selective scan of (u, delta, A, Bm, Cm, D), h0 = 0
 *   out    = BitLinear_out(y)
 *   The codes fed to dt_down/B/C and to dt_up are decided on the int32
 *   accumulator rows of the projection before them (in real arithmetic the
 *   same codes as those of the rescaled rows; exact in float32 because
 *   |acc| < 2^24).
 * A16 (W1.58A16 form): the same graph with every BitLinear in A16 form.
 * Requirements: d_state == 16; d_model and d_inner multiples of 16;
 * A8: d_inner <= 512; A16: d_model, d_inner multiples of 64.
 * ws: bitssm_workspace_size bytes.
 * --------------------------------------------------------------------- */
int bitssm_workspace_size(const bitssm_layer* p, int B, int L, int dtype, int act_mode,
                          size_t* bytes);
int bitssm_forward(const bitssm_layer* p, const void* x, void* out, const void* residual, int B,
                   int L, int dtype, int act_mode, void* ws, size_t ws_bytes, void* stream);

/* Number of kernels one bitssm_forward call over B sequences of length L
 * launches for this layer and act mode, or -1 for a bad argument.  A8 with
 * d_model in {128, 256}, d_inner in {256, 512} and dt_rank + 2 d_state <= 64:
 * 3 (pre = quantise x + in_proj + x_proj; scan with Delta-up fused; post =
 * quantise y + out_proj), or 4 when B * d_inner is small (below 24 x the SM
 * count): pre, Delta-up + softplus as an int8 GEMM writing delta, the scan
 * reading it, post.  Other A8 shapes: 6 (quantise x, in_proj, x_proj, scan,
 * quantise y, out_proj).  A16: 7 (RMS of x, in_proj, x_proj, dt_proj, scan,
 * RMS of y, out_proj).  A8 block form (d_conv != 0): 8 (quantise x,
 * in_proj, z_proj, conv + SiLU + quantise u, x_proj, scan, gate + quantise
 * y, out_proj).  Plus 1 (first) for the weight expansion when `prepared`
 * is NULL. */
int bitssm_forward_launches(const bitssm_layer* p, int B, int L, int act_mode);

/* bitssm_forward, additionally recording events[i] (cudaEvent_t handles
 * created by the caller, passed as void*) on `stream` before the i-th kernel
 * and events[n] after the last of the n = bitssm_forward_launches() kernels,
 * for per-kernel timing.  n_events must be at least n + 1.  Same results and
 * errors as bitssm_forward. */
int bitssm_forward_timed(const bitssm_layer* p, const void* x, void* out, const void* residual,
                         int B, int L, int dtype, int act_mode, void* ws, size_t ws_bytes,
                         void* const* events, int n_events, void* stream);

/* ---------------------------------------------------------------------
 * SSD scan (Mamba-2): the selective recurrence with one decay per head
 * ("Ternary Mamba" abstract: the W1.58A16 model is Mamba-2 1.3B; "SSDi8"
 * abstract: SSD, the state space duality of Mamba-2).  For sequence b, head
 * h of H with head dimension P, and B/C group g = h / (H / G) of G:
 *   S_t = exp(dt_t[h] A[h]) S_{t-1} + dt_t[h] x_t[h] (outer) B_t[g]
 *   y_t[h] = S_t C_t[g] + D[h] x_t[h]            (S: [P, N] per head)
 * x, y: float [B, L, H, P]; dt: float [B, L, H], the step after its softplus
 * (> 0); A: float [H] (< 0); Bm, Cm: float [B, L, G, N]; D: float [H] or
 * NULL (zero); S0: float [B, H, P, N] starting state or NULL (zero);
 * S_last: float [B, H, P, N] or NULL, receives the state after the last step
 * (may alias S0: each state is read before it is written, by one thread).
 * Supported: N = 16 * 2^k up to 512 and P * N / 16 a multiple of 32 up to
 * 1024 (for example P = 64, N = 128), B <= 65535; otherwise
 * BITSSM_ERR_UNSUPPORTED_SHAPE.  H % G != 0, a negative size or (with
 * B > 0) a NULL required pointer: BITSSM_ERR_INVALID_ARG; B = 0 does
 * nothing.  The exp is the exp2 unit's
 * approximation of exp2(dt A log2 e) (relative error ~2^-22); the
 * recurrence is float32.
 * --------------------------------------------------------------------- */
int ssd_scan_forward(const float* x, const float* dt, const float* A, const float* Bm,
                     const float* Cm, const float* D, const float* S0, float* y, float* S_last,
                     int B, int L, int H, int P, int G, int N, void* stream);

/* ---------------------------------------------------------------------
 * Forward with a carried state: the recurrent form of the same layer
 * ("Ternary Mamba" abstract: SSMs offer linear-time inference; the state h
 * is all that links one step to the next).  h [B, d_inner, d_state] float:
 * the scan starts from h (instead of zero) and h is overwritten with the
 * state after the last step.  Every other stage is token-local, so running
 * a sequence in pieces (or one token at a time) with the same h gives the
 * results of one call over the whole sequence.  Arguments otherwise as
 * bitssm_forward (same workspace size for the same B and L); h must not
 * alias x, out or the workspace.  Errors as bitssm_forward; a NULL h is
 * BITSSM_ERR_INVALID_ARG; a block-form layer (d_conv != 0, whose conv would
 * also need the last d_conv - 1 inputs carried) is
 * BITSSM_ERR_UNSUPPORTED_SHAPE.
 * bitssm_step is the decode step: L = 1, x and out [B, d_model].
 * --------------------------------------------------------------------- */
int bitssm_forward_state(const bitssm_layer* p, const void* x, void* out, const void* residual,
                         float* h, int B, int L, int dtype, int act_mode, void* ws, size_t ws_bytes,
                         void* stream);
int bitssm_step(const bitssm_layer* p, const void* x, void* out, const void* residual, float* h,
                int B, int dtype, int act_mode, void* ws, size_t ws_bytes, void* stream);

/* Residual stack (TriSSM README Overview table: 12 layers at d = 256):
 * out = x; for each layer l: out = out + mixer_l(out), rounded to `dtype`.
 * `layers` is a host array of n_layers layer structs of identical shapes.
 * ws: bitssm_workspace_size bytes of one layer. */
int bitssm_stack_forward(const bitssm_layer* layers, int n_layers, const void* x, void* out,
                         int B, int L, int dtype, int act_mode, void* ws, size_t ws_bytes,
                         void* stream);

/* ---------------------------------------------------------------------
 * The forward on host buffers, copies overlapped with the computation.
 * n_layers == 1: out = mixer(x) as bitssm_forward (no residual);
 * n_layers > 1: the residual stack as bitssm_stack_forward.
 * x_host, out_host: [B, L, d_model] of `dtype` in host memory (page-locked,
 * e.g. cudaHostAlloc, for the copies to overlap; pageable memory gives the
 * same results, serialised).  x_dev, out_dev: caller-owned device buffers of
 * the same size (the copies' staging; out_dev also holds the result).
 * The batch is cut into n_chunks (1..16) groups of whole sequences; chunk
 * i's host-to-device copy, forward and device-to-host copy run on a helper
 * stream, `stream` and a second helper stream, ordered by events, so copies
 * of neighbouring chunks overlap the forward (sequences are independent, so
 * the result equals one call over the whole batch).  ws: bitssm_workspace_size
 * for one chunk (ceil(B / n_chunks) sequences) is enough.  Everything queued
 * on `stream` before the call happens first; the work of the call is
 * complete when `stream` reaches the point after it.  The two helper streams
 * and their events are created on the first call on each device and kept;
 * calls from several host threads are serialised inside.  Weights should be
 * prepared (bitssm_prepare_weights): otherwise every chunk expands them.
 * Errors: BITSSM_ERR_INVALID_ARG (NULL buffers, n_chunks out of range,
 * dtype), the errors of bitssm_forward, BITSSM_ERR_CUDA for a failed copy or
 * stream operation (bitssm_last_error has the message).  The pages give no
 * interface for this; it is the host-facing form of the same forward.
 * --------------------------------------------------------------------- */
int bitssm_forward_host(const bitssm_layer* layers, int n_layers, const void* x_host,
                        void* out_host, int B, int L, int dtype, int act_mode, void* x_dev,
                        void* out_dev, void* ws, size_t ws_bytes, int n_chunks, void* stream);

/* Expanded weights: the six ternary matrices of a layer expanded once to
 * tensor-core operand form (A8: int8 {-1,0,1}; A16: bf16 w * bf16(s)).
 * bitssm_prepare_weights fills `dst` (bitssm_prepared_size bytes, device,
 * 256-byte aligned); a layer whose `prepared` field points to it skips the
 * per-call expansion.  The buffer stays valid while the packed weights do
 * not change. */
int bitssm_prepared_size(const bitssm_layer* p, int act_mode, size_t* bytes);
int bitssm_prepare_weights(const bitssm_layer* p, int act_mode, void* dst, size_t dst_bytes,
                           void* stream);

/* Inspection of the forward's intermediates inside a workspace (for
 * stage-by-stage checks).  Fills byte offsets into the workspace, or
 * (size_t)-1 for a buffer the forward does not write (the A8 codes q_x,
 * q_u and q_y are written only with BITSSM_KEEP_CODES when the layer runs
 * as the fused kernels), and the row pitch in elements of each buffer.
 *   A8:  q_x int8 [T, ld_qx], deq_x float [T], u [T, E] of u_dtype (float,
 *        or, in the fused kernels, the exact int16 in_proj accumulators with
 *        u = u_i16 * u_scale[t], u_scale float [T]),
 *        q_u int8 [T, ld_qu], deq_u float [T], Bm float [T, N],
 *        Cm float [T, N], q_dt int8 [T, ld_qdt], deq_dt float [T],
 *        y float [T, E], q_y int8 [T, ld_qu], deq_y float [T]; delta float
 *        [T, E] only when the forward forms it by a GEMM before the scan
 *        (see bitssm_forward_launches); block form only: u_pre float
 *        [T, E] (in_proj output before the conv; u then holds the float u
 *        after conv + SiLU), z float [T, E] (the gate branch); y is the scan
 *        output before the gate
 *   A16: r_x float [T], u bf16 [T, E], dt_low bf16 [T, R], r_dt float [T],
 *        Bm, Cm float [T, N], delta float [T, E] (= softplus(delta_raw +
 *        dt_bias), formed in the dt_proj epilogue), y bf16 [T, E],
 *        r_y float [T]
 * deq_* is the per-token factor m * r / 127 of the absmax codes; r_* the
 * RMSNorm factor. */
typedef struct bitssm_ws_view {
  size_t q_x, deq_x, u, q_u, deq_u, Bm, Cm, q_dt, deq_dt, y, q_y, deq_y;
  size_t r_x, dt_low, r_dt, delta_raw, r_y;
  size_t u_scale, delta;
  size_t u_pre, z;
  int ld_qx, ld_qu, ld_qdt;
  int u_dtype;
} bitssm_ws_view;
int bitssm_workspace_layout(const bitssm_layer* p, int B, int L, int dtype, int act_mode,
                            bitssm_ws_view* view);

#ifdef __cplusplus
}
#endif

#endif /* BITSSM_H */
