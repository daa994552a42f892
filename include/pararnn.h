/*
 * pararnn.h -- C ABI of libpararnn.so: parallel-in-time Newton solves of
 * nonlinear RNN recurrences on one NVIDIA B200 (sm_100a).
 *
 * What is computed (page titles and passages):
 *  - "ParaRNN: Unlocking Parallel Training of Nonlinear RNNs for Large Language
 *    Models", TL;DR and Abstract: the recurrence h_t = f(h_{t-1}, x_t) over a
 *    whole sequence is one nonlinear system, solved by Newton's iterations; each
 *    iteration solves a block bi-diagonal linear system by a parallel reduction.
 *    Figure 2 caption: diagonal Jacobians (ParaGRU) and 2x2 block-diagonal ones
 *    (ParaLSTM).  Figure 4 caption: the residual is the max over the batch.
 *  - DEER summary ("Recasting nonlinear recurrences as quadratically convergent
 *    fixed-point iterations with parallel scans"): the converged result equals
 *    sequential evaluation; a tolerance of 1e-4 suffices in float32; Newton may
 *    diverge far from the solution (no damping here: that is reported, not fixed).
 *
 * Conventions shared by every entry point
 *  - Every array pointer is a DEVICE pointer owned by the caller.  The library
 *    never allocates, frees or synchronises; each call only enqueues work on
 *    `stream` (a cudaStream_t passed as void*, NULL = legacy default stream)
 *    and returns.
 *  - Layouts are C order with the channel axis D innermost.  A "channel" is
 *    one (b, d) pair; channels are independent problems.
 *  - Outputs must not alias inputs.  Arrays must be naturally aligned for their
 *    element type (4 B for float, 2 B for bf16); the 2x2 scan additionally needs
 *    A 16-byte aligned and b, x, x0 8-byte aligned.
 *  - `ws` is caller-owned device scratch of at least pararnn_workspace_size()
 *    bytes, 256-byte aligned.  Its contents need no initialisation and are
 *    meaningless after the call.  Concurrent calls need distinct workspaces.
 *  - The return value reports host-side validation and launch errors only.
 *    What happens on the device (iteration count, convergence, a timed-out
 *    wait, a non-finite residual) is written to a caller-owned device struct
 *    that is valid once `stream` has been synchronised.
 *  - Every device-side wait (look-back between time chunks, the grid barrier
 *    between sweeps) is bounded; on expiry the kernel stops, reports
 *    PARARNN_ERR_DEVICE_TIMEOUT and leaves the CUDA context usable.
 */
#ifndef PARARNN_H_
#define PARARNN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PARARNN_VERSION 1
/* Largest max_iters a solve accepts (the info struct keeps every residual). */
#define PARARNN_MAX_ITERS 127

typedef enum {
  PARARNN_OK = 0,
  PARARNN_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, misalignment, bad dtype */
  PARARNN_ERR_UNSUPPORTED = 2,      /* no kernel for this device (needs sm_100a) */
  PARARNN_ERR_CUDA = 3,             /* a CUDA runtime call failed (launch, memset) */
  PARARNN_ERR_DEVICE_TIMEOUT = 4,   /* device side: a bounded wait expired */
  PARARNN_ERR_NONFINITE = 5,        /* device side: a residual was NaN or Inf */
  PARARNN_ERR_WORKSPACE = 6         /* ws is NULL, too small or misaligned */
} pararnn_status_t;

typedef enum { PARARNN_F32 = 0, PARARNN_BF16 = 1 } pararnn_dtype_t;

typedef enum {
  PARARNN_OP_SCAN_DIAG = 0,
  PARARNN_OP_SCAN_BLOCK2 = 1,
  PARARNN_OP_GRU = 2,
  PARARNN_OP_LSTM = 3,
  PARARNN_OP_GRU_BACKWARD = 4,
  PARARNN_OP_LSTM_BACKWARD = 5,
  PARARNN_OP_MHGRU = 6,
  PARARNN_OP_GRU_PROJECTED = 7,
  PARARNN_OP_MHGRU_STRIDED = 8
} pararnn_op_t;

/* Device-side outcome of a solve (caller-owned DEVICE memory, written by the
 * kernel; read it after synchronising the stream).
 *  iterations   : Newton semantics -- the first k with rho_k <= tol, or
 *                 max_iters if none (then converged = 0).
 *  converged    : 1 if some rho_k <= tol.
 *  status       : a pararnn_status_t for the device side (OK, DEVICE_TIMEOUT,
 *                 NONFINITE).
 *  updates      : Newton updates contained in the returned trajectory.  The
 *                 kernel evaluates m iterations per sweep over memory, so a
 *                 converged solve may return h^{k+j} (j >= 1 further updates
 *                 after the certified iterate h^k); an unconverged one returns
 *                 exactly h^{max_iters}.
 *  passes       : sweeps over the inputs in HBM.
 *  max_residual : rho at `iterations`.
 *  rho[k]       : rho_k = max over (b, t, d, component) of |f(h^k_{t-1}) - h^k_t|
 *                 for every k evaluated (k <= iterations at least); others 0. */
typedef struct {
  int32_t iterations;
  int32_t converged;
  int32_t status;
  int32_t updates;
  int32_t passes;
  int32_t reserved;
  float max_residual;
  float rho[PARARNN_MAX_ITERS + 1];
} pararnn_solve_info_t;

/* Optional tuning and test hooks (host struct; pass NULL for defaults).
 *  iters_first : Newton iterations evaluated in the first sweep
 *                (0 = 4 for GRU, 5 for LSTM).
 *  iters_next  : Newton iterations per later sweep (0 = 2).
 *  wait_timeout_ns : bound on every device-side wait (0 = 1e9, i.e. 1 s).
 *  debug_stall_unit: FOR TESTS ONLY -- leave at -1 (off) in any other use.
 *                 The work unit with this index never publishes its look-back
 *                 status, so the units after it run their bounded waits out;
 *                 the call must then report PARARNN_ERR_DEVICE_TIMEOUT
 *                 (look-back regime only).  It exists so that the test suite
 *                 can check the bounded waits without faulting a GPU.
 *  regime      : how the time chunks of a channel tile are chained.  (For the
 *                multi-head solves: 1 = one lane per time segment holding
 *                whole 8x8 maps, 2 = 8 lanes per head and segment, 0 = the
 *                first without strides, the second with them.)
 *                0 = automatic; 1 = look-back (chunks of a tile on different
 *                CTAs, chained through global memory); 2 = walk (one CTA walks
 *                a tile's chunks in order, no traffic between CTAs).  Both give
 *                the same result up to fp32 rounding; in walk mode at most 8
 *                iterations are evaluated per sweep.
 *  walk_warps  : warps per CTA in the walk regime with 32-channel tiles:
 *                0 = automatic (16 for the diagonal scan below 512 tiles,
 *                else 8), 4, 8 or 16.
 *  walk_width  : channels per tile of the walk regime's tensor-copy walker for
 *                the GRU / LSTM solves: 0 = automatic (8 when 32-channel tiles
 *                would be fewer than 4 per SM and L >= 2048 -- finer tiles
 *                balance the SMs once sequences are long enough to repay their
 *                start-up -- else 32), 8 or 32.  The scans always use 32. */
typedef struct {
  int32_t iters_first;
  int32_t iters_next;
  int64_t wait_timeout_ns;
  int64_t debug_stall_unit;
  int32_t regime;
  int32_t walk_warps;
  int32_t walk_width;
  int32_t reserved;
} pararnn_options_t;

/* Bytes of workspace the call with the same arguments needs. 0 on bad sizes. */
size_t pararnn_workspace_size(pararnn_op_t op, int64_t B, int64_t L, int64_t D,
                              int32_t max_iters, const pararnn_options_t* opts);

/* Diagonal affine scan (the linear solve of one Newton step, diagonal case;
 * ParaRNN Figure 2 left):  h_t = A_t * h_{t-1} + b_t  for t = 1..L.
 *  A, b : [B, L, D] fp32.      h0 : [B, D] fp32 or NULL (= 0).
 *  h    : [B, L, D] fp32 output (t = 1..L; h0 is not repeated).
 *  status_dev : optional device int32 receiving the device-side status. */
pararnn_status_t pararnn_scan_diag(const float* A, const float* b, const float* h0, float* h,
                                   int64_t B, int64_t L, int64_t D, void* ws, size_t ws_bytes,
                                   int32_t* status_dev, const pararnn_options_t* opts,
                                   void* stream);

/* 2x2 block affine scan (ParaLSTM's linear solve; ParaRNN Figure 2 left):
 *  x_t = A_t x_{t-1} + b_t,  A : [B, L, D, 2, 2] row-major ((0,0),(0,1),(1,0),(1,1)),
 *  b : [B, L, D, 2],  x0 : [B, D, 2] or NULL,  x : [B, L, D, 2] output. */
pararnn_status_t pararnn_scan_block2(const float* A, const float* b, const float* x0, float* x,
                                     int64_t B, int64_t L, int64_t D, void* ws, size_t ws_bytes,
                                     int32_t* status_dev, const pararnn_options_t* opts,
                                     void* stream);

/* ParaGRU Newton solve (ParaRNN Abstract; Figure 2 right, Figure 5 left).
 * Cell, per channel, with diagonal recurrence weights:
 *   z = sig(Pz + az h), r = sig(Pr + ar h), c = tanh(Pc + ac (r h)),
 *   h' = (1 - z) h + z c.
 *  P  : [B, L, 3, D] projected pre-activations, gate order (z, r, c); fp32 or
 *       bf16 (p_dtype); state, Jacobians and scan are fp32 either way.
 *  a  : [3, D] fp32 (az, ar, ac).     h0 : [B, D] fp32 or NULL (= 0).
 *  h  : [B, L, D] fp32 output trajectory, t = 1..L.
 *  tol: stop at the first k with rho_k <= tol (1e-4 per the DEER summary).
 *  max_iters : 0..PARARNN_MAX_ITERS.   info : device struct (required).
 * Newton starts from h^0 = 0 and applies no damping. */
pararnn_status_t pararnn_solve_gru(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                   const float* h0, float* h, int64_t B, int64_t L, int64_t D,
                                   float tol, int32_t max_iters, void* ws, size_t ws_bytes,
                                   pararnn_solve_info_t* info, const pararnn_options_t* opts,
                                   void* stream);

/* ParaLSTM Newton solve with per-channel state (c, h) and a 2x2 Jacobian
 * (ParaRNN Figure 2 caption; Figure 5 right).  Cell (diagonal recurrence on h):
 *   i = sig(Pi + ai h), f = sig(Pf + af h), g = tanh(Pg + ag h),
 *   o = sig(Po + ao h), c' = f c + i g, h' = o tanh(c').
 *  P : [B, L, 4, D] gate order (i, f, g, o), fp32 or bf16.   a : [4, D] fp32.
 *  c0, h0 : [B, D] fp32 or NULL (= 0).   c, h : [B, L, D] fp32 outputs.
 *  The residual max runs over both components.  Other arguments as for GRU. */
pararnn_status_t pararnn_solve_lstm(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                    const float* c0, const float* h0, float* c, float* h,
                                    int64_t B, int64_t L, int64_t D, float tol, int32_t max_iters,
                                    void* ws, size_t ws_bytes, pararnn_solve_info_t* info,
                                    const pararnn_options_t* opts, void* stream);

/* Backward pass of the ParaGRU solve: gradients of a loss through the solved
 * trajectory (DEER summary: "forward plus gradients"; ParaRNN trains with
 * them).  With g_t = dl/dh_t given, the total gradient lambda_t obeys the
 * adjoint recursion lambda_t = g_t + J_{t+1}^T lambda_{t+1} -- the transposed
 * bi-diagonal system of a Newton step, run backwards in time -- and
 *   dP_t = lambda_t df/dP_t,  da = sum over (b, t) of lambda_t df/da,
 *   dh0 = J_1^T lambda_1,
 * with every derivative taken at the forward solution.  One pass, no Newton
 * iterations.
 *  P, p_dtype, a, h0 : as given to pararnn_solve_gru.
 *  h  : [B, L, D] fp32, the forward solution (t = 1..L).
 *  dh : [B, L, D] fp32 upstream gradient dl/dh_t.
 *  dP : [B, L, 3, D] fp32 output.   da : [3, D] fp32 output (overwritten; the
 *       sum over b and t is accumulated with atomics, so its last bits depend
 *       on the order of addition).   dh0 : [B, D] fp32 output or NULL.
 *  status_dev : optional device int32 for the device-side status.
 *  ws : pararnn_workspace_size(PARARNN_OP_GRU_BACKWARD, B, L, D, 0, opts). */
pararnn_status_t pararnn_solve_gru_backward(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                            const float* h0, const float* h, const float* dh,
                                            float* dP, float* da, float* dh0, int64_t B,
                                            int64_t L, int64_t D, void* ws, size_t ws_bytes,
                                            int32_t* status_dev, const pararnn_options_t* opts,
                                            void* stream);

/* Backward pass of the ParaLSTM solve, state (c, h) and 2x2 transposed
 * Jacobians.  c, h : the forward solution.  dc, dh : upstream gradients
 * dl/dc_t and dl/dh_t (either may be NULL = 0, not both).  Outputs dP
 * [B, L, 4, D], da [4, D] (overwritten, atomically accumulated), dc0 and dh0
 * [B, D] (each may be NULL).  Workspace for PARARNN_OP_LSTM_BACKWARD. */
pararnn_status_t pararnn_solve_lstm_backward(const void* P, pararnn_dtype_t p_dtype,
                                             const float* a, const float* c0, const float* h0,
                                             const float* c, const float* h, const float* dc,
                                             const float* dh, float* dP, float* da, float* dc0,
                                             float* dh0, int64_t B, int64_t L, int64_t D,
                                             void* ws, size_t ws_bytes, int32_t* status_dev,
                                             const pararnn_options_t* opts, void* stream);

/* One cell step for every channel: h_next = f(h_prev, P) -- a decode step when
 * generating token by token (ParaRNN Figure 3 caption: generation
 * throughput).  P : [B, 3, D] (z, r, c) for one time step, fp32 or bf16;
 * a : [3, D]; h_prev : [B, D] or NULL (= 0); h_next : [B, D].  No workspace;
 * h_next may not alias h_prev's storage of another step being read. */
pararnn_status_t pararnn_step_gru(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                  const float* h_prev, float* h_next, int64_t B, int64_t D,
                                  void* stream);
/* ParaLSTM decode step: P : [B, 4, D]; (c_prev, h_prev) -> (c_next, h_next). */
pararnn_status_t pararnn_step_lstm(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                   const float* c_prev, const float* h_prev, float* c_next,
                                   float* h_next, int64_t B, int64_t D, void* stream);

/* Sequential application of the cell over the whole sequence on the GPU, one
 * thread per channel walking t = 1..L in order (the "sequential application"
 * that ParaRNN's abstract and the DEER summary compare the parallel solve
 * against).  Same arguments and layout as pararnn_solve_gru / _lstm without
 * tol, max_iters, workspace or info.  Its time is L times the cell's
 * dependency chain, independent of B * D up to the GPU's thread count.  When D
 * is a multiple of 32 and P 16-byte aligned, each warp stages its channels'
 * upcoming inputs through shared memory (with D = 1, each thread its own
 * contiguous inputs); measured on B200 that is about 110 ns per step, so for
 * more than roughly 15 000 channels (B * D) the rollout takes less time than
 * the Newton solve, and for fewer it takes more (422x more at B = 16, D = 1,
 * L = 2^20). */
pararnn_status_t pararnn_rollout_gru(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                     const float* h0, float* h, int64_t B, int64_t L, int64_t D,
                                     void* stream);
pararnn_status_t pararnn_rollout_lstm(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                      const float* c0, const float* h0, float* c, float* h,
                                      int64_t B, int64_t L, int64_t D, void* stream);

/* Newton solve of the multi-head GRU whose recurrence is block-diagonal with
 * dense 8x8 blocks, one per head of 8 channels (the dense-block case that the
 * DEER summary's caveats price at O(n^3) per step).  Per head, elementwise:
 *   z = sig(P_z + U_z h), r = sig(P_r + U_r h), c = tanh(P_c + r (U_c h)),
 *   h' = (1 - z) h + z c   -- the ParaGRU cell when every block is diagonal.
 * Same method, stopping rule, info and status semantics as pararnn_solve_gru;
 * each Newton step solves a block bi-diagonal system with dense 8x8 blocks.
 *   P  : [B, L, 3, D] (z, r, c), fp32 or bf16, D = 8 H, 16-byte aligned;
 *   U  : [3, H, 8, 8] fp32: gate, head, row (output channel), column (input);
 *   h0 : [B, D] or NULL (= 0);  h : [B, L, D], 16-byte aligned: the iterate,
 *        updated in place, and the result (must not overlap P, U or h0);
 *   ws : pararnn_workspace_size(PARARNN_OP_MHGRU, B, L, 8 H, max_iters, opts).
 * The kernel is cooperative (every CTA resident), one warp per (b, head). */
pararnn_status_t pararnn_solve_mhgru(const void* P, pararnn_dtype_t p_dtype, const float* U,
                                     const float* h0, float* h, int64_t B, int64_t L,
                                     int64_t H, float tol, int32_t max_iters, void* ws,
                                     size_t ws_bytes, pararnn_solve_info_t* info,
                                     const pararnn_options_t* opts, void* stream);

/* The multi-head GRU with a time stride per head (DEER summary, caveats
 * paragraph: heads of 8 channels with exponentially increasing strides, i.e.
 * shorter effective sequences).  Head g recurs on h_{t - s_g}:
 *   h_t[head g] = cell_g(P_t, h_{t - s_g}[head g]),   h_{t - s_g} = h0 for t < s_g,
 * so a head at stride s is s independent interleaved sequences (t = r, r + s,
 * ...), each of about L / s steps; the Newton solve, its stopping rule and its
 * outputs are otherwise those of pararnn_solve_mhgru (which is this call with
 * every stride 1).
 *  strides : [H] int32 in DEVICE memory, each >= 1 (a stride of L or more makes
 *            every step of the head depend on h0 only).  A stride below 1 is
 *            found on the device: the call then does no work and info.status
 *            reads PARARNN_ERR_INVALID_ARGUMENT.  NULL is rejected.
 *  ws      : pararnn_workspace_size(PARARNN_OP_MHGRU_STRIDED, B, L, 8 H, max_iters,
 *            opts) bytes (it also holds the heads' stride offsets).
 * Requires H L < 2^31; other arguments and errors as pararnn_solve_mhgru. */
pararnn_status_t pararnn_solve_mhgru_strided(const void* P, pararnn_dtype_t p_dtype,
                                             const float* U, const int32_t* strides,
                                             const float* h0, float* h, int64_t B, int64_t L,
                                             int64_t H, float tol, int32_t max_iters, void* ws,
                                             size_t ws_bytes, pararnn_solve_info_t* info,
                                             const pararnn_options_t* opts, void* stream);

/* Sequential application of the multi-head GRU on the GPU: each (batch row,
 * head) sequence walks t = 1..L in order, 8 lanes per sequence (lane i =
 * channel i of the head, the head's state exchanged by shuffles each step).
 * The baseline the Newton solve of the same system is compared with (the DEER
 * summary's caveat: dense blocks make each Newton step O(n^3) per step, while
 * the sequential cell is O(n^2)).  Arguments and layouts as pararnn_solve_mhgru
 * (every head at stride 1) without tol, max_iters, workspace or info; P needs
 * only its element alignment.  Requires 8 B H <= 2^31.  Errors:
 * PARARNN_ERR_INVALID_ARGUMENT (bad sizes, dtype, NULL or misaligned
 * pointers), PARARNN_ERR_CUDA (launch failure).  B, L or H = 0: no work. */
pararnn_status_t pararnn_rollout_mhgru(const void* P, pararnn_dtype_t p_dtype, const float* U,
                                       const float* h0, float* h, int64_t B, int64_t L,
                                       int64_t H, void* stream);

/* One multi-head GRU step for every (batch row, head): h_next = f(h_prev, P),
 * the decode step of the multi-head cell.  P : [B, 3, D] (z, r, c) for one time
 * step, fp32 or bf16, D = 8 H; U : [3, H, 8, 8]; h_prev : [B, D] or NULL (= 0);
 * h_next : [B, D] (must not overlap h_prev).  Errors as pararnn_rollout_mhgru
 * (it is that call with L = 1). */
pararnn_status_t pararnn_step_mhgru(const void* P, pararnn_dtype_t p_dtype, const float* U,
                                    const float* h_prev, float* h_next, int64_t B, int64_t H,
                                    void* stream);

/* Input projection P = x W^T + bias on the tensor cores (tcgen05, bf16 inputs,
 * fp32 accumulation): the projected gate pre-activations that the cells take
 * as inputs (ParaRNN TL;DR: the recurrence keeps only diagonal weights, the
 * dense weights act on the inputs; Figure 2 caption).  For a layer of G gates
 * and D channels, N = G * D and P is [M, N] = [B, L, G, D] with M = B * L, the
 * layout pararnn_solve_gru / _lstm read.
 *   x    : [M, K] bf16, row-major (K contiguous), 16-byte aligned;
 *   W    : [N, K] bf16, row-major (the nn.Linear weight layout), 16-byte aligned;
 *   bias : [N] fp32 or NULL (= 0), 16-byte aligned;
 *   P    : [M, N], fp32 (p_dtype = PARARNN_F32) or bf16 (round to nearest even),
 *          16-byte aligned; must not overlap x, W or bias.
 * N and K must be multiples of 8 (16-byte rows for the tensor copies) and M, N,
 * K below 2^31; otherwise PARARNN_ERR_INVALID_ARGUMENT.  K = 0 writes the bias
 * (or zeros).  No workspace.  status_dev (optional, zeroed by the call) reads 4
 * if a device-side wait ran out.  Needs sm_100a (PARARNN_ERR_UNSUPPORTED). */
pararnn_status_t pararnn_input_projection(const void* x, const void* W, const float* bias,
                                          void* P, pararnn_dtype_t p_dtype, int64_t M,
                                          int64_t N, int64_t K, int32_t* status_dev,
                                          void* stream);

/* ParaGRU layer from its inputs: the input projection P = x W^T + bias fused
 * with the Newton solve, so that P is never written to HBM (ParaRNN, TL;DR and
 * Abstract: dense weights act on the inputs of an LM layer, the recurrence
 * keeps diagonal ones).  The result is the one of pararnn_input_projection
 * with fp32 P followed by pararnn_solve_gru on that P, up to the order of
 * floating-point rounding.
 *  x    : [B, L, K] bf16 (row b L + t = input at step t + 1 of batch row b),
 *         16-byte aligned.
 *  W    : [3 D, K] bf16, the nn.Linear layout: rows 0..D-1 give the z gate,
 *         D..2D-1 the r gate, 2D..3D-1 the c gate; 16-byte aligned.
 *  bias : [3 D] fp32 or NULL (zero), same row order.
 *  a, h0, h, tol, max_iters, info, opts: as in pararnn_solve_gru (h0 [B, D]
 *         or NULL, h [B, L, D] fp32 output, info device memory).
 *  ws   : workspace of pararnn_workspace_size(PARARNN_OP_GRU_PROJECTED, ...)
 *         bytes (a few hundred; zeroed by the call), 256-byte aligned.
 * The projection runs on the tensor cores (bf16 operands, fp32 accumulation);
 * each chunk of P stays in TMEM and shared memory.  A solve that needs more
 * than one sweep of the default 4 Newton iterations recomputes the projection
 * for each later sweep.  opts->regime selects how many work items a CTA walks
 * at once: 1 = one (16 walker warps), otherwise two (two groups of 8 warps);
 * the result does not depend on it beyond rounding order.  Requirements: K > 0 and
 * K % 8 == 0, B L < 2^31; otherwise PARARNN_ERR_INVALID_ARGUMENT.  Needs sm_100a. */
pararnn_status_t pararnn_solve_gru_projected(const void* x, const void* W, const float* bias,
                                             const float* a, const float* h0, float* h,
                                             int64_t B, int64_t L, int64_t D, int64_t K,
                                             float tol, int32_t max_iters, void* ws,
                                             size_t ws_bytes, pararnn_solve_info_t* info,
                                             const pararnn_options_t* opts, void* stream);

/* Allocation-free variant of pararnn_solve_gru (the pages have no counterpart:
 * this is an interface convenience of this library).
 * For callers that cannot allocate device memory where they solve -- their
 * device memory is fully reserved by another allocator, they sit behind a
 * plug-in interface that passes inputs and outputs but no workspace, or they
 * run in a latency-critical loop where an allocation (which may synchronise
 * the device) is not allowed.  Same arguments and results as
 * pararnn_solve_gru without ws / ws_bytes: the scratch is a device array of
 * PARARNN_NOALLOC_SCRATCH_BYTES inside the library, present on every GPU that
 * loads it until the process exits.
 *  - Problems whose pararnn_workspace_size(PARARNN_OP_GRU, ...) exceeds
 *    PARARNN_NOALLOC_SCRATCH_BYTES are rejected with PARARNN_ERR_WORKSPACE
 *    before any work is enqueued.  (In the walk regime -- the automatic
 *    choice once there are at least 200 tiles of 32 channels -- the scratch
 *    needed stays under 4 KB whatever L is.)
 *  - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *    library routine.  The part of the scratch that must start at zero is
 *    cleared on the stream at every call.
 *  - The first call on a device looks up the array's device address with that
 *    device current (a one-time set-up per device); make that first call
 *    before any stream capture.  The address belongs to the device's context:
 *    after cudaDeviceReset the next call finds a new context (by the driver's
 *    context id) and looks the address up again, so it is never stale; that
 *    call, too, should come before any capture.
 *  - Every call on a device shares the one array, which keeps what the last
 *    call left: calls whose kernels may overlap on the GPU (different streams
 *    without ordering, several host threads) race on it and must be
 *    serialised by the caller. */
#define PARARNN_NOALLOC_SCRATCH_BYTES (4u << 20)
pararnn_status_t pararnn_solve_gru_noalloc(const void* P, pararnn_dtype_t p_dtype, const float* a,
                                           const float* h0, float* h, int64_t B, int64_t L,
                                           int64_t D, float tol, int32_t max_iters,
                                           pararnn_solve_info_t* info,
                                           const pararnn_options_t* opts, void* stream);

/* Throughput probe: a measurement aid with no counterpart in the pages.  It
 * enqueues on `stream` one launch of a kernel that keeps one functional-unit
 * pipe of every SM busy (many independent dependency chains per thread, all
 * CTAs resident) and stores in *ops (host memory) the number of operations
 * that launch performs.  Timing the launch with events gives the measured
 * peak that a kernel bound by that pipe is reported against:
 *  pipe 0: the special-function pipe, as one base-2 exponential and one
 *          reciprocal per step (ex2.approx + rcp.approx, the pair each
 *          sigmoid and tanh of the ParaGRU / ParaLSTM cells takes);
 *          *ops counts both.
 *  pipe 1: fp32 fused multiply-add; *ops counts FMAs (2 flops each).
 * iters (> 0) sets the launch's length: 32 * iters chain steps per thread.
 * sink: device memory of at least 4 bytes; it is written only if the chains
 * hit a value they never reach (so the work cannot be optimised away).
 * Errors: PARARNN_ERR_INVALID_ARGUMENT (pipe, iters, NULL pointers),
 * PARARNN_ERR_UNSUPPORTED (not sm_100a), PARARNN_ERR_CUDA (launch). */
pararnn_status_t pararnn_probe_rate(int32_t pipe, int32_t iters, float* sink, int64_t* ops,
                                    void* stream);

/* Static description of a status code (never NULL). */
const char* pararnn_status_string(pararnn_status_t status);

/* PARARNN_VERSION of the loaded library. */
int32_t pararnn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PARARNN_H_ */
