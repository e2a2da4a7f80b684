/*
 * wkv.h -- C ABI of libwkv.so, the B200 (sm_100a) RWKV WKV operator.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers: CUDA device memory owned by the caller, contiguous, row-major,
 *    16-byte aligned.  [B,T,C] arrays hold token t of batch b, channel c at
 *    ((b*T + t)*C + c); channel c = h*N + i belongs to head h, row i.
 *    u and du are [C] (= [H][N]).  Outputs are fully overwritten, never
 *    accumulated into.  Inputs and outputs must not overlap.
 *  - Head size N = C / H.  This build supports N == 64 (WKV_ERR_HEADSIZE otherwise).
 *  - stream: a cudaStream_t (NULL = legacy default stream).  Every call only
 *    enqueues work on that stream and returns; none synchronises, none
 *    allocates device memory (scratch is passed in by the caller).
 *  - Return value: WKV_OK (0) or a negative WKV_ERR_* code.  On an argument
 *    error nothing is launched and no output is touched.  WKV_ERR_CUDA means
 *    the launch itself failed (cudaGetLastError after the launch).
 *  - Device-side waits (on TMA completion) are bounded by a one-second limit;
 *    a wait that runs out makes the kernel stop early and records
 *    WKV_FAULT_TIMEOUT in a device word that wkv_take_device_faults() reads.
 *  - B == 0 or T == 0 is a valid empty problem: nothing is launched, except
 *    that wkv6_bwd zeroes du when B*T == 0.
 *
 * Library builds
 * --------------
 * libwkv.so runs one fixed algorithm per entry point: the chunked tensor-core
 * forms where an entry point has one.  The same sources built with
 * -DWKV_RECURRENCE_PATHS=1 give libwkv_recurrence.so, a test and comparison
 * build with this same ABI in which wkv6_fwd, wkv6_fwd_bf16, wkv6_bidir_fwd,
 * wkv6_fwd_fused, wkv6_fwd_state, wkv5_fwd, wkv5_fwd_bf16, wkv6_bwd,
 * wkv6_bwd_bf16 and wkv5_bwd run the token-by-token recurrence kernels instead
 * (the kernels wkv6_bwd_noalloc uses in both builds).  Results agree within the
 * tolerances stated below; nothing is selected at run time.  A third build,
 * libwkv_debug.so (-DWKV_DEVICE_CHECKS=1), is libwkv.so with an index check on
 * every global store of every kernel (and every L2 prefetch of an output row):
 * an index outside the array skips the access and records WKV_FAULT_INDEX
 * (nothing traps), and every entry point then waits for its kernels and returns
 * WKV_ERR_DEVICE_CHECK (or WKV_ERR_TIMEOUT for a bounded wait that ran out)
 * instead of WKV_OK.
 *
 * RWKV-6 log-decay
 * ----------------
 * The decay argument w of the RWKV-6 entry points is the log-decay
 * ew = -exp(w_raw) <= 0 that the reference's autograd wrapper hands its kernel
 * ("How the WKV (Weighted Key Value) Mechanism in RWKV Processes Images",
 * CUDA Wrapper (Image Side)); the kernel exponentiates it on the fly
 * ("How Custom CUDA Kernels (wkv6_cuda.cu) Implement the WKV Operation",
 * Kernel Architecture and Launch Configuration: w is "exponentiated
 * on-the-fly"), so state row i of head h decays by d_t[i] = exp(ew_t[h*N+i]).
 */
#ifndef WKV_H_
#define WKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *wkv_stream_t; /* identical to cudaStream_t */

enum {
    WKV_OK = 0,
    WKV_ERR_ARG = -1,        /* B, T < 0; C, H < 1; C != H*N; a required pointer is NULL */
    WKV_ERR_HEADSIZE = -2,   /* N = C/H is not a compiled head size (64) */
    WKV_ERR_ALIGN = -3,      /* a pointer is not 16-byte aligned */
    WKV_ERR_WORKSPACE = -4,  /* workspace NULL or smaller than the *_workspace_bytes query */
    WKV_ERR_CUDA = -5,       /* a CUDA runtime call or the launch failed */
    WKV_ERR_DEVICE = -6,     /* the current device is not sm_100 (B200) */
    WKV_ERR_TOO_LARGE = -7,  /* a size exceeds a documented limit (B*T*C >= 2^31 elements) */
    WKV_ERR_DEVICE_CHECK = -8, /* debug build: a kernel's index check failed (WKV_FAULT_INDEX) */
    WKV_ERR_TIMEOUT = -9     /* debug build: a kernel's bounded wait ran out (WKV_FAULT_TIMEOUT) */
};

/* Bits of the device fault word (see wkv_take_device_faults). */
#define WKV_FAULT_TIMEOUT 0x1u   /* a bounded device-side wait ran out */
#define WKV_FAULT_INDEX 0x2u     /* debug build: a kernel's store index was out of range (store skipped) */

/*
 * wkv6_fwd -- causal RWKV-6 WKV forward, fp32 inputs, fp32 state and output.
 *
 * Operation ("RWKV Architecture: How Receptance Weighted Key Value Combines RNN
 * Linear Inference with Transformer Parallel Training", RWKV-5 "Eagle" matrix
 * state and RWKV-6 "Finch" dynamic decay; "How Custom CUDA Kernels
 * (wkv6_cuda.cu) ...", Past-to-Future Pass, y += r*(u*x + s) with s = s*w + x):
 * per (b, h), with S_{-1} = 0 (N x N),
 *     y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),   S_t = diag(exp(w_t)) S_{t-1} + k_t^T v_t.
 * Arguments follow the reference launcher cuda_forward(B, T, C, H, r, k, v, w, u, y)
 * ("How Custom CUDA Kernels ...", Kernel Architecture and Launch Configuration).
 *   r, k, v, w : [B,T,C] float, inputs (w = log-decay, see above)
 *   u          : [C] float, bonus for the current token
 *   y          : [B,T,C] float, output
 * Algorithm: the chunked form ("RWKV Architecture ...", Parallel Training
 * Formulation) on the tensor cores, every fp32 operand split exactly into three
 * bf16 terms (relative L2 error about 2e-7).  (In the test build, see "Library
 * builds" above, the token-by-token recurrence.)
 */
int wkv6_fwd(int B, int T, int C, int H, const float *r, const float *k, const float *v,
             const float *w, const float *u, float *y, wkv_stream_t stream);

/*
 * wkv6_fwd_bf16 -- wkv6_fwd with bfloat16 r, k, v, w (raw IEEE bf16 bit patterns,
 * uint16_t); u, the state and y stay fp32.  Same operation and layout.
 */
int wkv6_fwd_bf16(int B, int T, int C, int H, const uint16_t *r, const uint16_t *k,
                  const uint16_t *v, const uint16_t *w, const float *u, float *y, wkv_stream_t stream);

/*
 * wkv6_bidir_fwd -- bidirectional RWKV-6 WKV forward, fp32 ("How Custom CUDA
 * Kernels (wkv6_cuda.cu) ...", Forward Pass Implementation: a future-to-past
 * pass without the bonus, then a past-to-future pass that adds the bonus u):
 *     y_t = r_t S^b_{t+1} + r_t (S_{t-1} + diag(u) k_t^T v_t),
 *     S^b_t = diag(exp(w_t)) S^b_{t+1} + k_t^T v_t,  S^b_T = 0,
 * i.e. every other token contributes once with the decay accumulated between
 * the two positions and the current token once with u.  Same arguments as wkv6_fwd.
 */
int wkv6_bidir_fwd(int B, int T, int C, int H, const float *r, const float *k, const float *v,
                   const float *w, const float *u, float *y, wkv_stream_t stream);

/*
 * wkv6_fwd_state -- wkv6_fwd carrying the recurrent state across calls, so that a
 * sequence can be processed in pieces (streaming, recurrent inference: "RWKV
 * Architecture ...", Recurrent Inference Formulation -- the N x N state is all a
 * step needs from the past).  Same operation with S_{-1} = s0 instead of 0:
 *     y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),   S_t = diag(exp(w_t)) S_{t-1} + k_t^T v_t.
 *   r, k, v, w, u, y : as in wkv6_fwd (fp32, causal)
 *   s0 : [B,H,N,N] float, the initial state of each (b, h): element (i, j) at
 *        ((b*H + h)*N + i)*N + j, row i = key channel, column j = value channel;
 *        NULL means the zero state
 *   sT : [B,H,N,N] float, output: the state S_{T-1} after the last token (s0, or
 *        zero, when T == 0); NULL if not wanted.  s0 and sT may be the same buffer
 *        (updated in place); neither may overlap the other arguments.
 * Running wkv6_fwd_state on tokens [0, t) and then on [t, T) with the first
 * call's sT as the second call's s0 gives the same y and final state as one call
 * on [0, T) (up to fp32 rounding).  Errors: as wkv6_fwd, plus WKV_ERR_ALIGN for a
 * misaligned s0 or sT and WKV_ERR_TOO_LARGE when B*H*N*N >= 2^31.
 * Algorithm: the chunked tensor-core form of wkv6_fwd, with s0 loaded into tensor
 * memory before the first chunk and the state stored after the last.  (In the test
 * build, the token-by-token recurrence.)
 */
int wkv6_fwd_state(int B, int T, int C, int H, const float *r, const float *k, const float *v,
                   const float *w, const float *u, const float *s0, float *y, float *sT,
                   wkv_stream_t stream);

/*
 * wkv6_decode -- one recurrent step for B independent sequences (token-by-token
 * generation; the same recurrence as wkv6_fwd_state with T = 1, s0 = sT = state):
 *     y_b = r_b (S_b + diag(u) k_b^T v_b),   S_b <- diag(exp(w_b)) S_b + k_b^T v_b.
 *   r, k, v, w : [B,C] float, this step's token of each sequence (w = log-decay)
 *   u          : [C] float
 *   state      : [B,H,N,N] float, in/out, layout as s0 of wkv6_fwd_state
 *   y          : [B,C] float, output
 * Errors: WKV_ERR_ARG, WKV_ERR_HEADSIZE, WKV_ERR_ALIGN, WKV_ERR_TOO_LARGE
 * (B*H*N*N >= 2^31), WKV_ERR_DEVICE, WKV_ERR_CUDA; B == 0 launches nothing.
 */
int wkv6_decode(int B, int C, int H, const float *r, const float *k, const float *v, const float *w,
                const float *u, float *state, float *y, wkv_stream_t stream);

/*
 * wkv6_bwd -- gradients of L = sum(dy * y) for wkv6_fwd (bidirectional == 0) or
 * wkv6_bidir_fwd (bidirectional != 0), fp32 ("How Custom CUDA Kernels
 * (wkv6_cuda.cu) ...", Backward Pass Gradient Computation; arguments follow the
 * reference backward(B, T, C, H, r, k, v, ew, u, gy, gr, gk, gv, gw, gu)).
 *   r, k, v, w, dy     : [B,T,C] float, inputs
 *   u                  : [C] float, input
 *   dr, dk, dv, dw     : [B,T,C] float, outputs (dw is the gradient with respect
 *                        to the log-decay w passed in)
 *   du                 : [C] float, output, summed over B and T in a fixed
 *                        order (bitwise reproducible run to run)
 *   workspace          : device scratch of at least wkv6_bwd_workspace_bytes(...)
 *                        bytes, 16-byte aligned, owned by the caller; its content
 *                        on entry is ignored and on exit undefined.
 * Algorithm: the chunked form on the tensor cores in two kernels (one carrying
 * the forward state, one the adjoint), operands split into two bf16 terms
 * (relative L2 error about 1e-5 on every gradient); in the test build, the
 * two-sweep recurrence.  Both write every output element; only the order of
 * additions differs, and each is bitwise reproducible run to run.
 */
int wkv6_bwd(int B, int T, int C, int H, int bidirectional, const float *r, const float *k,
             const float *v, const float *w, const float *u, const float *dy, float *dr, float *dk,
             float *dv, float *dw, float *du, void *workspace, size_t workspace_bytes,
             wkv_stream_t stream);

/*
 * wkv6_bwd_bf16 -- wkv6_bwd with bfloat16 r, k, v, w and dy (raw IEEE bf16 bit
 * patterns, uint16_t) for bf16 training: the same gradients, computed in fp32
 * from the bf16 values, with u and every gradient (dr, dk, dv, dw, du) in fp32.
 * Same layouts, workspace (wkv6_bwd_workspace_bytes), algorithms and errors
 * as wkv6_bwd.
 */
int wkv6_bwd_bf16(int B, int T, int C, int H, int bidirectional, const uint16_t *r, const uint16_t *k,
                  const uint16_t *v, const uint16_t *w, const float *u, const uint16_t *dy, float *dr,
                  float *dk, float *dv, float *dw, float *du, void *workspace, size_t workspace_bytes,
                  wkv_stream_t stream);

/* Scratch bytes wkv6_bwd needs for these sizes: 2*B*C floats (per-batch du
 * partials, and the per-channel totals that the tensor-core backward carries
 * from its first kernel to its second). */
size_t wkv6_bwd_workspace_bytes(int B, int T, int C, int H, int bidirectional);

/*
 * wkv6_bwd_noalloc -- wkv6_bwd without a workspace argument, for callers that
 * cannot allocate device memory: for example code that runs inside another
 * framework's callback or plugin which hands it no scratch buffer, or a
 * serving process that reserves all of its device memory at start-up and may
 * not call cudaMalloc afterwards (cudaMalloc can synchronise the device and
 * fragments a planned memory pool).  The source pages have no counterpart to
 * this entry point; it exists for those callers.
 *
 * Same operation, arguments (minus workspace) and layouts as wkv6_bwd, computed
 * by the two-sweep recurrence kernel (the results agree with wkv6_bwd's within
 * the fp32 gradient tolerance; wkv6_bwd runs the tensor-core kernels by default).
 * Its scratch is a fixed 1 MiB device array inside libwkv.so, which every GPU
 * that loads the library holds until the process exits; the call itself
 * allocates nothing.
 *   Limit: B*C <= 262144, else WKV_ERR_TOO_LARGE and nothing is launched.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept with the context it was
 *   looked up in: after a cudaDeviceReset (a new context, into which the
 *   library's device code is loaded anew) the next call looks it up again, so
 *   that call too must come before any stream capture.
 *   All calls share the one array: calls that may overlap on the GPU (on
 *   different streams, or from several host threads) race and must be
 *   serialised by the caller.  Nothing in the array needs clearing between
 *   calls: each call writes every entry it later reads.
 */
int wkv6_bwd_noalloc(int B, int T, int C, int H, int bidirectional, const float *r, const float *k,
                     const float *v, const float *w, const float *u, const float *dy, float *dr, float *dk,
                     float *dv, float *dw, float *du, wkv_stream_t stream);

/*
 * wkv6_fwd_fused -- RWKV-6 forward (causal, or bidirectional when
 * bidirectional != 0) with its decay prologue and its output epilogue fused
 * in, fp32.  RWKV-6 computes the decay pre-activation from a base and a
 * low-rank term, w_t = w_base + tanh(x_t W1) W2 ("RWKV Architecture ...",
 * RWKV-6 "Finch"), the kernel's log-decay is ew = -exp(w_t) ("How the WKV ...
 * Processes Images", CUDA wrapper), and each head's output is group-normalised
 * and multiplied by the SiLU gate (RWKV-5 "Eagle": multi-head normalisation and
 * SiLU output gating; the spatial-mix block passes y and g on together).  The
 * dense projections stay with the caller; this call takes their results:
 *   r, k, v    : [B,T,C] float
 *   ww         : [B,T,C] float, the low-rank term tanh(x W1) W2
 *   w_base     : [C] float;   u : [C] float (bonus)
 *   g          : [B,T,C] float, the gate (e.g. silu(x W_g))
 *   gn_weight, gn_bias : [C] float;   eps : float > 0
 *   out        : [B,T,C] float, overwritten with
 *     out[b,t,c] = ((y[b,t,c] - mu) / sqrt(var + eps) * gn_weight[c] + gn_bias[c]) * g[b,t,c]
 *   where y is wkv6_fwd (or wkv6_bidir_fwd) at w = -exp(w_base + ww), and mu and
 *   var are the mean and the (biased) variance of y over the N channels of c's
 *   head at (b, t).  Neither the log-decay nor y is written to memory.
 * Same sizes, pointer rules, algorithms and errors as wkv6_fwd; eps <= 0 or not finite gives WKV_ERR_ARG.  On the tensor-core path
 * the prologue runs where the chunk is transformed and the norm and gate in the
 * last sweep's epilogue.
 */
int wkv6_fwd_fused(int B, int T, int C, int H, int bidirectional, const float *r, const float *k, const float *v,
                   const float *ww, const float *w_base, const float *u, const float *g, const float *gn_weight,
                   const float *gn_bias, float eps, float *out, wkv_stream_t stream);

/*
 * wkv5_fwd -- RWKV-5 WKV forward, fp32 ("RWKV Architecture ...", RWKV-5
 * "Eagle": the matrix state decays by a static, per-channel factor):
 *     S_t = diag(exp(-w)) S_{t-1} + k_t^T v_t,   y_t = r_t (S_{t-1} + diag(u) k_t^T v_t),
 * S_{-1} = 0; i.e. wkv6_fwd with the log-decay ew_t = -w at every token.
 *   r, k, v, y : [B,T,C] float, y overwritten;  w, u : [C] float, w >= 0
 *   (state row i of head h decays by exp(-w[h*N + i]) per token).
 * Same sizes, pointer rules, stream semantics and errors as wkv6_fwd.
 * Algorithm: the chunked tensor-core form of wkv6_fwd with the constant log-decay
 * in place of the loaded one (no w tensor is read).  (In the test build, the
 * token-by-token recurrence.)
 */
int wkv5_fwd(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
             const float *u, float *y, wkv_stream_t stream);

/*
 * wkv5_fwd_bf16 -- wkv5_fwd with bfloat16 r, k, v (raw IEEE bf16 bit patterns,
 * uint16_t); w, u and y stay fp32, and the state is fp32.  Errors as wkv5_fwd.
 */
int wkv5_fwd_bf16(int B, int T, int C, int H, const uint16_t *r, const uint16_t *k, const uint16_t *v,
                  const float *w, const float *u, float *y, wkv_stream_t stream);

/*
 * wkv5_bwd -- gradients of L = sum(dy * y) for wkv5_fwd (causal), fp32:
 *   dr, dk, dv : [B,T,C] overwritten;  dw, du : [C] overwritten, summed over B
 *   and T in a fixed order (deterministic).  dw is w.r.t. the decay rate w of
 *   wkv5_fwd (dL/dw = -sum_{b,t} dL/d(ew_t)).
 * workspace: at least wkv5_bwd_workspace_bytes(B,T,C,H) bytes of device memory,
 * 16-byte aligned, caller-owned.  Errors as wkv6_bwd.
 * Algorithm: the chunked tensor-core backward of wkv6_bwd (causal) with the
 * constant log-decay -w in place of loaded decays; each token's decay gradient is
 * added into per-(b, c) totals in double instead of being stored, and dw is their
 * sum over b.  (The test build runs the recurrence backward on a [B,T,C] copy of
 * the log-decay and folds its per-token dw over b and t.)
 */
int wkv5_bwd(int B, int T, int C, int H, const float *r, const float *k, const float *v, const float *w,
             const float *u, const float *dy, float *dr, float *dk, float *dv, float *dw, float *du,
             void *workspace, size_t workspace_bytes, wkv_stream_t stream);

/* Scratch bytes wkv5_bwd needs: 24*B*C (product build; 4 * (2*B*T*C + 2*B*C) in
 * the recurrence test build). */
size_t wkv5_bwd_workspace_bytes(int B, int T, int C, int H);

/*
 * wkv4_fwd -- RWKV-4 WKV forward, fp32 ("RWKV Architecture ...", The
 * Fundamental Mathematical Duality and The Recurrent Inference Formulation):
 *     y_t = (sum_{s<t} e^{-(t-1-s) w + k_s} v_s + e^{u + k_t} v_t)
 *         / (sum_{s<t} e^{-(t-1-s) w + k_s}     + e^{u + k_t}),
 * evaluated as the a/b recurrence carried in log space with a running maximum
 * exponent (yarian.com RWKV overview, 3.2: log-space time decay).
 *   k, v : [B,T,C] float inputs;  w : [C] float, w >= 0 (per-step decay e^{-w});
 *   u    : [C] float bonus;       y : [B,T,C] float output.
 * The receptance gate sigma(r) is applied outside the operator, as on the page.
 */
int wkv4_fwd(int B, int T, int C, const float *k, const float *v, const float *w, const float *u,
             float *y, wkv_stream_t stream);

/*
 * wkv4_bwd -- gradients of L = sum(dy * y) for wkv4_fwd ("RWKV Architecture ...",
 * The Fundamental Mathematical Duality: y_t = N_t / D_t, a ratio of decayed sums;
 * its derivatives with respect to k_s, v_s, w and u).
 *   k, v, dy   : [B,T,C] float inputs;  w (> 0), u : [C] float inputs
 *   dk, dv     : [B,T,C] float outputs
 *   dw, du     : [C] float outputs, summed over B and T in a fixed order
 *                (bitwise reproducible run to run)
 *   workspace  : device scratch of at least wkv4_bwd_workspace_bytes(B, T, C) bytes,
 *                16-byte aligned, owned by the caller; content ignored on entry.
 * dk and dv also serve as scratch during the call (they are fully written).
 * Errors: WKV_ERR_ARG, WKV_ERR_ALIGN, WKV_ERR_WORKSPACE, WKV_ERR_TOO_LARGE
 * (B*T*C >= 2^31), WKV_ERR_DEVICE, WKV_ERR_CUDA.  B == 0 or T == 0 zeroes dw, du.
 */
int wkv4_bwd(int B, int T, int C, const float *k, const float *v, const float *w, const float *u,
             const float *dy, float *dk, float *dv, float *dw, float *du, void *workspace,
             size_t workspace_bytes, wkv_stream_t stream);

/* Scratch bytes wkv4_bwd needs: B*T*C floats (one per step) plus 2*B*C floats of partials. */
size_t wkv4_bwd_workspace_bytes(int B, int T, int C);

/* Static description of a status code (never NULL). */
const char *wkv_status_string(int status);

/*
 * wkv_take_device_faults -- synchronise the current device, copy the device
 * fault word (WKV_FAULT_* bits set by kernels whose bounded waits ran out) to
 * *faults, and clear it.  Returns WKV_OK or WKV_ERR_CUDA.  Diagnostic call:
 * unlike the entry points above it does synchronise.
 */
int wkv_take_device_faults(unsigned *faults);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int wkv_version(void);

/*
 * wkv_selftest_wait_timeout -- exercise the failure path of the bounded waits
 * (the mbarrier waits every tensor-core and TMA kernel here uses, each limited
 * to one second).  Launches one CTA on `stream` whose thread waits on an
 * mbarrier that nothing arrives on; after the limit the wait gives up, sets
 * WKV_FAULT_TIMEOUT in the device fault word and the kernel returns, so the
 * context stays usable.  A caller then sees the bit through
 * wkv_take_device_faults().  Takes about a second of GPU time; for tests and
 * health checks only.  Returns WKV_OK, WKV_ERR_DEVICE or WKV_ERR_CUDA.
 */
int wkv_selftest_wait_timeout(wkv_stream_t stream);

/*
 * wkv_selftest_index_check -- exercise the failure path of the kernels' index
 * checks.  Launches one thread that attempts a store whose index equals the size
 * of the array it targets; the check skips the store, records WKV_FAULT_INDEX in
 * the device fault word and the kernel returns.  The product build returns WKV_OK
 * (read the bit with wkv_take_device_faults); the debug build, which waits for
 * its kernels, returns WKV_ERR_DEVICE_CHECK and clears the bit.  For tests only.
 */
int wkv_selftest_index_check(wkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WKV_H_ */
