/*
 * e2ttt.h -- C ABI of the E2-TTT chunk-parallel closed-form fast-weight update
 * on NVIDIA B200 (sm_100a).
 *
 * Method: "Rethinking Expressivity and Efficiency in Test-Time Training"
 * (E2-TTT, arXiv 2608.21308). Its abstract states that, with gradients taken
 * at the chunk-start weights, a closed-form state transition reproduces
 * exactly the chunk-end fast-weight and momentum states of the per-token
 * recurrence; its "Approach" summary (atlas.scime.ai) says the transition is
 * built from two scalar kernels (a momentum kernel and a weight kernel) made
 * with log-space cumulative sums, and two weighted gradient aggregations; the
 * "Limitations" summaries say the chunk output is taken at the chunk-start
 * weights.
 *
 * Semantics implemented here, per batch row b and head h, for the chunk of
 * tokens t = 1..C (chunk i holds tokens [iC, (i+1)C); the last may be short):
 *   per-token recurrence (gates: eta = lr, mu = mom, lam = decay)
 *       M_t = mu_t M_{t-1} - eta_t g_t ,   W_t = lam_t W_{t-1} + M_t
 *   with g_t = grad_W l(W0; k_t, v_t) at the chunk-start weights W0, and
 *       l = 1/2 |f_W(k) - v|^2   (E2TTT_LOSS_MSE)   or   -<f_W(k), v>   (E2TTT_LOSS_NEG_DOT)
 *       f_W(x) = W x                          (E2TTT_LINEAR,  W  [d_v, d_k])
 *       f_W(x) = W2 (silu(W1 x) * (W3 x))     (E2TTT_SWIGLU,  W1, W3 [d_h, d_k], W2 [d_v, d_h])
 *       f_W(x) = W2 gelu(W1 x)                (E2TTT_GELU_MLP, W1 [d_h, d_k], W2 [d_v, d_h])
 *   closed form (what the library computes):
 *       a_t = eta_t U(t+1,C),  b_t = eta_t sum_{j=t..C} L(j+1,C) U(t+1,j)
 *       M_end = U(1,C) M0 - sum_t a_t g_t
 *       W_end = L(1,C) W0 + (sum_j L(j+1,C) U(1,j)) M0 - sum_t b_t g_t
 *       out_t = f_{W0}(q_t)
 *   where U(i,j) = prod_{s=i..j} mu_s and L(i,j) = prod_{s=i..j} lam_s.
 *   W_end / M_end of a chunk are the W0 / M0 of the next one.
 *
 * Layouts (all row-major, contiguous, caller-owned DEVICE memory):
 *   q, k        [B, H, T, d_k]   activation dtype (shape->act)
 *   v, out      [B, H, T, d_v]   activation dtype
 *   lr, mom, decay              [B, H, T] fp32 gate VALUES (not logits)
 *   W0, M0, W_end, M_end        [B, H, S] fp32, S = e2ttt_state_elems(shape):
 *        linear: W [d_v, d_k];  SwiGLU: [W1 | W3 | W2] concatenated;
 *        GELU MLP: [W1 | W2] concatenated
 *   saved_states                [n_chunks, B, H, 2, S] fp32: (W, M) at the
 *                               start of every chunk (written by the forward,
 *                               read by the backward); with shape->save_acts
 *                               = 1 followed by the forward's per-chunk
 *                               activations (e2ttt_saved_bytes(shape) bytes in
 *                               all)
 *
 * Conventions:
 *   - The library allocates no memory at run time. Scratch comes from
 *     `workspace` (device memory of at least e2ttt_workspace_bytes(shape,
 *     for_bwd) bytes, 256-byte aligned); its contents on entry do not matter.
 *     One exception is made at load time: the library holds a 32 MiB static
 *     __device__ array on every GPU where its kernels are loaded, for the life
 *     of the process; only e2ttt_chunk_scan_fwd_noalloc (and
 *     e2ttt_noalloc_status) use it.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream). Argument checks run on the host
 *     before anything is launched and return E2TTT_ERR_INVALID_ARG or
 *     E2TTT_ERR_UNSUPPORTED synchronously, with nothing written.
 *     A failed launch returns E2TTT_ERR_CUDA. The library never exits, aborts
 *     or traps; e2ttt_last_error() describes the last failure of the calling
 *     thread.
 *   - Outputs must not overlap inputs or each other (E2TTT_ERR_INVALID_ARG).
 *   - Results are deterministic: no atomics in any reduction.
 */
#ifndef E2TTT_H
#define E2TTT_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  E2TTT_OK = 0,
  E2TTT_ERR_INVALID_ARG = 1,   /* null pointer, bad size, overlap, short workspace   */
  E2TTT_ERR_UNSUPPORTED = 2,   /* valid but not implemented (see each entry point)    */
  E2TTT_ERR_CUDA = 3,          /* a CUDA call or kernel launch failed                 */
  E2TTT_ERR_TIMEOUT = 4        /* a device-side bounded wait gave up                  */
} e2ttt_status;

/* Fast weight f_W: LINEAR W x; SWIGLU W2 (silu(W1 x) * (W3 x)); GELU_MLP
 * W2 gelu(W1 x) with the exact GELU z Phi(z) (the MLP variant, "E2-TTT_MLP" in
 * the atlas.scime.ai summary, "Key results"). */
typedef enum { E2TTT_LINEAR = 0, E2TTT_SWIGLU = 1, E2TTT_GELU_MLP = 2 } e2ttt_fast_kind;
typedef enum { E2TTT_F32 = 0, E2TTT_BF16 = 1 } e2ttt_dtype;
typedef enum { E2TTT_LOSS_MSE = 0, E2TTT_LOSS_NEG_DOT = 1 } e2ttt_loss;
/* Momentum / weight kernels. PER_TOKEN: a_t, b_t of every token (the method).
 * CHUNK_MEAN: the chunk-averaged variant ("Rethinking Expressivity and
 * Efficiency in Test-Time Training", atlas.scime.ai summary, "Surprising
 * findings": per-token factors collapsed to chunk scalars), every token of a
 * chunk carrying the chunk means of a_t and b_t; the chunk scalars U(1,n),
 * L(1,n), c are unchanged. Forward and backward honour it. */
typedef enum { E2TTT_COEF_PER_TOKEN = 0, E2TTT_COEF_CHUNK_MEAN = 1 } e2ttt_coef;
/* Momentum. E2TTT_NO_MOMENTUM runs the recurrence without momentum,
 * W_t = lam_t W_{t-1} - eta_t g_t (mu = 0; the pages' repository names a
 * no-momentum kernel builder): no momentum state exists, so mom, M0 and M_end
 * must be NULL in the forward (saved states then hold zero M), and mom, dM_end,
 * dmom and dM0 must be NULL in the backward. The forward moves only W through
 * HBM (about half the state traffic). */
typedef enum { E2TTT_MOMENTUM = 0, E2TTT_NO_MOMENTUM = 1 } e2ttt_momentum;
/* GEMM precision. AUTO: bf16 activations of tensor-core shapes (C, d_k, d_v,
 * d_h multiples of 128, 16-byte aligned pointers) run on the tcgen05 tensor
 * cores with bf16 operands (activations and bf16 copies of the chunk-start
 * weights) and fp32 accumulation; everything else on the fp32 CUDA-core
 * kernels. FP32: always the fp32 CUDA-core kernels (the bf16 activations are
 * widened, the weights stay fp32), forward and backward: for problems whose
 * gradients are sensitive to rounding the weights to bf16 (a GELU MLP fast
 * weight with a non-zero M0 and upstream state gradients moves its exact
 * gradients by 5-15 % under that rounding). Slower. */
typedef enum { E2TTT_GEMM_AUTO = 0, E2TTT_GEMM_FP32 = 1 } e2ttt_gemm;

/* Saved activations (save_acts). 0: saved_states holds the chunk-start states
 * only, and the backward recomputes the forward's per-chunk intermediates it
 * needs. 1 (SwiGLU and GELU MLPs on the tensor-core path only): the forward
 * also keeps, for every chunk, the residual E of the key rows and the hidden
 * gradient dH of the inner loss (bf16) in saved_states after the states, in
 * place of its per-call scratch (no extra memory traffic), and the backward
 * reads them instead of recomputing them. The forward and the backward of one
 * step must be given the same shape, save_acts included. */
typedef enum { E2TTT_RECOMPUTE_ACTS = 0, E2TTT_SAVE_ACTS = 1 } e2ttt_acts;

/* Problem description. kind/act/loss/coef/momentum/gemm/save_acts hold
 * e2ttt_fast_kind / e2ttt_dtype / e2ttt_loss / e2ttt_coef / e2ttt_momentum /
 * e2ttt_gemm / e2ttt_acts values (zero-initialised gemm and save_acts fields
 * are E2TTT_GEMM_AUTO and E2TTT_RECOMPUTE_ACTS). d_h is ignored (may be 0)
 * for E2TTT_LINEAR.
 * Limits: all sizes >= 1; B*H <= 65535; B*H*T*max(d_k, d_v, 2 d_h) < 2^31
 * (d_h counted for the MLPs only); 1 <= C <= 1024. */
typedef struct {
  int B, H, T, C;
  int d_k, d_v, d_h;
  int kind;
  int act;
  int loss;
  int coef;
  int momentum;
  int gemm;
  int save_acts;
} e2ttt_shape;

/* Fast-weight state size S per (b, h): d_v*d_k (linear), 2*d_h*d_k + d_v*d_h
 * (SwiGLU, [W1 | W3 | W2]) or d_h*d_k + d_v*d_h (GELU MLP, [W1 | W2]). Returns
 * 0 for an invalid shape. */
size_t e2ttt_state_elems(const e2ttt_shape* shape);

/* Bytes of device scratch the forward (for_bwd = 0) or backward (for_bwd = 1)
 * needs for `shape`. Returns 0 for an invalid shape. */
size_t e2ttt_workspace_bytes(const e2ttt_shape* shape, int for_bwd);

/* Number of chunks, ceil(T / C); 0 for an invalid shape. */
int e2ttt_num_chunks(const e2ttt_shape* shape);

/* Bytes of saved_states for `shape`: n_chunks * B * H * 2 * S * 4, plus with
 * save_acts = 1 the per-chunk activations ([n_chunks, B, H, C, d_v] bf16 E,
 * then [n_chunks, B, H, C, 2 d_h] (SwiGLU) or [.., d_h] (GELU MLP) bf16 dH;
 * each region 256-byte aligned). 0 for an invalid shape. The backward only
 * reads saved_states. */
size_t e2ttt_saved_bytes(const e2ttt_shape* shape);

/* 1 if e2ttt_chunk_scan_fwd runs `shape` on the tcgen05 tensor cores (given
 * 16-byte aligned pointers), 0 if on the fp32 CUDA-core kernels (always 0 with
 * gemm = E2TTT_GEMM_FP32), -1 if the shape is invalid. */
int e2ttt_fwd_uses_tensor_cores(const e2ttt_shape* shape);

/* The two scalar kernels of every chunk (atlas.scime.ai summary, "Approach":
 * the token-wise recurrence with momentum and decay, unrolled over a chunk,
 * gives a momentum kernel and a weight kernel, computed from sums of logarithms;
 * arxivlens "Results": their cost is sums over the tokens after t, taken in log
 * space, and sums of ratios of gate products).
 *   a[b,h,t] = eta_t U(t+1,C)                       momentum kernel
 *   b[b,h,t] = eta_t sum_{j=t..C} L(j+1,C) U(t+1,j) weight kernel
 *   chunk_scalars [3, B, H, n_chunks]: U(1,C), L(1,C), sum_j L(j+1,C) U(1,j)
 * t counts from the start of its chunk. Inputs lr/mom/decay [B,H,T] fp32
 * (mom NULL, i.e. mu = 0, in no-momentum mode); outputs a, b [B,H,T] fp32.
 * Device pointers; asynchronous on `stream`. */
e2ttt_status e2ttt_chunk_coeffs(const e2ttt_shape* shape,
                                const float* lr, const float* mom, const float* decay,
                                float* a, float* b, float* chunk_scalars,
                                void* stream);

/* Forward over all T tokens (abstract: closed-form chunk state transition;
 * "Limitations": output at the chunk-start weights).
 *   Inputs:  q, k, v (act dtype), lr, mom, decay, W0 (fp32), M0 (fp32; may be
 *            NULL, meaning a zero momentum state).
 *   Outputs: out (act dtype), W_end, M_end (fp32, the states after the last
 *            chunk), saved_states (may be NULL; needed by the backward).
 *   No-momentum mode (shape->momentum = E2TTT_NO_MOMENTUM): mom, M0 and M_end
 *   must be NULL; saved_states then hold W and a zero M for every chunk.
 *   Paths: bf16 activations with C % 128 == 0 and d_k, d_v (and d_h for the
 *   SwiGLU and GELU MLPs) multiples of 128 run on the tcgen05 tensor cores
 *   (bf16 operands, fp32 accumulation and state); a shorter last chunk
 *   (T % C != 0) runs there padded to C tokens, its padding rows adding
 *   nothing. Every other shape and fp32 activations run on fp32 CUDA-core
 *   kernels. */
e2ttt_status e2ttt_chunk_scan_fwd(const e2ttt_shape* shape,
                                  const void* q, const void* k, const void* v,
                                  const float* lr, const float* mom, const float* decay,
                                  const float* W0, const float* M0,
                                  void* out, float* W_end, float* M_end,
                                  float* saved_states,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/* e2ttt_chunk_scan_fwd for callers that cannot allocate device memory: the
 * same forward, same arguments minus the workspace, with the scratch taken from
 * a 32 MiB array owned by the library (no counterpart in the paper; this is a
 * deployment convenience). Callers such as applications whose device memory is
 * already claimed by their own pool allocator, C hosts without a device
 * allocator, or loops that cannot afford cudaMalloc's implicit synchronisation
 * use it instead of providing a workspace.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The array lives in device memory of every GPU on which the library's
 *     kernels are loaded, for the life of the process.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     Calls outside capture look it up again, so a context made anew on the
 *     device (after cudaDeviceReset) gets its own address; calls under capture
 *     reuse the address the last uncaptured call found, so after a reset make
 *     one uncaptured call before capturing again.
 *   - Shapes whose workspace (e2ttt_workspace_bytes(shape, 0)) exceeds 32 MiB
 *     return E2TTT_ERR_INVALID_ARG with the sizes in e2ttt_last_error(); the
 *     tiny linear and the d=128 SwiGLU workloads fit, the 1.3B layer does not.
 *   - All calls share the array and it keeps the last call's contents; calls
 *     that overlap on the GPU (several streams or host threads) race on it and
 *     must be serialised by the caller.
 *   - The status of the device-side bounded waits is read with
 *     e2ttt_noalloc_status (the caller never sees the array's address). */
e2ttt_status e2ttt_chunk_scan_fwd_noalloc(const e2ttt_shape* shape,
                                          const void* q, const void* k, const void* v,
                                          const float* lr, const float* mom, const float* decay,
                                          const float* W0, const float* M0,
                                          void* out, float* W_end, float* M_end,
                                          float* saved_states, void* stream);

/* Status of the device-side bounded waits of the last
 * e2ttt_chunk_scan_fwd_noalloc call on the current device (the no-allocation
 * counterpart of e2ttt_workspace_status, whose status word lives in the
 * library's static array): synchronizes `stream`, then returns
 * E2TTT_ERR_TIMEOUT if a tensor-core kernel gave up waiting (that call's
 * outputs are then invalid), else E2TTT_OK; E2TTT_ERR_CUDA if there is no
 * usable current device. Not for use under stream capture. No counterpart in
 * the paper. */
e2ttt_status e2ttt_noalloc_status(void* stream);

/* Backward of e2ttt_chunk_scan_fwd for the scalar objective
 *     L = sum_t <dout_t, out_t> + <dW_end, W_end> + <dM_end, M_end>
 * (abstract: with the closed form, training proceeds chunk by chunk with all
 * tokens of a chunk in parallel). Chunks run in reverse;
 * the gradient of the chunk-end states flows into the previous chunk. Second
 * order terms through g_t(W0, k_t, v_t) are included (no stop-gradient).
 *   Inputs:  q, k, v, lr, mom, decay, saved_states (from the forward), dout
 *            (act dtype), dW_end, dM_end (fp32 [B,H,S]; may be NULL = zero).
 *   Outputs: dq, dk, dv (act dtype), dlr, dmom, ddecay (fp32 [B,H,T]),
 *            dW0, dM0 (fp32 [B,H,S]).
 *   No-momentum mode: mom, dM_end, dmom and dM0 must be NULL.
 *   Paths: the SwiGLU and GELU MLP backward with bf16 activations (shapes as
 *   for the forward's tensor-core path, a shorter last chunk included) runs on
 *   the tensor cores; the linear fast weight and fp32 activations run on fp32
 *   CUDA cores. */
e2ttt_status e2ttt_chunk_scan_bwd(const e2ttt_shape* shape,
                                  const void* q, const void* k, const void* v,
                                  const float* lr, const float* mom, const float* decay,
                                  const float* saved_states, const void* dout,
                                  const float* dW_end, const float* dM_end,
                                  void* dq, void* dk, void* dv,
                                  float* dlr, float* dmom, float* ddecay,
                                  float* dW0, float* dM0,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Status of the device-side bounded waits of the last compute call that used
 * `workspace`: synchronizes `stream`, then returns E2TTT_ERR_TIMEOUT if a
 * tensor-core kernel gave up waiting (its outputs are then invalid; the CUDA
 * context stays usable), else E2TTT_OK. The status word is the first 4 bytes
 * of the workspace and is reset by every compute call. */
e2ttt_status e2ttt_workspace_status(const void* workspace, void* stream);

/* Failure-detection test hook (no counterpart in the paper). on = 1 arms it:
 * the next e2ttt_chunk_scan_fwd that runs on the tensor cores makes one CTA of
 * its first GEMM launch wait on an mbarrier that nothing ever completes, and
 * limits every wait of that launch to 1 ms instead of 1 s. The wait runs out,
 * the CTA records the failure in the workspace status word, waits (bounded) for
 * its own copies in flight, frees its tensor memory and exits; no memory access
 * is changed. e2ttt_workspace_status then returns E2TTT_ERR_TIMEOUT, that call's
 * outputs are invalid, and the CUDA context stays usable: the next call runs
 * normally. The hook disarms itself once used; on = 0 disarms it. */
void e2ttt_test_stall_next_forward(int on);

/* Launch tracing. While enabled, every kernel the library launches is
 * bracketed by a pair of CUDA events recorded on its launch stream (events are
 * created by the library and reused; no device memory is allocated).
 * e2ttt_trace_enable(1) starts a fresh record, (0) stops and discards it.
 * e2ttt_trace_summary() waits for the recorded events, returns a JSON object
 * {"launches": N, "kernels": {name: {"launches": n, "total_ms": t}}} and
 * starts a fresh record; the string stays valid until the next call. */
void e2ttt_trace_enable(int on);
const char* e2ttt_trace_summary(void);

/* Static description of a status code. */
const char* e2ttt_status_string(e2ttt_status status);

/* Human-readable detail of the last failed call on the calling thread ("" if
 * none). The pointer stays valid until the thread's next library call. */
const char* e2ttt_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* E2TTT_H */
