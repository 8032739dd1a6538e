/*
 * ss.h -- C ABI of the B200 (sm_100a) selective-scan library (libss.so).
 *
 * The operation is Mamba's selective state-space scan (S6):
 *     Delta_t = softplus(delta_t + bias)         (or delta_t + bias)
 *     h_t     = exp(Delta_t * A) (.) h_{t-1} + Delta_t * B_t * u_t
 *     y_t     = (C_t . h_t + D * u_t) * SiLU(z_t)
 * per (batch, channel), with an N-wide diagonal state per channel.
 * Definitions: "Mamba" (stanleyjacob.dev/oss/mamba), Part IV Stage 3 (Delta,
 * A = -exp(A_log)), Stage 4 (zero-order hold for A, Euler rule for B), Stage 5
 * (selective_scan_fn argument list and shapes), Stage 6 (skip, then SiLU(z)
 * gate), Stage 7 (backward by recomputation; decode as one in-place step).
 * Checkpoints every 64 steps: "Mamba, on a laptop GPU." (anamaya.fyi), "The
 * state lives in registers".  Final state for decode continuation:
 * "mamba-metal" README, "Long-context prompts (parallel prefill)".
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, dense and
 *     row-major (the last index fastest).  The library allocates no memory.
 *   - Shapes: u, delta, z, y, dy, du, ddelta, dz: (batch, dim, seqlen);
 *     A: (dim, dstate); B, C: (batch, dstate, seqlen) -- shared by all
 *     channels of a batch row; D, delta_bias: (dim,); states: (batch, dim,
 *     dstate); checkpoints: (batch, dim, ceil(seqlen/64), dstate).
 *   - dtype (ss_dtype) is the storage type of u, delta, z, B, C, y, dy, du,
 *     ddelta, dz.  A, D, delta_bias, states, checkpoints, dA, dB, dC, dD and
 *     ddelta_bias are always fp32.  All arithmetic is fp32 with fp32 state.
 *   - Pointers must be aligned to their element size; 16-byte aligned rows
 *     take the vectorised path.  z, D, delta_bias may be NULL (no gate, zero
 *     skip, zero bias).  dstate must be 16.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns once its kernels are enqueued.  Launch
 *     errors are reported as SS_ERR_CUDA.  Invalid arguments are rejected
 *     before anything is enqueued.  A non-OK status sets a thread-local
 *     message readable with ss_last_error().  No C++ exception crosses the ABI.
 *   - Testing error paths: with the environment variable SS_FAIL_LAUNCH set
 *     (to anything but "0"), every call that would launch kernels returns
 *     SS_ERR_CUDA instead, with nothing enqueued and a message naming the
 *     injection.  SS_BWD_VARIANT (0..3) forces the reverse-walk variant of
 *     ss_bwd (see ss_bwd_path); variant 3 is honoured only where it applies.
 *   - There is no silent fallback: an unsupported shape or dtype is an error.
 *   - Results are bitwise reproducible run to run (no floating-point atomics).
 */
#ifndef SS_H_
#define SS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SS_API __attribute__((visibility("default")))
#else
#define SS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ss_dtype { SS_F32 = 0, SS_BF16 = 1, SS_F16 = 2 } ss_dtype;

typedef enum ss_status {
  SS_OK = 0,
  SS_ERR_INVALID_ARG = 1,  /* null required pointer, non-positive size, bad dtype */
  SS_ERR_UNSUPPORTED = 2,  /* valid but not implemented here (e.g. dstate != 16)   */
  SS_ERR_ALIGNMENT = 3,    /* a pointer not aligned to its element size           */
  SS_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than the size query says  */
  SS_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed         */
  SS_ERR_INTERNAL = 6
} ss_status;

#define SS_CHECKPOINT_CHUNK 64 /* steps between state checkpoints */

/* Library version (major*10000 + minor*100 + patch). */
SS_API int ss_version(void);

/* Message for the last non-OK status returned on the calling thread. */
SS_API const char* ss_last_error(void);

/* Static name of a status code. */
SS_API const char* ss_status_string(int status);

/*
 * Which forward path a problem takes on the current device:
 *   0 = per-channel scan (one pass over L per channel),
 *   1 = chunk-parallel scan (L split into *num_segments segments, a
 *       (decay, increment) carry scan across them, then a second pass).
 * The choice depends only on batch*dim, seqlen and the SM count.
 * Returns -1 (and sets ss_last_error) on invalid arguments.
 */
SS_API int ss_fwd_path(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                int64_t* num_segments);

/* Bytes of device workspace ss_fwd needs for this problem on the current
 * device (0 on the per-channel path).  (size_t)-1 on invalid arguments. */
SS_API size_t ss_fwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen);

/*
 * Forward scan ("Mamba", Part IV Stages 4-6; Part V "the hardware-aware scan
 * kernel").  Reads u, delta, z, A, B, C, D, delta_bias; writes
 *   y            (batch, dim, seqlen), dtype                     required
 *   final_state  (batch, dim, dstate) fp32, state after step L-1  or NULL
 *   checkpoints  (batch, dim, ceil(seqlen/64), dstate) fp32      or NULL
 *                entry k = state after step min(64k+63, L-1); the backward
 *                needs them, inference may pass NULL.
 * workspace: device memory of at least ss_fwd_workspace_size() bytes (may be
 * NULL when that size is 0); its contents need not be initialised.
 */
SS_API ss_status ss_fwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                 const void* u, const void* delta, const void* z, const float* A,
                 const void* B, const void* C, const float* D, const float* delta_bias,
                 int delta_softplus, void* y, float* final_state, float* checkpoints,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * ss_fwd with an initial state and packed documents.
 *   h0       (batch, dim, dstate) fp32, 16-byte aligned, or NULL (zero state)
 *   seq_idx  (batch, seqlen) int32 document ids, or NULL (one document per row).
 *            Wherever the id changes between step t-1 and t, the state
 *            restarts from zero before step t, so a packed row equals its
 *            documents run one by one (niverel-mamba README, "seq_idx strict
 *            reset").  Step 0 starts from h0.
 * Running a sequence in pieces -- each piece's h0 the previous piece's
 * final_state -- gives the same y and states as one call over the whole
 * sequence (chunked prefill: the mlx-mamba3 README, "Supported Features" and
 * "Verification & Status"; the prefill state handed to decode: the
 * "mamba-metal" README, "Long-context prompts").  Checkpoints are the states
 * after each 64-step chunk of this call's own sequence.
 */
SS_API ss_status ss_fwd_with_state(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                   int dtype, const void* u, const void* delta, const void* z,
                                   const float* A, const void* B, const void* C, const float* D,
                                   const float* delta_bias, int delta_softplus, const float* h0,
                                   const int32_t* seq_idx, void* y, float* final_state,
                                   float* checkpoints, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * ss_fwd_noalloc -- the forward scan for callers that cannot allocate device
 * memory.  (An addition of this library: the pages have no counterpart.)
 *
 * Some callers cannot hand ss_fwd a workspace: code that must not call
 * cudaMalloc because it synchronises the device and can fail mid-run (a
 * real-time decode loop, a memory planner that owns every byte of the GPU),
 * or a host that links this library but gives it no allocator.  This entry
 * point takes the same arguments as ss_fwd minus the workspace, and uses a
 * scratch area compiled into the library instead: a fixed
 * SS_FWD_NOALLOC_SCRATCH_BYTES array in device memory, which every GPU that
 * loads the library keeps until the process exits.  Only the chunk-parallel
 * path needs scratch; a problem whose ss_fwd_workspace_size() exceeds the
 * array is rejected with SS_ERR_WORKSPACE (nothing is enqueued).
 *
 * - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * - Every call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress, which allocates nothing), so the address stays
 *   right across device resets and contexts.  Make the first call on a device
 *   before any stream capture: that call loads the module onto the device.
 * - All calls share the one array and it keeps the last call's contents.
 *   Nothing in it needs clearing: every word the kernels read is written
 *   earlier in the same call.  Calls whose work overlaps on the GPU (other
 *   streams, other host threads) race on it: order them on one stream or with
 *   events.
 * Results are identical to ss_fwd on the same inputs.
 */
#define SS_FWD_NOALLOC_SCRATCH_BYTES (4u << 20)
SS_API ss_status ss_fwd_noalloc(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                int dtype, const void* u, const void* delta, const void* z,
                                const float* A, const void* B, const void* C, const float* D,
                                const float* delta_bias, int delta_softplus, void* y,
                                float* final_state, float* checkpoints, void* stream);

/* Bytes of device workspace ss_bwd needs.  (size_t)-1 on invalid arguments.
 * The size covers the most chunk groups the reverse walk may use (below), so
 * it depends on the problem only, not on the device. */
SS_API size_t ss_bwd_workspace_size(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen);

/*
 * How ss_bwd walks a problem on the current device.  Returns the walk variant
 *   0 = one channel per 4-lane group (16 channels per 64-thread block),
 *   1 = two channels per 4-lane group, 32 channels per block,
 *   2 = two channels per 4-lane group, 16 channels per one-warp block,
 * and stores in *num_groups (if non-NULL) how many groups of whole 64-step
 * chunks are walked in parallel (1..16).  With more than one group, the
 * states pass also composes each chunk's map of the reverse gradient carry,
 * c -> P_k c + e_k (P_k the product of the chunk's decays, e_k the carry the
 * chunk's own steps produce), and a scan over those maps gives each group
 * the carry entering its last step.  The result assumes 16-byte aligned
 * rows; -1 (with ss_last_error) on invalid arguments.
 */
SS_API int ss_bwd_path(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                int64_t* num_groups);

/*
 * Backward scan for the loss <dy, y> ("Mamba", Part IV Stage 7: recompute the
 * states rather than store them; gradients for u, Delta, A, B, C, D, z).
 * States are recomputed chunk by chunk from `checkpoints` written by ss_fwd on
 * the same inputs ("Mamba, on a laptop GPU.", "The state lives in registers":
 * walk the chunks in reverse, carry the state gradient across boundaries).
 * Outputs (all overwritten, never accumulated into):
 *   du, ddelta   (batch, dim, seqlen) dtype          required
 *   dz           (batch, dim, seqlen) dtype          required iff z != NULL
 *   dA           (dim, dstate) fp32                  required
 *   dB, dC       (batch, dstate, seqlen) fp32        required
 *   dD           (dim,) fp32 = sum dy*SiLU(z)*u      or NULL
 *   ddelta_bias  (dim,) fp32 = sum over batch, time of ddelta   or NULL
 * ddelta is the gradient with respect to delta (before bias and softplus).
 * Channel sums (dB, dC) and batch sums (dA, dD, ddelta_bias) are formed in a
 * fixed order in `workspace` (>= ss_bwd_workspace_size() bytes) by separate
 * reduction kernels: deterministic, no atomics.  The reverse walk may run in
 * parallel over groups of 64-step chunks (see ss_bwd_path); the result does
 * not depend on the device beyond fp32 rounding order, and is bitwise
 * repeatable on a given device.
 */
SS_API ss_status ss_bwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                 const void* u, const void* delta, const void* z, const float* A,
                 const void* B, const void* C, const float* D, const float* delta_bias,
                 int delta_softplus, const void* dy, const float* checkpoints,
                 void* du, void* ddelta, void* dz, float* dA, float* dB, float* dC,
                 float* dD, float* ddelta_bias, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * ss_bwd for a piece of a longer sequence, the adjoint of ss_fwd_with_state:
 *   h0      (batch, dim, dstate) fp32, the forward's initial state, or NULL
 *   dfinal  (batch, dim, dstate) fp32, the gradient reaching this piece's
 *           final state from later pieces (their dh0), or NULL (zero)
 *   dh0     (batch, dim, dstate) fp32 output, the gradient of the loss with
 *           respect to h0, or NULL (not written)
 *   seq_idx (batch, seqlen) int32 or NULL: as in the forward; no gradient
 *           crosses a document start.
 * The loss is <dy, y> + <dfinal, final_state>.  The states are 16-byte
 * aligned.  Walking the pieces last to first, each piece's dfinal the next
 * piece's dh0, reproduces the one-call gradients (dA, dD, ddelta_bias summed
 * over the pieces by the caller).
 */
SS_API ss_status ss_bwd_with_state(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                   int dtype, const void* u, const void* delta, const void* z,
                                   const float* A, const void* B, const void* C, const float* D,
                                   const float* delta_bias, int delta_softplus, const float* h0,
                                   const int32_t* seq_idx, const void* dy, const float* dfinal,
                                   const float* checkpoints,
                                   void* du, void* ddelta, void* dz, float* dA, float* dB,
                                   float* dC, float* dD, float* ddelta_bias, float* dh0,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Causal depthwise conv1d + SiLU, the step before the scan ("Mamba", Part IV
 * Stage 2: each of the d_inner channels has its own width-d_conv filter,
 * padded on the left only, so position t sees t-(W-1) .. t; then a SiLU).
 *   pre[b,d,t] = bias[d] + sum_{k<W} w[d,k] xin[b,d,t-(W-1)+k]
 *   u[b,d,t]   = silu ? pre * sigmoid(pre) : pre
 * xin is x for t >= 0 and, before t = 0, the window state_in (the W-1 inputs
 * preceding this call's sequence, oldest first) or zero when state_in is NULL.
 *   x, u       (batch, dim, seqlen) dtype
 *   w          (dim, width) fp32;  bias (dim,) fp32 or NULL;  width in 1..4
 *   state_in   (batch, dim, width-1) fp32 or NULL
 *   state_out  (batch, dim, width-1) fp32 or NULL: the last width-1 inputs,
 *              the window a continuation or ss_conv1d_step starts from
 *   seq_idx    (batch, seqlen) int32 or NULL: packed documents; the window
 *              restarts from zero at every change of id, so no input reaches
 *              an output of another document, and state_out keeps only the
 *              last document's inputs
 * u is an input of x_proj (which produces delta, B, C), so it is computed
 * here, before the scan, rather than inside the scan's prologue.
 */
SS_API ss_status ss_conv1d_fwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t width, int dtype,
                               const void* x, const float* w, const float* bias,
                               const float* state_in, const int32_t* seq_idx, int silu, void* u,
                               float* state_out, void* stream);

/* Bytes of device workspace ss_conv1d_bwd needs.  (size_t)-1 on invalid arguments. */
SS_API size_t ss_conv1d_bwd_workspace_size(int64_t batch, int64_t dim, int64_t seqlen, int64_t width);

/*
 * Adjoint of ss_conv1d_fwd for the loss <du, u> + <dstate_out, state_out>:
 *   dx         (batch, dim, seqlen) dtype           required
 *   dw         (dim, width) fp32, summed over batch and time     required
 *   dbias      (dim,) fp32 or NULL
 *   dstate_in  (batch, dim, width-1) fp32 or NULL: gradient of state_in
 * dstate_out (nullable) is the gradient reaching state_out from a later piece
 * (its dstate_in).  dw and dbias are summed in a fixed order through
 * `workspace` (>= ss_conv1d_bwd_workspace_size() bytes): deterministic.
 */
SS_API ss_status ss_conv1d_bwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t width, int dtype,
                               const void* x, const float* w, const float* bias,
                               const float* state_in, const int32_t* seq_idx, int silu,
                               const void* du, const float* dstate_out, void* dx, float* dw,
                               float* dbias,
                               float* dstate_in, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * One decode step of the convolution ("Mamba", Part II and Part IV Stage 7:
 * the step path advances the small convolution window): u = SiLU(bias +
 * w . [window, x]), then the window drops its oldest input and appends x.
 *   state  (batch, dim, width-1) fp32, in/out (NULL only when width == 1)
 *   x, u   (batch, dim) dtype
 */
SS_API ss_status ss_conv1d_step(int64_t batch, int64_t dim, int64_t width, int dtype, float* state,
                                const void* x, const float* w, const float* bias, int silu, void* u,
                                void* stream);

/*
 * Mamba-2 SSD forward ("Mamba", Part V, "Deep dive: Mamba-2 and state-space
 * duality": A a scalar per head, multi-head with B and C shared by groups of
 * heads; computed as a masked quadratic form inside 64-step chunks and a
 * recurrence between chunks, on the tensor cores).  Per batch b, head h (group
 * g = h / (nheads / ngroups)):
 *   Delta_t = softplus(dt_t + dt_bias_h)   (dt_t + dt_bias_h without softplus)
 *   H_t     = exp(Delta_t A_h) H_{t-1} + Delta_t x_t B_t^T      H: headdim x dstate
 *   y_t     = (H_t C_t + D_h x_t) * SiLU(z_t)                    (no gate: z NULL)
 * Time-major layouts (as in Mamba-2):
 *   x, z, y      (batch, seqlen, nheads, headdim)  dtype (bf16 or fp16)
 *   dt           (batch, seqlen, nheads)           dtype
 *   B, C         (batch, seqlen, ngroups, dstate)  dtype
 *   A, D, dt_bias (nheads,) fp32; D, dt_bias may be NULL
 *   h0, final_state (batch, nheads, headdim, dstate) fp32 or NULL
 * headdim 64, dstate 64 or 128 (else SS_ERR_UNSUPPORTED).  x, z, y, B, C and
 * the states are 16-byte aligned.  The inter-chunk read-out uses a bf16/fp16
 * copy of the state as its tensor-core operand; the state itself is fp32.
 * The products run as tcgen05 MMAs with TMEM accumulators and TMA-loaded
 * operand tiles; with the environment variable SS_SSD_VARIANT=mma they run
 * on the warp-level mma.sync kernel instead (same arithmetic, kept for
 * comparison).  The tcgen05 kernel bounds every wait on its copies and
 * products: a wait that runs out sets a bit in the device fault word
 * (ss_device_fault) and the kernel returns early with y incomplete, after
 * waiting (bounded) for its copies and products in flight and freeing its
 * TMEM.  Test hook: with SS_INJECT_WAIT_TIMEOUT set, the first chunk's copy
 * wait runs out on a barrier nothing arrives on.
 */
SS_API ss_status ss_ssd_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                            int64_t ngroups, int64_t dstate, int dtype, const void* x, const void* dt,
                            const float* A, const void* B, const void* C, const float* D,
                            const void* z, const float* dt_bias, int dt_softplus, const float* h0,
                            void* y, float* final_state, void* stream);

/*
 * Sequence sharding ("mamba-metal" README, "Long-context prompts (parallel
 * prefill)": the state passed between pieces of a long sequence).  A segment
 * of the scan run from an initial state h0 ends in h_end = P o h0 + E, where
 * E is its end state from zero and P its diagonal state transition
 *   P[b][d][n] = prod_t exp(Delta_t A[d][n]) = exp(A[d][n] sum_t Delta_t),
 *   Delta_t = softplus(delta_t + delta_bias_d) (without softplus: delta + bias).
 * ss_segment_decay writes P (batch, dim, dstate) fp32 for the segment given
 * by delta (batch, dim, seqlen) dtype; A (dim, dstate) fp32, delta_bias (dim,)
 * fp32 or NULL.  The sum runs over each row in a fixed order.  Packed
 * documents (seq_idx) are not covered: a document start inside a segment
 * would zero P.
 * ss_state_chain chains nseg segments elementwise (count elements each; P, E,
 * out: (nseg, count) fp32, init: (count,) fp32 or NULL for zero):
 *   reverse = 0:  out[0] = init,        out[s+1] = P[s] o out[s] + E[s]
 *                 (the state entering each segment, E = end states from zero)
 *   reverse = 1:  out[nseg-1] = init,   out[s-1] = P[s] o out[s] + E[s]
 *                 (the adjoint leaving each segment, E = dh0 of each segment
 *                 run with a zero adjoint at its end)
 * Both are asynchronous on `stream`; SS_ERR_INVALID_ARG for missing pointers
 * or non-positive sizes, SS_ERR_ALIGNMENT for misaligned fp32 pointers,
 * SS_ERR_UNSUPPORTED beyond batch * dim < 2^31 (segment_decay) or count <=
 * 2^38, nseg <= 65536 (state_chain).
 */
SS_API ss_status ss_segment_decay(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, int dtype,
                                  const void* delta, const float* A, const float* delta_bias,
                                  int delta_softplus, float* P, void* stream);
SS_API ss_status ss_state_chain(int64_t count, int64_t nseg, const float* P, const float* E,
                                const float* init, int reverse, float* out, void* stream);

/* Which SSD forward kernel ss_ssd_fwd launches (reads SS_SSD_VARIANT). */
#define SS_SSD_PATH_TCGEN05 0
#define SS_SSD_PATH_MMA 1
SS_API int ss_ssd_fwd_path(void);

/*
 * Device fault word of the kernels that bound their waits (the tcgen05 SSD
 * forward): 0 when no wait ran out since the last clear; bit 0 a copy-wait
 * timeout, bit 1 a product-wait timeout, bit 2 a drain timeout at exit.
 * Synchronizes the current device first; clear != 0 resets the word.
 * Returns -1 (and sets ss_last_error) when the device reports an error.
 */
SS_API int ss_device_fault(int clear);

/*
 * Mamba-2 SSD backward: the gradient of the loss <dy, y> + <dfinal, final_state>
 * of ss_ssd_fwd with respect to every input ("Mamba", Part IV Stage 7, the
 * backward of the scan, applied to the Part V recurrence).  Per (b, h) with
 * dout_t = dy_t SiLU(z_t) and G_t = dL/dH_t:
 *   G_t    = exp(Delta_{t+1} A_h) G_{t+1} + dout_t C_t^T      (G_{L-1} from dfinal)
 *   dx_t   = Delta_t G_t B_t + D_h dout_t
 *   dB_t   = sum over the group's heads of Delta_t G_t^T x_t;   dC_t likewise of H_t^T dout_t
 *   dDelta = x_t^T G_t B_t + A_h <G_t, exp(Delta_t A_h) H_{t-1}>;  ddt = dDelta sigmoid(dt + dt_bias)
 *            with softplus (dDelta without);  dA_h, dD_h, ddt_bias_h summed over b, t
 *   dz_t   = dy_t (H_t C_t + D_h x_t) sigmoid(z_t) (1 + z_t (1 - sigmoid(z_t)))
 *   dh0    = G before step 0 (the adjoint of h0)
 * Inputs as in ss_ssd_fwd, plus dy (batch, seqlen, nheads, headdim) dtype and
 * dfinal (batch, nheads, headdim, dstate) fp32 or NULL (zero).  Outputs, all
 * overwritten, device memory owned by the caller:
 *   dx (like x), ddt (like dt): dtype;  dz (like z) dtype, or NULL (not written;
 *   must be NULL without z);  dB, dC (batch, seqlen, ngroups, dstate) fp32;
 *   dA (nheads) fp32;  dD, ddt_bias (nheads) fp32 or NULL;  dh0 like h0, or NULL.
 * The work runs chunk by chunk (64 steps): the chunk maps of the state and the
 * adjoint, one pass over the chunks per state element, then every chunk's
 * gradient; dB, dC are summed over heads and dA, dD, ddt_bias over chunks in a
 * fixed order, so results are bitwise reproducible.  The maps and the chunk
 * gradients are tcgen05 products with fp32 accumulation on fp16 operands
 * (11-bit significand; bf16 inputs are converted exactly, derived operands such
 * as dout and the decayed masks are rounded to fp16), and the state/adjoint
 * slabs and the dB/dC partials in the workspace are stored as fp16 (every
 * recurrence and sum runs in fp32), so |values| beyond the fp16 range, 65504,
 * overflow there; SS_SSD_VARIANT=mma runs tf32 mma.sync kernels on fp32
 * slabs instead.  A chunk-gradient CTA takes up to 8 heads of one group at the
 * same chunk (the largest divisor of the heads per group that still gives
 * every SM a CTA) and sums their dB/dC in its fp32 accumulators before it
 * stores one fp16 partial; SS_SSD_HEADS_PER_CTA=max (or =n) takes the largest
 * divisor up to 8 (up to n) whatever the grid (a test and tuning switch).
 * Bounded waits report through ss_device_fault.  `workspace`: device memory
 * of at least ss_ssd_bwd_workspace_size() bytes, 256-byte aligned.  Same
 * size limits and error codes as ss_ssd_fwd; SS_ERR_WORKSPACE when the
 * workspace is missing or too small.
 */
SS_API size_t ss_ssd_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                        int64_t ngroups, int64_t dstate);
SS_API ss_status ss_ssd_bwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                            int64_t ngroups, int64_t dstate, int dtype, const void* x, const void* dt,
                            const float* A, const void* B, const void* C, const float* D,
                            const void* z, const float* dt_bias, int dt_softplus, const float* h0,
                            const void* dy, const float* dfinal, void* dx, void* ddt, float* dA,
                            float* dB, float* dC, float* dD, void* dz, float* ddt_bias, float* dh0,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step on a cached state, in place ("Mamba", Part IV Stage 7: one
 * token in, a fixed-size state updated in place, one token out; "mamba-metal"
 * README, "O(1) per token via state caching").  Exactly one iteration of the
 * forward recurrence:
 *   state (batch, dim, dstate) fp32  in/out
 *   u, delta, z, y (batch, dim) dtype;  B, C (batch, dstate) dtype
 * Capturable in a CUDA graph (a single kernel, no host synchronisation).
 */
SS_API ss_status ss_state_update(int64_t batch, int64_t dim, int64_t dstate, int dtype,
                          float* state, const void* u, const void* delta, const void* z,
                          const float* A, const void* B, const void* C, const float* D,
                          const float* delta_bias, int delta_softplus, void* y,
                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SS_H_ */
