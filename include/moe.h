/*
 * moe.h -- C ABI of libmoe.so: a deterministic mixture-of-experts layer
 * (forward and backward) on one B200 GPU.
 *
 * The operation is the MoE layer described by "Cursor open-sources
 * Mixture-of-Kittens (MoK): a deterministic MoE training megakernel"
 * (page 1, sections "MoE layer as the bottleneck" and "Three design decisions
 * that matter"): tokens are routed to their top-k experts, dispatched into an
 * expert-contiguous layout, run through SwiGLU experts as expert-grouped
 * GEMMs, and combined back with their gate weights; the backward mirrors it
 * (reverse-combine, grouped dgrad/wgrad, reverse-dispatch), with the router
 * weight gradient taken inside the SwiGLU backward.  The pages print no
 * formula; the arithmetic is the plain top-k softmax-gated SwiGLU mixture:
 *
 *   l = X W_r + b,  S_t = top-k(l_t) (descending, ties -> lower expert id)
 *   g_t,e = softmax over the k selected logits
 *   H = silu(X_t W_gate[e]) * (X_t W_up[e]),   Y_t = sum_{e in S_t} g_t,e H W_down[e]
 *
 * Conventions for every entry point
 * ---------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller; the library
 *   never allocates, frees or keeps them after the call returns.
 * - bf16 tensors are row-major, 16-byte aligned, and passed as void*.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is only
 *   enqueued: no entry point except moe_get_error synchronises the stream or
 *   reads device memory on the host.
 * - Argument errors are returned synchronously and nothing is enqueued.
 * - Device-side errors (a bounded wait that ran out, non-finite router logits)
 *   set a status word inside `ctx`; moe_get_error reads it.  moe_fwd clears it.
 * - Results are bit-reproducible: fixed reduction orders, no float atomics.
 *
 * Limits: 1 <= E <= 512; 1 <= top_k <= min(E, 16); d and I multiples of 256;
 * 0 <= T and T * top_k < 2^31; 0 <= first_local_expert,
 * first_local_expert + num_local_experts <= E.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,          /* null pointer, bad shape, misaligned tensor */
  MOE_ERR_UNSUPPORTED = 2,          /* shape or mode outside the limits above */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3,  /* ctx or workspace smaller than the *_size() call says */
  MOE_ERR_CUDA = 4,                 /* a CUDA runtime call failed (launch, attribute, ...) */
  MOE_ERR_DEVICE_TIMEOUT = 5,       /* a bounded device-side wait ran out */
  MOE_ERR_NONFINITE = 6,            /* a router logit was NaN or +-Inf */
  MOE_ERR_EXCHANGE = 7              /* expert-parallel exchange buffers held tables that do not fit
                                       together (routing of another step, or not published) */
} moe_status;

typedef enum moe_precision {
  MOE_BF16 = 0,  /* bf16 operands, fp32 accumulation */
  MOE_MXFP8 = 1,  /* E4M3 operands with one E8M0 scale per 32 along each GEMM's contraction dim:
                     use moe_prepare_weights + moe_fwd_mx / moe_bwd_mx (moe_fwd / moe_bwd refuse it).
                     The gate/up, down and both dgrad GEMMs are MXFP8; the weight-gradient GEMMs
                     contract over tokens from the bf16 operands */
  MOE_MXFP8_ALL = 2  /* MOE_MXFP8 with the two weight-gradient GEMMs on MXFP8 as well: their
                        operands (X, dA, dB, Hg = g H and dY of each expert) quantised along the
                        expert's rows, one scale per 32 rows from its first row, pad rows zero.
                        Same entry points; a larger workspace (moe_workspace_size of this shape) */,
  MOE_NVFP4 = 3  /* moe_fwd_nvfp4 / moe_bwd_nvfp4: E2M1 operands with one E4M3 scale per 16 values
                    along each GEMM's contraction dim and one fp32 scale per tensor */
} moe_precision;

typedef enum moe_wgrad_dtype {
  MOE_WGRAD_BF16 = 0,  /* dW_gate / dW_up / dW_down in bf16, the weights' type (round to nearest even
                          of the fp32 sum) */
  MOE_WGRAD_FP32 = 1   /* the same fp32 sums, unrounded: for optimisers that keep fp32 gradients */
} moe_wgrad_dtype;

/* Layer shape.  Experts [first_local_expert, first_local_expert + num_local_experts)
 * are computed here (num_local_experts = 0 means all E).  Assignments to other
 * experts belong to another rank: they add nothing to Y or to the expert part of dX.
 * wgrad_dtype (moe_wgrad_dtype) is the element type of the expert weight gradients
 * that moe_bwd, moe_bwd_mx and moe_bwd_stream write; the other entry points ignore it
 * (buffer sizes do not depend on it), and any value but 0 or 1 makes the shape invalid. */
typedef struct moe_shape {
  int64_t T;       /* tokens */
  int32_t d;       /* model (hidden) dimension */
  int32_t E;       /* experts the router scores (router width) */
  int32_t I;       /* expert SwiGLU intermediate dimension */
  int32_t top_k;   /* experts per token */
  int32_t prec;    /* moe_precision */
  int32_t first_local_expert;
  int32_t num_local_experts;
  int32_t wgrad_dtype;
} moe_shape;

/* Bytes of the saved-for-backward context that moe_fwd writes and moe_bwd reads
 * (routing table, dispatched tokens, SwiGLU pre-activations, status word).
 * Depends on the shape only.  0 for an invalid shape. */
size_t moe_ctx_size(const moe_shape* shape);

/* Bytes of scratch workspace moe_fwd / moe_bwd need (worst case over routings:
 * padded rows <= T*k + 127*num_local).  0 for an invalid shape. */
size_t moe_workspace_size(const moe_shape* shape);

/* Forward.
 *   X       [T, d]   bf16   tokens
 *   W_r     [d, E]   bf16   router weight
 *   bias    [E]      fp32   router bias added before selection and gating; may be NULL
 *   W_gate  [El, d, I] bf16, W_up [El, d, I] bf16, W_down [El, I, d] bf16  (El = local experts)
 *   Y       [T, d]   bf16   output (written)
 *   ctx     ctx_bytes        saved for moe_bwd (written)
 *   ws      ws_bytes         scratch
 * Implements: router GEMM, top-k + softmax gating, histogram + prefix sums,
 * stable scatter/dispatch (page 1, "Three design decisions", pull dispatch),
 * grouped gate/up GEMM + SwiGLU, grouped down GEMM with the gate multiply,
 * combine (push combine). */
moe_status moe_fwd(const moe_shape* shape, const void* X, const void* W_r, const float* bias,
                   const void* W_gate, const void* W_up, const void* W_down, void* Y,
                   void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes, void* stream);

/* Forward with its two grouped GEMMs in one persistent launch (page 1, the opening paragraph
 * and "Three design decisions that matter": one megakernel fusing the MoE steps, its work
 * scheduled through Cluster Launch Control).  Same arguments, results and ctx as moe_fwd, bit
 * for bit; bf16 mode, one batch (no ring stream).  The routing and dispatch launches of moe_fwd
 * run first and the combine launch last; between them one kernel runs every gate/up tile
 * (SwiGLU epilogue) and then every down tile (gate multiply) as work units that CTAs take in
 * one global order.  A down tile waits, bounded (about 2 s, then MOE_ERR_DEVICE_TIMEOUT in
 * ctx's status word), until every gate/up tile of its 128 rows has stored H, so down tiles
 * start while the last gate/up tiles run.  CTAs of the launch that have not started yet are
 * cancelled by running CTAs, which take over their work (Cluster Launch Control). */
moe_status moe_fwd_persistent(const moe_shape* shape, const void* X, const void* W_r, const float* bias,
                              const void* W_gate, const void* W_up, const void* W_down, void* Y,
                              void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes, void* stream);

/* Backward of the last moe_fwd that wrote `ctx` (same shape, X, W_r, weights).
 *   dY      [T, d]   bf16   upstream gradient
 *   dX      [T, d]   bf16   written
 *   dW_gate, dW_up [El, d, I], dW_down [El, I, d]   written (not accumulated); bf16, or
 *                    fp32 when shape->wgrad_dtype is MOE_WGRAD_FP32
 *   dW_r    [d, E]   fp32   written
 * Implements the mirror of the forward (page 1, "Three design decisions":
 * pull reverse-combine, push reverse-dispatch), grouped dgrad and wgrad with
 * fixed-order reductions, and the router-weight gradient computed inside the
 * SwiGLU backward from <dY W_down^T, H> ("SonicMoE-style", same page). */
moe_status moe_bwd(const moe_shape* shape, const void* X, const void* W_r, const void* W_gate,
                   const void* W_up, const void* W_down, const void* dY, void* ctx, size_t ctx_bytes,
                   void* dX, void* dW_gate, void* dW_up, void* dW_down, float* dW_r,
                   void* ws, size_t ws_bytes, void* stream);

/* Backward with its two dgrad GEMMs in one persistent launch, as moe_fwd_persistent does for the
 * forward: every tile of the dgrad of W_down (SwiGLU backward and router-gate gradient
 * epilogue), then every tile of the dgrad of gate/up, which waits (bounded) for the dgrad of
 * W_down's tiles of its 128 rows.  The router backward runs after that launch instead of
 * between the two GEMMs.  Same arguments and results as moe_bwd, bit for bit; bf16 mode, one
 * batch.  Follows either forward. */
moe_status moe_bwd_persistent(const moe_shape* shape, const void* X, const void* W_r, const void* W_gate,
                              const void* W_up, const void* W_down, const void* dY, void* ctx,
                              size_t ctx_bytes, void* dX, void* dW_gate, void* dW_up, void* dW_down,
                              float* dW_r, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns the device status word held in `ctx`
 * (MOE_OK if no device error since the last moe_fwd), and clears it.
 * Returns MOE_ERR_CUDA if the synchronisation itself failed. */
moe_status moe_get_error(void* ctx, void* stream);

/* Test hook: copies the routing table of the last moe_fwd into caller buffers
 * (device pointers; any may be NULL to skip), local experts only:
 *   ids [T, k] int32, gates [T, k] fp32, counts [El] int32, offsets [El+1] int32,
 *   padded_offsets [El+1] int32 (segments padded to 128 rows), perm [sum counts] int32
 *   (token of each row, ascending token id inside an expert), slot_row [T, k] int32
 *   (padded row of each assignment, -1 for a non-local expert). */
moe_status moe_debug_routing(const moe_shape* shape, const void* ctx, int32_t* ids, float* gates,
                             int32_t* counts, int32_t* offsets, int32_t* padded_offsets,
                             int32_t* perm, int32_t* slot_row, void* stream);

/* Test hook: copies the fp32 router logits [T, E] (bias included) that the last
 * moe_fwd computed in `ws` into `logits` (device pointer). */
moe_status moe_debug_logits(const moe_shape* shape, const void* ws, float* logits, void* stream);

/* Test hook: copies the router-logit gradient of the last moe_bwd that used
 * `ws` into `dl` [T, k] fp32 (device pointer): dl[t, j] = dL/dl_{t, ids[t, j]},
 * the only nonzeros of dL/dlogits (dW_r = X^T dl scattered to the ids). */
moe_status moe_debug_router_grad(const moe_shape* shape, const void* ws, float* dl, void* stream);

/* Test hook for the device-side failure path (no counterpart on the pages):
 * clears ctx's status word, then launches one kernel on `stream` whose mbarrier
 * wait is never satisfied.  The wait is the same bounded wait every GEMM role
 * uses: it gives up after its spin limit (about 2 s), records
 * MOE_ERR_DEVICE_TIMEOUT in ctx's status word and the kernel returns, so the
 * context stays usable; moe_get_error then reports (and clears) the status.
 * ctx as sized by moe_ctx_size(shape).  Returns MOE_ERR_INVALID_ARG for a NULL
 * or misaligned ctx, MOE_ERR_WORKSPACE_TOO_SMALL for a short one, MOE_ERR_CUDA
 * if the launch fails. */
moe_status moe_debug_bounded_wait(const moe_shape* shape, void* ctx, size_t ctx_bytes, void* stream);

/* Test hook for the persistent GEMM pairs' cross-CTA waits (no counterpart on the pages): runs
 * moe_fwd_persistent with the gate/up tiles left out of the persistent launch, so every down
 * tile waits for H rows that nobody writes.  The first wait to reach its limit (about 2 s)
 * records MOE_ERR_DEVICE_TIMEOUT in ctx's status word; every other wait, and every CTA that
 * starts later, sees the status and stops, and the kernel ends.  Y is not valid afterwards;
 * the context stays usable.  Same arguments and argument errors as moe_fwd_persistent. */
moe_status moe_debug_pair_wait(const moe_shape* shape, const void* X, const void* W_r, const float* bias,
                               const void* W_gate, const void* W_up, const void* W_down, void* Y, void* ctx,
                               size_t ctx_bytes, void* ws, size_t ws_bytes, void* stream);

/* Benchmark support (no counterpart on the pages).  When enabled, every
 * kernel launch of the library is bracketed by two CUDA events recorded on the
 * launch stream.  moe_profile_read synchronises the device, writes per kernel
 * id the summed milliseconds and launch counts recorded since the last read
 * (arrays of max_kernels entries; either may be NULL), clears the records and
 * returns the number of kernel ids (or -1 if the synchronisation failed).
 * moe_kernel_name gives a kernel id's name; moe_kernel_launches counts every
 * kernel this library has launched in the process.  Not thread-safe against
 * concurrent enabling. */
moe_status moe_profile_enable(int on);
int moe_profile_read(int max_kernels, double* total_ms, int* launches);
const char* moe_kernel_name(int kernel_id);
unsigned long long moe_kernel_launches(void);

/* ---------------------------------------------------------------------------
 * MXFP8 mode (page 1, closing paragraph of "Three design decisions that matter": the layer
 * has a BF16 and an MXFP8 precision mode).  Shapes
 * carry prec = MOE_MXFP8.  E4M3 codes with one E8M0 scale per 32 values along
 * each GEMM's contraction dimension (OCP MX: scale exponent = floor(log2 amax)
 * - 8; codes rounded to nearest even, saturating at +-448).  The gate/up and
 * down GEMMs and both dgrad GEMMs run on kind::mxf8f6f4 block-scaled tensor
 * cores with both operands quantised; the two weight-gradient GEMMs contract
 * over tokens and stay bf16 (MOE_MXFP8), or (MOE_MXFP8_ALL) run on the same
 * tensor cores with X, dA, dB, Hg and dY quantised along each expert's rows in
 * blocks of 32 rows from its first row.  The router stays bf16, so routing is
 * the same in every mode; all outputs are bf16 (dW_r fp32; the expert weight
 * gradients fp32 with wgrad_dtype = MOE_WGRAD_FP32).
 *
 * moe_prepare_weights quantises the bf16 master weights once (e.g. after each
 * optimiser step) into `wq` (moe_weights_size bytes), laid out as ten regions,
 * each starting on a 256-byte boundary:
 *   [Wgu codes][Wgu scales] [Wd2 ..][..] [Wd3 ..][..] [Wg4 ..][..] [Wu4 ..][..]
 *   Wgu [El*2I, d]: W_gate / W_up with K = d, rows per expert in blocks of 128 =
 *        64 W_gate columns then the same 64 W_up columns;
 *   Wd2 [El*d, I]: W_down transposed (K = I);   Wd3 [El*I, d]: W_down (K = d);
 *   Wg4 [El*d, I]: W_gate (K = I);              Wu4 [El*d, I]: W_up (K = I).
 * Codes are row-major bytes; the scales of a [R, K] region sit in 512-byte
 * chunks, byte (r%32)*16 + ((r%128)/32)*4 + (k%128)/32 of chunk
 * (r/128)*(K/128) + k/128 (the order the block-scaled MMA reads them in).
 * moe_fwd_mx / moe_bwd_mx take the same arguments as moe_fwd / moe_bwd with
 * wq in place of the bf16 expert weights; ctx and ws are sized by
 * moe_ctx_size / moe_workspace_size of the MXFP8 shape (MOE_MXFP8 and
 * MOE_MXFP8_ALL share ctx and prepared weights; the workspace differs). */
size_t moe_weights_size(const moe_shape* shape);

/* Test hook (MOE_MXFP8_ALL): copies one weight-gradient operand quantised along the
 * rows by the last moe_fwd_mx (X_perm, saved in ctx) or moe_bwd_mx (in ws): which = 0
 * X_perm, 1 dY_perm (C = d),
 * 2 dA, 3 dB, 4 Hg (C = I).  RP = the padded-row capacity (moe_padded_rows).  codes
 * (RP*C bytes) are K-major in 128-row tiles: byte ((R/128)*C + c)*128 + R%128 is the
 * code of padded row R, column c; scales (RP*C/32 bytes) sit in 512-byte chunks,
 * byte (c%32)*16 + ((c%128)/32)*4 + (R%128)/32 of chunk (R/128)*(C/128) + c/128.
 * Tiles past an expert's real rows hold whatever the buffer held.  Device pointers;
 * MOE_ERR_INVALID_ARG for another precision or `which`.  One-batch buffers (moe_fwd_mx /
 * moe_bwd_mx) only: a ring-streamed layer's ctx and ws are laid out for its minibatches. */
moe_status moe_debug_mx_wgrad_operand(const moe_shape* shape, const void* ctx, const void* ws, int32_t which,
                                      void* codes, void* scales, void* stream);
/* Padded-row capacity RP of a shape (rows of X_perm and the other row buffers); 0 if invalid. */
int64_t moe_padded_rows(const moe_shape* shape);
moe_status moe_prepare_weights(const moe_shape* shape, const void* W_gate, const void* W_up, const void* W_down,
                               void* wq, size_t wq_bytes, void* stream);
moe_status moe_fwd_mx(const moe_shape* shape, const void* X, const void* W_r, const float* bias, const void* wq,
                      size_t wq_bytes, void* Y, void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes,
                      void* stream);
moe_status moe_bwd_mx(const moe_shape* shape, const void* X, const void* W_r, const void* wq, size_t wq_bytes,
                      const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate, void* dW_up,
                      void* dW_down, float* dW_r, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * NVFP4 mode (page 1, "MoE layer as the bottleneck": NVFP4 training kernels
 * named as earlier work; the format is NVIDIA's published NVFP4).  Shapes carry
 * prec = MOE_NVFP4.  Each GEMM operand is E2M1 (values 0, 0.5, 1, 1.5, 2, 3, 4,
 * 6 and their negatives) with one E4M3 scale per 16 values along the GEMM's
 * contraction dimension and one fp32 global scale per tensor:
 *   gs = 2688 / amax(tensor)  (1 for an all-zero tensor),
 *   block scale s = e4m3((amax_block / 6) * gs), codes q = e2m1(v * (gs / s)),
 *   value = q * s / gs,
 * every step in fp32 with round-to-nearest-even and saturation (6, 448); a block
 * whose scale rounds to 0 holds zeros.  The tensors are X [T, d] (along d), the
 * local experts' W_gate, W_up (along d) and W_down (along I), and H [rows, I]
 * over every assigned row (along I); the gate/up and down GEMMs run on
 * kind::mxf4nvf4 block-scaled tensor cores (K = 64 per MMA) and multiply their
 * fp32 accumulators by 1 / (gs_A gs_B).  H = silu(A) B is formed in fp32 by the
 * gate/up GEMM, its amax sets its global scale, then it is quantised.  Routing
 * is the bf16 router's, Y is bf16.  The forward keeps A, B (bf16) and X_perm (bf16) in ctx.
 *
 * moe_bwd_nvfp4 runs both dgrad GEMMs on NVFP4 operands: dY [T, d] along d (its own global
 * scale) with W_down along d; [dA | dB] along I with [W_gate | W_up] along I, each pair one
 * tensor with one global scale (the GEMM sums over both halves, K = 2I).  dA and dB are formed
 * in fp32 by the dgrad of W_down's epilogue (SwiGLU backward from the saved bf16 A, B), their
 * joint amax sets their scale, then they are quantised.  The weight gradients contract the bf16
 * operands (X_perm, dA, dB, g H, dY_perm) on the bf16 engine, as in MOE_MXFP8; dW_r fp32.
 *
 * moe_prepare_weights with an MOE_NVFP4 shape quantises W_gate, W_up, W_down
 * (the local experts' [El, d, I], [El, d, I], [El, I, d] bf16) into wq
 * (moe_weights_size of that shape): the five MXFP8 regions (Wgu, Wd2, Wd3, Wg4,
 * Wu4, each codes then scales) at half a byte per value, then the global
 * scales, each region on a 256-byte boundary; two codes per byte, value 2i in
 * the low nibble of byte i; scale byte (r%32)*16 + ((r%128)/32)*4 + (k%64)/16 of
 * 512-byte chunk (r/128)*(K/64) + k/64; the global scales are four fp32: gate,
 * up, down, and [gate | up] (the backward's Wg4 / Wu4 share it).
 * moe_fwd_nvfp4 / moe_bwd_nvfp4 take moe_fwd_mx's / moe_bwd_mx's arguments; ctx
 * and ws are sized by moe_ctx_size / moe_workspace_size of the MOE_NVFP4 shape;
 * d and I multiples of 256 as everywhere.  Errors as for moe_fwd_mx /
 * moe_bwd_mx; moe_get_error reads the device status. */
moe_status moe_fwd_nvfp4(const moe_shape* shape, const void* X, const void* W_r, const float* bias, const void* wq,
                         size_t wq_bytes, void* Y, void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes,
                         void* stream);
moe_status moe_bwd_nvfp4(const moe_shape* shape, const void* X, const void* W_r, const void* wq, size_t wq_bytes,
                         const void* dY, void* ctx, size_t ctx_bytes, void* dX, void* dW_gate, void* dW_up,
                         void* dW_down, float* dW_r, void* ws, size_t ws_bytes, void* stream);
/* Test hook: byte offsets of the NVFP4 buffers (out has room for 23).  out[0..1]: X codes and
 * scales in ctx; out[2..5]: H codes, H scales, fp32 H [RP, I] and eight scale words (amax X,
 * amax H as fp32 bits, gs_X, gs_H, amax dY, amax [dA | dB], gs_dY, gs_[dA | dB]) in ws;
 * out[6..10]: Wgu codes, Wgu scales, Wd2 codes, Wd2 scales and the four weight global scales
 * in wq; out[11..16]: dY, dA, dB codes and scales in ws; out[17..22]: Wd3, Wg4, Wu4 codes and
 * scales in wq.  Host only; MOE_ERR_INVALID_ARG for another precision or a NULL out. */
moe_status moe_debug_nv_offsets(const moe_shape* shape, int64_t* out);

/* ---------------------------------------------------------------------------
 * Ring-streamed layer (page 1, "Three design decisions that matter", bullet 3:
 * a fixed ring token buffer cycled at minibatch granularity, dispatch and
 * combine interleaved at macrobatch boundaries, walked in reverse in the
 * backward so that little forward activation has to be replayed).
 *
 * One call processes M minibatches of shape->T tokens each (X, Y, dY, dX are
 * [M*T, d]).  The result is the layer of moe_fwd / moe_bwd over all M*T tokens;
 * only where the dispatched token rows (X_perm) live changes: in the caller's
 * ring of ring_bytes (ring_bytes / (2 d) rows) instead of ctx.
 *   - The device groups consecutive minibatches into macrobatches: a macrobatch
 *     closes once its padded rows give the gate/up grouped GEMM two full waves
 *     of 128 x 256 tiles ((rows / 128) * (I / 128) >= 2 * SMs), or before a
 *     minibatch that would not fit in the ring with it.
 *   - Forward: each macrobatch's rows are dispatched at the ring's write
 *     pointer (a segment that would run past the end restarts at row 0), then
 *     its grouped GEMMs and its combine run.
 *   - Backward: the dgrad path runs over all rows; the gate/up weight gradient
 *     walks the macrobatches in reverse, reusing those still intact in the ring
 *     and re-dispatching (replaying) older ones chunk by chunk.
 * No host synchronisation and no dropped tokens: all sizes are decided on the
 * device; the host enqueues a fixed number of launches per minibatch.
 * Requirements: shape->T a multiple of 16; 1 <= M <= 256; ring_bytes at least
 * moe_stream_min_ring_bytes(shape) (one minibatch's worst case), else
 * MOE_ERR_WORKSPACE_TOO_SMALL.  moe_fwd_stream / moe_bwd_stream take bf16 weights
 * (MOE_BF16 shapes); moe_fwd_stream_mx / moe_bwd_stream_mx below run MOE_MXFP8 shapes
 * (wgrad_dtype applies as in moe_bwd).  The size calls accept either. */
size_t moe_stream_ctx_size(const moe_shape* shape, int32_t num_minibatches);
size_t moe_stream_workspace_size(const moe_shape* shape, int32_t num_minibatches);
size_t moe_stream_min_ring_bytes(const moe_shape* shape);
moe_status moe_fwd_stream(const moe_shape* shape, int32_t num_minibatches, const void* X, const void* W_r,
                          const float* bias, const void* W_gate, const void* W_up, const void* W_down, void* Y,
                          void* ctx, size_t ctx_bytes, void* ring, size_t ring_bytes, void* ws, size_t ws_bytes,
                          void* stream);
moe_status moe_bwd_stream(const moe_shape* shape, int32_t num_minibatches, const void* X, const void* W_r,
                          const void* W_gate, const void* W_up, const void* W_down, const void* dY, void* ctx,
                          size_t ctx_bytes, void* dX, void* dW_gate, void* dW_up, void* dW_down, float* dW_r,
                          void* ring, size_t ring_bytes, void* ws, size_t ws_bytes, void* stream);
/* Test hook: copies the plan of the last moe_fwd_stream (int32 words, device
 * pointer): [16 header words: macrobatches, backward chunks, padded rows,
 * replayed rows, resident rows, ring rows, 0...] then mb_of[M],
 * seg_poff[M*El+1], cum[M*El], mb_range[2M], shift_fwd[M], shift_bwd[M],
 * replay[M], chunk[4M] ({m_lo, m_hi, valid, mode}), ring_start[M]. */
/* MXFP8 ring-streamed layer (shape->prec = MOE_MXFP8 or MOE_MXFP8_ALL): the same plan and ring as
 * moe_fwd_stream / moe_bwd_stream, with the gate/up, down and both dgrad GEMMs on MXFP8 from the
 * prepared weights `wq` (moe_prepare_weights of this shape).  MOE_MXFP8: bf16 weight gradients as in
 * the bf16 stream (ring replay, backward chunks); a ring row holds the bf16 row, its E4M3 codes along
 * d and their scales (2d + d + d/32 bytes).  MOE_MXFP8_ALL: MXFP8 weight gradients over every
 * segment of the stream, the operands quantised along the rows in blocks of 32 rows of each
 * (macrobatch, expert) segment, X's codes along the rows kept at the padded rows of the stream (ctx),
 * so nothing is replayed; a ring row holds the codes along d and their scales (d + d/32 bytes).  The
 * ring holds R = ring_bytes / (row bytes) rows rounded down to a multiple of 128, laid out as R bf16
 * rows (MOE_MXFP8 only), R code rows, then the codes' scale chunks.  ctx / ws / minimum ring sizes:
 * the moe_stream_* size calls of this shape.  Same errors as the bf16 stream. */
moe_status moe_fwd_stream_mx(const moe_shape* shape, int32_t num_minibatches, const void* X, const void* W_r,
                             const float* bias, const void* wq, size_t wq_bytes, void* Y, void* ctx, size_t ctx_bytes,
                             void* ring, size_t ring_bytes, void* ws, size_t ws_bytes, void* stream);
moe_status moe_bwd_stream_mx(const moe_shape* shape, int32_t num_minibatches, const void* X, const void* W_r,
                             const void* wq, size_t wq_bytes, const void* dY, void* ctx, size_t ctx_bytes, void* dX,
                             void* dW_gate, void* dW_up, void* dW_down, float* dW_r, void* ring, size_t ring_bytes,
                             void* ws, size_t ws_bytes, void* stream);
moe_status moe_debug_stream_plan(const moe_shape* shape, int32_t num_minibatches, const void* ctx, int32_t* tables,
                                 void* stream);

/* Router GEMM + top-k gating that allocates nothing.  The pages have no
 * counterpart of this call: it exists for callers that must not allocate
 * device memory while they run -- code executing inside an allocator or
 * memory-planner callback (where cudaMalloc would re-enter the allocator), or
 * a service whose device memory was all handed to its own pool at start-up.
 *   X [T, d] bf16, W_r [d, E] bf16, bias [E] fp32 or NULL     (inputs)
 *   ids [T, k] int32, gates [T, k] fp32                       (outputs: the same
 *       values moe_fwd puts in its routing table)
 *   status: one int32 in device memory, or NULL; cleared, then set to a
 *       moe_status code by a device-side error (non-finite logit, timeout)
 * Its scratch (W_r transposed, split-K partial logits, logits, per-block
 * histograms) is a static device array of MOE_STATIC_SCRATCH_BYTES = 32 MiB
 * inside the library; every GPU that loads the library holds it until the
 * process exits.  Shapes needing more (about E*d*2 + (S+1)*T*E*4 +
 * ceil(T/16)*E*4 bytes, S = K splits of the router GEMM) are refused with
 * MOE_ERR_WORKSPACE_TOO_SMALL.
 * Set-up: CUDA loads the library's kernels and this array lazily (unless
 * CUDA_MODULE_LOADING=EAGER), and loading commits device memory.  The first
 * call on each device (any T, T = 0 included) does the set-up with that device
 * current: it looks up the array's device address (cudaGetSymbolAddress) and
 * loads every kernel the call launches.  So make one call on each device
 * before entering the region that must not allocate, and before any stream
 * capture; after it, calls allocate nothing.  No call synchronises.  The
 * address is kept for the life of the process and does not survive
 * cudaDeviceReset (after a reset, do not call this again in that process).
 * All calls share the one array: calls that overlap on the GPU race on it and
 * must be serialised by the caller. */
moe_status moe_route_static(const moe_shape* shape, const void* X, const void* W_r, const float* bias,
                            int32_t* ids, float* gates, int32_t* status, void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism across R ranks (page 1, "Three design decisions that
 * matter", bullet 1: the rank that owns an expert pulls the tokens it needs
 * from the senders' memory, so senders need not signal arrival; expert outputs
 * are pushed back to the token's rank; the backward mirrors both; one schedule
 * table serves all four phases).
 *
 * Rank q of R holds shape->T tokens of its own and the experts
 * [q E/R, (q+1) E/R) (E a multiple of R, 1 <= R <= 64); shape->first_local_expert
 * and num_local_experts are ignored.  Every rank owns an exchange buffer of
 * moe_ep_buffer_size bytes (256-byte aligned, zeroed once before the first
 * step) that all ranks can address: `bufs` lists the R buffers' addresses in this
 * process (peer mappings across GPUs, or all on one device), bufs[rank] its own.
 * Peers read a rank's routing table, X and dY from it and write expert outputs,
 * dX rows and router-gate gradients into it, with plain loads and stores; the
 * only signals are one ready flag per rank and step phase, and one done flag
 * per (owner, source) pair, each wait bounded (about 2 s, then
 * MOE_ERR_DEVICE_TIMEOUT in ctx's status word).  `epoch` numbers the step (a
 * new value every step, not 0).
 *
 * A step is six calls per rank, in this order on its stream; each call of a
 * phase may wait for the earlier phases of every rank of the same step:
 *   moe_ep_fwd_route    route this rank's tokens (router GEMM, top-k, the table
 *                       over all E experts) and publish them with X
 *   moe_ep_fwd_experts  pull the local experts' rows from every rank (ranks in
 *                       order, tokens ascending: the one-device layer's order for
 *                       the rank-major concatenation of the ranks' tokens), run
 *                       the grouped gate/up + SwiGLU and down GEMMs, push each
 *                       output row back to its source's slot
 *   moe_ep_fwd_combine  Y [T, d] = the pushed rows, summed over the k slots in order
 *   moe_ep_bwd_publish  publish dY [T, d]
 *   moe_ep_bwd_experts  pull dY rows, dgrad + SwiGLU backward, push each row's
 *                       router-gate gradient and its dX row back, then the local
 *                       experts' weight gradients dW_gate, dW_up [E/R, d, I],
 *                       dW_down [E/R, I, d] (bf16, or fp32 by wgrad_dtype)
 *   moe_ep_bwd_finish   router backward of this rank's tokens: dX [T, d] and this
 *                       rank's part of dW_r [d, E] (fp32; the full dW_r is the sum
 *                       over ranks, as for any replicated weight)
 * Y, dX and the expert weight gradients equal the one-device layer's on the
 * rank-major concatenation wherever the router GEMM's fixed K split is the same
 * for T and R T tokens (bit for bit; see router_splits in the sources).
 * ctx / ws are this rank's (moe_ep_ctx_size / moe_ep_workspace_size bytes); ctx
 * leads with the status word moe_get_error reads.  bf16 mode only.  Argument
 * errors return synchronously; an R, rank or E that does not fit gives
 * MOE_ERR_INVALID_ARG, an exchange buffer not 256-byte aligned too. */
size_t moe_ep_buffer_size(const moe_shape* shape, int32_t num_ranks);
size_t moe_ep_ctx_size(const moe_shape* shape, int32_t num_ranks);
size_t moe_ep_workspace_size(const moe_shape* shape, int32_t num_ranks);
moe_status moe_ep_fwd_route(const moe_shape* shape, int32_t num_ranks, int32_t rank, void* const* bufs, const void* X,
                            const void* W_r, const float* bias, void* ctx, size_t ctx_bytes, void* ws,
                            size_t ws_bytes, int32_t epoch, void* stream);
moe_status moe_ep_fwd_experts(const moe_shape* shape, int32_t num_ranks, int32_t rank, void* const* bufs,
                              const void* W_gate, const void* W_up, const void* W_down, void* ctx, size_t ctx_bytes,
                              void* ws, size_t ws_bytes, int32_t epoch, void* stream);
moe_status moe_ep_fwd_combine(const moe_shape* shape, int32_t num_ranks, int32_t rank, void* const* bufs, void* Y,
                              void* ctx, size_t ctx_bytes, int32_t epoch, void* stream);
moe_status moe_ep_bwd_publish(const moe_shape* shape, int32_t num_ranks, int32_t rank, void* const* bufs,
                              const void* dY, void* ctx, size_t ctx_bytes, int32_t epoch, void* stream);
moe_status moe_ep_bwd_experts(const moe_shape* shape, int32_t num_ranks, int32_t rank, void* const* bufs,
                              const void* W_gate, const void* W_up, const void* W_down, void* dW_gate, void* dW_up,
                              void* dW_down, void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes, int32_t epoch,
                              void* stream);
moe_status moe_ep_bwd_finish(const moe_shape* shape, int32_t num_ranks, int32_t rank, void* const* bufs,
                             const void* X, const void* W_r, void* dX, float* dW_r, void* ctx, size_t ctx_bytes,
                             void* ws, size_t ws_bytes, int32_t epoch, void* stream);
/* Test hook: the owner side of the last moe_ep_fwd_experts (device pointers, any may be NULL):
 * counts [E/R] rows per local expert, padded_offsets [E/R + 1], row_src [rows] for every
 * padded row: source rank * T * top_k + that rank's assignment index (token * top_k + slot),
 * or -1 / -2 for pad rows; `rows` = R T min(top_k, E/R) + 127 E/R rounded up to 128. */
moe_status moe_ep_debug_plan(const moe_shape* shape, int32_t num_ranks, int32_t rank, const void* ctx,
                             int32_t* counts, int32_t* padded_offsets, int32_t* row_src, void* stream);

/* Static string naming a status code. */
const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
