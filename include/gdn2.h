/*
 * gdn2.h -- C ABI of the Gated DeltaNet-2 recurrence library (libgdn2.so), sm_100a.
 *
 * The operation (page "NVIDIA представила Gated DeltaNet-2 с канал-wise гейтами ...",
 * section "Техническая схема", the state-update equation), per batch element and head:
 *
 *     S_t = (I - k_t (b_t ⊙ k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t ⊙ v_t)^T
 *     o_t = S_t^T q_t
 *
 * S in R^{d_k x d_v} (fp32).  b_t in [0,1]^{d_k} is the erase gate on the key axis,
 * w_t in [0,1]^{d_v} the write gate on the value axis, alpha_t in (0,1]^{d_k} the
 * channel-wise decay.  The read-out uses the post-update state and no 1/sqrt(d_k)
 * scale.  Collapsing b and w to one scalar per token gives KDA; collapsing alpha to a
 * scalar as well gives Gated DeltaNet (page "NVIDIA улучшила память LLM ...", the
 * quoted remark on special cases): pass such gates as broadcast (materialised) tensors.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers to contiguous, row-major buffers, each
 *     16-byte aligned.  The caller owns every buffer; the library allocates nothing
 *     and keeps no state between calls, except gdn2_chunk_fwd_noalloc, whose fixed
 *     scratch array (below) is library-owned device memory shared by all its calls.
 *   - Kernels launch on the calling thread's current CUDA device, which must own every
 *     pointer of the call (and `stream`, if given).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream).  The return value reports argument checking and launch
 *     errors only; device-side errors are read with gdn2_workspace_status().
 *   - Nothing throws across the ABI.  Every entry point returns a gdn2_status.
 *   - d_k, d_v in {64, 128}.  Token dtype (q, k, v, b, w and o) is fp32 or bf16;
 *     alpha and the states are always fp32.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_NULL = -1,         /* a required pointer is NULL                        */
    GDN2_ERR_SHAPE = -2,        /* a size is negative or inconsistent                */
    GDN2_ERR_DTYPE = -3,        /* unknown dtype code                                */
    GDN2_ERR_UNSUPPORTED = -4,  /* valid but unsupported (d_k/d_v not 64/128, C!=64) */
    GDN2_ERR_WORKSPACE = -5,    /* workspace NULL or smaller than required           */
    GDN2_ERR_CUDA = -6,         /* a CUDA runtime call or kernel launch failed       */
    GDN2_ERR_ALIGN = -7,        /* a pointer is not 16-byte aligned                  */
    GDN2_ERR_DEVICE = -8,       /* a kernel reported an internal error (bounded wait
                                   expired); read by gdn2_workspace_status           */
    GDN2_ERR_NOALLOC_LIMIT = -9 /* gdn2_chunk_fwd_noalloc: the problem needs more
                                   scratch than GDN2_NOALLOC_SCRATCH_BYTES           */
} gdn2_status;

typedef enum { GDN2_F32 = 0, GDN2_BF16 = 1 } gdn2_dtype;

/* Bytes of device workspace gdn2_chunk_fwd needs for these sizes (0 on bad sizes is
 * never returned: at least the 256-byte status header is always required).
 * Depends only on its arguments. */
GDN2_API size_t gdn2_chunk_fwd_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C, int dtype);

/*
 * Chunkwise-parallel prefill over T tokens (page "NVIDIA представила Gated DeltaNet-2 ...",
 * the paragraph on the chunkwise WY form with chunk size C = 64).
 *
 *   q, k, b       [B, T, H, d_k]   token dtype
 *   v, w          [B, T, H, d_v]   token dtype
 *   alpha         [B, T, H, d_k]   fp32, each value in (0, 1]
 *   S0            [B, H, d_k, d_v] fp32 initial state, or NULL for a zero state
 *   o   (out)     [B, T, H, d_v]   token dtype
 *   S_T (out)     [B, H, d_k, d_v] fp32 final state; may alias S0 (in-place resume)
 *   C             chunk size; must be 64
 *   workspace     device scratch of at least gdn2_chunk_fwd_workspace_bytes(...) bytes,
 *                 16-byte aligned; its first 256 bytes hold the device status words
 *                 (see gdn2_workspace_status) and must have been zeroed once by the
 *                 caller before first use (cudaMemset), after which calls keep them.
 *   T = 0 copies S0 (or zeros) to S_T; the token and o pointers are then not read and
 *   may be NULL.  A last partial chunk (T % C != 0) is handled.
 */
GDN2_API int gdn2_chunk_fwd(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                   const void *w, const float *S0, void *o, float *S_T, int B, int H, int T, int d_k,
                   int d_v, int C, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * The same prefill with the layer's input and output edges fused into the kernel (page
 * "NVIDIA представила Gated DeltaNet-2 ...", the paragraph on the layer: q and k pass an L2
 * norm, the gates are sigmoid projections, the output goes through RMSNorm).  Per (b, t, h):
 *
 *   q = q_raw / max(|q_raw|_2, 1e-6),   k = k_raw / max(|k_raw|_2, 1e-6)
 *   b = sigmoid(b_logit),   w = sigmoid(w_logit),   alpha = exp(-softplus(a_logit))
 *   o = recurrence output; if o_weight != NULL:  o <- o / sqrt(mean_v(o^2) + 1e-6) * o_weight
 *
 *   q_raw, k_raw, b_logit [B, T, H, d_k]  bf16
 *   v, w_logit            [B, T, H, d_v]  bf16
 *   a_logit               [B, T, H, d_k]  fp32
 *   o_weight              [d_v] fp32 RMSNorm weight shared by the heads, or NULL (no norm)
 * Everything else as gdn2_chunk_fwd, except the workspace: at least
 * gdn2_chunk_fwd_edges_workspace_bytes(...) bytes (gdn2_chunk_fwd's plus 128 KB per thread
 * block, B*H blocks, or B*H*segments when few long chains are split in time: the ring in which
 * the kernel passes the decay rows of the next four chunks between its warps).  A workspace
 * serves one call at a time.  Only bf16 tokens with d_k = d_v = 128 and C = 64 are supported
 * (GDN2_ERR_UNSUPPORTED otherwise).
 */
GDN2_API size_t gdn2_chunk_fwd_edges_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C);
GDN2_API int gdn2_chunk_fwd_edges(const void *q_raw, const void *k_raw, const void *v, const float *a_logit,
                                  const void *b_logit, const void *w_logit, const float *S0,
                                  const float *o_weight, void *o, float *S_T, int B, int H, int T, int d_k,
                                  int d_v, int C, int dtype, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * The layer's edge maps on their own, as one elementwise kernel: the maps gdn2_chunk_fwd_edges
 * applies inside the prefill (same page and paragraph), for callers that keep the recurrence's
 * inputs mapped, and to measure the fused prefill against the unfused layer.  Per (b, t, h):
 *   q = q_raw / max(|q_raw|_2, 1e-6),  k = k_raw / max(|k_raw|_2, 1e-6)
 *   b = sigmoid(b_logit),  w = sigmoid(w_logit),  alpha = exp(-softplus(a_logit))
 * Inputs as gdn2_chunk_fwd_edges (bf16, a_logit fp32); outputs q, k, b [B, T, H, d_k] bf16,
 * w [B, T, H, d_v] bf16, alpha [B, T, H, d_k] fp32 -- the inputs of gdn2_chunk_fwd.  d_k, d_v in
 * {64, 128}; outputs must not alias inputs.
 */
GDN2_API int gdn2_layer_edge_maps(const void *q_raw, const void *k_raw, const float *a_logit, const void *b_logit,
                                  const void *w_logit, void *q, void *k, float *alpha, void *b, void *w, int B, int T,
                                  int H, int d_k, int d_v, void *stream);

/* RMSNorm of the layer output in place: o <- o / sqrt(mean_v(o^2) + 1e-6) * weight, per row of d_v.
 * o [rows, d_v] bf16, weight [d_v] fp32; d_v in {64, 128}. */
GDN2_API int gdn2_rms_norm(void *o, const float *weight, long long rows, int d_v, void *stream);

/*
 * One decode token per sequence, state updated in place (constant memory per token,
 * page "NVIDIA улучшила память LLM ...", section "Контекст").
 *
 *   q, k, b       [B, H, d_k]      token dtype
 *   v, w          [B, H, d_v]      token dtype
 *   alpha         [B, H, d_k]      fp32
 *   S   (in/out)  [B, H, d_k, d_v] fp32, read and overwritten
 *   o   (out)     [B, H, d_v]      token dtype
 */
GDN2_API int gdn2_decode_step(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                     const void *w, float *S, void *o, int B, int H, int d_k, int d_v, int dtype,
                     void *stream);

/* Bytes of device workspace gdn2_chunk_bwd needs (0 on bad sizes).  Depends only on its
 * arguments: two fp32 [B, T, H, d_v] buffers, the fp32 state at every 64th step of every
 * chain, one fp32 d_k vector per 64 steps per chain, and, when few chains split their value
 * columns over blocks (2*B*H <= 148), one fp32 [B, T, H, d_k] buffer of partial row sums. */
GDN2_API size_t gdn2_chunk_bwd_workspace_bytes(int B, int H, int T, int d_k, int d_v);

/*
 * Backward pass of the recurrence: the gradients of a scalar loss L with respect to every
 * input of gdn2_chunk_fwd, given the loss's gradients at its outputs (page "NVIDIA
 * представила Gated DeltaNet-2 ...", the paragraph on the chunkwise kernels: the backward
 * needs gradients that account for the per-channel gates).
 *
 *   q, k, v, alpha, b, w, S0   the forward's inputs, same layouts and dtypes (S0 may be NULL)
 *   dO        [B, T, H, d_v]   token dtype, dL/do
 *   dS_T      [B, H, d_k, d_v] fp32, dL/dS_T, or NULL for zero
 *   dq, dk, db, dalpha (out)   [B, T, H, d_k] fp32
 *   dv, dw             (out)   [B, T, H, d_v] fp32
 *   dS0                (out)   [B, H, d_k, d_v] fp32, dL/dS0, or NULL if not wanted
 *   workspace  device scratch of at least gdn2_chunk_bwd_workspace_bytes(...) bytes, 16-byte
 *              aligned, no initialisation needed (no status header: these kernels never wait)
 *
 * Every gradient is computed and written in fp32 whatever the token dtype.  dalpha is
 * formed as d(log alpha) / alpha with alpha floored at FLT_MIN.  T = 0 writes dS0 = dS_T
 * (or zeros) and reads no token pointer.  d_k, d_v in {64, 128}.  The output buffers must
 * not alias the inputs or each other.  Three kernel launches on `stream`; with few chains
 * (2*B*H <= 148) each chain's value columns are split over several blocks, which adds zero fills of
 * dq, dk and workspace buffers and a fourth, small kernel.  Results are deterministic in the
 * unsplit case; in the split case the row sums are added in an unspecified order (fp32 rounding).
 */
GDN2_API int gdn2_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                            const void *w, const float *S0, const void *dO, const float *dS_T, float *dq,
                            float *dk, float *dv, float *dalpha, float *db, float *dw, float *dS0, int B, int H,
                            int T, int d_k, int d_v, int dtype, void *workspace, size_t workspace_bytes,
                            void *stream);

/* Bytes of device workspace gdn2_chunk_bwd_tc needs (0 on bad or unsupported sizes): the 256-byte
 * status header, then per chunk of 64 steps of every chain a 75,776-byte record of the forward's chunk
 * factors and a 124,928-byte side record of the backward, the fp32 state at the end of every chain,
 * and, when few chains are long (B*H <= 64 and at least 32 chunks), three fp32 states per time segment
 * of each chain.  About 200 KB per 64 steps per chain; T = 0 needs the header only. */
GDN2_API size_t gdn2_chunk_bwd_tc_workspace_bytes(int B, int H, int T, int d_k, int d_v);

/*
 * Backward pass on the tensor cores: the same gradients as gdn2_chunk_bwd (same arguments, layouts
 * and output dtypes), for bf16 tokens with d_k = d_v = 128 (GDN2_ERR_UNSUPPORTED otherwise).  The
 * chunkwise WY form with C = 64 (page "NVIDIA представила Gated DeltaNet-2 ...", the paragraph on the
 * chunkwise kernels) is differentiated product by product: a forward replay by the two-stage prefill's
 * kernels keeps each chunk's factors, one block per chain walks the chunks backwards with the state
 * gradient resident in tensor memory, and one kernel over every chunk-head forms the token gradients
 * from five tcgen05 products and the gate and decay terms.
 *
 * Accuracy: the products take bf16 operands (the chunk factors, the state and its gradient, dO) with
 * fp32 accumulation, so each gradient carries the bf16 relative error of the forward's tensor-core
 * path (about 1e-2 of the tensor's largest magnitude) rather than gdn2_chunk_bwd's fp32 one.  The state
 * gradient is carried from chunk to chunk in fp32; d(ln alpha) sums fp32 terms over at most 64 steps.
 *
 *   workspace  device scratch of at least gdn2_chunk_bwd_tc_workspace_bytes(...) bytes, 16-byte
 *              aligned, whose first 256 bytes are a status header zeroed once by the caller (the
 *              kernels' bounded waits report there; read it with gdn2_workspace_status)
 *
 * T = 0 writes dS0 = dS_T (or zeros).  The output buffers must not alias the inputs or each other.
 * Five to eight kernel launches on `stream`; results are deterministic.
 */
GDN2_API int gdn2_chunk_bwd_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                               const void *w, const float *S0, const void *dO, const float *dS_T, float *dq,
                               float *dk, float *dv, float *dalpha, float *db, float *dw, float *dS0, int B, int H,
                               int T, int d_k, int d_v, int dtype, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * Measurement aid (not part of the recurrence): runs the tensor-core products of one chunk of the
 * chunkwise prefill -- G1 [A; P] = [Ê; Q̂] K̃^T (M128 N64 K128), G2 (2 x M128 N128 K64), G3 (M128 N128
 * K128), G4 and G5 (2 x M128 N128 K64), with the prefill kernels' shapes and shared-memory operand
 * layouts -- `reps` chunks in a row on each of `nctas` CTAs (one per SM), on operands that stay in
 * shared memory; 14,680,064 flops per chunk as issued.  mode 0 issues every product back to back
 * (the tensor pipe's rate on these shapes); mode 1 lets each group wait for the completion of the
 * one before it, as the prefill's data flow does.  Time it with events on `stream`.  The workspace
 * holds only the 256-byte status header (zeroed once); a bounded wait that expires sets it.
 */
#define GDN2_PHASE_PROBE_FLOPS_PER_CHUNK 14680064.0
GDN2_API int gdn2_gemm_phase_probe(int mode, int reps, int nctas, void *workspace, size_t workspace_bytes,
                                   void *stream);

/* Reads the device status word of a workspace (synchronises `stream` first).
 * *out receives 0 when every kernel that used this workspace finished normally, or a
 * nonzero code naming the first internal error.  With clear != 0 the word is reset.
 * Returns GDN2_OK, or GDN2_ERR_NULL / GDN2_ERR_CUDA. */
GDN2_API int gdn2_workspace_status(void *workspace, int clear, int *out, void *stream);

/* Static description of a status code (never NULL). */
GDN2_API const char *gdn2_status_str(int status);

/*
 * Prefill for callers that cannot allocate device memory.  (The pages have no
 * counterpart: this is a deployment convenience of this library.)
 *
 * Who needs it: hosts that own all device memory (a framework's pool allocator or a
 * fixed per-process budget) and do not let a plugin call cudaMalloc, and callers that
 * forbid allocation on a latency-critical path because cudaMalloc can synchronise the
 * device.  They cannot hand gdn2_chunk_fwd a workspace.
 *
 * Same arguments and results as gdn2_chunk_fwd without the workspace; it always runs
 * the CUDA-core (SIMT) chunkwise path.  Its scratch is one fixed array of
 * GDN2_NOALLOC_SCRATCH_BYTES (32 MiB) in the library's device memory, reserved on every
 * GPU that loads the library until the process exits.  The call allocates nothing.
 *   - Limit: 256 + 4 * B * H * ceil(T/64) * (3*64*d_k + 64*d_v + 64*64 + d_k) bytes must
 *     not exceed GDN2_NOALLOC_SCRATCH_BYTES (e.g. B*H*ceil(T/64) <= 226 chunk-heads at
 *     d_k = d_v = 128); larger problems return GDN2_ERR_NOALLOC_LIMIT and launch nothing.
 *   - The first call on a device looks up the array's device address on that device
 *     (cudaGetSymbolAddress, with that device current); make that first call before any
 *     stream capture.  The address is kept per device and context: after a device reset
 *     (cudaDeviceReset) the next call looks it up again in the new context.
 *   - All calls share the one array and it keeps the last call's contents (nothing in it
 *     needs to start at zero).  Calls that overlap on the GPU -- on different streams or
 *     from different host threads -- race on it: serialise them.
 *   - The CUDA-core path it runs has no bounded waits and reports no device-side status:
 *     there is no workspace, and gdn2_workspace_status does not apply.  The return value
 *     reports argument checks and launch errors.
 */
#define GDN2_NOALLOC_SCRATCH_BYTES (32u << 20)
GDN2_API int gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                                    const void *b, const void *w, const float *S0, void *o, float *S_T, int B,
                                    int H, int T, int d_k, int d_v, int C, int dtype, void *stream);

/* Which prefill implementation gdn2_chunk_fwd selects for these sizes:
 * 0 = SIMT two-kernel path (fp32 FMA; fp32 tokens, or d_k / d_v = 64);
 * 1 = fused tcgen05 kernel, one CTA per (b, h) chain (bf16, d_k = d_v = 128, B*H <= 64; long
 *     sequences are cut into segments in time and composed);
 * 2 = two-stage tcgen05 path (bf16, d_k = d_v = 128, B*H > 64): the intra-chunk work runs in
 *     parallel over every chunk of every chain, then one CTA per chain walks the state. */
GDN2_API int gdn2_chunk_fwd_path(int B, int H, int T, int d_k, int d_v, int C, int dtype);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
