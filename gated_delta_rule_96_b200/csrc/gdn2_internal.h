// Host-side launchers shared between the ABI layer and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdn2 {

// Status header at the start of every prefill workspace (device status words).
constexpr size_t kStatusBytes = 256;

// Decode: one token per (b, h); S updated in place.
int launch_decode(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                  const void *w, float *S, void *o, int B, int H, int K, int V, int bf16, cudaStream_t st);

// SIMT two-kernel prefill (fp32 FMA everywhere; any token dtype).
size_t simt_workspace_bytes(int B, int H, int T, int K, int V, int C);
int launch_chunk_simt(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                      const void *w, const float *S0, void *o, float *ST, int B, int H, int T, int K, int V,
                      int C, int bf16, void *ws, cudaStream_t st);

// Fused tcgen05 prefill (bf16 tokens, d_k = d_v = 128, C = 64).
bool tc_supported(int B, int H, int T, int K, int V, int C, int bf16);
// edges != 0: the layer-edge variant's ring (RING_SLOTS x 80 KB per block) is included
size_t tc_workspace_bytes(int B, int H, int T, int K, int V, int C, int edges = 0);
// edges != 0: q, k, b, w, alpha are the layer's raw inputs (see gdn2_chunk_fwd_edges); onorm, if
// not null, is the RMSNorm weight applied to o.
int launch_chunk_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                    const void *w, const float *S0, void *o, float *ST, int B, int H, int T, int K, int V,
                    int C, void *ws, cudaStream_t st, int edges = 0, const float *onorm = nullptr);

// Two-stage tcgen05 prefill (bf16 tokens, d_k = d_v = 128, C = 64): the intra-chunk work in parallel
// over every chunk-head, then the state chain; long sequences in windows, few long chains cut into
// segments in time.
size_t split_workspace_bytes(int B, int H, int T);
// edges != 0: q, k, b, w, alpha are the layer's raw inputs (see gdn2_chunk_fwd_edges); onorm, if not
// null, is the RMSNorm weight applied to o.
int launch_chunk_split(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                       const void *w, const float *S0, void *o, float *ST, int B, int H, int T, void *ws,
                       cudaStream_t st, int edges = 0, const float *onorm = nullptr);

// Measurement kernel of the prefill's tensor-core phases (mode 0: back to back; 1: each group waits
// for the previous one), `reps` chunks per CTA on `nctas` CTAs.
int launch_phase_probe(int mode, int reps, int nctas, unsigned int *status, cudaStream_t st);

// S_g = M_(g-1) S_(g-1) + N_(g-1) along nseg segments of each chain (fp32; M, N, Sg [chains][nseg][128][128],
// S0 [chains][128][128] or null for zero).
int launch_segment_scan(const float *M, const float *N, const float *S0, float *Sg, int chains, int nseg,
                        cudaStream_t st);

// The layer's edge maps on their own (bf16 tokens, d in {64, 128}; rows = B*T*H).
int launch_edge_maps(const void *q_raw, const void *k_raw, const float *a_logit, const void *b_logit,
                     const void *w_logit, void *q, void *k, float *alpha, void *b, void *w, long long rows, int K, int V,
                     cudaStream_t st);
int launch_rms_norm(void *o, const float *weight, long long rows, int V, cudaStream_t st);

// Backward pass (three sequential passes per chain; fp32 gradients; d_k, d_v in {64, 128}).
size_t bwd_workspace_bytes(int B, int H, int T, int K, int V);
int launch_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                     const float *S0, const void *dO, const float *dST, float *dq, float *dk, float *dv,
                     float *dalpha, float *db, float *dw, float *dS0, int B, int H, int T, int K, int V, int bf16,
                     void *ws, cudaStream_t st);

// Tensor-core backward (bf16 tokens, d_k = d_v = 128): forward replay by the two-stage prefill's kernels,
// reverse walk of the state gradient, gradient kernel over every chunk-head.
size_t chunk_bwd_tc_workspace_bytes(int B, int H, int T);
int launch_chunk_bwd_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                        const float *S0, const void *dO, const float *dST, float *dq, float *dk, float *dv,
                        float *dalpha, float *db, float *dw, float *dS0, int B, int H, int T, void *ws,
                        cudaStream_t st);

}  // namespace gdn2
