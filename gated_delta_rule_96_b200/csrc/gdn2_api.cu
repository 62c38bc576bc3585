// extern "C" boundary of libgdn2: argument checking, path selection, launches.
// Declarations and the meaning of every argument: include/gdn2.h.
#include <stdint.h>

#include "gdn2.h"
#include "gdn2_internal.h"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d == 64 || d == 128; }

int check_common(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                 const void *o, int B, int H, int K, int V, int dtype) {
    if (B < 0 || H < 0 || K <= 0 || V <= 0) return GDN2_ERR_SHAPE;
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (!dim_ok(K) || !dim_ok(V)) return GDN2_ERR_UNSUPPORTED;
    if (!q || !k || !v || !alpha || !b || !w || !o) return GDN2_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(b) || !aligned16(w) ||
        !aligned16(o))
        return GDN2_ERR_ALIGN;
    return GDN2_OK;
}

bool use_tc(int B, int H, int T, int K, int V, int C, int dtype) {
    return gdn2::tc_supported(B, H, T, K, V, C, dtype == GDN2_BF16 ? 1 : 0);
}

// Implementation for these sizes: 0 = CUDA-core two-kernel path; 1 = fused tcgen05 kernel (one CTA
// per chain), for up to 64 chains of fewer than 32 chunks; 2 = two-stage tcgen05 path (intra-chunk
// work parallel over every chunk-head, then the state chain, cut into segments in time when there
// are few long chains), for everything else.
int select_path(int B, int H, int T, int K, int V, int C, int dtype) {
    if (!use_tc(B, H, T, K, V, C, dtype)) return 0;
    const long long chains = (long long)B * H, NC = (T + 63) / 64;
    return chains > 64 || NC >= 32 ? 2 : 1;
}

}  // namespace

extern "C" {

size_t gdn2_chunk_fwd_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C, int dtype) {
    if (B < 0 || H < 0 || T < 0 || !dim_ok(d_k) || !dim_ok(d_v) || C != 64) return gdn2::kStatusBytes;
    switch (select_path(B, H, T, d_k, d_v, C, dtype)) {
        case 2: return gdn2::split_workspace_bytes(B, H, T);
        case 1: return gdn2::tc_workspace_bytes(B, H, T, d_k, d_v, C);
        default: return gdn2::simt_workspace_bytes(B, H, T, d_k, d_v, C);
    }
}

size_t gdn2_chunk_fwd_edges_workspace_bytes(int B, int H, int T, int d_k, int d_v, int C) {
    if (B < 0 || H < 0 || T < 0 || !use_tc(B, H, T, d_k, d_v, C, GDN2_BF16)) return gdn2::kStatusBytes;
    if (select_path(B, H, T, d_k, d_v, C, GDN2_BF16) == 2) return gdn2::split_workspace_bytes(B, H, T);
    return gdn2::tc_workspace_bytes(B, H, T, d_k, d_v, C, 1);
}

int gdn2_chunk_fwd_path(int B, int H, int T, int d_k, int d_v, int C, int dtype) {
    if (B < 0 || H < 0 || T < 0) return 0;
    return select_path(B, H, T, d_k, d_v, C, dtype);
}

int gdn2_chunk_fwd(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                   const float *S0, void *o, float *S_T, int B, int H, int T, int d_k, int d_v, int C, int dtype,
                   void *workspace, size_t workspace_bytes, void *stream) {
    if (T < 0) return GDN2_ERR_SHAPE;
    int rc;
    if (T == 0) {
        // no tokens: token and output pointers are not read (empty tensors may be NULL)
        if (B < 0 || H < 0) return GDN2_ERR_SHAPE;
        if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
        if (!dim_ok(d_k) || !dim_ok(d_v)) return GDN2_ERR_UNSUPPORTED;
    } else {
        rc = check_common(q, k, v, alpha, b, w, o, B, H, d_k, d_v, dtype);
        if (rc != GDN2_OK) return rc;
    }
    if (C != 64) return GDN2_ERR_UNSUPPORTED;
    if (!S_T) return GDN2_ERR_NULL;
    if (!aligned16(S_T) || (S0 && !aligned16(S0))) return GDN2_ERR_ALIGN;
    if (!workspace) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    if (workspace_bytes < gdn2_chunk_fwd_workspace_bytes(B, H, T, d_k, d_v, C, dtype)) return GDN2_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (B == 0 || H == 0) return GDN2_OK;
    const size_t state_bytes = sizeof(float) * (size_t)B * H * d_k * d_v;
    if (T == 0) {
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, st))
                           : cudaMemsetAsync(S_T, 0, state_bytes, st);
        return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
    }
    const int bf16 = dtype == GDN2_BF16 ? 1 : 0;
    const int path = select_path(B, H, T, d_k, d_v, C, dtype);
    if (path == 2)
        rc = gdn2::launch_chunk_split(q, k, v, alpha, b, w, S0, o, S_T, B, H, T, workspace, st);
    else if (path == 1)
        rc = gdn2::launch_chunk_tc(q, k, v, alpha, b, w, S0, o, S_T, B, H, T, d_k, d_v, C, workspace, st);
    else
        rc = gdn2::launch_chunk_simt(q, k, v, alpha, b, w, S0, o, S_T, B, H, T, d_k, d_v, C, bf16, workspace, st);
    return rc;
}

int gdn2_chunk_fwd_edges(const void *q_raw, const void *k_raw, const void *v, const float *a_logit,
                         const void *b_logit, const void *w_logit, const float *S0, const float *o_weight, void *o,
                         float *S_T, int B, int H, int T, int d_k, int d_v, int C, int dtype, void *workspace,
                         size_t workspace_bytes, void *stream) {
    if (T < 0) return GDN2_ERR_SHAPE;
    if (T == 0) return gdn2_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, S0, nullptr, S_T, B, H,
                                      0, d_k, d_v, C, dtype, workspace, workspace_bytes, stream);
    int rc = check_common(q_raw, k_raw, v, a_logit, b_logit, w_logit, o, B, H, d_k, d_v, dtype);
    if (rc != GDN2_OK) return rc;
    if (C != 64 || !use_tc(B, H, T, d_k, d_v, C, dtype)) return GDN2_ERR_UNSUPPORTED;
    if (!S_T) return GDN2_ERR_NULL;
    if (!aligned16(S_T) || (S0 && !aligned16(S0)) || (o_weight && !aligned16(o_weight))) return GDN2_ERR_ALIGN;
    if (!workspace) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    if (workspace_bytes < gdn2_chunk_fwd_edges_workspace_bytes(B, H, T, d_k, d_v, C)) return GDN2_ERR_WORKSPACE;
    if (B == 0 || H == 0) return GDN2_OK;
    if (select_path(B, H, T, d_k, d_v, C, dtype) == 2)
        return gdn2::launch_chunk_split(q_raw, k_raw, v, a_logit, b_logit, w_logit, S0, o, S_T, B, H, T, workspace,
                                        reinterpret_cast<cudaStream_t>(stream), 1, o_weight);
    return gdn2::launch_chunk_tc(q_raw, k_raw, v, a_logit, b_logit, w_logit, S0, o, S_T, B, H, T, d_k, d_v, C,
                                 workspace, reinterpret_cast<cudaStream_t>(stream), 1, o_weight);
}

int gdn2_decode_step(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                     float *S, void *o, int B, int H, int d_k, int d_v, int dtype, void *stream) {
    int rc = check_common(q, k, v, alpha, b, w, o, B, H, d_k, d_v, dtype);
    if (rc != GDN2_OK) return rc;
    if (!S) return GDN2_ERR_NULL;
    if (!aligned16(S)) return GDN2_ERR_ALIGN;
    if (B == 0 || H == 0) return GDN2_OK;
    return gdn2::launch_decode(q, k, v, alpha, b, w, S, o, B, H, d_k, d_v, dtype == GDN2_BF16 ? 1 : 0,
                               reinterpret_cast<cudaStream_t>(stream));
}

size_t gdn2_chunk_bwd_workspace_bytes(int B, int H, int T, int d_k, int d_v) {
    if (B < 0 || H < 0 || T < 0 || !dim_ok(d_k) || !dim_ok(d_v)) return 0;
    return gdn2::bwd_workspace_bytes(B, H, T, d_k, d_v);
}

int gdn2_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                   const float *S0, const void *dO, const float *dS_T, float *dq, float *dk, float *dv,
                   float *dalpha, float *db, float *dw, float *dS0, int B, int H, int T, int d_k, int d_v,
                   int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (T < 0 || B < 0 || H < 0) return GDN2_ERR_SHAPE;
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (!dim_ok(d_k) || !dim_ok(d_v)) return GDN2_ERR_UNSUPPORTED;
    if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0))) return GDN2_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t state_bytes = sizeof(float) * (size_t)B * H * d_k * d_v;
    if (T == 0) {   // S_T = S0: dS0 = dS_T; no token gradients
        if (!dS0 || B == 0 || H == 0) return GDN2_OK;
        const cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(dS0, 0, state_bytes, st);
        return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
    }
    int rc = check_common(q, k, v, alpha, b, w, dO, B, H, d_k, d_v, dtype);
    if (rc != GDN2_OK) return rc;
    if (!dq || !dk || !dv || !dalpha || !db || !dw) return GDN2_ERR_NULL;
    if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dalpha) || !aligned16(db) ||
        !aligned16(dw))
        return GDN2_ERR_ALIGN;
    if (!workspace) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    if (workspace_bytes < gdn2_chunk_bwd_workspace_bytes(B, H, T, d_k, d_v)) return GDN2_ERR_WORKSPACE;
    if (B == 0 || H == 0) return GDN2_OK;
    return gdn2::launch_chunk_bwd(q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, B, H, T,
                                  d_k, d_v, dtype == GDN2_BF16 ? 1 : 0, workspace, st);
}

size_t gdn2_chunk_bwd_tc_workspace_bytes(int B, int H, int T, int d_k, int d_v) {
    if (B < 0 || H < 0 || T < 0 || d_k != 128 || d_v != 128) return 0;
    return gdn2::chunk_bwd_tc_workspace_bytes(B, H, T);
}

int gdn2_chunk_bwd_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                      const float *S0, const void *dO, const float *dS_T, float *dq, float *dk, float *dv,
                      float *dalpha, float *db, float *dw, float *dS0, int B, int H, int T, int d_k, int d_v,
                      int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (T < 0 || B < 0 || H < 0) return GDN2_ERR_SHAPE;
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (dtype != GDN2_BF16 || d_k != 128 || d_v != 128) return GDN2_ERR_UNSUPPORTED;
    if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0))) return GDN2_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {   // S_T = S0: dS0 = dS_T; no token gradients
        if (!dS0 || B == 0 || H == 0) return GDN2_OK;
        const size_t state_bytes = sizeof(float) * (size_t)B * H * d_k * d_v;
        const cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(dS0, 0, state_bytes, st);
        return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
    }
    int rc = check_common(q, k, v, alpha, b, w, dO, B, H, d_k, d_v, dtype);
    if (rc != GDN2_OK) return rc;
    if (!dq || !dk || !dv || !dalpha || !db || !dw) return GDN2_ERR_NULL;
    if (!aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dalpha) || !aligned16(db) ||
        !aligned16(dw))
        return GDN2_ERR_ALIGN;
    if (!workspace) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    if (workspace_bytes < gdn2_chunk_bwd_tc_workspace_bytes(B, H, T, d_k, d_v)) return GDN2_ERR_WORKSPACE;
    if (B == 0 || H == 0) return GDN2_OK;
    return gdn2::launch_chunk_bwd_tc(q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, B, H, T,
                                     workspace, st);
}

int gdn2_layer_edge_maps(const void *q_raw, const void *k_raw, const float *a_logit, const void *b_logit,
                         const void *w_logit, void *q, void *k, float *alpha, void *b, void *w, int B, int T, int H,
                         int d_k, int d_v, void *stream) {
    if (B < 0 || T < 0 || H < 0) return GDN2_ERR_SHAPE;
    if (!dim_ok(d_k) || !dim_ok(d_v)) return GDN2_ERR_UNSUPPORTED;
    const long long rows = (long long)B * T * H;
    if (rows == 0) return GDN2_OK;
    const void *ptrs[10] = {q_raw, k_raw, a_logit, b_logit, w_logit, q, k, alpha, b, w};
    for (const void *p : ptrs) {
        if (!p) return GDN2_ERR_NULL;
        if (!aligned16(p)) return GDN2_ERR_ALIGN;
    }
    return gdn2::launch_edge_maps(q_raw, k_raw, a_logit, b_logit, w_logit, q, k, alpha, b, w, rows, d_k, d_v,
                                  reinterpret_cast<cudaStream_t>(stream));
}

int gdn2_rms_norm(void *o, const float *weight, long long rows, int d_v, void *stream) {
    if (rows < 0) return GDN2_ERR_SHAPE;
    if (!dim_ok(d_v)) return GDN2_ERR_UNSUPPORTED;
    if (rows == 0) return GDN2_OK;
    if (!o || !weight) return GDN2_ERR_NULL;
    if (!aligned16(o) || !aligned16(weight)) return GDN2_ERR_ALIGN;
    return gdn2::launch_rms_norm(o, weight, rows, d_v, reinterpret_cast<cudaStream_t>(stream));
}

int gdn2_gemm_phase_probe(int mode, int reps, int nctas, void *workspace, size_t workspace_bytes, void *stream) {
    if ((mode != 0 && mode != 1) || reps < 1 || nctas < 1) return GDN2_ERR_SHAPE;
    if (!workspace) return GDN2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDN2_ERR_ALIGN;
    if (workspace_bytes < gdn2::kStatusBytes) return GDN2_ERR_WORKSPACE;
    return gdn2::launch_phase_probe(mode, reps, nctas, reinterpret_cast<unsigned int *>(workspace),
                                    reinterpret_cast<cudaStream_t>(stream));
}

int gdn2_workspace_status(void *workspace, int clear, int *out, void *stream) {
    if (!workspace || !out) return GDN2_ERR_NULL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GDN2_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDN2_ERR_CUDA;
    *out = (int)word;
    if (clear && word) {
        if (cudaMemsetAsync(workspace, 0, gdn2::kStatusBytes, st) != cudaSuccess) return GDN2_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return GDN2_ERR_CUDA;
    }
    return GDN2_OK;
}

const char *gdn2_status_str(int status) {
    switch (status) {
        case GDN2_OK: return "ok";
        case GDN2_ERR_NULL: return "a required pointer is NULL";
        case GDN2_ERR_SHAPE: return "a size is negative or inconsistent";
        case GDN2_ERR_DTYPE: return "unknown dtype code";
        case GDN2_ERR_UNSUPPORTED: return "unsupported size (d_k and d_v must be 64 or 128, C must be 64)";
        case GDN2_ERR_WORKSPACE: return "workspace missing or too small";
        case GDN2_ERR_CUDA: return "CUDA runtime or launch error";
        case GDN2_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case GDN2_ERR_DEVICE: return "a kernel reported an internal error";
        case GDN2_ERR_NOALLOC_LIMIT:
            return "problem needs more scratch than the no-allocation entry point's fixed array";
        default: return "unknown status";
    }
}

}  // extern "C"
