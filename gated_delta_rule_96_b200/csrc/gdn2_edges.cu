// The layer's edge maps as stand-alone elementwise kernels (sm_100a): the maps that
// gdn2_chunk_fwd_edges fuses into the prefill, run on their own so that the unfused layer
// (maps -> gdn2_chunk_fwd -> RMSNorm) can be measured against the fused one.
//
// Page "NVIDIA представила Gated DeltaNet-2 ...", the paragraph on the layer: q and k pass an L2
// norm, the gates are sigmoid projections, the decay comes from its projection, the output passes
// RMSNorm.  Per (b, t, h):
//   q = q_raw / max(|q_raw|, 1e-6), k likewise; b = sigmoid(b_logit), w = sigmoid(w_logit);
//   alpha = exp(-softplus(a_logit)) = 1 / (1 + e^a);  o <- o / sqrt(mean(o^2) + 1e-6) * weight.
// One warp per row; bf16 tokens, fp32 alpha, d in {64, 128}.
#include "gdn2_common.cuh"
#include "gdn2_internal.h"

namespace gdn2 {
namespace edges {

constexpr float NORM_EPS = 1e-6f, RMS_EPS = 1e-6f;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}
// sigmoid and the decay from its logit, in the numerically safe forms for either sign
__device__ __forceinline__ float sigmoidf_(float x) {
    const float e = __expf(-fabsf(x));
    return x >= 0.f ? 1.f / (1.f + e) : e / (1.f + e);
}

// 2 or 4 bf16 of one lane as one load / store (d = 64: 2 channels a lane, d = 128: 4)
template <int P>
struct Vec;
template <>
struct Vec<2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&x)[2]) {
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(p);
        x[0] = __low2float(v); x[1] = __high2float(v);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&x)[2]) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x[0], x[1]);
    }
    static __device__ __forceinline__ void loadf(const float *p, float (&x)[2]) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        x[0] = v.x; x[1] = v.y;
    }
    static __device__ __forceinline__ void storef(float *p, const float (&x)[2]) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    }
};
template <>
struct Vec<4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&x)[4]) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&u.x), b = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
        x[0] = __low2float(a); x[1] = __high2float(a); x[2] = __low2float(b); x[3] = __high2float(b);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&x)[4]) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
        *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
    }
    static __device__ __forceinline__ void loadf(const float *p, float (&x)[4]) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static __device__ __forceinline__ void storef(float *p, const float (&x)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

template <int DK, int DV>
__global__ void __launch_bounds__(256) edge_maps_kernel(const __nv_bfloat16 *__restrict__ q_raw,
                                                        const __nv_bfloat16 *__restrict__ k_raw,
                                                        const float *__restrict__ a_logit,
                                                        const __nv_bfloat16 *__restrict__ b_logit,
                                                        const __nv_bfloat16 *__restrict__ w_logit,
                                                        __nv_bfloat16 *__restrict__ q, __nv_bfloat16 *__restrict__ k,
                                                        float *__restrict__ alpha, __nv_bfloat16 *__restrict__ b,
                                                        __nv_bfloat16 *__restrict__ w, long long rows) {
    constexpr int PK = DK / 32, PV = DV / 32;   // channels per lane
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
        const size_t ok = (size_t)r * DK + PK * lane, ov = (size_t)r * DV + PV * lane;
        float qx[PK], kx[PK], bx[PK], ax[PK], wx[PV], sq = 0.f, sk = 0.f;
        Vec<PK>::load(q_raw + ok, qx);
        Vec<PK>::load(k_raw + ok, kx);
        Vec<PK>::load(b_logit + ok, bx);
        Vec<PK>::loadf(a_logit + ok, ax);
        Vec<PV>::load(w_logit + ov, wx);
#pragma unroll
        for (int i = 0; i < PK; ++i) {
            sq += qx[i] * qx[i];
            sk += kx[i] * kx[i];
        }
        const float iq = 1.f / fmaxf(sqrtf(warp_sum(sq)), NORM_EPS), ik = 1.f / fmaxf(sqrtf(warp_sum(sk)), NORM_EPS);
#pragma unroll
        for (int i = 0; i < PK; ++i) {
            qx[i] *= iq;
            kx[i] *= ik;
            bx[i] = sigmoidf_(bx[i]);
            ax[i] = sigmoidf_(-ax[i]);   // 1 / (1 + e^a)
        }
#pragma unroll
        for (int i = 0; i < PV; ++i) wx[i] = sigmoidf_(wx[i]);
        Vec<PK>::store(q + ok, qx);
        Vec<PK>::store(k + ok, kx);
        Vec<PK>::store(b + ok, bx);
        Vec<PK>::storef(alpha + ok, ax);
        Vec<PV>::store(w + ov, wx);
    }
}

template <int DV>
__global__ void __launch_bounds__(256) rms_norm_kernel(__nv_bfloat16 *__restrict__ o, const float *__restrict__ weight,
                                                       long long rows) {
    constexpr int PV = DV / 32;
    const int lane = threadIdx.x & 31;
    const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
    float wt[PV];
    Vec<PV>::loadf(weight + PV * lane, wt);
    for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nwarps) {
        const size_t off = (size_t)r * DV + PV * lane;
        float x[PV], ss = 0.f;
        Vec<PV>::load(o + off, x);
#pragma unroll
        for (int i = 0; i < PV; ++i) ss += x[i] * x[i];
        const float scale = rsqrtf(warp_sum(ss) * (1.f / DV) + RMS_EPS);
#pragma unroll
        for (int i = 0; i < PV; ++i) x[i] *= scale * wt[i];
        Vec<PV>::store(o + off, x);
    }
}

int grid_for(long long rows) {
    const long long warps = rows, blocks = (warps + 7) / 8;
    return (int)(blocks < 148 * 16 ? (blocks > 0 ? blocks : 1) : 148 * 16);
}

}  // namespace edges

int launch_edge_maps(const void *q_raw, const void *k_raw, const float *a_logit, const void *b_logit,
                     const void *w_logit, void *q, void *k, float *alpha, void *b, void *w, long long rows, int K, int V,
                     cudaStream_t st) {
    using bf = __nv_bfloat16;
    auto go = [&](auto kern) {
        kern<<<edges::grid_for(rows), 256, 0, st>>>((const bf *)q_raw, (const bf *)k_raw, a_logit, (const bf *)b_logit,
                                                     (const bf *)w_logit, (bf *)q, (bf *)k, alpha, (bf *)b, (bf *)w, rows);
    };
    if (K == 128 && V == 128) go(edges::edge_maps_kernel<128, 128>);
    else if (K == 128 && V == 64) go(edges::edge_maps_kernel<128, 64>);
    else if (K == 64 && V == 128) go(edges::edge_maps_kernel<64, 128>);
    else if (K == 64 && V == 64) go(edges::edge_maps_kernel<64, 64>);
    else return -4;
    return launch_status();
}

int launch_rms_norm(void *o, const float *weight, long long rows, int V, cudaStream_t st) {
    if (V == 128)
        edges::rms_norm_kernel<128><<<edges::grid_for(rows), 256, 0, st>>>((__nv_bfloat16 *)o, weight, rows);
    else if (V == 64)
        edges::rms_norm_kernel<64><<<edges::grid_for(rows), 256, 0, st>>>((__nv_bfloat16 *)o, weight, rows);
    else
        return -4;
    return launch_status();
}

}  // namespace gdn2
