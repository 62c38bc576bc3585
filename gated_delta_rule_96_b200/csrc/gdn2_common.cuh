// Shared device helpers of libgdn2 (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn2 {

// token element <-> fp32
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_tok(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_tok(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <typename Tok>
__device__ __forceinline__ float ld_tok(const Tok *p) {
    return to_f32(*p);
}

// fp32 state streamed once per call: evict-first loads/stores
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

// Launch-error helper used by the host launchers.
inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? 0 : -6;
}

}  // namespace gdn2
