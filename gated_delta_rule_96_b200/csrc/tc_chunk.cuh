// Device helpers shared by the tensor-core prefill kernels (sm_100a): fast exponentials, packed
// bf16 products, warp-level tf32 tile products and the 64 x 64 unit-lower-triangular inverse of
// the chunkwise WY form (page "NVIDIA представила Gated DeltaNet-2 ...", the paragraph on the
// chunkwise WY kernels with C = 64: T = (I + A)^-1 turns the chunk's rank-1 updates into
// products).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tc_ptx.cuh"

namespace gdn2 {
namespace tcc {

using namespace gdn2::tc;

constexpr int LDA = 68;   // fp32 row stride of the A/T scratch: conflict-free mma fragment loads

// hardware base-2 exponential and logarithm (approximate, flush-to-zero): the operands they
// feed are rounded to bf16 right after, far coarser than the approximation error
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_log2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    __nv_bfloat162 p = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return make_float2(__low2float(p), __high2float(p));
}
// product of two packed bf16 pairs, rounded to bf16 (the exact product of two bf16 values is
// representable in fp32, so this is one rounding of the exact product)
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}
// tf32 operand of mma.sync: the fp32 bit pattern (the tensor core reads the top 19 bits, i.e.
// truncates the mantissa to 10 bits; T ends up in bf16, far coarser)
__device__ __forceinline__ uint32_t tf32(float x) { return __float_as_uint(x); }
// D(16x8) += A(16x8) B(8x8), tf32 inputs, fp32 accumulate (warp-level)
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// 16x8 tile of L(16 x 8k) * R(8k x 8), L and R fp32 [.][ld] in shared memory, k-steps ks..ke-1
__device__ __forceinline__ void tile_mm(float (&d)[4], const float *Lm, int ldl, int l0, int lc0, const float *Rm,
                                        int ldr, int rr0, int rc0, int ks, int ke, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    for (int s = ks; s < ke; ++s) {
        const int kc = 8 * s;
        const uint32_t a0 = tf32(Lm[(l0 + gq) * ldl + lc0 + kc + tq]);
        const uint32_t a1 = tf32(Lm[(l0 + gq + 8) * ldl + lc0 + kc + tq]);
        const uint32_t a2 = tf32(Lm[(l0 + gq) * ldl + lc0 + kc + tq + 4]);
        const uint32_t a3 = tf32(Lm[(l0 + gq + 8) * ldl + lc0 + kc + tq + 4]);
        const uint32_t b0 = tf32(Rm[(rr0 + kc + tq) * ldr + rc0 + gq]);
        const uint32_t b1 = tf32(Rm[(rr0 + kc + tq + 4) * ldr + rc0 + gq]);
        mma_tf32(d, a0, a1, a2, a3, b0, b1);
    }
}
__device__ __forceinline__ void tile_store(float *Dm, int ld, int r0, int c0, const float (&d)[4], float sc,
                                           int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    Dm[(r0 + gq) * ld + c0 + 2 * tq] = sc * d[0];
    Dm[(r0 + gq) * ld + c0 + 2 * tq + 1] = sc * d[1];
    Dm[(r0 + gq + 8) * ld + c0 + 2 * tq] = sc * d[2];
    Dm[(r0 + gq + 8) * ld + c0 + 2 * tq + 1] = sc * d[3];
}

// The same 16x8 fragment, scaled, into a bf16 [64 x 64] swizzled tile (two columns per store).
__device__ __forceinline__ void tile_store_bf16(unsigned char *tile, int r0, int c0, const float (&d)[4], float sc,
                                                int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    *reinterpret_cast<uint32_t *>(tile + sw_off(r0 + gq, c0 + 2 * tq, 64)) = pack_bf16(sc * d[0], sc * d[1]);
    *reinterpret_cast<uint32_t *>(tile + sw_off(r0 + gq + 8, c0 + 2 * tq, 64)) = pack_bf16(sc * d[2], sc * d[3]);
}

// T is kept transposed on and above the diagonal of the A scratch (A is strictly lower):
// T[x][y] (x >= y) lives at AS[y * LDA + x]; entries with x < y are zero and read as zero.
__device__ __forceinline__ float t_at(const float *AS, int x, int y) { return x >= y ? AS[y * LDA + x] : 0.f; }
// 16x8 tile of L(16 x 8k) * T(8k x 8), T rows rr0.., columns rc0.. (B operand from T^T)
__device__ __forceinline__ void tile_mm_tb(float (&d)[4], const float *Lm, int ldl, int l0, int lc0, const float *AS,
                                           int rr0, int rc0, int ks, int ke, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    for (int s = ks; s < ke; ++s) {
        const int kc = 8 * s;
        const uint32_t a0 = tf32(Lm[(l0 + gq) * ldl + lc0 + kc + tq]);
        const uint32_t a1 = tf32(Lm[(l0 + gq + 8) * ldl + lc0 + kc + tq]);
        const uint32_t a2 = tf32(Lm[(l0 + gq) * ldl + lc0 + kc + tq + 4]);
        const uint32_t a3 = tf32(Lm[(l0 + gq + 8) * ldl + lc0 + kc + tq + 4]);
        const uint32_t b0 = tf32(t_at(AS, rr0 + kc + tq, rc0 + gq));
        const uint32_t b1 = tf32(t_at(AS, rr0 + kc + tq + 4, rc0 + gq));
        mma_tf32(d, a0, a1, a2, a3, b0, b1);
    }
}
// 16x8 tile of T(16 x 8k) * R(8k x 8), T rows l0.., columns lc0.. (A operand from T^T)
__device__ __forceinline__ void tile_mm_ta(float (&d)[4], const float *AS, int l0, int lc0, const float *Rm, int ldr,
                                           int rr0, int rc0, int ks, int ke, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    for (int s = ks; s < ke; ++s) {
        const int kc = 8 * s;
        const uint32_t a0 = tf32(t_at(AS, l0 + gq, lc0 + kc + tq));
        const uint32_t a1 = tf32(t_at(AS, l0 + gq + 8, lc0 + kc + tq));
        const uint32_t a2 = tf32(t_at(AS, l0 + gq, lc0 + kc + tq + 4));
        const uint32_t a3 = tf32(t_at(AS, l0 + gq + 8, lc0 + kc + tq + 4));
        const uint32_t b0 = tf32(Rm[(rr0 + kc + tq) * ldr + rc0 + gq]);
        const uint32_t b1 = tf32(Rm[(rr0 + kc + tq + 4) * ldr + rc0 + gq]);
        mma_tf32(d, a0, a1, a2, a3, b0, b1);
    }
}
// the 16x8 fragment (scaled) as a block of T at rows r0.., columns c0.. (r0 > c0 + 7)
__device__ __forceinline__ void tile_store_t(float *AS, int r0, int c0, const float (&d)[4], float sc, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
    AS[(c0 + 2 * tq) * LDA + r0 + gq] = sc * d[0];
    AS[(c0 + 2 * tq + 1) * LDA + r0 + gq] = sc * d[1];
    AS[(c0 + 2 * tq) * LDA + r0 + gq + 8] = sc * d[2];
    AS[(c0 + 2 * tq + 1) * LDA + r0 + gq + 8] = sc * d[3];
}

// Layer edges fused into the prefill (the layer around the recurrence: q and k L2-normalised per
// token and head, b and w sigmoid gates, the decay from a logit, the output through RMSNorm).
constexpr float EDGE_NORM_EPS = 1e-6f;   // q / max(|q|, eps), likewise k
constexpr float EDGE_RMS_EPS = 1e-6f;    // o / sqrt(mean(o^2) + eps) * weight
__device__ __forceinline__ float fast_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// sigmoid(x) = 1 / (1 + 2^(-x log2 e)); the exponential saturates to +inf (result 0) or 0 (result 1)
__device__ __forceinline__ float sigmoid_f(float x) { return fast_rcp(1.f + fast_exp2(-1.4426950408889634f * x)); }
// alpha = exp(-softplus(a)) = 1 / (1 + e^a) = sigmoid(-a) (0 past fp32's range: the caller floors it)
__device__ __forceinline__ float alpha_of_logit(float a) { return fast_rcp(1.f + fast_exp2(1.4426950408889634f * a)); }
__device__ __forceinline__ uint32_t bsigmoid2(uint32_t a) {
    const float2 f = unpack2(a);
    return pack_bf16(sigmoid_f(f.x), sigmoid_f(f.y));
}

// T = (I + A)^-1 for the strictly lower-triangular 64 x 64 matrix A held in AS (fp32, row stride
// LDA, zeros on and above the diagonal).  On return T^T is on and above AS's diagonal (A stays
// below it) and T, in bf16, is in the swizzled 64 x 64 tile Tt, whose blocks above the diagonal
// must already be zero.  128 threads (tid2 = 0..127) take part, synchronised on the named barrier
// `bar`; XS is 4 KB of per-warp scratch.  The last step's writes are not followed by a barrier:
// the caller synchronises before reading Tt or AS.
//   Diagonal 16 x 16 blocks by column-oriented forward substitution (64 threads, one column
//   each), then two doubling steps on mma.sync tf32: the 16 x 16 blocks (1,0) and (3,2) as
//   T_RI = -T_RR (A_RI T_II), then the 32 x 32 block below the diagonal likewise.
__device__ __forceinline__ void solve_unit_lower(float *AS, float *XS, unsigned char *Tt, int tid2, uint32_t bar) {
    const int pw = tid2 >> 5, lane = tid2 & 31;
    // ---------------------------------------------------------------- T = (I + A)^-1
    // The bf16 T tile is written block by block as T is formed (G2 of the previous chunk,
    // its reader, has completed); its blocks above the diagonal stay zero.
    if (tid2 < 64) {   // diagonal 16x16 blocks, one column per thread
        // column-oriented substitution: as soon as T[i][j] is known its contribution is
        // subtracted from every later row, so the dependent chain is one FMA per row
        const int J = tid2 >> 4, j = tid2 & 15, o16 = 16 * J;
        const float *Ab = AS + o16 * LDA + o16;
        float nacc[16], col[16];   // nacc[r] = -sum_{i<r} A[r][i] T[i][j]
#pragma unroll
        for (int r = 0; r < 16; ++r) nacc[r] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float t = i == j ? 1.f : (i < j ? 0.f : nacc[i]);
            col[i] = t;
#pragma unroll
            for (int r = i + 1; r < 16; ++r) nacc[r] = fmaf(-Ab[r * LDA + i], t, nacc[r]);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            if (r >= j) AS[(o16 + j) * LDA + o16 + r] = col[r];   // T^T, on and above the diagonal
            *reinterpret_cast<__nv_bfloat16 *>(Tt + sw_off(o16 + r, o16 + j, 64)) = __float2bfloat16_rn(col[r]);
        }
    }
    group_sync(bar, 128);
    if (pw < 2) {   // blocks (1,0) and (3,2): T_RI = -T_RR (A_RI T_II), within one warp
        const int R = 16 * (2 * pw + 1), I = 16 * (2 * pw);
        float *X = XS + pw * 384;   // 16 x 16 (row stride 24), private to this warp
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            tile_mm_tb(d, AS, LDA, R, I, AS, I, I + 8 * nt, 0, 2, lane);
            tile_store(X, 24, 0, 8 * nt, d, 1.f, lane);
        }
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            tile_mm_ta(d, AS, R, R, X, 24, 0, 8 * nt, 0, 2, lane);
            tile_store_t(AS, R, I + 8 * nt, d, -1.f, lane);
            tile_store_bf16(Tt, R, I + 8 * nt, d, -1.f, lane);
        }
    }
    group_sync(bar, 128);
    {   // rows 32..63 x cols 8pw..8pw+7: T = -T_hi (A_hi,lo T_lo), within one warp
        const int nt = pw;
        float *X = XS + pw * 256;   // 32 x 8, private to this warp
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {   // block (0,1) of T is zero: skipped for columns >= 16
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            tile_mm_tb(d, AS, LDA, 32 + 16 * mt, 0, AS, 0, 8 * nt, nt >= 2 ? 2 : 0, 4, lane);
            tile_store(X, 8, 16 * mt, 0, d, 1.f, lane);
        }
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {   // block (2,3) of T is zero: skipped for rows < 48
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            tile_mm_ta(d, AS, 32 + 16 * mt, 32, X, 8, 0, 0, 0, mt == 0 ? 2 : 4, lane);
            tile_store_bf16(Tt, 32 + 16 * mt, 8 * nt, d, -1.f, lane);
        }
    }}

}  // namespace tcc
}  // namespace gdn2
