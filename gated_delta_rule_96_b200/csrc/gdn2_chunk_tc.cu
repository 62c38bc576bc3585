// Fused chunkwise prefill on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
// bf16 tokens, d_k = d_v = 128, chunk C = 64.  One CTA owns one (b, h) chain and walks
// its chunks in order; the state never leaves the SM and no intermediate goes to global
// memory.
//
// Per chunk (page "NVIDIA представила Gated DeltaNet-2 ...": the update equation of
// section "Техническая схема" evaluated in the chunkwise WY form with C = 64 named on
// the same page).  g = per-channel prefix of log alpha inside the chunk, e = b ⊙ k,
// u = w ⊙ v, m = per-channel midpoint of g over the chunk, g_C = g at the chunk's end:
//
//   build   Ê = e ⊙ exp(g-m), Q̂ = q ⊙ exp(g-m), K̃ = k ⊙ exp(m-g), U = u    (bf16 smem)
//   G1      [A; P] = [Ê; Q̂] K̃^T                    A_ri = sum_c e_rc k_ic exp(g_rc - g_ic)
//   solve   T = (I + A)^-1        (fp32; 16x16 diagonal blocks, doubling on mma.sync tf32)
//   G2      [W'; *] = [T; P] Ê,  [U~; *] = [T; P] U    (W = exp(m) ⊙ W' = T (exp(g) ⊙ E))
//   G3      [Delta; O] = [U~; 0] + [-W'; Q̂] Z       Z = Diag(exp(m)) S (bf16 copy)
//   G4/G5   O += P Delta,   Z += K̃^T Delta          (Z accumulates in TMEM, fp32)
//   next    S' = Diag(exp(g_C - m)) Z,  Z' = Diag(exp(m')) S'
//
// The state is kept in TMEM as Z = Diag(exp(m)) S for the chunk about to be processed:
// then S' = Diag(exp(g_C)) S + K^T Delta = Diag(exp(g_C - m)) (Z + K̃^T Delta), so G5
// accumulates straight into the state and one TMEM round trip per chunk rescales it.
//
// The cumulative channel decay is absorbed into the rank-1 factors around m: every
// factor exp(±(g - m)) lies in [e^-60, e^60] while the chunk's log-decay span
// g_0 - g_63 stays <= 120 in every channel, and each product exp(g_r - g_i) that A and P
// need is formed by the tensor core from two representable factors.  A chunk with a
// wider span computes A and P on CUDA cores from exp(g_r - g_i) <= 1 per element and
// uses unscaled factors elsewhere (m = 0), so any alpha in (0, 1] is handled.
//
// Warp roles (16 warps, registers rebalanced per warpgroup with setmaxnreg):
//   warps 0-3   state group (56 regs): rescales Z, writes its bf16 copy, Delta and o
//               epilogues
//   warps 4-11  chunk group (200 regs): loads, build, A/P readout, triangular solve, -W'
//               epilogue for chunk n+1 while the state group finishes chunk n
//   warp 12     MMA issuer (56 regs): one thread issues every tcgen05.mma as its inputs
//               become ready (mbarrier signals), in any order the dependencies allow
//   warp 13     producer (56 regs): stages alpha of the next chunk into shared memory with
//               bulk asynchronous copies
//   warps 14-15 value group (56 regs): U = w ⊙ v of the next chunk
// Every wait is bounded; on expiry the block sets the workspace status word and exits.
#include "gdn2_common.cuh"
#include "gdn2_internal.h"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace tcfwd {

using namespace gdn2::tc;

constexpr int C = 64, KD = 128, VD = 128;
constexpr int NT = 512;                       // 16 warps
constexpr int STATE_THREADS = 128, CHUNK_THREADS = 256;
constexpr uint32_t BAR_STATE = 1, BAR_CHUNK = 2;   // named barrier ids
constexpr float SPAN_MAX_LOG2 = 173.123f;     // 120 nats in log2 units
constexpr uint32_t WAIT_LIMIT = 1u << 22;
constexpr uint32_t POLL_LIMIT = 1u << 26;

// TMEM columns (512 allocated)
constexpr uint32_t TM_D2 = 0;                 // [W'; *] (128); [A; P] (64) in its first columns
constexpr uint32_t TM_D1 = 0;
constexpr uint32_t TM_D3 = 128;               // [U~ -> Delta; O], two buffers of 128
constexpr uint32_t TM_Z = 384;                // Z fp32 (128)
constexpr uint32_t TM_COLS = 512;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t SM_S = 0;                      // Z in bf16 [c x v], B of G3 (MN-major)
constexpr uint32_t SM_EQ = 32768;                 // [Ê -> -W'; Q̂] 128 x 128 (K-major A of G1 / G3)
constexpr uint32_t SM_KT = 65536;                 // K̃ [i x c] 64 x 128
constexpr uint32_t SM_U = 81920;                  // U [i x v] 64 x 128
constexpr uint32_t SM_DL = 98304;                 // Delta [i x v] 64 x 128
constexpr uint32_t SM_T = 114688;                 // T [r x i] 64 x 64, followed by
constexpr uint32_t SM_P = 122880;                 // P [r x i]: [T; P] is one K-major 128-row operand
constexpr int LDA = 68;                           // fp32 row stride: conflict-free mma fragment loads
constexpr uint32_t SM_AS = 131072;                // A fp32 [64][LDA]
constexpr uint32_t SM_TF = SM_AS + 64 * LDA * 4;  // T fp32 [64][LDA]
constexpr uint32_t SM_VEC = SM_TF + 64 * LDA * 4;  // [2 chunks][sS, sZ, sPost] + g_0 (7 x 128 fp32)
constexpr uint32_t SM_WT = SM_VEC + 3584;         // fp32 [8][128] warp totals / solve scratch
constexpr uint32_t SM_ALPHA = SM_WT + 4096;       // alpha of the next chunk, fp32 [64][128]
constexpr uint32_t SM_MISC = SM_ALPHA + 32768;    // mbarriers, TMEM slot, flags
constexpr uint32_t SM_BYTES = SM_MISC + 256 + 1024;
constexpr uint32_t SM_G32 = SM_DL;                // wide-span chunks: g fp32 [64][128] over Delta, T, P

// mbarriers (byte offsets inside SM_MISC)
enum : uint32_t {
    MB_BUILD = 0, MB_G1 = 8, MB_SOLVE = 16, MB_G2 = 24, MB_S1DONE = 32, MB_VEC = 40, MB_STILDE = 48,
    MB_G3 = 56, MB_DELTA = 64, MB_G45 = 72, MB_D3FREE0 = 80, MB_D3FREE1 = 88, MB_AFULL = 96, MB_AEMPTY = 104,
    MB_U = 112, MB_COUNT = 15
};
constexpr uint32_t MISC_TSLOT = 128, MISC_ABORT = 132;

constexpr uint32_t ID_G1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G2 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G3 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G4 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G5 = idesc_bf16(128, 128, 1, 1);

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
__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
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

struct Ctx {
    unsigned char *sm;
    uint32_t tmem, misc;
    const __nv_bfloat16 *q, *k, *v, *b, *w;
    const float *alpha;
    __nv_bfloat16 *o;
    int T, H, bb, h, NC;
};

__device__ __forceinline__ uint32_t mbar(const Ctx &c, uint32_t off) { return c.misc + off; }
__device__ __forceinline__ volatile uint32_t *abort_flag(const Ctx &c) {
    return reinterpret_cast<volatile uint32_t *>(c.sm + SM_MISC + MISC_ABORT);
}

// Group-collective bounded wait: every thread of the group gets the same verdict.
__device__ __forceinline__ bool group_wait(const Ctx &c, uint32_t mb, uint32_t parity, uint32_t bar,
                                           uint32_t nthreads) {
    bool ok = mbar_wait(mb, parity, WAIT_LIMIT);
    if (*abort_flag(c)) ok = false;
    const bool fail = group_or(bar, nthreads, !ok);
    fence_after();
    if (fail) *abort_flag(c) = 1u;
    return !fail;
}

// ============================================================================ chunk group
__device__ void chunk_group(const Ctx &c, int tid1) {
    unsigned char *sm = c.sm;
    float *AS = reinterpret_cast<float *>(sm + SM_AS);
    float *TF = reinterpret_cast<float *>(sm + SM_TF);
    float *vec = reinterpret_cast<float *>(sm + SM_VEC);
    float *v_g0 = vec + 768;
    float *WT = reinterpret_cast<float *>(sm + SM_WT);
    float *G32 = reinterpret_cast<float *>(sm + SM_G32);
    const int sw = tid1 >> 5, lane = tid1 & 31;       // chunk-group warp 0..7
    const int quarter = sw & 3, chalf = sw >> 2;      // TMEM lane quarter, column half
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
    const int crow = quarter * 32 + lane;
    const int c4 = lane * 4, p0 = sw * 8;
    const int T = c.T, H = c.H, bb = c.bb, h = c.h;

    for (int i = tid1; i < 512; i += CHUNK_THREADS)   // T tile: blocks above the diagonal stay zero
        reinterpret_cast<uint4 *>(sm + SM_T)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int n = 0; n < c.NC; ++n) {
        const int t0 = n * C, L = min(C, T - t0);
        const uint32_t par = (uint32_t)(n & 1);
        // ---------------------------------------------------------------- loads and log-decay prefix
        float al[8][4];   // alpha (1 past the end of the sequence)
        uint2 rq[8], rk[8], rb[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int t = min(p0 + p, L - 1);
            const size_t row = ((size_t)bb * T + t0 + t) * H + h;
            rq[p] = __ldg(reinterpret_cast<const uint2 *>(c.q + row * KD + c4));
            rk[p] = __ldg(reinterpret_cast<const uint2 *>(c.k + row * KD + c4));
            rb[p] = __ldg(reinterpret_cast<const uint2 *>(c.b + row * KD + c4));
        }
        // alpha of this chunk, staged in shared memory by the producer warp
        if (!group_wait(c, mbar(c, MB_AFULL), par, BAR_CHUNK, CHUNK_THREADS)) return;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float4 a4 = *reinterpret_cast<const float4 *>(sm + SM_ALPHA + (p0 + p) * 512 + c4 * 4);
            al[p][0] = a4.x; al[p][1] = a4.y; al[p][2] = a4.z; al[p][3] = a4.w;
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
#pragma unroll
            for (int j = 0; j < 4; ++j)   // past the end: alpha = 1; subnormal alpha: smallest normal
                al[p][j] = p0 + p >= L ? 1.f : fmaxf(al[p][j], 1.17549435e-38f);
            if (p0 + p >= L) rq[p] = rk[p] = rb[p] = make_uint2(0u, 0u);
        }
        // log2 of the product of this thread's 8 alphas per channel: sum of the exponent fields plus
        // log2 of the product of the mantissas (in [1, 256): cannot under- or overflow)
        float lw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int ex = 0;
            float mp = 1.f;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint32_t u = __float_as_uint(al[p][j]);
                ex += (int)(u >> 23) - 127;
                mp *= __uint_as_float((u & 0x7FFFFFu) | 0x3F800000u);
            }
            lw[j] = (float)ex + fast_log2(mp);
        }
        *reinterpret_cast<float4 *>(WT + sw * 128 + c4) = make_float4(lw[0], lw[1], lw[2], lw[3]);
        if (sw == 0)
            *reinterpret_cast<float4 *>(v_g0 + c4) = make_float4(fast_log2(al[0][0]), fast_log2(al[0][1]),
                                                                 fast_log2(al[0][2]), fast_log2(al[0][3]));
        group_sync(BAR_CHUNK, CHUNK_THREADS);
        if (tid1 == 0) mbar_arrive(mbar(c, MB_AEMPTY));   // the alpha buffer may be refilled
        float pre[4] = {0.f, 0.f, 0.f, 0.f}, gC[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w2 = 0; w2 < 8; ++w2) {
            const float4 t4 = *reinterpret_cast<const float4 *>(WT + w2 * 128 + c4);
            const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                gC[j] += tv[j];
                if (w2 < sw) pre[j] += tv[j];
            }
        }
        const float4 g04 = *reinterpret_cast<const float4 *>(v_g0 + c4);
        const float g0[4] = {g04.x, g04.y, g04.z, g04.w};
        int wide = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) wide |= (g0[j] - gC[j] > SPAN_MAX_LOG2);
        const bool slow = group_or(BAR_CHUNK, CHUNK_THREADS, wide != 0);   // WT and v_g0 reads done
        float m2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) m2[j] = slow ? 0.f : 0.5f * (g0[j] + gC[j]);

        // ---------------------------------------------------------------- wait for the state group
        // EQ, K̃, [T; P], Delta and the vector slot of chunk n-2 are free once G3 and G4/G5 of
        // chunk n-1 have completed.
        if (n > 0) {
            if (!group_wait(c, mbar(c, MB_G3), par ^ 1u, BAR_CHUNK, CHUNK_THREADS)) return;
            if (!group_wait(c, mbar(c, MB_G45), par ^ 1u, BAR_CHUNK, CHUNK_THREADS)) return;
        }
        if (sw == 0) {   // per-channel factors of this chunk for the state group
            // sS: scale of the bf16 state operand of G3 (exp(m)); sZ: scale of the TMEM state that
            // G5 accumulates into; sPost: factor that turns the accumulated Z into the next state.
            // Tensor-core chunk: sS = sZ = exp(m), sPost = exp(g_C - m) (G5 uses K̃).
            // Wide-span chunk:   sS = 1, sZ = exp(g_C), sPost = 1 (G5 uses K^ = exp(g_C - g) ⊙ K).
            float *vs = vec + (n & 1) * 384;
            float sS[4], sZ[4], sP[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sS[j] = slow ? 1.f : exp2f(m2[j]);
                sZ[j] = slow ? exp2f(gC[j]) : sS[j];
                sP[j] = slow ? 1.f : exp2f(gC[j] - m2[j]);
            }
            *reinterpret_cast<float4 *>(vs + c4) = make_float4(sS[0], sS[1], sS[2], sS[3]);
            *reinterpret_cast<float4 *>(vs + 128 + c4) = make_float4(sZ[0], sZ[1], sZ[2], sZ[3]);
            *reinterpret_cast<float4 *>(vs + 256 + c4) = make_float4(sP[0], sP[1], sP[2], sP[3]);
            mbar_arrive(mbar(c, MB_VEC));   // 32 arrivals
        }
        // ---------------------------------------------------------------- build
        if (!slow) {
            // exp(g - m) and exp(m - g) at the 8 positions from one exponential at each end of the
            // thread's span and running products of alpha: exp(g_p - m) = exp(g_(p-1) - m) alpha_p
            float f1[4], f2[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f1[j] = fast_exp2(pre[j] - m2[j]);             // before the first position
                f2[j] = fast_exp2(m2[j] - (pre[j] + lw[j]));   // at the last position
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int r = p0 + p;
                const float2 q01 = unpack2(rq[p].x), q23 = unpack2(rq[p].y);
                const float2 k01 = unpack2(rk[p].x), k23 = unpack2(rk[p].y);
                const float2 b01 = unpack2(rb[p].x), b23 = unpack2(rb[p].y);
                const float qq[4] = {q01.x, q01.y, q23.x, q23.y}, kk[4] = {k01.x, k01.y, k23.x, k23.y};
                const float bv[4] = {b01.x, b01.y, b23.x, b23.y};
                float E[4], Qh[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    f1[j] *= al[p][j];
                    E[j] = bv[j] * kk[j] * f1[j];
                    Qh[j] = qq[j] * f1[j];
                }
                *reinterpret_cast<uint2 *>(sm + SM_EQ + sw_off(r, c4, 128)) =
                    make_uint2(pack_bf16(E[0], E[1]), pack_bf16(E[2], E[3]));
                *reinterpret_cast<uint2 *>(sm + SM_EQ + sw_off(64 + r, c4, 128)) =
                    make_uint2(pack_bf16(Qh[0], Qh[1]), pack_bf16(Qh[2], Qh[3]));
            }
#pragma unroll
            for (int p = 7; p >= 0; --p) {
                const int r = p0 + p;
                const float2 k01 = unpack2(rk[p].x), k23 = unpack2(rk[p].y);
                *reinterpret_cast<uint2 *>(sm + SM_KT + sw_off(r, c4, 64)) =
                    make_uint2(pack_bf16(k01.x * f2[0], k01.y * f2[1]), pack_bf16(k23.x * f2[2], k23.y * f2[3]));
#pragma unroll
                for (int j = 0; j < 4; ++j) f2[j] *= al[p][j];
            }
        } else {
            float run[4] = {pre[0], pre[1], pre[2], pre[3]};
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int r = p0 + p;
                const float2 q01 = unpack2(rq[p].x), q23 = unpack2(rq[p].y);
                const float2 k01 = unpack2(rk[p].x), k23 = unpack2(rk[p].y);
                const float2 b01 = unpack2(rb[p].x), b23 = unpack2(rb[p].y);
                const float qq[4] = {q01.x, q01.y, q23.x, q23.y}, kk[4] = {k01.x, k01.y, k23.x, k23.y};
                const float bv[4] = {b01.x, b01.y, b23.x, b23.y};
                float E[4], Qh[4], Kt[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    run[j] += fast_log2(al[p][j]);
                    const float gam = exp2f(run[j]);
                    E[j] = bv[j] * kk[j] * gam;
                    Qh[j] = qq[j] * gam;
                    Kt[j] = kk[j] * exp2f(gC[j] - run[j]);
                }
                *reinterpret_cast<uint2 *>(sm + SM_EQ + sw_off(r, c4, 128)) =
                    make_uint2(pack_bf16(E[0], E[1]), pack_bf16(E[2], E[3]));
                *reinterpret_cast<uint2 *>(sm + SM_EQ + sw_off(64 + r, c4, 128)) =
                    make_uint2(pack_bf16(Qh[0], Qh[1]), pack_bf16(Qh[2], Qh[3]));
                *reinterpret_cast<uint2 *>(sm + SM_KT + sw_off(r, c4, 64)) =
                    make_uint2(pack_bf16(Kt[0], Kt[1]), pack_bf16(Kt[2], Kt[3]));
                *reinterpret_cast<float4 *>(G32 + r * 128 + c4) = make_float4(run[0], run[1], run[2], run[3]);
            }
        }
        fence_async_smem();
        group_sync(BAR_CHUNK, CHUNK_THREADS);

        // ---------------------------------------------------------------- A (fp32 smem) and P (bf16 tile)
        if (tid1 == 0) mbar_arrive(mbar(c, MB_BUILD));   // on a wide-span chunk G1 runs but is not read
        if (!group_wait(c, mbar(c, MB_G1), par, BAR_CHUNK, CHUNK_THREADS)) return;
        if (!slow) {
            uint32_t r32[32];
            tmem_ld32(c.tmem + lrow + TM_D1 + 32 * chalf, r32);
            wait_ld();
            if (quarter < 2) {   // rows 0..63: A, strictly lower
                const int r = crow;
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const int col = 32 * chalf + i;
                    float4 x;
                    x.x = col < r ? __uint_as_float(r32[i]) : 0.f;
                    x.y = col + 1 < r ? __uint_as_float(r32[i + 1]) : 0.f;
                    x.z = col + 2 < r ? __uint_as_float(r32[i + 2]) : 0.f;
                    x.w = col + 3 < r ? __uint_as_float(r32[i + 3]) : 0.f;
                    *reinterpret_cast<float4 *>(AS + r * LDA + col) = x;
                }
            } else {             // rows 64..127: P, lower with diagonal -> bf16 tile
                const int r = crow - 64;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int c0 = 32 * chalf + 8 * u + 2 * i;
                        const float x0 = c0 <= r ? __uint_as_float(r32[8 * u + 2 * i]) : 0.f;
                        const float x1 = c0 + 1 <= r ? __uint_as_float(r32[8 * u + 2 * i + 1]) : 0.f;
                        pk[i] = pack_bf16(x0, x1);
                    }
                    *reinterpret_cast<uint4 *>(sm + SM_P + sw_off(r, 32 * chalf + 8 * u, 64)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        } else {
            // wide-span chunk: A_ri = sum_c e_rc k_ic 2^(g_rc - g_ic) (i < r), P (i <= r) on CUDA cores;
            // raw tokens are re-read from global memory (resident in L2), P goes through TF first.
            for (int r = sw; r < 64; r += 8) {
                const bool rv_ok = r < L;
                float er[4], qr[4], gr[4];
                const size_t rowr = ((size_t)bb * T + t0 + r) * H + h;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int cc = lane + 32 * u;
                    er[u] = rv_ok ? __bfloat162float(c.b[rowr * KD + cc]) * __bfloat162float(c.k[rowr * KD + cc]) : 0.f;
                    qr[u] = rv_ok ? __bfloat162float(c.q[rowr * KD + cc]) : 0.f;
                    gr[u] = G32[r * 128 + cc];
                }
                for (int i = 0; i < 64; ++i) {
                    float a = 0.f, pp = 0.f;
                    if (i <= r && i < L) {
                        const size_t rowi = ((size_t)bb * T + t0 + i) * H + h;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int cc = lane + 32 * u;
                            const float kd = __bfloat162float(c.k[rowi * KD + cc]) * exp2f(gr[u] - G32[i * 128 + cc]);
                            a += er[u] * kd;
                            pp += qr[u] * kd;
                        }
#pragma unroll
                        for (int msk = 16; msk > 0; msk >>= 1) {
                            a += __shfl_xor_sync(0xffffffffu, a, msk);
                            pp += __shfl_xor_sync(0xffffffffu, pp, msk);
                        }
                    }
                    if (lane == 0) {
                        AS[r * LDA + i] = i < r ? a : 0.f;
                        TF[r * LDA + i] = i <= r ? pp : 0.f;
                    }
                }
            }
            group_sync(BAR_CHUNK, CHUNK_THREADS);
            {
                const int r = tid1 >> 2, i0 = 16 * (tid1 & 3);
                uint32_t pk[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(TF[r * LDA + i0 + 2 * i], TF[r * LDA + i0 + 2 * i + 1]);
                *reinterpret_cast<uint4 *>(sm + SM_P + sw_off(r, i0, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4 *>(sm + SM_P + sw_off(r, i0 + 8, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
        group_sync(BAR_CHUNK, CHUNK_THREADS);

        // ---------------------------------------------------------------- T = (I + A)^-1
        // The bf16 tile is written block by block as T is formed; its blocks above the diagonal
        // stay zero (set once, and again after a wide-span chunk reused the space).
        if (slow) {
            for (int i = tid1; i < 512; i += CHUNK_THREADS)
                reinterpret_cast<uint4 *>(sm + SM_T)[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (tid1 < 64) {   // diagonal 16x16 blocks, one column per thread
            const int J = tid1 >> 4, j = tid1 & 15, o16 = 16 * J;
            float col[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == j) ? 1.f : 0.f;
                if (r > j) {
                    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
                    for (int i = 0; i < r; i += 4) {
                        s0 += AS[(o16 + r) * LDA + o16 + i] * col[i];
                        if (i + 1 < r) s1 += AS[(o16 + r) * LDA + o16 + i + 1] * col[i + 1];
                        if (i + 2 < r) s2 += AS[(o16 + r) * LDA + o16 + i + 2] * col[i + 2];
                        if (i + 3 < r) s3 += AS[(o16 + r) * LDA + o16 + i + 3] * col[i + 3];
                    }
                    acc = -((s0 + s1) + (s2 + s3));
                }
                col[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                TF[(o16 + r) * LDA + o16 + j] = col[r];
                *reinterpret_cast<__nv_bfloat16 *>(sm + SM_T + sw_off(o16 + r, o16 + j, 64)) = __float2bfloat16_rn(col[r]);
            }
        }
        group_sync(BAR_CHUNK, CHUNK_THREADS);
        if (sw < 2) {   // blocks (1,0) and (3,2): T_RI = -T_RR (A_RI T_II), within one warp
            const int R = 16 * (2 * sw + 1), I = 16 * (2 * sw);
            float *X = WT + sw * 384;   // 16 x 16 (row stride 24), private to this warp
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_mm(d, AS, LDA, R, I, TF, LDA, I, I + 8 * nt, 0, 2, lane);
                tile_store(X, 24, 0, 8 * nt, d, 1.f, lane);
            }
            __syncwarp();
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_mm(d, TF, LDA, R, R, X, 24, 0, 8 * nt, 0, 2, lane);
                tile_store(TF, LDA, R, I + 8 * nt, d, -1.f, lane);
                tile_store_bf16(sm + SM_T, R, I + 8 * nt, d, -1.f, lane);
            }
        }
        group_sync(BAR_CHUNK, CHUNK_THREADS);
        if (sw < 4) {   // rows 32..63 x cols 8sw..8sw+7: T = -T_hi (A_hi,lo T_lo), within one warp
            const int nt = sw;
            float *X = WT + sw * 256;   // 32 x 8, private to this warp
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {   // block (0,1) of T is zero: skipped for columns >= 16
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_mm(d, AS, LDA, 32 + 16 * mt, 0, TF, LDA, 0, 8 * nt, nt >= 2 ? 2 : 0, 4, lane);
                tile_store(X, 8, 16 * mt, 0, d, 1.f, lane);
            }
            __syncwarp();
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {   // block (2,3) of T is zero: skipped for rows < 48
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_mm(d, TF, LDA, 32 + 16 * mt, 32, X, 8, 0, 0, 0, mt == 0 ? 2 : 4, lane);
                tile_store_bf16(sm + SM_T, 32 + 16 * mt, 8 * nt, d, -1.f, lane);
            }
        }
        fence_async_smem();
        group_sync(BAR_CHUNK, CHUNK_THREADS);
        if (tid1 == 0) mbar_arrive(mbar(c, MB_SOLVE));

        // ---------------------------------------------------------------- -W' over Ê; zero the O rows of D3
        if (!group_wait(c, mbar(c, MB_G2), par, BAR_CHUNK, CHUNK_THREADS)) return;
        if (quarter < 2) {
            const int r = crow;
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
                uint32_t r32[32];
                tmem_ld32(c.tmem + lrow + TM_D2 + 64 * chalf + 32 * u2, r32);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int cc = 64 * chalf + 32 * u2 + 8 * u;
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        pk[i] = pack_bf16(-__uint_as_float(r32[8 * u + 2 * i]), -__uint_as_float(r32[8 * u + 2 * i + 1]));
                    *reinterpret_cast<uint4 *>(sm + SM_EQ + sw_off(r, cc, 128)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        } else {
            uint32_t z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0u;
            const uint32_t d3 = TM_D3 + 128 * (n & 1);
            tmem_st32(c.tmem + lrow + d3 + 64 * chalf, z);
            tmem_st32(c.tmem + lrow + d3 + 64 * chalf + 32, z);
            wait_st();
        }
        fence_async_smem();
        fence_before();
        group_sync(BAR_CHUNK, CHUNK_THREADS);
        if (tid1 == 0) mbar_arrive(mbar(c, MB_S1DONE));
    }
}

// ============================================================================ state group
__device__ void state_group(const Ctx &c, int tid, float *ST, size_t chain) {
    unsigned char *sm = c.sm;
    const float *vec = reinterpret_cast<const float *>(sm + SM_VEC);
    const int warp = tid >> 5;
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const int crow = tid;   // TMEM lane = row c of Z (and row r of D3)
    const int T = c.T, H = c.H;
    float egm_prev = 1.f;

    for (int n = 0; n < c.NC; ++n) {
        const uint32_t par = (uint32_t)(n & 1);
        const int t0 = n * C, L = min(C, T - t0);
        // ---------------------------------------------------------------- S_n = sPost_n-1 Z; Z <- sZ_n S_n; bf16(sS_n S_n)
        if (!group_wait(c, mbar(c, MB_VEC), par, BAR_STATE, STATE_THREADS)) return;
        if (n > 0 && !group_wait(c, mbar(c, MB_G45), par ^ 1u, BAR_STATE, STATE_THREADS)) return;
        const float *vs = vec + (n & 1) * 384;
        const float ssc = vs[crow] * egm_prev;         // scale of the bf16 operand
        const float zsc = vs[128 + crow] * egm_prev;   // scale of the TMEM state
        egm_prev = vs[256 + crow];
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
            uint32_t r32[32];
            tmem_ld32(c.tmem + lrow + TM_Z + 32 * u2, r32);
            wait_ld();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int vv = 32 * u2 + 8 * u;
                const float *x = reinterpret_cast<const float *>(r32) + 8 * u;
                uint4 pk;
                pk.x = pack_bf16(ssc * x[0], ssc * x[1]);
                pk.y = pack_bf16(ssc * x[2], ssc * x[3]);
                pk.z = pack_bf16(ssc * x[4], ssc * x[5]);
                pk.w = pack_bf16(ssc * x[6], ssc * x[7]);
                *reinterpret_cast<uint4 *>(sm + SM_S + sw_off(crow, vv, 128)) = pk;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(zsc * __uint_as_float(r32[i]));
            tmem_st32(c.tmem + lrow + TM_Z + 32 * u2, r32);
        }
        wait_st();
        fence_async_smem();
        fence_before();
        group_sync(BAR_STATE, STATE_THREADS);
        if (tid == 0) mbar_arrive(mbar(c, MB_STILDE));

        // ---------------------------------------------------------------- Delta rows -> bf16 tile
        if (!group_wait(c, mbar(c, MB_G3), par, BAR_STATE, STATE_THREADS)) return;
        const uint32_t d3 = TM_D3 + 128 * (n & 1);
        if (warp < 2) {
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(c.tmem + lrow + d3 + 32 * u2, r32);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int vv = 32 * u2 + 8 * u;
                    uint4 pk;
                    pk.x = pack_bf16(__uint_as_float(r32[8 * u]), __uint_as_float(r32[8 * u + 1]));
                    pk.y = pack_bf16(__uint_as_float(r32[8 * u + 2]), __uint_as_float(r32[8 * u + 3]));
                    pk.z = pack_bf16(__uint_as_float(r32[8 * u + 4]), __uint_as_float(r32[8 * u + 5]));
                    pk.w = pack_bf16(__uint_as_float(r32[8 * u + 6]), __uint_as_float(r32[8 * u + 7]));
                    *reinterpret_cast<uint4 *>(sm + SM_DL + sw_off(crow, vv, 64)) = pk;
                }
            }
        }
        fence_async_smem();
        fence_before();
        group_sync(BAR_STATE, STATE_THREADS);
        if (tid == 0) mbar_arrive(mbar(c, MB_DELTA));

        // ---------------------------------------------------------------- o rows (16-byte stores)
        if (!group_wait(c, mbar(c, MB_G45), par, BAR_STATE, STATE_THREADS)) return;
        if (warp >= 2) {
            const int r = crow - 64;
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(c.tmem + lrow + d3 + 32 * u2, r32);
                wait_ld();
                if (r < L) {
                    __nv_bfloat16 *dst = c.o + (((size_t)c.bb * T + t0 + r) * H + c.h) * VD + 32 * u2;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 pk;
                        pk.x = pack_bf16(__uint_as_float(r32[8 * u]), __uint_as_float(r32[8 * u + 1]));
                        pk.y = pack_bf16(__uint_as_float(r32[8 * u + 2]), __uint_as_float(r32[8 * u + 3]));
                        pk.z = pack_bf16(__uint_as_float(r32[8 * u + 4]), __uint_as_float(r32[8 * u + 5]));
                        pk.w = pack_bf16(__uint_as_float(r32[8 * u + 6]), __uint_as_float(r32[8 * u + 7]));
                        *reinterpret_cast<uint4 *>(dst + 8 * u) = pk;
                    }
                }
            }
        }
        fence_before();
        group_sync(BAR_STATE, STATE_THREADS);
        if (tid == 0) mbar_arrive(mbar(c, (n & 1) ? MB_D3FREE1 : MB_D3FREE0));
    }
    // S_T = Diag(sPost) Z of the last chunk
    float *dst = ST + (chain * KD + crow) * VD;
#pragma unroll
    for (int u2 = 0; u2 < 4; ++u2) {
        uint32_t r32[32];
        tmem_ld32(c.tmem + lrow + TM_Z + 32 * u2, r32);
        wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(dst + 32 * u2 + i) =
                make_float4(egm_prev * __uint_as_float(r32[i]), egm_prev * __uint_as_float(r32[i + 1]),
                            egm_prev * __uint_as_float(r32[i + 2]), egm_prev * __uint_as_float(r32[i + 3]));
    }
}

// ============================================================================ producer
// Stages alpha of chunk n into shared memory (bulk copies completing on MB_AFULL) once the
// chunk group has consumed chunk n-1's.
__device__ void producer(const Ctx &c, int lane) {
    const uint32_t dst = smem_u32(c.sm + SM_ALPHA);
    const int T = c.T, H = c.H, bb = c.bb, h = c.h;
    for (int n = 0; n < c.NC; ++n) {
        const int t0 = n * C, L = min(C, T - t0);
        if (n > 0) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(mbar(c, MB_AEMPTY), (uint32_t)((n - 1) & 1), WAIT_LIMIT) && !*abort_flag(c);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) *abort_flag(c) = 1u;
                return;
            }
        }
        if (lane == 0) mbar_arrive_expect_tx(mbar(c, MB_AFULL), (uint32_t)L * 512u);
        __syncwarp();
        for (int r = lane; r < L; r += 32)   // one 512-byte row per copy, spread over the warp
            bulk_g2s(dst + (uint32_t)r * 512u, c.alpha + (((size_t)bb * T + t0 + r) * H + h) * KD, 512u,
                     mbar(c, MB_AFULL));
    }
}

// ============================================================================ value group
// U = w ⊙ v of chunk n, written once G2 of chunk n-1 (its last reader) has completed;
// signals MB_U (64 arrivals).  Warps 14-15: lane l holds channels 4l..4l+3, warp half
// picks positions; rows past the end of the sequence are zero.
__device__ void value_group(const Ctx &c, int tid2) {
    const int vw = tid2 >> 5, lane = tid2 & 31, c4 = lane * 4;
    const int T = c.T, H = c.H, bb = c.bb, h = c.h;
    for (int n = 0; n < c.NC; ++n) {
        const int t0 = n * C, L = min(C, T - t0);
        if (n > 0) {
            bool ok = mbar_wait(mbar(c, MB_G2), (uint32_t)((n - 1) & 1), WAIT_LIMIT) && !*abort_flag(c);
            if (!__all_sync(0xffffffffu, ok)) {
                *abort_flag(c) = 1u;
                return;
            }
            fence_after();
        }
#pragma unroll 1
        for (int p0 = 32 * vw; p0 < 32 * vw + 32; p0 += 8) {
            uint2 rv[8], rw[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int t = min(p0 + p, L - 1);
                const size_t row = ((size_t)bb * T + t0 + t) * H + h;
                rv[p] = __ldg(reinterpret_cast<const uint2 *>(c.v + row * VD + c4));
                rw[p] = __ldg(reinterpret_cast<const uint2 *>(c.w + row * VD + c4));
            }
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float2 v01 = unpack2(rv[p].x), v23 = unpack2(rv[p].y);
                const float2 w01 = unpack2(rw[p].x), w23 = unpack2(rw[p].y);
                const bool ok = p0 + p < L;
                *reinterpret_cast<uint2 *>(c.sm + SM_U + sw_off(p0 + p, c4, 64)) =
                    ok ? make_uint2(pack_bf16(w01.x * v01.x, w01.y * v01.y), pack_bf16(w23.x * v23.x, w23.y * v23.y))
                       : make_uint2(0u, 0u);
            }
        }
        fence_async_smem();
        mbar_arrive(mbar(c, MB_U));
    }
}

// ============================================================================ MMA issuer
__device__ void mma_issuer(const Ctx &c) {
    const uint32_t aS = smem_u32(c.sm + SM_S), aEQ = smem_u32(c.sm + SM_EQ), aKT = smem_u32(c.sm + SM_KT),
                   aU = smem_u32(c.sm + SM_U), aDL = smem_u32(c.sm + SM_DL), aTP = smem_u32(c.sm + SM_T);
    const uint32_t tm = c.tmem;
    int i1 = 0, i2 = 0, i3 = 0, i45 = 0;
    uint32_t idle = 0;
    while (i45 < c.NC) {
        bool did = false;
        if (i1 < c.NC && mbar_test(mbar(c, MB_BUILD), (uint32_t)(i1 & 1))) {
            fence_after();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ss(tm + TM_D1, desc_kmajor(aEQ, 128, j), desc_kmajor(aKT, 64, j), ID_G1, j > 0);
            mma_commit(mbar(c, MB_G1));
            ++i1;
            did = true;
        }
        if (i2 < i1 && mbar_test(mbar(c, MB_SOLVE), (uint32_t)(i2 & 1)) && mbar_test(mbar(c, MB_U), (uint32_t)(i2 & 1)) &&
            (i2 < 2 || mbar_test(mbar(c, (i2 & 1) ? MB_D3FREE1 : MB_D3FREE0), (uint32_t)(((i2 - 2) >> 1) & 1)))) {
            fence_after();
            const uint32_t d3 = TM_D3 + 128 * (i2 & 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tm + TM_D2, desc_kmajor(aTP, 128, j), desc_mnmajor(aEQ, 128, j), ID_G2, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tm + d3, desc_kmajor(aTP, 128, j), desc_mnmajor(aU, 64, j), ID_G2, j > 0);
            mma_commit(mbar(c, MB_G2));
            ++i2;
            did = true;
        }
        if (i3 < i2 && mbar_test(mbar(c, MB_S1DONE), (uint32_t)(i3 & 1)) &&
            mbar_test(mbar(c, MB_STILDE), (uint32_t)(i3 & 1))) {
            fence_after();
            const uint32_t d3 = TM_D3 + 128 * (i3 & 1);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ss(tm + d3, desc_kmajor(aEQ, 128, j), desc_mnmajor(aS, 128, j), ID_G3, 1);
            mma_commit(mbar(c, MB_G3));
            ++i3;
            did = true;
        }
        if (i45 < i3 && mbar_test(mbar(c, MB_DELTA), (uint32_t)(i45 & 1))) {
            fence_after();
            const uint32_t d3 = TM_D3 + 128 * (i45 & 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tm + d3, desc_kmajor(aTP, 128, j), desc_mnmajor(aDL, 64, j), ID_G4, 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tm + TM_Z, desc_mnmajor(aKT, 64, j), desc_mnmajor(aDL, 64, j), ID_G5, 1);
            mma_commit(mbar(c, MB_G45));
            ++i45;
            did = true;
        }
        if (did) {
            idle = 0;
        } else if (++idle > POLL_LIMIT || *abort_flag(c)) {
            *abort_flag(c) = 1u;
            return;
        }
    }
}

__global__ void __launch_bounds__(NT)
    chunk_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const float *__restrict__ alpha,
                    const __nv_bfloat16 *__restrict__ b, const __nv_bfloat16 *__restrict__ w,
                    const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ ST, int H,
                    int T, unsigned int *__restrict__ status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int chain = blockIdx.x;
    Ctx c;
    c.sm = sm;
    c.misc = smem_u32(sm + SM_MISC);
    c.q = q; c.k = k; c.v = v; c.b = b; c.w = w; c.alpha = alpha; c.o = o;
    c.T = T; c.H = H; c.bb = chain / H; c.h = chain % H; c.NC = (T + C - 1) / C;

    if (warp == 12) tmem_alloc(c.misc + MISC_TSLOT, TM_COLS);
    if (tid == 0) {
        for (uint32_t i = 0; i < MB_COUNT; ++i)
            mbar_init(c.misc + 8 * i, i * 8 == MB_VEC ? 32u : i * 8 == MB_U ? 64u : 1u);
        *reinterpret_cast<volatile uint32_t *>(sm + SM_MISC + MISC_ABORT) = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    c.tmem = *reinterpret_cast<volatile uint32_t *>(sm + SM_MISC + MISC_TSLOT);

    if (warp < 4) {   // Z <- S0 (the first rescale multiplies by exp(m) of chunk 0)
        regs_dec<56>();
        const int crow = tid;
        const uint32_t lrow = (uint32_t)(warp * 32) << 16;
        const float *src = S0 ? S0 + ((size_t)chain * KD + crow) * VD : nullptr;
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
            uint32_t r32[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 x = src ? *reinterpret_cast<const float4 *>(src + 32 * u2 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                r32[i] = __float_as_uint(x.x); r32[i + 1] = __float_as_uint(x.y);
                r32[i + 2] = __float_as_uint(x.z); r32[i + 3] = __float_as_uint(x.w);
            }
            tmem_st32(c.tmem + lrow + TM_Z + 32 * u2, r32);
        }
        wait_st();
        fence_before();
        group_sync(BAR_STATE, STATE_THREADS);
        fence_after();
        state_group(c, tid, ST, (size_t)chain);
    } else if (warp < 12) {
        regs_inc<200>();
        chunk_group(c, tid - 128);
    } else {
        regs_dec<56>();
        if (warp == 12 && (tid & 31) == 0) mma_issuer(c);
        if (warp == 13) producer(c, tid & 31);
        if (warp >= 14) value_group(c, tid - 448);
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0 && *reinterpret_cast<volatile uint32_t *>(sm + SM_MISC + MISC_ABORT)) atomicOr(status, 1u);
    if (warp == 12) tmem_dealloc(c.tmem, TM_COLS);
}

}  // namespace tcfwd

bool tc_supported(int B, int H, int T, int K, int V, int C, int bf16) {
    (void)B; (void)H; (void)T;
    return bf16 && K == 128 && V == 128 && C == 64;
}

size_t tc_workspace_bytes(int, int, int, int, int, int) { return kStatusBytes; }

int launch_chunk_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                    const float *S0, void *o, float *ST, int B, int H, int T, int K, int V, int C, void *ws,
                    cudaStream_t st) {
    if (!tc_supported(B, H, T, K, V, C, 1)) return -4;
    const int smem = (int)tcfwd::SM_BYTES;
    if (cudaFuncSetAttribute(tcfwd::chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return -6;
    tcfwd::chunk_tc_kernel<<<B * H, tcfwd::NT, smem, st>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, alpha,
        (const __nv_bfloat16 *)b, (const __nv_bfloat16 *)w, S0, (__nv_bfloat16 *)o, ST, H, T,
        reinterpret_cast<unsigned int *>(ws));
    return launch_status();
}

}  // namespace gdn2
