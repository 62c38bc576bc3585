// Two-stage chunkwise prefill on the tensor cores (tcgen05 + TMEM + TMA), sm_100a.
// bf16 tokens, d_k = d_v = 128, chunk C = 64.
//
// The update equation of page "NVIDIA представила Gated DeltaNet-2 ..." (section "Техническая
// схема") is evaluated in the chunkwise WY form with C = 64 that the same page names.  Everything
// in that form that depends only on a chunk's own tokens -- the log-decay prefix, the decay
// absorbed into the rank-1 factors, the Gram matrices, the triangular solve and the WY factors --
// is independent from chunk to chunk; only the state update is a chain.  So:
//
//   stage 1, prep_kernel: fully parallel over every (batch, chunk, head), two CTAs per SM.  The
//     token tiles arrive by TMA tensor copies straight into the swizzled operand layout; per
//     chunk (g = per-channel log-decay prefix, m = its midpoint, e = b ⊙ k, u = w ⊙ v):
//       build  Ê = e ⊙ exp(g - m), Q̂ = q ⊙ exp(g - m), K̃ = k ⊙ exp(m - g), U = u   (in place)
//       G1     [A; P] = [Ê; Q̂] K̃^T                        (tcgen05, TMEM)
//       solve  T = (I + A)^-1                               (fp32 + mma.sync tf32)
//       G2     W' = T Ê,  Ũ = T U                           (tcgen05, TMEM)
//     and stores one record per chunk: the operand images [-W'; Q̂], K̃, Ũ, P (bf16, already in
//     the swizzled layout the second stage's tensor-core reads use) and the per-channel frame
//     factors, by bulk copies.
//   stage 2, walk_kernel: one CTA per (batch, head) chain walks its chunks with the state
//     resident in TMEM as Z = Diag(exp(m)) S; each record arrives by one bulk copy into a
//     double-buffered slot:
//       G3     [-W'Z̃; Q̂Z̃] = [-W'; Q̂] Z̃                      (Z̃ = bf16 copy of the framed state)
//       Delta  = Ũ - W'Z̃
//       G4/G5  O = Q̂Z̃ + P Delta,   Z += K̃^T Delta
//       next   S' = Diag(exp(g_C - m)) Z,  Z' = Diag(exp(m')) S'
//     and writes o by TMA tensor stores.
// A chunk whose log-decay span exceeds 120 nats in some channel forms A and P on CUDA cores from
// exp(g_r - g_i) <= 1 per element and uses unscaled factors (m = 0), exactly as the fused kernel;
// the second stage only sees the factors stored with the record.
//
// Long sequences are processed in windows of chunks so the record buffer stays bounded; the state
// passes from one window to the next through S_T.  Every wait is bounded; on expiry a kernel sets
// the workspace status word and stops.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "gdn2_common.cuh"
#include "gdn2_internal.h"
#include "tc_chunk.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace split {

using namespace gdn2::tc;
using namespace gdn2::tcc;

constexpr int C = 64, KD = 128, VD = 128;
constexpr float SPAN_MAX_LOG2 = 173.123f;   // 120 nats in log2 units
constexpr uint32_t WAIT_LIMIT = 1u << 22;
constexpr uint32_t STATUS_PREP = 2u, STATUS_WALK = 4u;

// ---------------------------------------------------------------------------- record (bytes)
constexpr uint32_t R_A3 = 0;        // [-W'; Q̂]: 128 x 128 K-major (A of G3)
constexpr uint32_t R_KT = 32768;    // K̃ [i x c]: 64 x 128 (MN-major A of G5)
constexpr uint32_t R_U = 49152;     // Ũ [i x v]: 64 x 128
constexpr uint32_t R_P = 65536;     // P [r x i]: 64 x 64, lower with the diagonal
constexpr uint32_t R_VEC = 73728;   // sS, sZ, sPost: 3 x 128 fp32
constexpr uint32_t R_COPY = R_VEC + 3 * 128 * 4;   // bytes moved per record
constexpr uint32_t R_BYTES = 75776;                // record stride (1024-aligned)

// ---------------------------------------------------------------------------- stage 1
constexpr int P1_NT = 256;
constexpr uint32_t P1_EQ = 0;                        // b -> Ê -> -W' (rows 0-63), q -> Q̂ (rows 64-127)
constexpr uint32_t P1_KT = 32768;                    // k -> K̃
constexpr uint32_t P1_U = 49152;                     // v -> U -> Ũ
constexpr uint32_t P1_W = 65536;                     // w; then [T; P] (128 rows, K = 64)
constexpr uint32_t P1_AS = 81920;                    // fp32 A / T^T [64][LDA]; first the prefix totals
constexpr uint32_t P1_X = P1_AS + 64 * LDA * 4;      // solve scratch (4 KB)
constexpr uint32_t P1_MISC = P1_X + 4096;
constexpr uint32_t P1_BYTES = P1_MISC + 256 + 1024;  // + alignment slack
enum : uint32_t { M1_LOAD = 0, M1_G1 = 8, M1_G2 = 16, M1_TSLOT = 32, M1_ABORT = 36 };
constexpr uint32_t P1_TM_D1 = 0, P1_TM_D2 = 0, P1_TM_D3 = 128, P1_TM_COLS = 256;

constexpr uint32_t ID_G1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G2 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G3 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G4 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G5 = idesc_bf16(128, 128, 1, 1);

struct TokMaps {   // [B, T, H, 128] bf16 token tensors as 4-D maps (d, H, T, B), box 64 x 1 x 64 x 1
    CUtensorMap q, k, b, v, w;
};

// Block-wide bounded wait: every thread gets the same verdict.
__device__ __forceinline__ bool block_wait(uint32_t mb, uint32_t parity, volatile uint32_t *abort) {
    bool ok = mbar_wait(mb, parity, WAIT_LIMIT) && !*abort;
    const bool fail = __syncthreads_or(!ok) != 0;
    if (fail) *abort = 1u;
    return !fail;
}

// Wide-span chunk: A_ri = sum_c e_rc k_ic exp2(g_rc - g_ic) (i < r) and P_ri likewise with q
// (i <= r), one row per thread (threads 0-63 rows of A, 64-127 rows of P: the TMEM lanes G1 would
// have written).  The exponent is summed from log2 alpha while i walks down from r, so it never
// leaves [-inf, 0]; rows are read again from global memory.
__device__ __forceinline__ void wide_span_ap(uint32_t tmem_d1, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                             const __nv_bfloat16 *b, const float *alpha, size_t row0, size_t stride,
                                             int tid, int L) {
    const int r = tid & 63;
    const bool isP = tid >= 64;
    const uint32_t lane_base = tmem_d1 + ((uint32_t)((tid >> 5) * 32) << 16);
    const int rc = min(r, L - 1);
    const size_t rowr = row0 + (size_t)rc * stride;
    auto row = [&](int t) { return row0 + (size_t)t * stride; };
    auto log2a = [&](int t, int cc) { return fast_log2(fmaxf(alpha[row(t) * KD + cc], 1.17549435e-38f)); };
#pragma unroll 1
    for (int i0 = 0; i0 < 64; i0 += 16) {
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.f;
        if (r < L && i0 <= r) {
#pragma unroll 1
            for (int cc = 0; cc < KD; ++cc) {
                const float x = isP ? __bfloat162float(q[rowr * KD + cc])
                                    : __bfloat162float(b[rowr * KD + cc]) * __bfloat162float(k[rowr * KD + cc]);
                const int itop = min(i0 + 15, r);
                float d = 0.f;
#pragma unroll 1
                for (int jj = r; jj > itop; --jj) d += log2a(jj, cc);
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    if (i0 + i <= itop) {
                        acc[i] += x * __bfloat162float(k[row(i0 + i) * KD + cc]) * exp2f(d);
                        d += log2a(i0 + i, cc);
                    }
                }
            }
        }
        uint32_t r16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int col = i0 + i;
            const bool keep = r < L && (isP ? col <= r : col < r);
            r16[i] = __float_as_uint(keep ? acc[i] : 0.f);
        }
        tmem_st16(lane_base + i0, r16);
    }
    wait_st();
}

__global__ void __launch_bounds__(P1_NT, 2)
    prep_kernel(const __grid_constant__ TokMaps maps, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                const __nv_bfloat16 *b, const float *__restrict__ alpha, unsigned char *records, int H, int T,
                int NC, int n0, int nw, int nch, unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t misc = smem_u32(sm + P1_MISC);
    volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sm + P1_MISC + M1_ABORT);
    const uint32_t aEQ = smem_u32(sm + P1_EQ), aKT = smem_u32(sm + P1_KT), aU = smem_u32(sm + P1_U),
                   aW = smem_u32(sm + P1_W);
    float *AS = reinterpret_cast<float *>(sm + P1_AS);
    float *WT = AS;              // [8][128] per-warp log2 totals, then g_0 [128]
    float *v_g0 = WT + 8 * 128;

    if (warp == 0) tmem_alloc(misc + M1_TSLOT, P1_TM_COLS);
    if (tid == 0) {
        mbar_init(misc + M1_LOAD, 1);
        mbar_init(misc + M1_G1, 1);
        mbar_init(misc + M1_G2, 1);
        *abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.b);
        prefetch_tmap(&maps.v); prefetch_tmap(&maps.w);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + P1_MISC + M1_TSLOT);

    const int c4 = lane * 4, p0 = warp * 8;   // build mapping: 8 positions x 4 channels per thread
    int it = 0;
    for (int ch = blockIdx.x; ch < nch; ch += gridDim.x, ++it) {
        // chunk-heads of the window in (batch, chunk, head) order: neighbouring CTAs read adjacent heads
        const int h = ch % H, nl = (ch / H) % nw, bb = ch / (H * nw), n = n0 + nl;
        const int t0 = n * C, L = min(C, T - t0);
        unsigned char *rec = records + (size_t)ch * R_BYTES;
        const uint32_t par = (uint32_t)(it & 1);

        // ------------------------------------------------------------------ token tiles by TMA
        if (tid == 0) {
            bulk_wait_read_all();   // the previous chunk-head's record stores have read their sources
            mbar_arrive_expect_tx(misc + M1_LOAD, 10u * 8192u);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tma_load_4d(aEQ + hf * 16384, &maps.b, 64 * hf, h, t0, bb, misc + M1_LOAD);
                tma_load_4d(aEQ + hf * 16384 + 8192, &maps.q, 64 * hf, h, t0, bb, misc + M1_LOAD);
                tma_load_4d(aKT + hf * 8192, &maps.k, 64 * hf, h, t0, bb, misc + M1_LOAD);
                tma_load_4d(aU + hf * 8192, &maps.v, 64 * hf, h, t0, bb, misc + M1_LOAD);
                tma_load_4d(aW + hf * 8192, &maps.w, 64 * hf, h, t0, bb, misc + M1_LOAD);
            }
        }
        // ------------------------------------------------------------------ alpha and the log-decay prefix
        const size_t row0 = ((size_t)bb * T + t0) * H + h;
        float al[8][4];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(alpha + (row0 + (size_t)min(p0 + p, L - 1) * H) * KD + c4));
            al[p][0] = a4.x; al[p][1] = a4.y; al[p][2] = a4.z; al[p][3] = a4.w;
        }
#pragma unroll
        for (int p = 0; p < 8; ++p)
#pragma unroll
            for (int j = 0; j < 4; ++j)   // past the end: alpha = 1; subnormal alpha: smallest normal
                al[p][j] = p0 + p >= L ? 1.f : fmaxf(al[p][j], 1.17549435e-38f);
        // log2 of the product of the thread's 8 alphas per channel: the exponent fields plus log2 of
        // the product of the mantissas (in [1, 256))
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
        *reinterpret_cast<float4 *>(WT + warp * 128 + c4) = make_float4(lw[0], lw[1], lw[2], lw[3]);
        if (warp == 0)
            *reinterpret_cast<float4 *>(v_g0 + c4) =
                make_float4(fast_log2(al[0][0]), fast_log2(al[0][1]), fast_log2(al[0][2]), fast_log2(al[0][3]));
        __syncthreads();
        float pre[4] = {0.f, 0.f, 0.f, 0.f}, gC[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w2 = 0; w2 < 8; ++w2) {
            const float4 t4 = *reinterpret_cast<const float4 *>(WT + w2 * 128 + c4);
            const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                gC[j] += tv[j];
                if (w2 < warp) pre[j] += tv[j];
            }
        }
        const float4 g04 = *reinterpret_cast<const float4 *>(v_g0 + c4);
        const float g0[4] = {g04.x, g04.y, g04.z, g04.w};
        int wide_l = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) wide_l |= (g0[j] - gC[j] > SPAN_MAX_LOG2);
        const bool wide = __syncthreads_or(wide_l) != 0;   // also: WT and v_g0 reads done
        float m2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) m2[j] = wide ? 0.f : 0.5f * (g0[j] + gC[j]);
        if (warp == 0) {
            // sS: scale of the bf16 state operand (exp(m)); sZ: scale of the TMEM state that G5
            // accumulates into; sPost: the factor that turns the accumulated Z into the next state.
            // Tensor-core chunk: sS = sZ = exp(m), sPost = exp(g_C - m).  Wide-span chunk: sS = 1,
            // sZ = exp(g_C), sPost = 1 (K̃ is then exp(g_C - g) ⊙ k).
            float sS[4], sZ[4], sP[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sS[j] = wide ? 1.f : fast_exp2(m2[j]);
                sZ[j] = wide ? fast_exp2(gC[j]) : sS[j];
                sP[j] = wide ? 1.f : fast_exp2(gC[j] - m2[j]);
            }
            float *vec = reinterpret_cast<float *>(rec + R_VEC);
            *reinterpret_cast<float4 *>(vec + c4) = make_float4(sS[0], sS[1], sS[2], sS[3]);
            *reinterpret_cast<float4 *>(vec + 128 + c4) = make_float4(sZ[0], sZ[1], sZ[2], sZ[3]);
            *reinterpret_cast<float4 *>(vec + 256 + c4) = make_float4(sP[0], sP[1], sP[2], sP[3]);
        }

        // ------------------------------------------------------------------ build (in place)
        if (!block_wait(misc + M1_LOAD, par, abort)) break;
        {
            uint2 rq[8], rk[8], rb[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int r = p0 + p;
                rb[p] = *reinterpret_cast<const uint2 *>(sm + P1_EQ + sw_off(r, c4, 128));
                rq[p] = *reinterpret_cast<const uint2 *>(sm + P1_EQ + sw_off(64 + r, c4, 128));
                rk[p] = *reinterpret_cast<const uint2 *>(sm + P1_KT + sw_off(r, c4, 64));
                const uint2 rv = *reinterpret_cast<const uint2 *>(sm + P1_U + sw_off(r, c4, 64));
                const uint2 rw = *reinterpret_cast<const uint2 *>(sm + P1_W + sw_off(r, c4, 64));
                *reinterpret_cast<uint2 *>(sm + P1_U + sw_off(r, c4, 64)) = make_uint2(bmul2(rw.x, rv.x), bmul2(rw.y, rv.y));
            }
            if (!wide) {
                // exp(g - m) from one exponential at the thread's first position and running
                // products of alpha after it; exp(m - g) backwards from one exponential at its last
                // position.  Both start inside the chunk, where every factor lies within
                // exp(+-span/2): a start before the first position (exp(-m) itself) can leave fp32's
                // range when the chunk's first alpha is tiny.  Packed bf16 arithmetic: each factor
                // and each product is rounded to bf16 once.
                float f1[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) f1[j] = fast_exp2(pre[j] + fast_log2(al[0][j]) - m2[j]);
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int r = p0 + p;
                    if (p > 0)
#pragma unroll
                        for (int j = 0; j < 4; ++j) f1[j] *= al[p][j];
                    const uint32_t F01 = pack_bf16(f1[0], f1[1]), F23 = pack_bf16(f1[2], f1[3]);
                    *reinterpret_cast<uint2 *>(sm + P1_EQ + sw_off(r, c4, 128)) =
                        make_uint2(bmul2(bmul2(rb[p].x, rk[p].x), F01), bmul2(bmul2(rb[p].y, rk[p].y), F23));
                    *reinterpret_cast<uint2 *>(sm + P1_EQ + sw_off(64 + r, c4, 128)) =
                        make_uint2(bmul2(rq[p].x, F01), bmul2(rq[p].y, F23));
                }
                float f2[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) f2[j] = fast_exp2(m2[j] - (pre[j] + lw[j]));
#pragma unroll
                for (int p = 7; p >= 0; --p) {
                    const int r = p0 + p;
                    *reinterpret_cast<uint2 *>(sm + P1_KT + sw_off(r, c4, 64)) =
                        make_uint2(bmul2(rk[p].x, pack_bf16(f2[0], f2[1])), bmul2(rk[p].y, pack_bf16(f2[2], f2[3])));
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
                    *reinterpret_cast<uint2 *>(sm + P1_EQ + sw_off(r, c4, 128)) =
                        make_uint2(pack_bf16(E[0], E[1]), pack_bf16(E[2], E[3]));
                    *reinterpret_cast<uint2 *>(sm + P1_EQ + sw_off(64 + r, c4, 128)) =
                        make_uint2(pack_bf16(Qh[0], Qh[1]), pack_bf16(Qh[2], Qh[3]));
                    *reinterpret_cast<uint2 *>(sm + P1_KT + sw_off(r, c4, 64)) =
                        make_uint2(pack_bf16(Kt[0], Kt[1]), pack_bf16(Kt[2], Kt[3]));
                }
                if (tid < 128) wide_span_ap(tmem + P1_TM_D1, q, k, b, alpha, row0, (size_t)H, tid, L);
            }
        }
        fence_async_smem();
        fence_before();
        __syncthreads();
        if (tid == 0) {
            fence_after();
            if (!wide) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    mma_ss(tmem + P1_TM_D1, desc_kmajor(aEQ, 128, j), desc_kmajor(aKT, 64, j), ID_G1, j > 0);
                mma_commit(misc + M1_G1);
            } else {
                mbar_arrive(misc + M1_G1);   // A and P were written into D1 directly
            }
            bulk_s2g(rec + R_KT, aKT, 16384);   // K̃ is final
        }
        // the T tile's blocks above the diagonal are zero (w, which shared the tile, is consumed)
        for (int i = tid; i < 512; i += P1_NT) reinterpret_cast<uint4 *>(sm + P1_W)[i] = make_uint4(0u, 0u, 0u, 0u);

        // ------------------------------------------------------------------ A (fp32) and P (bf16) out of TMEM
        if (!block_wait(misc + M1_G1, par, abort)) break;
        fence_after();
        {
            const int rowl = 32 * (warp & 3) + lane, col0 = 32 * (warp >> 2);
            uint32_t ra[32];
            tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + P1_TM_D1 + col0, ra);
            wait_ld();
            if (rowl < 64) {   // A: strictly lower
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 x;
                    x.x = col0 + i < rowl ? __uint_as_float(ra[i]) : 0.f;
                    x.y = col0 + i + 1 < rowl ? __uint_as_float(ra[i + 1]) : 0.f;
                    x.z = col0 + i + 2 < rowl ? __uint_as_float(ra[i + 2]) : 0.f;
                    x.w = col0 + i + 3 < rowl ? __uint_as_float(ra[i + 3]) : 0.f;
                    *reinterpret_cast<float4 *>(AS + rowl * LDA + col0 + i) = x;
                }
            } else {           // P: lower with the diagonal, rows 64-127 of the [T; P] tile
                const int r = rowl - 64;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int cc = col0 + 8 * u + 2 * i;
                        pk[i] = pack_bf16(cc <= r ? __uint_as_float(ra[8 * u + 2 * i]) : 0.f,
                                          cc + 1 <= r ? __uint_as_float(ra[8 * u + 2 * i + 1]) : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(sm + P1_W + sw_off(64 + r, col0 + 8 * u, 128)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
        fence_async_smem();
        fence_before();
        __syncthreads();
        // ------------------------------------------------------------------ T = (I + A)^-1 (warps 4-7)
        if (tid == 0) bulk_s2g(rec + R_P, aW + 8192, 8192);   // P is final
        if (warp >= 4) {
            solve_unit_lower(AS, reinterpret_cast<float *>(sm + P1_X), sm + P1_W, tid - 128, 1);
            fence_async_smem();
        }
        __syncthreads();
        // ------------------------------------------------------------------ G2: W' = T Ê, Ũ = T U
        if (tid == 0) {
            fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + P1_TM_D2, desc_kmajor(aW, 128, j), desc_mnmajor(aEQ, 128, j), ID_G2, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + P1_TM_D3, desc_kmajor(aW, 128, j), desc_mnmajor(aU, 64, j), ID_G2, j > 0);
            mma_commit(misc + M1_G2);
        }
        if (!block_wait(misc + M1_G2, par, abort)) break;
        fence_after();
        if ((warp & 3) < 2) {   // TMEM lanes 0-63: rows of W' (warps 0, 1) and of Ũ (warps 4, 5)
            const int i = 32 * (warp & 3) + lane;
            const bool isW = warp < 4;
            const uint32_t src = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (isW ? P1_TM_D2 : P1_TM_D3);
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(src + 32 * u2, r32);
                wait_ld();
                const float sg = isW ? -1.f : 1.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int cc = 32 * u2 + 8 * u;
                    const uint32_t *x = r32 + 8 * u;
                    const uint4 pk = make_uint4(pack_bf16(sg * __uint_as_float(x[0]), sg * __uint_as_float(x[1])),
                                                pack_bf16(sg * __uint_as_float(x[2]), sg * __uint_as_float(x[3])),
                                                pack_bf16(sg * __uint_as_float(x[4]), sg * __uint_as_float(x[5])),
                                                pack_bf16(sg * __uint_as_float(x[6]), sg * __uint_as_float(x[7])));
                    if (isW)
                        *reinterpret_cast<uint4 *>(sm + P1_EQ + sw_off(i, cc, 128)) = pk;
                    else
                        *reinterpret_cast<uint4 *>(sm + P1_U + sw_off(i, cc, 64)) = pk;
                }
            }
        }
        fence_async_smem();
        fence_before();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(rec + R_A3, aEQ, 32768);
            bulk_s2g(rec + R_U, aU, 16384);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();   // the record stores complete before the block exits
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0 && *abort) atomicOr(status, STATUS_PREP);
    if (warp == 0) tmem_dealloc(tmem, P1_TM_COLS);
}

// ---------------------------------------------------------------------------- stage 2
constexpr int W2_NT = 256;
constexpr uint32_t W2_S = 0;                          // Z̃ bf16 [c x v] (MN-major B of G3)
constexpr uint32_t W2_DL = 32768;                     // Delta bf16 [i x v]
constexpr uint32_t W2_SLOT = 49152;                   // 2 record slots
constexpr uint32_t W2_OST = W2_SLOT + 2 * R_BYTES;    // o rows staged for the TMA store (16 KB)
constexpr uint32_t W2_MISC = W2_OST + 16384;
constexpr uint32_t W2_BYTES = W2_MISC + 256 + 1024;
// mbarriers: FULL and G45 per slot, D3FREE per accumulator buffer, G3
enum : uint32_t { M2_FULL = 0, M2_G45 = 16, M2_D3FREE = 32, M2_G3 = 48, M2_TSLOT = 64, M2_ABORT = 68 };
constexpr uint32_t W2_TM_Z = 0, W2_TM_D3 = 128, W2_TM_COLS = 512;   // D3 buffers at 128 and 256
constexpr uint32_t BAR_STATE = 1, BAR_O = 2;

__device__ __forceinline__ bool group_wait2(uint32_t mb, uint32_t parity, uint32_t bar, uint32_t n,
                                            volatile uint32_t *abort) {
    bool ok = mbar_wait(mb, parity, WAIT_LIMIT) && !*abort;
    const bool fail = group_or(bar, n, !ok);
    fence_after();
    if (fail) *abort = 1u;
    return !fail;
}
__device__ __forceinline__ bool thread_wait(uint32_t mb, uint32_t parity, volatile uint32_t *abort) {
    if (!mbar_wait(mb, parity, WAIT_LIMIT) || *abort) {
        *abort = 1u;
        return false;
    }
    fence_after();
    return true;
}

__global__ void __launch_bounds__(W2_NT, 1)
    walk_kernel(const __grid_constant__ CUtensorMap map_o, const unsigned char *records, const float *S0, float *ST,
                int H, int T, int n0, int nw, unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chain = blockIdx.x, bb = chain / H, h = chain % H;
    const uint32_t misc = smem_u32(sm + W2_MISC);
    volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sm + W2_MISC + M2_ABORT);

    if (warp == 0) tmem_alloc(misc + M2_TSLOT, W2_TM_COLS);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(misc + M2_FULL + 8 * s, 1);
            mbar_init(misc + M2_G45 + 8 * s, 1);
            mbar_init(misc + M2_D3FREE + 8 * s, 64);
        }
        mbar_init(misc + M2_G3, 1);
        *abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&map_o);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + W2_MISC + M2_TSLOT);
    auto slot_addr = [&](int n) { return W2_SLOT + (uint32_t)(n & 1) * R_BYTES; };
    auto d3 = [&](int n) { return tmem + W2_TM_D3 + 128u * (uint32_t)(n & 1); };
    auto rec_of = [&](int nl) { return records + ((size_t)(bb * nw + nl) * H + h) * R_BYTES; };

    if (warp < 4) {
        // ------------------------------------------------------------------ state group: rows c of Z
        const int crow = tid;
        const uint32_t lrow = (uint32_t)(warp * 32) << 16;
        {   // Z <- S0 (or 0); the first rescale multiplies by chunk 0's exp(m)
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
                tmem_st32(tmem + lrow + W2_TM_Z + 32 * u2, r32);
            }
            wait_st();
        }
        float egm_prev = 1.f;
        bool ok = true;
        for (int nl = 0; nl < nw && ok; ++nl) {
            const uint32_t slot = slot_addr(nl);
            const float *vec = reinterpret_cast<const float *>(sm + slot + R_VEC);
            if (!group_wait2(misc + M2_FULL + 8 * (nl & 1), (uint32_t)((nl >> 1) & 1), BAR_STATE, 128, abort)) { ok = false; break; }
            if (nl > 0 && !group_wait2(misc + M2_G45 + 8 * ((nl - 1) & 1), (uint32_t)(((nl - 1) >> 1) & 1), BAR_STATE, 128, abort)) { ok = false; break; }
            // S_n = sPost_{n-1} Z, then Z <- sZ_n S_n and the bf16 operand sS_n S_n; the factors are
            // applied one after the other (their product alone can lie below fp32's range)
            const float post = egm_prev, ssc = vec[crow], zsc = vec[128 + crow];
            egm_prev = vec[256 + crow];
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(tmem + lrow + W2_TM_Z + 32 * u2, r32);
                wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(post * __uint_as_float(r32[i]));
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float *x = reinterpret_cast<const float *>(r32) + 8 * u;
                    const uint4 pk = make_uint4(pack_bf16(ssc * x[0], ssc * x[1]), pack_bf16(ssc * x[2], ssc * x[3]),
                                                pack_bf16(ssc * x[4], ssc * x[5]), pack_bf16(ssc * x[6], ssc * x[7]));
                    *reinterpret_cast<uint4 *>(sm + W2_S + sw_off(crow, 32 * u2 + 8 * u, 128)) = pk;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(zsc * __uint_as_float(r32[i]));
                tmem_st32(tmem + lrow + W2_TM_Z + 32 * u2, r32);
            }
            wait_st();
            fence_async_smem();
            fence_before();
            group_sync(BAR_STATE, 128);
            if (tid == 0) {   // G3: [-W'Z̃; Q̂Z̃] into D3 of this chunk, once its o rows of chunk n-2 are out
                fence_after();
                if (nl < 2 || thread_wait(misc + M2_D3FREE + 8 * (nl & 1), (uint32_t)(((nl - 2) >> 1) & 1), abort)) {
                    const uint32_t aA3 = smem_u32(sm + slot + R_A3), aS = smem_u32(sm + W2_S);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        mma_ss(d3(nl), desc_kmajor(aA3, 128, j), desc_mnmajor(aS, 128, j), ID_G3, j > 0);
                    mma_commit(misc + M2_G3);
                }
            }
            if (!group_wait2(misc + M2_G3, (uint32_t)(nl & 1), BAR_STATE, 128, abort)) { ok = false; break; }
            if (warp < 2) {   // Delta = Ũ - W'Z̃ (rows i < 64) -> bf16 tile
                const unsigned char *Ut = sm + slot + R_U;
#pragma unroll
                for (int u2 = 0; u2 < 4; ++u2) {
                    uint32_t r32[32];
                    tmem_ld32(d3(nl) + lrow + 32 * u2, r32);
                    wait_ld();
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int vv = 32 * u2 + 8 * u;
                        const uint4 ut = *reinterpret_cast<const uint4 *>(Ut + sw_off(crow, vv, 64));
                        const float2 a = unpack2(ut.x), b2 = unpack2(ut.y), c2 = unpack2(ut.z), d2 = unpack2(ut.w);
                        const float *x = reinterpret_cast<const float *>(r32) + 8 * u;
                        const uint4 pk = make_uint4(pack_bf16(a.x + x[0], a.y + x[1]), pack_bf16(b2.x + x[2], b2.y + x[3]),
                                                    pack_bf16(c2.x + x[4], c2.y + x[5]), pack_bf16(d2.x + x[6], d2.y + x[7]));
                        *reinterpret_cast<uint4 *>(sm + W2_DL + sw_off(crow, vv, 64)) = pk;
                    }
                }
            }
            fence_async_smem();
            fence_before();
            group_sync(BAR_STATE, 128);
            if (tid == 0) {   // G4: O += P Delta (rows 0-63 of the A tile are Ũ's bytes: their products
                              // land in the Delta rows of D3, already read); G5: Z += K̃^T Delta
                fence_after();
                const uint32_t aPA = smem_u32(sm + slot + R_P - 8192), aKT = smem_u32(sm + slot + R_KT),
                               aDL = smem_u32(sm + W2_DL);
#pragma unroll
                for (int j = 0; j < 4; ++j) mma_ss(d3(nl), desc_kmajor(aPA, 128, j), desc_mnmajor(aDL, 64, j), ID_G4, 1);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ss(tmem + W2_TM_Z, desc_mnmajor(aKT, 64, j), desc_mnmajor(aDL, 64, j), ID_G5, 1);
                mma_commit(misc + M2_G45 + 8 * (nl & 1));
            }
        }
        // S_T = Diag(sPost) Z of the last chunk, once its G4/G5 are complete
        if (ok && group_wait2(misc + M2_G45 + 8 * ((nw - 1) & 1), (uint32_t)(((nw - 1) >> 1) & 1), BAR_STATE, 128, abort)) {
            float *dst = ST + ((size_t)chain * KD + crow) * VD;
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(tmem + lrow + W2_TM_Z + 32 * u2, r32);
                wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4 *>(dst + 32 * u2 + i) =
                        make_float4(egm_prev * __uint_as_float(r32[i]), egm_prev * __uint_as_float(r32[i + 1]),
                                    egm_prev * __uint_as_float(r32[i + 2]), egm_prev * __uint_as_float(r32[i + 3]));
            }
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------------ producer: one bulk copy per record
        if (lane == 0) {
            for (int nl = 0; nl < nw; ++nl) {
                if (nl >= 2 && !thread_wait(misc + M2_G45 + 8 * (nl & 1), (uint32_t)(((nl - 2) >> 1) & 1), abort)) break;
                mbar_arrive_expect_tx(misc + M2_FULL + 8 * (nl & 1), R_COPY);
                bulk_g2s(smem_u32(sm + slot_addr(nl)), rec_of(nl), R_COPY, misc + M2_FULL + 8 * (nl & 1));
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------------ o group: TMEM lanes 64-127 of D3
        const int ot = tid - 192;   // O row of the chunk
        const uint32_t lrow = (uint32_t)(64 + 32 * (warp - 6)) << 16;
        for (int nl = 0; nl < nw; ++nl) {
            const int t0 = (n0 + nl) * C;
            if (!group_wait2(misc + M2_G45 + 8 * (nl & 1), (uint32_t)((nl >> 1) & 1), BAR_O, 64, abort)) break;
            if (ot == 0) bulk_wait_read_all();   // the previous chunk's o store has read the staging tile
            group_sync(BAR_O, 64);
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(d3(nl) + lrow + 32 * u2, r32);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t *x = r32 + 8 * u;
                    const uint4 pk = make_uint4(pack_bf16(__uint_as_float(x[0]), __uint_as_float(x[1])),
                                                pack_bf16(__uint_as_float(x[2]), __uint_as_float(x[3])),
                                                pack_bf16(__uint_as_float(x[4]), __uint_as_float(x[5])),
                                                pack_bf16(__uint_as_float(x[6]), __uint_as_float(x[7])));
                    *reinterpret_cast<uint4 *>(sm + W2_OST + sw_off(ot, 32 * u2 + 8 * u, 64)) = pk;
                }
            }
            fence_before();
            mbar_arrive(misc + M2_D3FREE + 8 * (nl & 1));
            fence_async_smem();
            group_sync(BAR_O, 64);
            if (ot == 0) {   // rows past the end of the sequence are clipped by the copy
                tma_store_4d(&map_o, 0, h, t0, bb, smem_u32(sm + W2_OST));
                tma_store_4d(&map_o, 64, h, t0, bb, smem_u32(sm + W2_OST + 8192));
                bulk_commit();
            }
        }
        if (ot == 0) bulk_wait_all();
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0 && *abort) atomicOr(status, STATUS_WALK);
    if (warp == 0) tmem_dealloc(tmem, W2_TM_COLS);
}

}  // namespace split

// ============================================================================ host side
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, fetched through the runtime (the library does not link libcuda)
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault) != cudaSuccess) p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// A [B, T, H, 128] bf16 token tensor as the 4-D map (d, H, T, B) with a 64 x 1 x 64 x 1 box in the
// 128-byte swizzle: one box is the 64 x 64 half-tile of the operand layout.  Rows past T read as zero.
bool token_map(CUtensorMap *m, const void *base, int B, int T, int H) {
    const EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {256, 256ull * H, 256ull * H * T};
    const cuuint32_t box[4] = {64, 1, 64, 1}, es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

constexpr int kWindowChunks = 64;   // chunks per window: bounds the record buffer

}  // namespace

size_t split_workspace_bytes(int B, int H, int T) {
    const int NC = (T + split::C - 1) / split::C, nw = std::min(NC, kWindowChunks);
    return kStatusBytes + (size_t)B * H * nw * split::R_BYTES;
}

int launch_chunk_split(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                       const float *S0, void *o, float *ST, int B, int H, int T, void *ws, cudaStream_t st) {
    split::TokMaps maps;
    CUtensorMap map_o;
    if (!token_map(&maps.q, q, B, T, H) || !token_map(&maps.k, k, B, T, H) || !token_map(&maps.b, b, B, T, H) ||
        !token_map(&maps.v, v, B, T, H) || !token_map(&maps.w, w, B, T, H) || !token_map(&map_o, o, B, T, H))
        return -6;
    const int smem1 = (int)split::P1_BYTES, smem2 = (int)split::W2_BYTES;
    if (cudaFuncSetAttribute(split::prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1) != cudaSuccess ||
        cudaFuncSetAttribute(split::walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2) != cudaSuccess)
        return -6;
    const int nsm = sm_count();
    if (nsm <= 0) return -6;
    unsigned int *status = reinterpret_cast<unsigned int *>(ws);
    unsigned char *records = static_cast<unsigned char *>(ws) + kStatusBytes;
    const int NC = (T + split::C - 1) / split::C;
    for (int n0 = 0; n0 < NC; n0 += kWindowChunks) {
        const int nw = std::min(kWindowChunks, NC - n0), nch = B * H * nw;
        split::prep_kernel<<<std::min(nch, 2 * nsm), split::P1_NT, smem1, st>>>(
            maps, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)b, alpha, records, H, T,
            NC, n0, nw, nch, status);
        split::walk_kernel<<<B * H, split::W2_NT, smem2, st>>>(map_o, records, n0 == 0 ? S0 : ST, ST, H, T, n0, nw,
                                                               status);
    }
    return launch_status();
}

}  // namespace gdn2
