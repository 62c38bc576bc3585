// Two-stage chunkwise prefill on the tensor cores (tcgen05 + TMEM + TMA), sm_100a.
// bf16 tokens, d_k = d_v = 128, chunk C = 64.
//
// The update equation of page "NVIDIA представила Gated DeltaNet-2 ..." (section "Техническая
// схема") is evaluated in the chunkwise WY form with C = 64 that the same page names.  Everything
// in that form that depends only on a chunk's own tokens -- the log-decay prefix, the decay
// absorbed into the rank-1 factors, the Gram matrices, the triangular solve and the WY factors --
// is independent from chunk to chunk; only the state update is a chain.  So:
//
//   stage 1, prep_kernel: fully parallel over every (batch, chunk, head), one persistent CTA per SM.  The
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
#include "split_layout.cuh"
#include "tc_chunk.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace split {

using namespace gdn2::tc;
using namespace gdn2::tcc;

constexpr float SPAN_MAX_LOG2 = 173.123f;   // 120 nats in log2 units
constexpr uint32_t WAIT_LIMIT = 1u << 22;
constexpr uint32_t STATUS_PREP = 2u, STATUS_WALK = 4u;

// ---------------------------------------------------------------------------- stage 1
// One persistent CTA per SM over the window's chunk-heads, three roles working on consecutive
// chunk-heads at once:
//   warps 0-7   build group: alpha prefix, decay factors and the bf16 operands of chunk-head j+1,
//               G1, then A (fp32, for the solve) and P (bf16, to the record) out of TMEM
//   warps 8-11  solve group: T = (I + A)^-1, G2 and the W', Ũ rows of chunk-head j
// The token tiles pass through a two-stage ring filled by TMA, alpha through one buffer.  The thread
// that frees a buffer refills it: the build group's first thread loads the next chunk-head's alpha as
// soon as the prefix has read it, and the solve group's first thread loads the tiles of chunk-head j+2
// into the stage of chunk-head j once the record's stores (K̃ and Q̂ as soon as G1 has run, -W' and Ũ at
// the end) have read it.  Twelve warps, three on each of the SM's four register sub-partitions, leave
// 168 registers per thread (a thirteenth, producer, warp would cut that to 128).
constexpr int P1_NT = 384;
constexpr uint32_t P1_STAGE = 81920;                 // per stage: EQ, KT, U, W tiles
constexpr uint32_t P1_EQ = 0;                        // b -> Ê -> -W' (rows 0-63), q -> Q̂ (rows 64-127)
constexpr uint32_t P1_KT = 32768;                    // k -> K̃
constexpr uint32_t P1_U = 49152;                     // v -> U -> Ũ
constexpr uint32_t P1_W = 65536;                     // w; then [T; T] (128 rows, K = 64)
constexpr uint32_t P1_A = 2 * P1_STAGE;              // alpha fp32 [64][128] (one buffer)
constexpr uint32_t P1_AS = P1_A + 32768;             // solve group: fp32 A / T^T [64][LDA]
constexpr uint32_t P1_X = P1_AS + 64 * LDA * 4;      // solve group scratch (4 KB)
constexpr uint32_t P1_WT = P1_X + 4096;              // build group: [8][128] log2 totals, then g_0 [128]
constexpr uint32_t P1_MISC = P1_WT + 4608;
constexpr uint32_t P1_BYTES = P1_MISC + 256 + 1024;  // + alignment slack
// mbarriers: FULL per stage; alpha full; G1; A ready / A scratch free; G2
enum : uint32_t {
    M1_FULL = 0, M1_AFULL = 32, M1_G1 = 48, M1_AREADY = 56, M1_ASFREE = 64, M1_G2 = 72, M1_TSLOT = 96,
    M1_ABORT = 100, M1_LAST = 104   // M1_LAST: three ints, the last job loaded into stage 0, stage 1, alpha
};
constexpr uint32_t P1_TM_D1 = 0, P1_TM_D2 = 128, P1_TM_D3 = 256, P1_TM_COLS = 512;
constexpr uint32_t BAR_A = 1, BAR_B = 2;   // named barriers: build group (256), solve group (128)

constexpr uint32_t ID_G1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G2 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G3 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G4 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G5 = idesc_bf16(128, 128, 1, 1);


// Bounded wait of a warp group (named barrier `bar`, n threads): every thread gets the same verdict.
__device__ __forceinline__ bool gwait(uint32_t mb, uint32_t parity, uint32_t bar, uint32_t n, volatile uint32_t *abort) {
    bool ok = mbar_wait(mb, parity, WAIT_LIMIT) && !*abort;
    const bool fail = group_or(bar, n, !ok);
    fence_after();
    if (fail) *abort = 1u;
    return !fail;
}

// Wide-span chunk: A_ri = sum_c e_rc k_ic exp2(g_rc - g_ic) (i < r) and P_ri likewise with q
// (i <= r), one row per thread (threads 0-63 rows of A, 64-127 rows of P: the TMEM lanes G1 would
// have written).  The exponent is summed from log2 alpha while i walks down from r, so it never
// leaves [-inf, 0]; rows are read again from global memory.  Layer-edge variant: q, k raw (their
// inverse norms applied here), b and alpha from their logits.
// (A rare correctness path: kept out of line so that it does not weigh on the build's registers.)
template <bool EDGES>
__device__ __noinline__ void wide_span_ap(uint32_t tmem_d1, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                             const __nv_bfloat16 *b, const float *alpha, size_t row0, size_t stride,
                                             int tid, int L) {
    const int r = tid & 63;
    const bool isP = tid >= 64;
    const uint32_t lane_base = tmem_d1 + ((uint32_t)((tid >> 5) * 32) << 16);
    const int rc = min(r, L - 1);
    const size_t rowr = row0 + (size_t)rc * stride;
    auto row = [&](int t) { return row0 + (size_t)t * stride; };
    auto log2a = [&](int t, int cc) {
        const float a = alpha[row(t) * KD + cc];
        return fast_log2(fmaxf(EDGES ? alpha_of_logit(a) : a, 1.17549435e-38f));
    };
    auto inv_norm = [&](const __nv_bfloat16 *x, size_t rw) {   // 1 / max(|x_row|, eps)
        float ss = 0.f;
        for (int cc = 0; cc < KD; ++cc) {
            const float v = __bfloat162float(x[rw * KD + cc]);
            ss += v * v;
        }
        return rsqrtf(fmaxf(ss, EDGE_NORM_EPS * EDGE_NORM_EPS));
    };
    const float sr = EDGES ? inv_norm(isP ? q : k, rowr) : 1.f;
#pragma unroll 1
    for (int i0 = 0; i0 < 64; i0 += 16) {
        float acc[16], sk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            acc[i] = 0.f;
            sk[i] = EDGES ? inv_norm(k, row(min(i0 + i, L - 1))) : 1.f;
        }
        if (r < L && i0 <= r) {
#pragma unroll 1
            for (int cc = 0; cc < KD; ++cc) {
                const float bg = EDGES ? sigmoid_f(__bfloat162float(b[rowr * KD + cc])) : __bfloat162float(b[rowr * KD + cc]);
                const float x = sr * (isP ? __bfloat162float(q[rowr * KD + cc]) : bg * __bfloat162float(k[rowr * KD + cc]));
                const int itop = min(i0 + 15, r);
                float d = 0.f;
#pragma unroll 1
                for (int jj = r; jj > itop; --jj) d += log2a(jj, cc);
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    if (i0 + i <= itop) {
                        acc[i] += x * sk[i] * __bfloat162float(k[row(i0 + i) * KD + cc]) * exp2f(d);
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

// Layer-edge variant (EDGES): the tensors are the layer's raw inputs -- q and k are divided by their
// L2 norms over the 128 channels, b and w pass a sigmoid, alpha = exp(-softplus(a)) comes from the decay
// logit -- folded into the build: the inverse norms join the decay factors before their one bf16
// rounding, so q and k are never rounded after normalisation.
// EXACT_F: each factor of a tensor-core chunk (Ê, Q̂, K̃) is one fp32 product rounded once to bf16,
// b ⊙ k included, instead of packed bf16 products of bf16-rounded frame factors.  The backward's
// replay builds its records this way: d(ln alpha) sums terms of both signs, and the bf16 rounding of
// the frame factors, a relative error that differs between Ê, Q̂ and K̃, doubles its error.
template <bool EDGES, bool EXACT_F = false>
__global__ void __launch_bounds__(P1_NT, 1)
    prep_kernel(const __grid_constant__ TokMaps maps, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                const __nv_bfloat16 *b, const float *alpha, unsigned char *records, unsigned char *aux, int H, int T,
                int n0, int nw, int nch, unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t misc = smem_u32(sm + P1_MISC);
    volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sm + P1_MISC + M1_ABORT);

    if (warp == 0) tmem_alloc(misc + M1_TSLOT, P1_TM_COLS);
    if (tid == 0) {
        for (int st = 0; st < 2; ++st) mbar_init(misc + M1_FULL + 8 * st, 1);
        mbar_init(misc + M1_AFULL, 1);
        for (int i = 0; i < 3; ++i) reinterpret_cast<volatile int *>(sm + P1_MISC + M1_LAST)[i] = -1;
        mbar_init(misc + M1_G1, 1);
        mbar_init(misc + M1_AREADY, 1);
        mbar_init(misc + M1_ASFREE, 1);
        mbar_init(misc + M1_G2, 1);
        *abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + P1_MISC + M1_TSLOT);
    // chunk-heads of the window in (batch, chunk, head) order: neighbouring CTAs read adjacent heads
    auto coords = [&](int ch, int &h, int &bb, int &n) {
        h = ch % H;
        n = n0 + (ch / H) % nw;
        bb = ch / (H * nw);
    };
    const int njobs = (int)blockIdx.x < nch ? (nch - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    auto rec_of = [&](int j) { return records + (size_t)(blockIdx.x + j * gridDim.x) * R_BYTES; };
    auto aux_of = [&](int j) { return aux + (size_t)(blockIdx.x + j * gridDim.x) * X_BYTES; };

    // loads of chunk-head job j: alpha into its buffer; the token tiles into stage j & 1
    auto load_alpha = [&](int j) {
        int h, bb, n;
        coords(blockIdx.x + j * gridDim.x, h, bb, n);
        mbar_arrive_expect_tx(misc + M1_AFULL, 32768u);
        tma_load_4d(smem_u32(sm + P1_A), &maps.alpha, 0, h, n * C, bb, misc + M1_AFULL);
    };
    auto load_tiles = [&](int j) {
        int h, bb, n;
        coords(blockIdx.x + j * gridDim.x, h, bb, n);
        const int t0 = n * C, stg = j & 1;
        const uint32_t st = smem_u32(sm + stg * P1_STAGE), fb = misc + M1_FULL + 8 * stg;
        mbar_arrive_expect_tx(fb, 10u * 8192u);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(st + P1_EQ + hf * 16384, &maps.b, 64 * hf, h, t0, bb, fb);
            tma_load_4d(st + P1_EQ + hf * 16384 + 8192, &maps.q, 64 * hf, h, t0, bb, fb);
            tma_load_4d(st + P1_KT + hf * 8192, &maps.k, 64 * hf, h, t0, bb, fb);
            tma_load_4d(st + P1_U + hf * 8192, &maps.v, 64 * hf, h, t0, bb, fb);
            tma_load_4d(st + P1_W + hf * 8192, &maps.w, 64 * hf, h, t0, bb, fb);
        }
    };
    // the last job each buffer was loaded for, whichever thread loaded it (for the exit: no copy may be
    // left in flight): stage 0, stage 1, alpha
    volatile int *last_ld = reinterpret_cast<volatile int *>(sm + P1_MISC + M1_LAST);
    if (tid == 0) {
        prefetch_tmap(&maps.q); prefetch_tmap(&maps.k); prefetch_tmap(&maps.b);
        prefetch_tmap(&maps.v); prefetch_tmap(&maps.w); prefetch_tmap(&maps.alpha);
        for (int j = 0; j < 2 && j < njobs; ++j) {
            load_tiles(j);
            last_ld[j] = j;
        }
        if (njobs > 0) {
            load_alpha(0);
            last_ld[2] = 0;
        }
    }

    if (warp < 8) {
        // ------------------------------------------------------------------ build group
        float *WT = reinterpret_cast<float *>(sm + P1_WT);
        float *v_g0 = WT + 8 * 128;
        const float *AL = reinterpret_cast<const float *>(sm + P1_A);
        const int c4 = lane * 4, p0 = warp * 8;   // 8 positions x 4 channels per thread
        for (int j = 0; j < njobs; ++j) {
            const int stg = j & 1;
            int h, bb, n;
            coords(blockIdx.x + j * gridDim.x, h, bb, n);
            const int t0 = n * C, L = min(C, T - t0);
            unsigned char *S = sm + stg * P1_STAGE;
            const uint32_t aEQ = smem_u32(S + P1_EQ), aKT = smem_u32(S + P1_KT);
            const uint32_t d1 = tmem + P1_TM_D1;

            // ---------------------------------------------------------------- alpha and the log-decay prefix
            if (!gwait(misc + M1_AFULL, (uint32_t)(j & 1), BAR_A, 256, abort)) break;
            float al[8][4];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                float4 a4 = *reinterpret_cast<const float4 *>(AL + (p0 + p) * KD + c4);
                if (EDGES) a4 = make_float4(alpha_of_logit(a4.x), alpha_of_logit(a4.y), alpha_of_logit(a4.z),
                                            alpha_of_logit(a4.w));
                // past the end: alpha = 1 (the copy filled zeros); subnormal alpha: smallest normal
                al[p][0] = p0 + p >= L ? 1.f : fmaxf(a4.x, 1.17549435e-38f);
                al[p][1] = p0 + p >= L ? 1.f : fmaxf(a4.y, 1.17549435e-38f);
                al[p][2] = p0 + p >= L ? 1.f : fmaxf(a4.z, 1.17549435e-38f);
                al[p][3] = p0 + p >= L ? 1.f : fmaxf(a4.w, 1.17549435e-38f);
            }
            // log2 of the product of the thread's 8 alphas per channel: the exponent fields plus log2 of
            // the product of the mantissas (in [1, 256))
            float lw[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                int ex = 0;
                float mp = 1.f;
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const uint32_t u = __float_as_uint(al[p][jj]);
                    ex += (int)(u >> 23) - 127;
                    mp *= __uint_as_float((u & 0x7FFFFFu) | 0x3F800000u);
                }
                lw[jj] = (float)ex + fast_log2(mp);
            }
            *reinterpret_cast<float4 *>(WT + warp * 128 + c4) = make_float4(lw[0], lw[1], lw[2], lw[3]);
            if (warp == 0)
                *reinterpret_cast<float4 *>(v_g0 + c4) =
                    make_float4(fast_log2(al[0][0]), fast_log2(al[0][1]), fast_log2(al[0][2]), fast_log2(al[0][3]));
            group_sync(BAR_A, 256);
            if (tid == 0 && j + 1 < njobs) {   // the alpha buffer has been read: the next chunk-head's in
                load_alpha(j + 1);
                last_ld[2] = j + 1;
            }
            float pre[4] = {0.f, 0.f, 0.f, 0.f}, gC[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w2 = 0; w2 < 8; ++w2) {
                const float4 t4 = *reinterpret_cast<const float4 *>(WT + w2 * 128 + c4);
                const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    gC[jj] += tv[jj];
                    if (w2 < warp) pre[jj] += tv[jj];
                }
            }
            const float4 g04 = *reinterpret_cast<const float4 *>(v_g0 + c4);
            const float g0[4] = {g04.x, g04.y, g04.z, g04.w};
            int wide_l = 0;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) wide_l |= (g0[jj] - gC[jj] > SPAN_MAX_LOG2);
            const bool wide = group_or(BAR_A, 256, wide_l != 0);   // also: WT and v_g0 reads done
            float m2[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) m2[jj] = wide ? 0.f : 0.5f * (g0[jj] + gC[jj]);
            if (warp == 0) {
                // sS: scale of the bf16 state operand (exp(m)); sZ: scale of the TMEM state that G5
                // accumulates into; sPost: the factor that turns the accumulated Z into the next state.
                // Tensor-core chunk: sS = sZ = exp(m), sPost = exp(g_C - m).  Wide-span chunk: sS = 1,
                // sZ = exp(g_C), sPost = 1 (K̃ is then exp(g_C - g) ⊙ k).
                float sS[4], sZ[4], sP[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    sS[jj] = wide ? 1.f : fast_exp2(m2[jj]);
                    sZ[jj] = wide ? fast_exp2(gC[jj]) : sS[jj];
                    sP[jj] = wide ? 1.f : fast_exp2(gC[jj] - m2[jj]);
                }
                float *vec = reinterpret_cast<float *>(rec_of(j) + R_VEC);
                *reinterpret_cast<float4 *>(vec + c4) = make_float4(sS[0], sS[1], sS[2], sS[3]);
                *reinterpret_cast<float4 *>(vec + 128 + c4) = make_float4(sZ[0], sZ[1], sZ[2], sZ[3]);
                *reinterpret_cast<float4 *>(vec + 256 + c4) = make_float4(sP[0], sP[1], sP[2], sP[3]);
                if (aux) {   // the frame exponents, for the backward: Ê = e 2^(g - ae), K̃ = k 2^(ak - g)
                    float *xe = reinterpret_cast<float *>(aux_of(j) + X_AE), *xk = reinterpret_cast<float *>(aux_of(j) + X_AK);
                    *reinterpret_cast<float4 *>(xe + c4) = make_float4(m2[0], m2[1], m2[2], m2[3]);
                    *reinterpret_cast<float4 *>(xk + c4) = wide ? make_float4(gC[0], gC[1], gC[2], gC[3])
                                                                : make_float4(m2[0], m2[1], m2[2], m2[3]);
                }
            }

            // ---------------------------------------------------------------- build (in place)
            if (!gwait(misc + M1_FULL + 8 * stg, (uint32_t)((j >> 1) & 1), BAR_A, 256, abort)) break;
            {
                uint2 rq[8], rk[8], rb[8];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int r = p0 + p;
                    rb[p] = *reinterpret_cast<const uint2 *>(S + P1_EQ + sw_off(r, c4, 128));
                    rq[p] = *reinterpret_cast<const uint2 *>(S + P1_EQ + sw_off(64 + r, c4, 128));
                    rk[p] = *reinterpret_cast<const uint2 *>(S + P1_KT + sw_off(r, c4, 64));
                    const uint2 rv = *reinterpret_cast<const uint2 *>(S + P1_U + sw_off(r, c4, 64));
                    uint2 rw = *reinterpret_cast<const uint2 *>(S + P1_W + sw_off(r, c4, 64));
                    if (EDGES) {
                        rw = make_uint2(bsigmoid2(rw.x), bsigmoid2(rw.y));
                        rb[p] = make_uint2(bsigmoid2(rb[p].x), bsigmoid2(rb[p].y));
                    }
                    *reinterpret_cast<uint2 *>(S + P1_U + sw_off(r, c4, 64)) = make_uint2(bmul2(rw.x, rv.x), bmul2(rw.y, rv.y));
                }
                // layer edges: inverse L2 norms of the warp's 8 q and k rows (a warp holds each row, 4
                // channels a lane), kept in the prefix scratch (read out by now) rather than in registers
                float *inv = WT + 16 * warp;   // [0, 8): q rows, [8, 16): k rows
                if (EDGES) {
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const float2 qa = unpack2(rq[p].x), qb = unpack2(rq[p].y), ka = unpack2(rk[p].x), kb = unpack2(rk[p].y);
                        float sq = qa.x * qa.x + qa.y * qa.y + qb.x * qb.x + qb.y * qb.y;
                        float sk = ka.x * ka.x + ka.y * ka.y + kb.x * kb.x + kb.y * kb.y;
#pragma unroll
                        for (int msk = 16; msk > 0; msk >>= 1) {
                            sq += __shfl_xor_sync(0xffffffffu, sq, msk);
                            sk += __shfl_xor_sync(0xffffffffu, sk, msk);
                        }
                        if (lane == p) inv[p] = rsqrtf(fmaxf(sq, EDGE_NORM_EPS * EDGE_NORM_EPS));
                        if (lane == 8 + p) inv[8 + p] = rsqrtf(fmaxf(sk, EDGE_NORM_EPS * EDGE_NORM_EPS));
                    }
                    __syncwarp();
                }
                auto iq = [&](int p) { return EDGES ? inv[p] : 1.f; };
                auto ik = [&](int p) { return EDGES ? inv[8 + p] : 1.f; };
                if (!wide) {
                    // exp(g - m) from one exponential at the thread's first position and running
                    // products of alpha after it; exp(m - g) backwards from one exponential at its last
                    // position.  Both start inside the chunk, where every factor lies within
                    // exp(+-span/2): a start before the first position (exp(-m) itself) can leave fp32's
                    // range when the chunk's first alpha is tiny.  Packed bf16 arithmetic: each factor
                    // and each product is rounded to bf16 once.
                    float f1[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) f1[jj] = fast_exp2(pre[jj] + fast_log2(al[0][jj]) - m2[jj]);
                    if (EXACT_F) {
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            const int r = p0 + p;
                            if (p > 0)
#pragma unroll
                                for (int jj = 0; jj < 4; ++jj) f1[jj] *= al[p][jj];
                            const float2 q01 = unpack2(rq[p].x), q23 = unpack2(rq[p].y);
                            const float2 k01 = unpack2(rk[p].x), k23 = unpack2(rk[p].y);
                            const float2 b01 = unpack2(rb[p].x), b23 = unpack2(rb[p].y);
                            const float sk = ik(p), sq = iq(p);
                            *reinterpret_cast<uint2 *>(S + P1_EQ + sw_off(r, c4, 128)) =
                                make_uint2(pack_bf16(b01.x * k01.x * (f1[0] * sk), b01.y * k01.y * (f1[1] * sk)),
                                           pack_bf16(b23.x * k23.x * (f1[2] * sk), b23.y * k23.y * (f1[3] * sk)));
                            *reinterpret_cast<uint2 *>(S + P1_EQ + sw_off(64 + r, c4, 128)) =
                                make_uint2(pack_bf16(q01.x * (f1[0] * sq), q01.y * (f1[1] * sq)),
                                           pack_bf16(q23.x * (f1[2] * sq), q23.y * (f1[3] * sq)));
                        }
                        float f2[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) f2[jj] = fast_exp2(m2[jj] - (pre[jj] + lw[jj]));
#pragma unroll
                        for (int p = 7; p >= 0; --p) {
                            const int r = p0 + p;
                            const float2 k01 = unpack2(rk[p].x), k23 = unpack2(rk[p].y);
                            const float sk = ik(p);
                            *reinterpret_cast<uint2 *>(S + P1_KT + sw_off(r, c4, 64)) =
                                make_uint2(pack_bf16(k01.x * (f2[0] * sk), k01.y * (f2[1] * sk)),
                                           pack_bf16(k23.x * (f2[2] * sk), k23.y * (f2[3] * sk)));
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) f2[jj] *= al[p][jj];
                        }
                    } else {
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const int r = p0 + p;
                        if (p > 0)
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) f1[jj] *= al[p][jj];
                        // layer edges: the inverse norms join the decay factors before their one rounding
                        const float sk = ik(p), sq = iq(p);
                        const uint32_t E01 = pack_bf16(f1[0] * sk, f1[1] * sk), E23 = pack_bf16(f1[2] * sk, f1[3] * sk);
                        const uint32_t F01 = pack_bf16(f1[0] * sq, f1[1] * sq), F23 = pack_bf16(f1[2] * sq, f1[3] * sq);
                        *reinterpret_cast<uint2 *>(S + P1_EQ + sw_off(r, c4, 128)) =
                            make_uint2(bmul2(bmul2(rb[p].x, rk[p].x), E01), bmul2(bmul2(rb[p].y, rk[p].y), E23));
                        *reinterpret_cast<uint2 *>(S + P1_EQ + sw_off(64 + r, c4, 128)) =
                            make_uint2(bmul2(rq[p].x, F01), bmul2(rq[p].y, F23));
                    }
                    float f2[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) f2[jj] = fast_exp2(m2[jj] - (pre[jj] + lw[jj]));
#pragma unroll
                    for (int p = 7; p >= 0; --p) {
                        const int r = p0 + p;
                        *reinterpret_cast<uint2 *>(S + P1_KT + sw_off(r, c4, 64)) =
                            make_uint2(bmul2(rk[p].x, pack_bf16(f2[0] * ik(p), f2[1] * ik(p))),
                                       bmul2(rk[p].y, pack_bf16(f2[2] * ik(p), f2[3] * ik(p))));
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) f2[jj] *= al[p][jj];
                    }
                    }
                } else {
                    float run[4] = {pre[0], pre[1], pre[2], pre[3]};
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const int r = p0 + p;
                        const float2 q01 = unpack2(rq[p].x), q23 = unpack2(rq[p].y);
                        const float2 k01 = unpack2(rk[p].x), k23 = unpack2(rk[p].y);
                        const float2 b01 = unpack2(rb[p].x), b23 = unpack2(rb[p].y);
                        const float sq = iq(p), sk = ik(p);
                        const float qq[4] = {q01.x * sq, q01.y * sq, q23.x * sq, q23.y * sq};
                        const float kk[4] = {k01.x * sk, k01.y * sk, k23.x * sk, k23.y * sk};
                        const float bv[4] = {b01.x, b01.y, b23.x, b23.y};
                        float E[4], Qh[4], Kt[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            run[jj] += fast_log2(al[p][jj]);
                            const float gam = exp2f(run[jj]);
                            E[jj] = bv[jj] * kk[jj] * gam;
                            Qh[jj] = qq[jj] * gam;
                            Kt[jj] = kk[jj] * exp2f(gC[jj] - run[jj]);
                        }
                        *reinterpret_cast<uint2 *>(S + P1_EQ + sw_off(r, c4, 128)) =
                            make_uint2(pack_bf16(E[0], E[1]), pack_bf16(E[2], E[3]));
                        *reinterpret_cast<uint2 *>(S + P1_EQ + sw_off(64 + r, c4, 128)) =
                            make_uint2(pack_bf16(Qh[0], Qh[1]), pack_bf16(Qh[2], Qh[3]));
                        *reinterpret_cast<uint2 *>(S + P1_KT + sw_off(r, c4, 64)) =
                            make_uint2(pack_bf16(Kt[0], Kt[1]), pack_bf16(Kt[2], Kt[3]));
                    }
                    // A and P straight into D1 (this group read the previous chunk-head's out of it)
                    if (tid < 128) wide_span_ap<EDGES>(d1, q, k, b, alpha, ((size_t)bb * T + t0) * H + h, (size_t)H, tid, L);
                }
            }
            fence_async_smem();
            fence_before();
            group_sync(BAR_A, 256);
            if (tid == 0) {
                if (!wide) {
                    fence_after();
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        mma_ss(d1, desc_kmajor(aEQ, 128, jj), desc_kmajor(aKT, 64, jj), ID_G1, jj > 0);
                    mma_commit(misc + M1_G1);
                } else {
                    mbar_arrive(misc + M1_G1);   // A and P were written into D1 directly
                }
            }
            // the T tile (w, which shared it, is consumed): zero rows 0-63, whose blocks above the diagonal
            // the solve leaves untouched
            for (int i = tid; i < 512; i += 256) reinterpret_cast<uint4 *>(S + P1_W)[i] = make_uint4(0u, 0u, 0u, 0u);
            fence_async_smem();
            // ---------------------------------------------------------------- A (fp32, for the solve) and P (bf16, to the record)
            if (!gwait(misc + M1_G1, (uint32_t)(j & 1), BAR_A, 256, abort)) break;
            if (j >= 1 && !gwait(misc + M1_ASFREE, (uint32_t)((j - 1) & 1), BAR_A, 256, abort)) break;
            {
                const int rowl = 32 * (warp & 3) + lane, col0 = 32 * (warp >> 2);
                uint32_t x[32];
                tmem_ld32(d1 + ((uint32_t)(32 * (warp & 3)) << 16) + col0, x);
                wait_ld();
                if (rowl < 64) {   // A: strictly lower
                    float *AS = reinterpret_cast<float *>(sm + P1_AS);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v;
                        v.x = col0 + i < rowl ? __uint_as_float(x[i]) : 0.f;
                        v.y = col0 + i + 1 < rowl ? __uint_as_float(x[i + 1]) : 0.f;
                        v.z = col0 + i + 2 < rowl ? __uint_as_float(x[i + 2]) : 0.f;
                        v.w = col0 + i + 3 < rowl ? __uint_as_float(x[i + 3]) : 0.f;
                        *reinterpret_cast<float4 *>(AS + rowl * LDA + col0 + i) = v;
                    }
                } else {           // P: lower with the diagonal, straight into the record's swizzled image
                    const int r = rowl - 64;
                    unsigned char *pdst = rec_of(j) + R_P;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int cc = col0 + 8 * u + 2 * i;
                            pk[i] = pack_bf16(cc <= r ? __uint_as_float(x[8 * u + 2 * i]) : 0.f,
                                              cc + 1 <= r ? __uint_as_float(x[8 * u + 2 * i + 1]) : 0.f);
                        }
                        *reinterpret_cast<uint4 *>(pdst + sw_off(r, col0 + 8 * u, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            }
            fence_before();
            group_sync(BAR_A, 256);
            if (tid == 0) mbar_arrive(misc + M1_AREADY);   // A is in the scratch, D1 may be overwritten
        }
    } else {
        // ------------------------------------------------------------------ solve group (warps 8-11)
        const int tb = tid - 256, wb = warp - 8;   // wb = TMEM lane quarter
        float *AS = reinterpret_cast<float *>(sm + P1_AS);
        for (int j = 0; j < njobs; ++j) {
            const int stg = j & 1;
            unsigned char *S = sm + stg * P1_STAGE;
            const uint32_t aEQ = smem_u32(S + P1_EQ), aU = smem_u32(S + P1_U), aW = smem_u32(S + P1_W);
            if (!gwait(misc + M1_AREADY, (uint32_t)(j & 1), BAR_B, 128, abort)) break;
            unsigned char *rec = rec_of(j);
            if (tb == 0) {   // K̃ and Q̂ are final: out by bulk copies while the chunk is solved
                bulk_s2g(rec + R_KT, smem_u32(S + P1_KT), 16384);
                bulk_s2g(rec + R_A3 + 8192, aEQ + 8192, 8192);       // Q̂: rows 64-127 of both column
                bulk_s2g(rec + R_A3 + 24576, aEQ + 24576, 8192);     // halves of [-W'; Q̂]
                if (aux) {   // Ê (rows 0-63 of both halves), for the backward
                    bulk_s2g(aux_of(j) + X_E, aEQ, 8192);
                    bulk_s2g(aux_of(j) + X_E + 8192, aEQ + 16384, 8192);
                }
            }
            // ---------------------------------------------------------------- T = (I + A)^-1, duplicated as [T; T]
            solve_unit_lower(AS, reinterpret_cast<float *>(sm + P1_X), S + P1_W, tb, BAR_B);
            group_sync(BAR_B, 128);
            if (tb == 0) mbar_arrive(misc + M1_ASFREE);   // the A scratch may take the next chunk-head's A
#pragma unroll
            for (int i = 0; i < 4; ++i) {   // rows 64-127 = rows 0-63: W' and Ũ land in all 128 TMEM lanes
                const int idx = tb + 128 * i;
                reinterpret_cast<uint4 *>(S + P1_W + 8192)[idx] = reinterpret_cast<const uint4 *>(S + P1_W)[idx];
            }
            fence_async_smem();
            group_sync(BAR_B, 128);
            // ---------------------------------------------------------------- G2: [W'; W'] = [T; T] Ê, [Ũ; Ũ] = [T; T] U
            if (tb == 0) {
                if (aux) bulk_s2g(aux_of(j) + X_T, aW, 8192);   // T, for the backward
                fence_after();
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    mma_ss(tmem + P1_TM_D2, desc_kmajor(aW, 128, jj), desc_mnmajor(aEQ, 128, jj), ID_G2, jj > 0);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    mma_ss(tmem + P1_TM_D3, desc_kmajor(aW, 128, jj), desc_mnmajor(aU, 64, jj), ID_G2, jj > 0);
                mma_commit(misc + M1_G2);
            }
            if (!gwait(misc + M1_G2, (uint32_t)(j & 1), BAR_B, 128, abort)) break;
            if (aux) {   // the copy of Ê has read rows 0-63 before -W' overwrites them
                if (tb == 0) {
                    bulk_commit();
                    bulk_wait_read_all();
                }
                group_sync(BAR_B, 128);
            }
            {   // lanes 0-63 (warps 8, 9): -W' rows into the [-W'; Q̂] tile; lanes 64-127 (warps 10, 11): the
                // same rows of Ũ into the U tile; bf16
                const int i = 32 * (wb & 1) + lane;
                const bool isW = wb < 2;
                const uint32_t src = tmem + ((uint32_t)(32 * wb) << 16) + (isW ? P1_TM_D2 : P1_TM_D3);
                unsigned char *dst = S + (isW ? P1_EQ : P1_U);
                const float sg = isW ? -1.f : 1.f;
#pragma unroll
                for (int u2 = 0; u2 < 4; u2 += 2) {
                    uint32_t x0[32], x1[32];
                    tmem_ld32(src + 32 * u2, x0);
                    tmem_ld32(src + 32 * u2 + 32, x1);
                    wait_ld();
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int cc = 32 * u2 + 8 * u;
                        const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
                        const uint4 pk = make_uint4(pack_bf16(sg * __uint_as_float(x[0]), sg * __uint_as_float(x[1])),
                                                    pack_bf16(sg * __uint_as_float(x[2]), sg * __uint_as_float(x[3])),
                                                    pack_bf16(sg * __uint_as_float(x[4]), sg * __uint_as_float(x[5])),
                                                    pack_bf16(sg * __uint_as_float(x[6]), sg * __uint_as_float(x[7])));
                        *reinterpret_cast<uint4 *>(dst + sw_off(i, cc, isW ? 128 : 64)) = pk;
                    }
                }
            }
            fence_async_smem();
            fence_before();
            group_sync(BAR_B, 128);
            if (tb == 0) {   // -W' (rows 0-63 of both column halves) and Ũ out; the stage is free once every
                             // store of the record has read it
                bulk_s2g(rec + R_A3, aEQ, 8192);
                bulk_s2g(rec + R_A3 + 16384, aEQ + 16384, 8192);
                bulk_s2g(rec + R_U, aU, 16384);
                bulk_commit();
                bulk_wait_read_all();
                if (j + 2 < njobs) {   // the stage is free: chunk-head j+2's tiles in
                    load_tiles(j + 2);
                    last_ld[stg] = j + 2;
                }
            }
        }
        if (tb == 0) {   // the record stores complete before the block exits
            bulk_commit();
            bulk_wait_all();
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0) {   // no tile or alpha load may be left in flight when the block exits (after an abort)
        for (int stg = 0; stg < 2; ++stg)
            if (last_ld[stg] >= 0) mbar_wait(misc + M1_FULL + 8 * stg, (uint32_t)((last_ld[stg] >> 1) & 1), WAIT_LIMIT);
        if (last_ld[2] >= 0) mbar_wait(misc + M1_AFULL, (uint32_t)(last_ld[2] & 1), WAIT_LIMIT);
        if (*abort) atomicOr(status, STATUS_PREP);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, P1_TM_COLS);
}

// ---------------------------------------------------------------------------- stage 2
// Warps 0-7 walk the chain: TMEM lane quarter w % 4, value-column half w / 4.  All eight rescale the
// state; warps 0, 1, 4, 5 (lanes 0-63) form Delta; warps 2, 3, 6, 7 (lanes 64-127) write the o rows
// of the previous chunk while Delta is formed.  Warp 8 issues the record copies.
constexpr int W2_NT = 288;
constexpr uint32_t W2_S = 0;                          // Z̃ bf16 [c x v] (MN-major B of G3)
constexpr uint32_t W2_DL = 32768;                     // Delta bf16 [i x v]
constexpr uint32_t W2_SLOT = 49152;                   // 2 record slots
constexpr uint32_t W2_OST = W2_SLOT + 2 * R_BYTES;    // o rows staged for the TMA store (16 KB)
constexpr uint32_t W2_MISC = W2_OST + 16384;
constexpr uint32_t W2_RMS = W2_MISC + 256;            // RMSNorm partial sums [64 rows][2 halves]
constexpr uint32_t W2_BYTES = W2_MISC + 768 + 1024;
// mbarriers: FULL and G45 per slot, G3
// G5 per slot completes before G4: the next chunk's rescale waits for G5 only, the o rows for G4/G5
enum : uint32_t { M2_FULL = 0, M2_G45 = 16, M2_G3 = 32, M2_ZST = 40, M2_G5 = 48, M2_TSLOT = 64, M2_ABORT = 68 };
constexpr uint32_t W2_TM_Z = 0, W2_TM_D3 = 128, W2_TM_COLS = 512;   // D3 buffers at 128 and 256
constexpr uint32_t BAR_ALL = 1, BAR_DELTA = 2, BAR_O = 3;            // named barriers (128 or 256 threads)

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

// o rows of one chunk (TMEM lanes 64-127 of its D3 buffer, value columns cb .. cb + 63) -> bf16 staging
// tile -> TMA store; rows past the end of the sequence are clipped by the copy.  ot: 0..127 over
// warps 2, 3, 6, 7.  With a weight (layer edges), each row passes RMSNorm first: the two column halves
// of a row sit in warps w and w + 4 and add their sums of squares through shared memory.
__device__ __forceinline__ void store_o(const CUtensorMap *map_o, unsigned char *sm, uint32_t d3, int ot, int r,
                                        int cb, int h, int t0, int bb, const float *onorm) {
    if (ot == 0) bulk_wait_read_all();   // the previous chunk's o store has read the staging tile
    group_sync(BAR_O, 128);
    uint32_t x0[32], x1[32];
    const uint32_t src = d3 + ((uint32_t)(64 + (r & ~31)) << 16) + cb;
    tmem_ld32(src, x0);
    tmem_ld32(src + 32, x1);
    wait_ld();
    if (onorm) {
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            ss += __uint_as_float(x0[i]) * __uint_as_float(x0[i]) + __uint_as_float(x1[i]) * __uint_as_float(x1[i]);
        float *part = reinterpret_cast<float *>(sm + W2_RMS);
        part[2 * r + (cb >> 6)] = ss;
        group_sync(BAR_O, 128);
        const float scale = rsqrtf((part[2 * r] + part[2 * r + 1]) * (1.f / VD) + EDGE_RMS_EPS);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            x0[i] = __float_as_uint(__uint_as_float(x0[i]) * scale * __ldg(onorm + cb + i));
            x1[i] = __float_as_uint(__uint_as_float(x1[i]) * scale * __ldg(onorm + cb + 32 + i));
        }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
        const uint4 pk = make_uint4(pack_bf16(__uint_as_float(x[0]), __uint_as_float(x[1])),
                                    pack_bf16(__uint_as_float(x[2]), __uint_as_float(x[3])),
                                    pack_bf16(__uint_as_float(x[4]), __uint_as_float(x[5])),
                                    pack_bf16(__uint_as_float(x[6]), __uint_as_float(x[7])));
        *reinterpret_cast<uint4 *>(sm + W2_OST + sw_off(r, cb + 8 * u, 64)) = pk;
    }
    fence_before();
    fence_async_smem();
    group_sync(BAR_O, 128);
    if (ot == 0) {
        tma_store_4d(map_o, 0, h, t0, bb, smem_u32(sm + W2_OST));
        tma_store_4d(map_o, 64, h, t0, bb, smem_u32(sm + W2_OST + 8192));
        bulk_commit();
    }
}


__global__ void __launch_bounds__(W2_NT, 1)
    walk_kernel(const __grid_constant__ CUtensorMap map_o, const unsigned char *records, unsigned char *aux,
                const float *S0, float *ST,
                int H, int T, int n0, int nw, int nseg, int seg_len, uint32_t flags, const float *onorm,
                unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chain = blockIdx.x / nseg, seg = blockIdx.x % nseg, bb = chain / H, h = chain % H;
    const int c0 = seg * seg_len, nc = min(nw, c0 + seg_len) - c0;   // this block's chunks of the window
    const bool zero_writes = (flags & WALK_ZERO_WRITES) != 0, store_out = (flags & WALK_SKIP_O) == 0;
    float *st_dst = (flags & WALK_ST_LAST) ? (seg == nseg - 1 ? ST + (size_t)chain * KD * VD : nullptr)
                                           : ST + (size_t)blockIdx.x * KD * VD;
    const uint32_t misc = smem_u32(sm + W2_MISC);
    volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sm + W2_MISC + M2_ABORT);

    if (warp == 0) tmem_alloc(misc + M2_TSLOT, W2_TM_COLS);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(misc + M2_FULL + 8 * s, 1);
            mbar_init(misc + M2_G45 + 8 * s, 1);
            mbar_init(misc + M2_G5 + 8 * s, 1);
        }
        mbar_init(misc + M2_G3, 1);
        mbar_init(misc + M2_ZST, 128);
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
    auto rec_of = [&](int nl) { return records + ((size_t)(bb * nw + c0 + nl) * H + h) * R_BYTES; };
    auto aux_of = [&](int nl) { return aux + ((size_t)(bb * nw + c0 + nl) * H + h) * X_BYTES; };

    if (warp < 8) {
        const int q4 = warp & 3, cb = 64 * (warp >> 2);   // TMEM lane quarter, value-column half
        const int crow = 32 * q4 + lane;                  // row c of Z (and row of D3)
        const uint32_t lq = (uint32_t)(32 * q4) << 16;
        const bool is_delta = q4 < 2;
        const int ot = 32 * (q4 - 2) + lane + 64 * (warp >> 2);   // o warps: 0..127
        {   // Z <- S0 (or 0, or I); the first rescale multiplies by chunk 0's exp(m)
            const float *src = S0 ? S0 + ((size_t)blockIdx.x * KD + crow) * VD + cb : nullptr;
            const bool ident = (flags & WALK_IDENTITY_S0) != 0;
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
                uint32_t r32[32];
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 x = src ? *reinterpret_cast<const float4 *>(src + 32 * u2 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                    r32[i] = __float_as_uint(x.x); r32[i + 1] = __float_as_uint(x.y);
                    r32[i + 2] = __float_as_uint(x.z); r32[i + 3] = __float_as_uint(x.w);
                }
                if (ident)
#pragma unroll
                    for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(cb + 32 * u2 + i == crow ? 1.f : 0.f);
                tmem_st32(tmem + lq + W2_TM_Z + cb + 32 * u2, r32);
            }
            wait_st();
        }
        float egm_prev = 1.f;
        bool ok = true;
        for (int nl = 0; nl < nc; ++nl) {
            const uint32_t slot = slot_addr(nl);
            // ---------------------------------------------------------------- record n in, chunk n-1 done
            {
                if (aux && tid == 0) bulk_wait_read_all();   // the copies of Z̃ and Delta have read them
                bool w_ok = mbar_wait(misc + M2_FULL + 8 * (nl & 1), (uint32_t)((nl >> 1) & 1), WAIT_LIMIT);
                if (nl > 0)
                    w_ok = w_ok && mbar_wait(misc + M2_G5 + 8 * ((nl - 1) & 1), (uint32_t)(((nl - 1) >> 1) & 1), WAIT_LIMIT);
                w_ok = w_ok && !*abort;
                const bool fail = group_or(BAR_ALL, 256, !w_ok);
                fence_after();
                if (fail) { *abort = 1u; ok = false; break; }
            }
            // ---------------------------------------------------------------- S_n = sPost_{n-1} Z; Z <- sZ_n S_n; Z̃ = bf16(sS_n S_n)
            // (the factors are applied one after the other: their product alone can lie below fp32's range)
            {
                const float *vec = reinterpret_cast<const float *>(sm + slot + R_VEC);
                const float post = egm_prev, ssc = vec[crow], zsc = vec[128 + crow];
                egm_prev = vec[256 + crow];
                uint32_t x0[32], x1[32];
                tmem_ld32(tmem + lq + W2_TM_Z + cb, x0);
                tmem_ld32(tmem + lq + W2_TM_Z + cb + 32, x1);
                wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x0[i] = __float_as_uint(post * __uint_as_float(x0[i]));
                    x1[i] = __float_as_uint(post * __uint_as_float(x1[i]));
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
                    const uint4 pk = make_uint4(pack_bf16(ssc * __uint_as_float(x[0]), ssc * __uint_as_float(x[1])),
                                                pack_bf16(ssc * __uint_as_float(x[2]), ssc * __uint_as_float(x[3])),
                                                pack_bf16(ssc * __uint_as_float(x[4]), ssc * __uint_as_float(x[5])),
                                                pack_bf16(ssc * __uint_as_float(x[6]), ssc * __uint_as_float(x[7])));
                    *reinterpret_cast<uint4 *>(sm + W2_S + sw_off(crow, cb + 8 * u, 128)) = pk;
                }
                // G3 needs only the bf16 copy: issue it first, then write Z back (G5, its next reader, is
                // issued once every thread's store is complete)
                fence_async_smem();
                fence_before();
                group_sync(BAR_ALL, 256);
                if (tid == 0) {   // G3: [-W'Z̃; Q̂Z̃] into this chunk's D3 buffer (its o rows of chunk n-2 are out)
                    fence_after();
                    const uint32_t aA3 = smem_u32(sm + slot + R_A3), aS = smem_u32(sm + W2_S);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        mma_ss(d3(nl), desc_kmajor(aA3, 128, j), desc_mnmajor(aS, 128, j), ID_G3, j > 0);
                    mma_commit(misc + M2_G3);
                    if (aux) {   // the state operand of the chunk, for the backward
                        bulk_s2g(aux_of(nl) + X_Z, aS, 32768);
                        bulk_commit();
                    }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x0[i] = __float_as_uint(zsc * __uint_as_float(x0[i]));
                    x1[i] = __float_as_uint(zsc * __uint_as_float(x1[i]));
                }
                tmem_st32(tmem + lq + W2_TM_Z + cb, x0);
                tmem_st32(tmem + lq + W2_TM_Z + cb + 32, x1);
                wait_st();
                fence_before();
                if (!is_delta) mbar_arrive(misc + M2_ZST);   // the o warps' rows of Z are written back
            }
            if (!is_delta) {
                // ------------------------------------------------------------ o rows of chunk n-1
                if (nl > 0 && store_out) {   // once G4 of chunk n-1 is complete
                    if (!group_wait2(misc + M2_G45 + 8 * ((nl - 1) & 1), (uint32_t)(((nl - 1) >> 1) & 1), BAR_O, 128, abort))
                        continue;
                    store_o(&map_o, sm, d3(nl - 1), ot, crow - 64, cb, h, (n0 + c0 + nl - 1) * C, bb, onorm);
                }
            } else {
                // ------------------------------------------------------------ Delta = Ũ - W'Z̃ -> bf16 tile; G4/G5
                const unsigned char *Ut = sm + slot + R_U;
                uint4 ut8[8];   // Ũ of this thread's row, read while G3 runs
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    ut8[u] = zero_writes ? make_uint4(0u, 0u, 0u, 0u)
                                         : *reinterpret_cast<const uint4 *>(Ut + sw_off(crow, cb + 8 * u, 64));
                if (!group_wait2(misc + M2_G3, (uint32_t)(nl & 1), BAR_DELTA, 128, abort)) continue;
                uint32_t x0[32], x1[32];
                tmem_ld32(d3(nl) + lq + cb, x0);
                tmem_ld32(d3(nl) + lq + cb + 32, x1);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int vv = cb + 8 * u;
                    const uint4 ut = ut8[u];
                    const float2 a = unpack2(ut.x), b2 = unpack2(ut.y), c2 = unpack2(ut.z), d2 = unpack2(ut.w);
                    const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
                    const uint4 pk = make_uint4(
                        pack_bf16(a.x + __uint_as_float(x[0]), a.y + __uint_as_float(x[1])),
                        pack_bf16(b2.x + __uint_as_float(x[2]), b2.y + __uint_as_float(x[3])),
                        pack_bf16(c2.x + __uint_as_float(x[4]), c2.y + __uint_as_float(x[5])),
                        pack_bf16(d2.x + __uint_as_float(x[6]), d2.y + __uint_as_float(x[7])));
                    *reinterpret_cast<uint4 *>(sm + W2_DL + sw_off(crow, vv, 64)) = pk;
                }
                fence_async_smem();
                fence_before();
                group_sync(BAR_DELTA, 128);
                if (aux && tid == 0) {   // Delta of the chunk, for the backward
                    bulk_s2g(aux_of(nl) + X_DL, smem_u32(sm + W2_DL), 16384);
                    bulk_commit();
                }
                if (tid == 0) {   // G4: O += P Delta (rows 0-63 of the A tile are Ũ's bytes: their products
                                  // land in the Delta rows of D3, already read); G5: Z += K̃^T Delta, once the
                                  // o warps' rows of Z are written back
                    const bool zs = thread_wait(misc + M2_ZST, (uint32_t)(nl & 1), abort);
                    fence_after();
                    if (zs) {
                    const uint32_t aPA = smem_u32(sm + slot + R_P - 8192), aKT = smem_u32(sm + slot + R_KT),
                                   aDL = smem_u32(sm + W2_DL);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_ss(tmem + W2_TM_Z, desc_mnmajor(aKT, 64, j), desc_mnmajor(aDL, 64, j), ID_G5, 1);
                    mma_commit(misc + M2_G5 + 8 * (nl & 1));
#pragma unroll
                    for (int j = 0; j < 4; ++j) mma_ss(d3(nl), desc_kmajor(aPA, 128, j), desc_mnmajor(aDL, 64, j), ID_G4, 1);
                    mma_commit(misc + M2_G45 + 8 * (nl & 1));
                    }
                }
            }
        }
        // the last chunk: its o rows, then S_T = Diag(sPost) Z, once its G4/G5 are complete
        ok = ok && nc > 0 &&
             group_wait2(misc + M2_G45 + 8 * ((nc - 1) & 1), (uint32_t)(((nc - 1) >> 1) & 1), BAR_ALL, 256, abort);
        if (ok && !is_delta && store_out) store_o(&map_o, sm, d3(nc - 1), ot, crow - 64, cb, h, (n0 + c0 + nc - 1) * C, bb, onorm);
        if (ok && st_dst) {
            float *dst = st_dst + (size_t)crow * VD + cb;
            uint32_t x0[32], x1[32];
            tmem_ld32(tmem + lq + W2_TM_Z + cb, x0);
            tmem_ld32(tmem + lq + W2_TM_Z + cb + 32, x1);
            wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                *reinterpret_cast<float4 *>(dst + i) =
                    make_float4(egm_prev * __uint_as_float(x0[i]), egm_prev * __uint_as_float(x0[i + 1]),
                                egm_prev * __uint_as_float(x0[i + 2]), egm_prev * __uint_as_float(x0[i + 3]));
                *reinterpret_cast<float4 *>(dst + 32 + i) =
                    make_float4(egm_prev * __uint_as_float(x1[i]), egm_prev * __uint_as_float(x1[i + 1]),
                                egm_prev * __uint_as_float(x1[i + 2]), egm_prev * __uint_as_float(x1[i + 3]));
            }
        }
        if (!is_delta && ot == 0) bulk_wait_all();   // the o stores complete before the block exits
        if (aux && tid == 0) bulk_wait_all();
    } else if (lane == 0) {
        // ------------------------------------------------------------------ producer: bulk copies per record
        // A walk that stores no o reads only -W' (rows 0-63 of both column halves of the G3 tile), K̃, Ũ
        // (not when the writes are off) and the factors: Q̂ and P feed only the o rows of D3, which it never
        // reads, so their products run on whatever the slot held before.
        const uint32_t part_ku = zero_writes ? 16384u : 32768u;
        const uint32_t bytes = store_out ? R_COPY : 2 * 8192u + part_ku + 3 * 128 * 4;
        for (int nl = 0; nl < nc; ++nl) {
            if (nl >= 2 && !thread_wait(misc + M2_G45 + 8 * (nl & 1), (uint32_t)(((nl - 2) >> 1) & 1), abort)) break;
            const uint32_t full = misc + M2_FULL + 8 * (nl & 1), dst = smem_u32(sm + slot_addr(nl));
            const unsigned char *src = rec_of(nl);
            mbar_arrive_expect_tx(full, bytes);
            if (store_out) {
                bulk_g2s(dst, src, R_COPY, full);
            } else {
                bulk_g2s(dst + R_A3, src + R_A3, 8192, full);
                bulk_g2s(dst + R_A3 + 16384, src + R_A3 + 16384, 8192, full);
                bulk_g2s(dst + R_KT, src + R_KT, part_ku, full);   // K̃, and Ũ right after it
                bulk_g2s(dst + R_VEC, src + R_VEC, 3 * 128 * 4, full);
            }
        }
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

}  // namespace

bool token_map(CUtensorMap *m, const void *base, int B, int T, int H, bool fp32) {
    const EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es_bytes = fp32 ? 4 : 2;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * es_bytes, 128 * es_bytes * H, 128 * es_bytes * H * T};
    const cuuint32_t box[4] = {fp32 ? 128u : 64u, 1, 64, 1}, es[4] = {1, 1, 1, 1};
    return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              fp32 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

namespace {

// Plan of a two-stage call.  The record buffer holds one window of chunks of every chain (at most
// 16,384 chunk-heads, 1.24 GB, and at least 64 chunks).  With few chains (B*H <= 64) each chain's
// window is cut into nseg segments walked in parallel: each segment's state map S_out = M S_in + N is
// found by two walks over its records (N from S_in = 0, M from S_in = I with the writes switched
// off), the maps are composed along the chain in fp32, and a final walk runs every segment from its
// true start state.
struct SplitPlan {
    int nw;     // chunks per window
    int nseg;   // segments per chain in a full window (1: plain walk)
};
// CTAs the segmented walks may use: one per SM of the B200 (148), so that every segment's walk runs at once.
constexpr int kSegCtas = 148;
SplitPlan split_plan(int B, int H, int T) {
    const int chains = B * H, NC = (T + split::C - 1) / split::C;
    int nw = chains > 0 ? std::max(64, 16384 / chains) : 64;
    nw = std::min(nw, std::max(NC, 1));
    int nseg = 1;
    if (chains <= 64 && nw >= 32) nseg = std::max(1, std::min(kSegCtas / std::max(chains, 1), nw / 8));
    return {nw, nseg};
}
constexpr size_t kStateBytes = sizeof(float) * 128 * 128;
// segments per chain of the backward's forward replay (one window of the whole sequence)
int replay_segments(int chains, int NC) {
    if (chains > 64 || NC < 32) return 1;
    return std::max(1, std::min(kSegCtas / std::max(chains, 1), NC / 8));
}

}  // namespace

size_t split_workspace_bytes(int B, int H, int T) {
    const SplitPlan p = split_plan(B, H, T);
    const size_t seg = p.nseg > 1 ? 3 * kStateBytes * (size_t)B * H * p.nseg : 0;
    return kStatusBytes + (size_t)B * H * p.nw * split::R_BYTES + seg;
}

int launch_chunk_split(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                       const float *S0, void *o, float *ST, int B, int H, int T, void *ws, cudaStream_t st, int edges,
                       const float *onorm) {
    split::TokMaps maps;
    CUtensorMap map_o;
    if (!token_map(&maps.q, q, B, T, H) || !token_map(&maps.k, k, B, T, H) || !token_map(&maps.b, b, B, T, H) ||
        !token_map(&maps.v, v, B, T, H) || !token_map(&maps.w, w, B, T, H) ||
        !token_map(&maps.alpha, alpha, B, T, H, true) || !token_map(&map_o, o, B, T, H))
        return -6;
    const int smem1 = (int)split::P1_BYTES, smem2 = (int)split::W2_BYTES;
    auto prep = edges ? split::prep_kernel<true> : split::prep_kernel<false>;
    if (!edges) onorm = nullptr;
    if (cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1) != cudaSuccess ||
        cudaFuncSetAttribute(split::walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2) != cudaSuccess)
        return -6;
    const int nsm = sm_count();
    if (nsm <= 0) return -6;
    const SplitPlan plan = split_plan(B, H, T);
    const int chains = B * H, NC = (T + split::C - 1) / split::C;
    unsigned int *status = reinterpret_cast<unsigned int *>(ws);
    unsigned char *records = static_cast<unsigned char *>(ws) + kStatusBytes;
    float *Nm = reinterpret_cast<float *>(records + (size_t)chains * plan.nw * split::R_BYTES);
    float *Mm = Nm + (size_t)chains * plan.nseg * 128 * 128, *Sg = Mm + (size_t)chains * plan.nseg * 128 * 128;
    for (int n0 = 0; n0 < NC; n0 += plan.nw) {
        const int nw = std::min(plan.nw, NC - n0), nch = chains * nw;
        const float *s_in = n0 == 0 ? S0 : ST;
        prep<<<std::min(nch, nsm), split::P1_NT, smem1, st>>>(
            maps, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)b, alpha, records, nullptr,
            H, T, n0, nw, nch, status);
        int nseg = plan.nseg > 1 && nw >= 16 ? std::min(plan.nseg, nw / 8) : 1;
        if (nseg <= 1) {
            split::walk_kernel<<<chains, split::W2_NT, smem2, st>>>(map_o, records, nullptr, s_in, ST, H, T, n0, nw, 1,
                                                                    nw, 0u, onorm, status);
            continue;
        }
        const int seg_len = (nw + nseg - 1) / nseg;
        nseg = (nw + seg_len - 1) / seg_len;   // every segment non-empty
        const uint32_t skip = split::WALK_SKIP_O;
        split::walk_kernel<<<chains * nseg, split::W2_NT, smem2, st>>>(map_o, records, nullptr, nullptr, Nm, H, T, n0,
                                                                       nw, nseg, seg_len, skip, onorm, status);
        split::walk_kernel<<<chains * nseg, split::W2_NT, smem2, st>>>(
            map_o, records, nullptr, nullptr, Mm, H, T, n0, nw, nseg, seg_len,
            skip | split::WALK_ZERO_WRITES | split::WALK_IDENTITY_S0, onorm, status);
        const int rc = launch_segment_scan(Mm, Nm, s_in, Sg, chains, nseg, st);
        if (rc != 0) return rc;
        split::walk_kernel<<<chains * nseg, split::W2_NT, smem2, st>>>(map_o, records, nullptr, Sg, ST, H, T, n0, nw,
                                                                       nseg, seg_len, split::WALK_ST_LAST, onorm, status);
    }
    return launch_status();
}

// Forward replay for the backward: the two stages over the whole sequence at once (one window), o not
// stored, every chunk-head's side record filled (Ê, T and the frame exponents by the first stage, Z̃ and
// Delta by the final walk), S_T written.  Few long chains walk in segments as in the prefill.
size_t replay_segment_bytes(int B, int H, int T) {
    const int chains = B * H, NC = (T + split::C - 1) / split::C;
    const int nseg = replay_segments(chains, NC);
    return nseg > 1 ? 3 * kStateBytes * (size_t)chains * nseg : 0;
}

int launch_split_replay(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                        const float *S0, float *ST, int B, int H, int T, unsigned char *records, unsigned char *aux,
                        float *seg, const CUtensorMap &any_map, unsigned int *status, cudaStream_t st) {
    split::TokMaps maps;
    if (!token_map(&maps.q, q, B, T, H) || !token_map(&maps.k, k, B, T, H) || !token_map(&maps.b, b, B, T, H) ||
        !token_map(&maps.v, v, B, T, H) || !token_map(&maps.w, w, B, T, H) ||
        !token_map(&maps.alpha, alpha, B, T, H, true))
        return -6;
    const int smem1 = (int)split::P1_BYTES, smem2 = (int)split::W2_BYTES;
    if (cudaFuncSetAttribute(split::prep_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1) != cudaSuccess ||
        cudaFuncSetAttribute(split::walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2) != cudaSuccess)
        return -6;
    const int nsm = sm_count();
    if (nsm <= 0) return -6;
    const int chains = B * H, NC = (T + split::C - 1) / split::C, nch = chains * NC;
    split::prep_kernel<false, true><<<std::min(nch, nsm), split::P1_NT, smem1, st>>>(
        maps, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)b, alpha, records, aux, H, T,
        0, NC, nch, status);
    int nseg = replay_segments(chains, NC);
    const uint32_t skip = split::WALK_SKIP_O;
    if (nseg <= 1) {
        split::walk_kernel<<<chains, split::W2_NT, smem2, st>>>(any_map, records, aux, S0, ST, H, T, 0, NC, 1, NC, skip,
                                                                nullptr, status);
        return launch_status();
    }
    const int seg_len = (NC + nseg - 1) / nseg;
    nseg = (NC + seg_len - 1) / seg_len;
    float *Nm = seg, *Mm = Nm + (size_t)chains * nseg * 128 * 128, *Sg = Mm + (size_t)chains * nseg * 128 * 128;
    split::walk_kernel<<<chains * nseg, split::W2_NT, smem2, st>>>(any_map, records, nullptr, nullptr, Nm, H, T, 0, NC,
                                                                   nseg, seg_len, skip, nullptr, status);
    split::walk_kernel<<<chains * nseg, split::W2_NT, smem2, st>>>(
        any_map, records, nullptr, nullptr, Mm, H, T, 0, NC, nseg, seg_len,
        skip | split::WALK_ZERO_WRITES | split::WALK_IDENTITY_S0, nullptr, status);
    const int rc = launch_segment_scan(Mm, Nm, S0, Sg, chains, nseg, st);
    if (rc != 0) return rc;
    split::walk_kernel<<<chains * nseg, split::W2_NT, smem2, st>>>(any_map, records, aux, Sg, ST, H, T, 0, NC, nseg,
                                                                   seg_len, skip | split::WALK_ST_LAST, nullptr, status);
    return launch_status();
}

}  // namespace gdn2
