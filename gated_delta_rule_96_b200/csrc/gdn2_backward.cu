// Backward pass of the GDN-2 recurrence (page "NVIDIA представила Gated DeltaNet-2 ...",
// section "Техническая схема": the state-update equation; the page's remark that the
// gradients must account for the per-channel gates).
//
// Given dO_t = dL/do_t and dS_T = dL/dS_T, the gradients of every input follow from the
// chain rule of one step, walked in reverse (e = b ⊙ k, u = w ⊙ v, Sbar_t = Diag(alpha_t)
// S_{t-1}, delta_t = u_t - Sbar_t^T e_t, G_t = dL/dS_t):
//
//   ddelta_t = G_t^T k_t            dv = w ⊙ ddelta, dw = v ⊙ ddelta
//   de_t = -Sbar_t ddelta_t         db = k ⊙ de
//   dk_t = G_t delta_t + b ⊙ de     dq_t = S_t dO_t
//   G_{t-1} = Diag(alpha_t)(G_t - e_t ddelta_t^T) + q_{t-1} dO_{t-1}^T,   dS0 = G_0
//
// Two observations shape the kernels.
//  * G's recurrence does not involve S (the update is linear in S), and S's does not
//    involve G.  So there is no need to hold S and G at the same step: three sequential
//    passes over the sequence, each carrying ONE d_k x d_v matrix in registers, do the
//    work: (1) forward over S: delta_t (kept) and dq_t = S_t dO_t, S at every chunk end;
//    (2) reverse over G: ddelta_t (kept), dv, dw, G_t delta_t, dS0; (3) forward over S
//    again: S_{t-1} ddelta_t, hence de, db and the complete dk.
//  * The decay gradient needs no state-sized product per step.  The loss depends on the
//    cumulative log-decay g_t = sum_{j<=t} log alpha_j only through exp(g_t) q_t,
//    exp(g_t) e_t and exp(-g_t) k_t (the chunkwise form of the recurrence with one chunk
//    spanning the sequence), so dL/dg_t = q ⊙ dq + e ⊙ de - k ⊙ (dk - b ⊙ de); and scaling
//    alpha_{s+1} is scaling S_s, so summing those from a chunk end s back to position j
//    gives d log alpha_j once rowsum(G_s^fut ⊙ S_s) is added, G_s^fut being dL/dS_s from
//    the steps after s.  Sums therefore run over at most one chunk (64 steps), from an
//    exact boundary term that pass (2) forms from the pass (1) state.
//
// Layout (one CTA per (b, h) chain, d_v / 8 warps): warp w owns the value columns
// 8w .. 8w+7 of the carried matrix, lane l the key rows KR*l .. KR*l+KR-1 (KR = d_k / 32);
// the matrix lives in registers.  Column sums over the key axis (feeding the recurrence)
// stay inside the warp (a shuffle reduce-scatter); row sums over the value axis (outputs
// only) go through shared memory and are flushed every NB steps.
#include <float.h>

#include "gdn2_common.cuh"
#include "gdn2_internal.h"

namespace gdn2 {
namespace bwd {

constexpr int C = 64;    // chunk length: checkpoint spacing and the span of the log-decay sums
constexpr int NB = 16;   // steps per flush of the row sums (divides C)
constexpr int PF = 16;   // steps of look-ahead for the L2 prefetch
static_assert(C % NB == 0, "chunk ends must be flush ends");

__device__ __forceinline__ float2 bf2(uint32_t u) {
    __nv_bfloat162 p = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return make_float2(__low2float(p), __high2float(p));
}

// KR consecutive token values (a lane's rows) as fp32
template <int KR>
__device__ __forceinline__ void ld_rows(const float *p, float (&x)[KR]) {
    if constexpr (KR == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    } else {
        const float2 a = __ldg(reinterpret_cast<const float2 *>(p));
        x[0] = a.x; x[1] = a.y;
    }
}
template <int KR>
__device__ __forceinline__ void ld_rows(const __nv_bfloat16 *p, float (&x)[KR]) {
    if constexpr (KR == 4) {
        const uint2 a = __ldg(reinterpret_cast<const uint2 *>(p));
        const float2 l = bf2(a.x), h = bf2(a.y);
        x[0] = l.x; x[1] = l.y; x[2] = h.x; x[3] = h.y;
    } else {
        const float2 l = bf2(__ldg(reinterpret_cast<const unsigned int *>(p)));
        x[0] = l.x; x[1] = l.y;
    }
}
// 8 consecutive values (a warp's columns) as fp32; every lane reads the same address
__device__ __forceinline__ void ld_cols8(const float *p, float (&x)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void ld_cols8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const float2 f0 = bf2(a.x), f1 = bf2(a.y), f2 = bf2(a.z), f3 = bf2(a.w);
    x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y; x[4] = f2.x; x[5] = f2.y; x[6] = f3.x; x[7] = f3.y;
}
// fp32 values written by an earlier pass of the same call (plain loads: not read-only data)
__device__ __forceinline__ void ld_ws8(const float *p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Sum over the 32 lanes of eight per-lane values p[0..7]; lane l receives the sum of
// p[(l >> 2) & 7].  Lanes differing in bit 4, then 3, then 2 exchange half of what they
// hold (4, 2, 1 values), then bits 1 and 0 finish: 9 shuffles instead of 40.
__device__ __forceinline__ float warp_colsum8(const float (&p)[8], int lane) {
    const bool h4 = (lane & 16) != 0, h3 = (lane & 8) != 0, h2 = (lane & 4) != 0;
    float a[4], c[2];
#pragma unroll
    for (int m = 0; m < 4; ++m)
        a[m] = (h4 ? p[m + 4] : p[m]) + __shfl_xor_sync(0xffffffffu, h4 ? p[m] : p[m + 4], 16);
#pragma unroll
    for (int m = 0; m < 2; ++m)
        c[m] = (h3 ? a[m + 2] : a[m]) + __shfl_xor_sync(0xffffffffu, h3 ? a[m] : a[m + 2], 8);
    float s = (h2 ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, h2 ? c[0] : c[1], 4);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    return s;
}

__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
// lane i of the calling warp prefetches the i-th 128-byte line of [p, p + bytes)
__device__ __forceinline__ void prefetch_row(const void *p, int bytes, int lane) {
    if (lane * 128 < bytes) prefetch_l2(static_cast<const char *>(p) + lane * 128);
}

__device__ __forceinline__ bool chunk_end(int t, int T) { return t == T - 1 || (t + 1) % C == 0; }

// Row sums of NB buffered steps: red[s][w][c] summed over the warps w.
template <int K, int NW>
__device__ __forceinline__ float red_sum(const float *red, int s, int c) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) acc += red[(s * NW + w) * K + c];
    return acc;
}

template <int KR>
__device__ __forceinline__ void st_red(float *red, int slot, int NW, int K, int warp, int r0, const float (&x)[KR]) {
    float *p = red + (slot * NW + warp) * K + r0;
    if constexpr (KR == 4) *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}

// ------------------------------------------------------------------------------------ pass 1
// Forward over S: delta_t -> workspace, dq_t = S_t dO_t -> dq, S at every chunk end -> ckpt.
template <int KR, int NW, typename Tok>
__global__ void __launch_bounds__(NW * 32, 1)
pass_forward(const Tok *__restrict__ k, const Tok *__restrict__ v, const float *__restrict__ alpha,
             const Tok *__restrict__ b, const Tok *__restrict__ w, const float *__restrict__ S0,
             const Tok *__restrict__ dO, float *__restrict__ dq, float *__restrict__ delta,
             float *__restrict__ ckpt, int H, int T, int NC) {
    constexpr int K = 32 * KR, V = 8 * NW, NT = NW * 32;
    extern __shared__ float red[];   // [NB][NW][K]
    const int chain = blockIdx.x, bb = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = KR * lane, c0 = 8 * warp, jm = (lane >> 2) & 7;

    float S[KR][8];
#pragma unroll
    for (int i = 0; i < KR; ++i) {
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (S0) ld_cols8(S0 + ((size_t)chain * K + r0 + i) * V + c0, x);
#pragma unroll
        for (int j = 0; j < 8; ++j) S[i][j] = x[j];
    }
    struct In { float al[KR], kk[KR], e[KR], u, g[8]; };
    auto load = [&](In &in, int t) {
        const size_t row = ((size_t)bb * T + t) * H + h;
        float bk[KR];
        ld_rows<KR>(alpha + row * K + r0, in.al);
        ld_rows<KR>(k + row * K + r0, in.kk);
        ld_rows<KR>(b + row * K + r0, bk);
#pragma unroll
        for (int i = 0; i < KR; ++i) in.e[i] = bk[i] * in.kk[i];
        in.u = to_f32(w[row * V + c0 + jm]) * to_f32(v[row * V + c0 + jm]);
        ld_cols8(dO + row * V + c0, in.g);
    };
    In cur, nxt;
    if (T > 0) load(cur, 0);
    for (int t = 0; t < T; ++t) {
        if (t + 1 < T) load(nxt, t + 1);
        if (warp == 0 && t + PF < T) {
            const size_t row = ((size_t)bb * T + t + PF) * H + h;
            prefetch_row(alpha + row * K, K * 4, lane);
            prefetch_row(k + row * K, K * (int)sizeof(Tok), lane);
            prefetch_row(b + row * K, K * (int)sizeof(Tok), lane);
            prefetch_row(v + row * V, V * (int)sizeof(Tok), lane);
            prefetch_row(w + row * V, V * (int)sizeof(Tok), lane);
            prefetch_row(dO + row * V, V * (int)sizeof(Tok), lane);
        }
        // Sbar = Diag(alpha) S; r = Sbar^T e (column sums); delta = u - r
        float pr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            pr[j] = 0.f;
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                S[i][j] *= cur.al[i];
                pr[j] = fmaf(S[i][j], cur.e[i], pr[j]);
            }
        }
        const float dmine = cur.u - warp_colsum8(pr, lane);
        const size_t rowt = ((size_t)bb * T + t) * H + h;
        if ((lane & 3) == 0) delta[rowt * V + c0 + jm] = dmine;
        float d[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) d[j] = __shfl_sync(0xffffffffu, dmine, 4 * j);
        // S_t = Sbar + k delta^T; row sums of S_t dO_t
        float x[KR];
#pragma unroll
        for (int i = 0; i < KR; ++i) {
            x[i] = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                S[i][j] = fmaf(cur.kk[i], d[j], S[i][j]);
                x[i] = fmaf(S[i][j], cur.g[j], x[i]);
            }
        }
        const int slot = t % NB;
        st_red<KR>(red, slot, NW, K, warp, r0, x);
        if (chunk_end(t, T)) {
            float *ck = ckpt + ((size_t)chain * NC + t / C) * K * V;
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                float4 *p = reinterpret_cast<float4 *>(ck + (size_t)(r0 + i) * V + c0);
                p[0] = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
                p[1] = make_float4(S[i][4], S[i][5], S[i][6], S[i][7]);
            }
        }
        if (slot == NB - 1 || t == T - 1) {
            __syncthreads();
            const int t0 = t - slot;
            for (int idx = tid; idx < (slot + 1) * K; idx += NT) {
                const int s = idx / K, c = idx % K;
                dq[(((size_t)bb * T + t0 + s) * H + h) * K + c] = red_sum<K, NW>(red, s, c);
            }
            __syncthreads();
        }
        cur = nxt;
    }
}

// ------------------------------------------------------------------------------------ pass 2
// Reverse over G: ddelta_t -> workspace, dv, dw, dk_t = G_t delta_t (completed by pass 3),
// rowsum(G^fut ⊙ S) at every chunk end -> bnd, dS0 = G_0.
template <int KR, int NW, typename Tok>
__global__ void __launch_bounds__(NW * 32, 1)
pass_reverse(const Tok *__restrict__ q, const Tok *__restrict__ k, const Tok *__restrict__ v,
             const float *__restrict__ alpha, const Tok *__restrict__ b, const Tok *__restrict__ w,
             const Tok *__restrict__ dO, const float *__restrict__ dST, const float *__restrict__ delta,
             const float *__restrict__ ckpt, float *__restrict__ ddelta, float *__restrict__ bnd,
             float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dw, float *__restrict__ dS0,
             int H, int T, int NC) {
    constexpr int K = 32 * KR, V = 8 * NW, NT = NW * 32;
    extern __shared__ float red[];   // [NB][NW][K], then [NW][K] for the chunk-end sums
    float *rbnd = red + NB * NW * K;
    const int chain = blockIdx.x, bb = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = KR * lane, c0 = 8 * warp, jm = (lane >> 2) & 7;

    float G[KR][8];
#pragma unroll
    for (int i = 0; i < KR; ++i) {
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (dST) ld_cols8(dST + ((size_t)chain * K + r0 + i) * V + c0, x);
#pragma unroll
        for (int j = 0; j < 8; ++j) G[i][j] = x[j];
    }
    struct In { float al[KR], kk[KR], e[KR], qq[KR], g[8], dl[8], vm, wm; };
    auto load = [&](In &in, int t) {
        const size_t row = ((size_t)bb * T + t) * H + h;
        float bk[KR];
        ld_rows<KR>(alpha + row * K + r0, in.al);
        ld_rows<KR>(k + row * K + r0, in.kk);
        ld_rows<KR>(b + row * K + r0, bk);
        ld_rows<KR>(q + row * K + r0, in.qq);
#pragma unroll
        for (int i = 0; i < KR; ++i) in.e[i] = bk[i] * in.kk[i];
        ld_cols8(dO + row * V + c0, in.g);
        ld_ws8(delta + row * V + c0, in.dl);
        in.vm = to_f32(v[row * V + c0 + jm]);
        in.wm = to_f32(w[row * V + c0 + jm]);
    };
    In cur, nxt;
    if (T > 0) load(cur, T - 1);
    for (int t = T - 1; t >= 0; --t) {
        if (t > 0) load(nxt, t - 1);
        if (warp == 0 && t - PF >= 0) {
            const size_t row = ((size_t)bb * T + t - PF) * H + h;
            prefetch_row(alpha + row * K, K * 4, lane);
            prefetch_row(k + row * K, K * (int)sizeof(Tok), lane);
            prefetch_row(b + row * K, K * (int)sizeof(Tok), lane);
            prefetch_row(q + row * K, K * (int)sizeof(Tok), lane);
            prefetch_row(v + row * V, V * (int)sizeof(Tok), lane);
            prefetch_row(w + row * V, V * (int)sizeof(Tok), lane);
            prefetch_row(dO + row * V, V * (int)sizeof(Tok), lane);
            prefetch_row(delta + row * V, V * 4, lane);
        }
        if (chunk_end(t, T)) {   // G here is dL/dS_t from the steps after t
            const int ci = t / C;
            const float *ck = ckpt + ((size_t)chain * NC + ci) * K * V;
            float y[KR];
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                float s[8];
                ld_ws8(ck + (size_t)(r0 + i) * V + c0, s);
                y[i] = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) y[i] = fmaf(G[i][j], s[j], y[i]);
            }
            st_red<KR>(rbnd, 0, NW, K, warp, r0, y);
            __syncthreads();
            for (int c = tid; c < K; c += NT) bnd[((size_t)chain * NC + ci) * K + c] = red_sum<K, NW>(rbnd, 0, c);
            __syncthreads();
        }
        // o_t = S_t^T q_t: G_t += q_t dO_t^T; ddelta = G_t^T k_t (column sums)
        float pr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            pr[j] = 0.f;
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                G[i][j] = fmaf(cur.qq[i], cur.g[j], G[i][j]);
                pr[j] = fmaf(G[i][j], cur.kk[i], pr[j]);
            }
        }
        const float ddm = warp_colsum8(pr, lane);
        const size_t rowt = ((size_t)bb * T + t) * H + h;
        if ((lane & 3) == 0) {
            ddelta[rowt * V + c0 + jm] = ddm;
            dv[rowt * V + c0 + jm] = ddm * cur.wm;
            dw[rowt * V + c0 + jm] = ddm * cur.vm;
        }
        float dd[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) dd[j] = __shfl_sync(0xffffffffu, ddm, 4 * j);
        // row sums of G_t delta_t; G_{t-1} = Diag(alpha_t)(G_t - e_t ddelta_t^T)
        float x[KR];
#pragma unroll
        for (int i = 0; i < KR; ++i) {
            x[i] = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                x[i] = fmaf(G[i][j], cur.dl[j], x[i]);
                G[i][j] = cur.al[i] * fmaf(-cur.e[i], dd[j], G[i][j]);
            }
        }
        const int slot = (T - 1 - t) % NB;
        st_red<KR>(red, slot, NW, K, warp, r0, x);
        if (slot == NB - 1 || t == 0) {
            __syncthreads();
            const int tf = t + slot;   // step of slot 0 (the latest of the group)
            for (int idx = tid; idx < (slot + 1) * K; idx += NT) {
                const int s = idx / K, c = idx % K;
                dk[(((size_t)bb * T + tf - s) * H + h) * K + c] = red_sum<K, NW>(red, s, c);
            }
            __syncthreads();
        }
        cur = nxt;
    }
    if (dS0) {
#pragma unroll
        for (int i = 0; i < KR; ++i) {
            float4 *p = reinterpret_cast<float4 *>(dS0 + ((size_t)chain * K + r0 + i) * V + c0);
            p[0] = make_float4(G[i][0], G[i][1], G[i][2], G[i][3]);
            p[1] = make_float4(G[i][4], G[i][5], G[i][6], G[i][7]);
        }
    }
}

// ------------------------------------------------------------------------------------ pass 3
// Forward over S with the kept delta: S_{t-1} ddelta_t gives de = -alpha ⊙ (S_{t-1} ddelta);
// then db, the complete dk, and per chunk the log-decay sums -> dalpha.
template <int KR, int NW, typename Tok>
__global__ void __launch_bounds__(NW * 32, 1)
pass_gates(const Tok *__restrict__ q, const Tok *__restrict__ k, const float *__restrict__ alpha,
           const Tok *__restrict__ b, const float *__restrict__ S0, const float *__restrict__ delta,
           const float *__restrict__ ddelta, const float *__restrict__ bnd, const float *__restrict__ dq,
           float *__restrict__ dk, float *__restrict__ db, float *__restrict__ dalpha, int H, int T, int NC) {
    constexpr int K = 32 * KR, V = 8 * NW, NT = NW * 32;
    extern __shared__ float red[];   // [NB][NW][K], then the chunk's dL/dg rows [C][K]
    float *hbuf = red + NB * NW * K;
    const int chain = blockIdx.x, bb = chain / H, h = chain % H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = KR * lane, c0 = 8 * warp;

    float S[KR][8];
#pragma unroll
    for (int i = 0; i < KR; ++i) {
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (S0) ld_cols8(S0 + ((size_t)chain * K + r0 + i) * V + c0, x);
#pragma unroll
        for (int j = 0; j < 8; ++j) S[i][j] = x[j];
    }
    struct In { float al[KR], kk[KR], dl[8], dd[8]; };
    auto load = [&](In &in, int t) {
        const size_t row = ((size_t)bb * T + t) * H + h;
        ld_rows<KR>(alpha + row * K + r0, in.al);
        ld_rows<KR>(k + row * K + r0, in.kk);
        ld_ws8(delta + row * V + c0, in.dl);
        ld_ws8(ddelta + row * V + c0, in.dd);
    };
    In cur, nxt;
    if (T > 0) load(cur, 0);
    for (int t = 0; t < T; ++t) {
        if (t + 1 < T) load(nxt, t + 1);
        if (warp == 0 && t + PF < T) {
            const size_t row = ((size_t)bb * T + t + PF) * H + h;
            prefetch_row(alpha + row * K, K * 4, lane);
            prefetch_row(k + row * K, K * (int)sizeof(Tok), lane);
            prefetch_row(delta + row * V, V * 4, lane);
            prefetch_row(ddelta + row * V, V * 4, lane);
        }
        float x[KR];
#pragma unroll
        for (int i = 0; i < KR; ++i) {
            x[i] = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                x[i] = fmaf(S[i][j], cur.dd[j], x[i]);                        // S_{t-1} ddelta_t
                S[i][j] = fmaf(cur.kk[i], cur.dl[j], cur.al[i] * S[i][j]);   // S_t
            }
        }
        const int slot = t % NB;
        st_red<KR>(red, slot, NW, K, warp, r0, x);
        if (slot == NB - 1 || t == T - 1) {
            __syncthreads();
            const int t0 = t - slot;
            for (int idx = tid; idx < (slot + 1) * K; idx += NT) {
                const int s = idx / K, c = idx % K;
                const size_t e = (((size_t)bb * T + t0 + s) * H + h) * K + c;
                const float a = alpha[e], kc = to_f32(k[e]), bc = to_f32(b[e]), qc = to_f32(q[e]);
                const float de = -a * red_sum<K, NW>(red, s, c);
                const float dkt = dk[e] + bc * de;
                dk[e] = dkt;
                db[e] = kc * de;
                // dL/dg_t = q dq + e de - k (dk - b de)
                hbuf[((t0 + s) % C) * K + c] = qc * dq[e] + 2.f * bc * kc * de - kc * dkt;
            }
            __syncthreads();
            if (chunk_end(t, T)) {
                const int ci = t / C, cs = ci * C;
                for (int c = tid; c < K; c += NT) {
                    float acc = bnd[((size_t)chain * NC + ci) * K + c];
                    for (int s = t - cs; s >= 0; --s) {
                        acc += hbuf[s * K + c];
                        const size_t e = (((size_t)bb * T + cs + s) * H + h) * K + c;
                        dalpha[e] = acc / fmaxf(alpha[e], FLT_MIN);
                    }
                }
                __syncthreads();
            }
        }
        cur = nxt;
    }
}

template <int KR, int NW, typename Tok>
int launch_all(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
               const float *S0, const void *dO, const float *dST, float *dq, float *dk, float *dv, float *dalpha,
               float *db, float *dw, float *dS0, int B, int H, int T, float *delta, float *ddelta, float *ckpt,
               float *bnd, cudaStream_t st) {
    constexpr int K = 32 * KR;
    const int NC = (T + C - 1) / C, NT = NW * 32, grid = B * H;
    const size_t red_bytes = sizeof(float) * NB * NW * K;
    const size_t sm1 = red_bytes, sm2 = red_bytes + sizeof(float) * NW * K, sm3 = red_bytes + sizeof(float) * C * K;
    auto f1 = pass_forward<KR, NW, Tok>;
    auto f2 = pass_reverse<KR, NW, Tok>;
    auto f3 = pass_gates<KR, NW, Tok>;
    if (cudaFuncSetAttribute(f1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1) != cudaSuccess ||
        cudaFuncSetAttribute(f2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2) != cudaSuccess ||
        cudaFuncSetAttribute(f3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3) != cudaSuccess)
        return -6;
    const Tok *tq = static_cast<const Tok *>(q), *tk = static_cast<const Tok *>(k), *tv = static_cast<const Tok *>(v);
    const Tok *tb = static_cast<const Tok *>(b), *tw = static_cast<const Tok *>(w), *tdo = static_cast<const Tok *>(dO);
    f1<<<grid, NT, sm1, st>>>(tk, tv, alpha, tb, tw, S0, tdo, dq, delta, ckpt, H, T, NC);
    f2<<<grid, NT, sm2, st>>>(tq, tk, tv, alpha, tb, tw, tdo, dST, delta, ckpt, ddelta, bnd, dk, dv, dw, dS0, H, T,
                              NC);
    f3<<<grid, NT, sm3, st>>>(tq, tk, alpha, tb, S0, delta, ddelta, bnd, dq, dk, db, dalpha, H, T, NC);
    return launch_status();
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace bwd

size_t bwd_workspace_bytes(int B, int H, int T, int K, int V) {
    const size_t ntok = (size_t)B * T * H, NC = (size_t)(T + bwd::C - 1) / bwd::C;
    return 2 * bwd::align256(sizeof(float) * ntok * V) + bwd::align256(sizeof(float) * B * H * NC * K * V) +
           bwd::align256(sizeof(float) * B * H * NC * K);
}

int launch_chunk_bwd(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                     const float *S0, const void *dO, const float *dST, float *dq, float *dk, float *dv,
                     float *dalpha, float *db, float *dw, float *dS0, int B, int H, int T, int K, int V, int bf16,
                     void *ws, cudaStream_t st) {
    const size_t ntok = (size_t)B * T * H, NC = (size_t)(T + bwd::C - 1) / bwd::C;
    char *p = static_cast<char *>(ws);
    float *delta = reinterpret_cast<float *>(p);
    p += bwd::align256(sizeof(float) * ntok * V);
    float *ddelta = reinterpret_cast<float *>(p);
    p += bwd::align256(sizeof(float) * ntok * V);
    float *ckpt = reinterpret_cast<float *>(p);
    p += bwd::align256(sizeof(float) * B * H * NC * K * V);
    float *bnd = reinterpret_cast<float *>(p);
#define GDN2_BWD(KR, NW, TOK)                                                                                    \
    return bwd::launch_all<KR, NW, TOK>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, B, H, \
                                        T, delta, ddelta, ckpt, bnd, st)
    if (bf16) {
        if (K == 128 && V == 128) GDN2_BWD(4, 16, __nv_bfloat16);
        if (K == 128 && V == 64) GDN2_BWD(4, 8, __nv_bfloat16);
        if (K == 64 && V == 128) GDN2_BWD(2, 16, __nv_bfloat16);
        if (K == 64 && V == 64) GDN2_BWD(2, 8, __nv_bfloat16);
    } else {
        if (K == 128 && V == 128) GDN2_BWD(4, 16, float);
        if (K == 128 && V == 64) GDN2_BWD(4, 8, float);
        if (K == 64 && V == 128) GDN2_BWD(2, 16, float);
        if (K == 64 && V == 64) GDN2_BWD(2, 8, float);
    }
#undef GDN2_BWD
    return -4;
}

}  // namespace gdn2
