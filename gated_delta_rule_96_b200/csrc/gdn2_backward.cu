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
// the matrix lives in registers as column pairs, updated with the packed two-wide fp32
// FMA of sm_100.  Column sums over the key axis (feeding the recurrence) stay inside the
// warp (a shuffle reduce-scatter); row sums over the value axis (outputs only) go through
// shared memory and are flushed every NB steps.  The token rows of each block of NB steps
// are copied into shared memory with cp.async two blocks ahead, so the step loop reads
// only registers and shared memory.
//
// Few chains: the value columns are independent in all three passes, so a chain's columns are
// split over up to 4 blocks (SPLIT instances); the row sums then accumulate with atomics and
// gates_finalize completes de, db, dk and the decay sums per chunk.
#include <float.h>

#include "gdn2_common.cuh"
#include "gdn2_internal.h"

namespace gdn2 {
namespace bwd {

constexpr int C = 64;   // chunk length: checkpoint spacing and the span of the log-decay sums
constexpr int NB = 8;   // steps per block: row-sum flush and cp.async staging unit (divides C)
static_assert(C % NB == 0, "chunk ends must be block ends");

__device__ __forceinline__ float2 bf2(uint32_t u) {
    __nv_bfloat162 p = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return make_float2(__low2float(p), __high2float(p));
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// all but the most recent group complete (this thread's copies)
__device__ __forceinline__ void cp_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// n consecutive steps' rows of one token tensor -> smem [n][E]: E elements from each source row
// (rows of `stride` elements, consecutive steps H rows apart)
template <int E, typename T>
__device__ __forceinline__ void stage_rows(T *dst, const T *src, size_t row0, int H, int n, int tid, int NT,
                                           int stride) {
    constexpr int PPR = E * (int)sizeof(T) / 16;   // 16-byte pieces per row
    for (int p = tid; p < n * PPR; p += NT) {
        const int s = p / PPR, c = p - s * PPR;
        cp_async16(reinterpret_cast<char *>(dst + s * E) + 16 * c,
                   reinterpret_cast<const char *>(src + (row0 + (size_t)s * H) * stride) + 16 * c);
    }
}

// a lane's KR consecutive values of a staged row, as fp32
template <int KR>
__device__ __forceinline__ void rows_of(const float *p, float (&x)[KR]) {
    if constexpr (KR == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    } else {
        const float2 a = *reinterpret_cast<const float2 *>(p);
        x[0] = a.x; x[1] = a.y;
    }
}
template <int KR>
__device__ __forceinline__ void rows_of(const __nv_bfloat16 *p, float (&x)[KR]) {
    if constexpr (KR == 4) {
        const uint2 a = *reinterpret_cast<const uint2 *>(p);
        const float2 l = bf2(a.x), h = bf2(a.y);
        x[0] = l.x; x[1] = l.y; x[2] = h.x; x[3] = h.y;
    } else {
        const float2 l = bf2(*reinterpret_cast<const uint32_t *>(p));
        x[0] = l.x; x[1] = l.y;
    }
}
// a warp's 8 consecutive values (every lane reads the same address), as 4 column pairs
__device__ __forceinline__ void cols_of(const float *p, float2 (&x)[4]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w); x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
}
__device__ __forceinline__ void cols_of(const __nv_bfloat16 *p, float2 (&x)[4]) {
    const uint4 a = *reinterpret_cast<const uint4 *>(p);
    x[0] = bf2(a.x); x[1] = bf2(a.y); x[2] = bf2(a.z); x[3] = bf2(a.w);
}
// global fp32 [8] at p (16-byte aligned) as column pairs
__device__ __forceinline__ void cols_global(const float *p, float2 (&x)[4]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p)), b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w); x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
}
__device__ __forceinline__ void store_cols(float *p, const float2 (&x)[4]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(x[0].x, x[0].y, x[1].x, x[1].y);
    reinterpret_cast<float4 *>(p)[1] = make_float4(x[2].x, x[2].y, x[3].x, x[3].y);
}
__device__ __forceinline__ float2 splat(float a) { return make_float2(a, a); }

// Sum over the 32 lanes of eight per-lane values p[0..7]; lane l receives the sum of
// p[(l >> 2) & 7].  Lanes differing in bit 4, then 3, then 2 exchange half of what they
// hold (4, 2, 1 values), then bits 1 and 0 finish: 9 shuffles instead of 40.
__device__ __forceinline__ float warp_colsum8(const float2 (&p2)[4], int lane) {
    const float p[8] = {p2[0].x, p2[0].y, p2[1].x, p2[1].y, p2[2].x, p2[2].y, p2[3].x, p2[3].y};
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
// the eight column values held by lanes 0, 4, ..., 28, as pairs in every lane
__device__ __forceinline__ void broadcast8(float mine, float2 (&d)[4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p)
        d[p] = make_float2(__shfl_sync(0xffffffffu, mine, 8 * p), __shfl_sync(0xffffffffu, mine, 8 * p + 4));
}

__device__ __forceinline__ bool chunk_end(int t, int T) { return t == T - 1 || (t + 1) % C == 0; }

// Row sums of a block: red[s][w][c] summed over the warps w.
template <int K, int NW>
__device__ __forceinline__ float red_sum(const float *red, int s, int c) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) acc += red[(s * NW + w) * K + c];
    return acc;
}
template <int KR>
__device__ __forceinline__ void st_red(float *red, int s, int NW, int K, int warp, int r0, const float (&x)[KR]) {
    float *p = red + (s * NW + warp) * K + r0;
    if constexpr (KR == 4) *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}

// The carried d_k x d_v matrix: a lane's KR rows x the warp's 8 columns, as column pairs.
template <int KR>
using Mat = float2[KR][4];

template <int KR>
__device__ __forceinline__ void load_mat(Mat<KR> &M, const float *src, int r0, int col, int stride) {
#pragma unroll
    for (int i = 0; i < KR; ++i) {
        if (src) cols_global(src + (size_t)(r0 + i) * stride + col, M[i]);
        else
#pragma unroll
            for (int p = 0; p < 4; ++p) M[i][p] = make_float2(0.f, 0.f);
    }
}

// Shared-memory staging areas of one block (per buffer), as byte offsets.
template <int K, int V, typename Tok>
struct Stage1 {   // pass 1: alpha, k, b | v, w, dO
    static constexpr int al = 0, kk = al + NB * K * 4, bk = kk + NB * K * (int)sizeof(Tok);
    static constexpr int vv = bk + NB * K * (int)sizeof(Tok), ww = vv + NB * V * (int)sizeof(Tok);
    static constexpr int go = ww + NB * V * (int)sizeof(Tok), bytes = go + NB * V * (int)sizeof(Tok);
};
template <int K, int V, typename Tok>
struct Stage2 {   // pass 2: alpha, k, b, q | v, w, dO, delta
    static constexpr int al = 0, kk = al + NB * K * 4, bk = kk + NB * K * (int)sizeof(Tok);
    static constexpr int qq = bk + NB * K * (int)sizeof(Tok), vv = qq + NB * K * (int)sizeof(Tok);
    static constexpr int ww = vv + NB * V * (int)sizeof(Tok), go = ww + NB * V * (int)sizeof(Tok);
    static constexpr int dl = go + NB * V * (int)sizeof(Tok), bytes = dl + NB * V * 4;
};
template <int K, int V, typename Tok>
struct Stage3 {   // pass 3: alpha, k, b, q, dq, dk | delta, ddelta
    static constexpr int al = 0, kk = al + NB * K * 4, bk = kk + NB * K * (int)sizeof(Tok);
    static constexpr int qq = bk + NB * K * (int)sizeof(Tok), dq = qq + NB * K * (int)sizeof(Tok);
    static constexpr int dk = dq + NB * K * 4, dl = dk + NB * K * 4, dd = dl + NB * V * 4;
    static constexpr int bytes = dd + NB * V * 4;
};

template <typename T>
__device__ __forceinline__ T *at(unsigned char *base, int off) { return reinterpret_cast<T *>(base + off); }

// ------------------------------------------------------------------------------------ pass 1
// Forward over S: delta_t -> workspace, dq_t = S_t dO_t -> dq, S at every chunk end -> ckpt.
template <int KR, int NW, typename Tok, bool SPLIT>
__global__ void __launch_bounds__(NW * 32, 1)
pass_forward(const Tok *__restrict__ k, const Tok *__restrict__ v, const float *__restrict__ alpha,
             const Tok *__restrict__ b, const Tok *__restrict__ w, const float *__restrict__ S0,
             const Tok *__restrict__ dO, float *__restrict__ dq, float *__restrict__ delta,
             float *__restrict__ ckpt, int H, int T, int NC, int Vt_arg, int ns_arg) {
    constexpr int K = 32 * KR, V = 8 * NW, NT = NW * 32;
    // unsplit: one block holds all V columns of its chain (stride and slice count are constants)
    const int Vt = SPLIT ? Vt_arg : V, ns = SPLIT ? ns_arg : 1;
    using L = Stage1<K, V, Tok>;
    extern __shared__ __align__(16) unsigned char smem[];
    float *red = reinterpret_cast<float *>(smem);                       // [NB][NW][K]
    unsigned char *stg = smem + NB * NW * K * 4;                         // [2][L::bytes]
    // block = (chain, slice of V columns); c0 is the warp's first column in the slice, cg in the state
    const int chain = blockIdx.x / ns, bb = chain / H, h = chain % H, cb = (blockIdx.x % ns) * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = KR * lane, c0 = 8 * warp, cg = cb + c0, jm = (lane >> 2) & 7;
    const int nblk = (T + NB - 1) / NB;

    auto stage = [&](int blk) {
        const int t0 = blk * NB, n = min(NB, T - t0);
        if (n <= 0) return;
        unsigned char *sb = stg + (blk & 1) * L::bytes;
        const size_t row0 = ((size_t)bb * T + t0) * H + h;
        stage_rows<K>(at<float>(sb, L::al), alpha, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::kk), k, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::bk), b, row0, H, n, tid, NT, K);
        stage_rows<V>(at<Tok>(sb, L::vv), v + cb, row0, H, n, tid, NT, Vt);
        stage_rows<V>(at<Tok>(sb, L::ww), w + cb, row0, H, n, tid, NT, Vt);
        stage_rows<V>(at<Tok>(sb, L::go), dO + cb, row0, H, n, tid, NT, Vt);
    };
    Mat<KR> S;
    load_mat<KR>(S, S0 ? S0 + (size_t)chain * K * Vt : nullptr, r0, cg, Vt);
    stage(0);
    cp_commit();
    stage(1);
    cp_commit();
    cp_wait_prev();
    __syncthreads();
    for (int blk = 0; blk < nblk; ++blk) {
        const int t0 = blk * NB, n = min(NB, T - t0);
        unsigned char *sb = stg + (blk & 1) * L::bytes;
        for (int s = 0; s < n; ++s) {
            const int t = t0 + s;
            float al[KR], kk[KR], bk[KR];
            rows_of<KR>(at<float>(sb, L::al) + s * K + r0, al);
            rows_of<KR>(at<Tok>(sb, L::kk) + s * K + r0, kk);
            rows_of<KR>(at<Tok>(sb, L::bk) + s * K + r0, bk);
            float2 g[4];
            cols_of(at<Tok>(sb, L::go) + s * V + c0, g);
            const float u = to_f32(at<Tok>(sb, L::ww)[s * V + c0 + jm]) * to_f32(at<Tok>(sb, L::vv)[s * V + c0 + jm]);
            // Sbar = Diag(alpha) S; r = Sbar^T e (column sums); delta = u - r
            float2 pr[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                const float2 a2 = splat(al[i]), e2 = splat(bk[i] * kk[i]);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    S[i][p] = __fmul2_rn(S[i][p], a2);
                    pr[p] = __ffma2_rn(S[i][p], e2, pr[p]);
                }
            }
            const float dmine = u - warp_colsum8(pr, lane);
            if ((lane & 3) == 0) delta[(((size_t)bb * T + t) * H + h) * Vt + cg + jm] = dmine;
            float2 d[4];
            broadcast8(dmine, d);
            // S_t = Sbar + k delta^T; row sums of S_t dO_t
            float x[KR];
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                const float2 k2 = splat(kk[i]);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    S[i][p] = __ffma2_rn(k2, d[p], S[i][p]);
                    acc = __ffma2_rn(S[i][p], g[p], acc);
                }
                x[i] = acc.x + acc.y;
            }
            st_red<KR>(red, s, NW, K, warp, r0, x);
            if (chunk_end(t, T)) {
                float *ck = ckpt + ((size_t)chain * NC + t / C) * K * Vt;
#pragma unroll
                for (int i = 0; i < KR; ++i) store_cols(ck + (size_t)(r0 + i) * Vt + cg, S[i]);
            }
        }
        __syncthreads();   // block done: row sums complete, its staging buffer free
        for (int idx = tid; idx < n * K; idx += NT) {
            const int s = idx / K, c = idx - s * K;
            float *d = dq + (((size_t)bb * T + t0 + s) * H + h) * K + c;
            if (ns > 1) atomicAdd(d, red_sum<K, NW>(red, s, c));   // the other slices' columns add in
            else *d = red_sum<K, NW>(red, s, c);
        }
        stage(blk + 2);
        cp_commit();
        cp_wait_prev();
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------ pass 2
// Reverse over G: ddelta_t -> workspace, dv, dw, dk_t = G_t delta_t (completed by pass 3),
// rowsum(G^fut ⊙ S) at every chunk end -> bnd, dS0 = G_0.  Blocks run from the end.
template <int KR, int NW, typename Tok, bool SPLIT>
__global__ void __launch_bounds__(NW * 32, 1)
pass_reverse(const Tok *__restrict__ q, const Tok *__restrict__ k, const Tok *__restrict__ v,
             const float *__restrict__ alpha, const Tok *__restrict__ b, const Tok *__restrict__ w,
             const Tok *__restrict__ dO, const float *__restrict__ dST, const float *__restrict__ delta,
             const float *__restrict__ ckpt, float *__restrict__ ddelta, float *__restrict__ bnd,
             float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dw, float *__restrict__ dS0,
             int H, int T, int NC, int Vt_arg, int ns_arg) {
    constexpr int K = 32 * KR, V = 8 * NW, NT = NW * 32;
    // unsplit: one block holds all V columns of its chain (stride and slice count are constants)
    const int Vt = SPLIT ? Vt_arg : V, ns = SPLIT ? ns_arg : 1;
    using L = Stage2<K, V, Tok>;
    extern __shared__ __align__(16) unsigned char smem[];
    float *red = reinterpret_cast<float *>(smem);                  // [NB][NW][K]
    float *rbnd = red + NB * NW * K;                                // [NW][K]
    unsigned char *stg = smem + (NB + 1) * NW * K * 4;              // [2][L::bytes]
    // block = (chain, slice of V columns); c0 is the warp's first column in the slice, cg in the state
    const int chain = blockIdx.x / ns, bb = chain / H, h = chain % H, cb = (blockIdx.x % ns) * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = KR * lane, c0 = 8 * warp, cg = cb + c0, jm = (lane >> 2) & 7;
    const int nblk = (T + NB - 1) / NB;
    // reverse block r holds steps lo(r) .. hi(r), hi(r) = T - 1 - r NB; staged at s = t - lo
    auto lo_of = [&](int r) { return max(T - (r + 1) * NB, 0); };
    auto stage = [&](int r) {
        if (r >= nblk) return;
        const int lo = lo_of(r), n = T - r * NB - lo;
        unsigned char *sb = stg + (r & 1) * L::bytes;
        const size_t row0 = ((size_t)bb * T + lo) * H + h;
        stage_rows<K>(at<float>(sb, L::al), alpha, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::kk), k, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::bk), b, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::qq), q, row0, H, n, tid, NT, K);
        stage_rows<V>(at<Tok>(sb, L::vv), v + cb, row0, H, n, tid, NT, Vt);
        stage_rows<V>(at<Tok>(sb, L::ww), w + cb, row0, H, n, tid, NT, Vt);
        stage_rows<V>(at<Tok>(sb, L::go), dO + cb, row0, H, n, tid, NT, Vt);
        stage_rows<V>(at<float>(sb, L::dl), delta + cb, row0, H, n, tid, NT, Vt);
    };
    Mat<KR> G;
    load_mat<KR>(G, dST ? dST + (size_t)chain * K * Vt : nullptr, r0, cg, Vt);
    stage(0);
    cp_commit();
    stage(1);
    cp_commit();
    cp_wait_prev();
    __syncthreads();
    for (int r = 0; r < nblk; ++r) {
        const int lo = lo_of(r), hi = T - 1 - r * NB;
        unsigned char *sb = stg + (r & 1) * L::bytes;
        for (int t = hi; t >= lo; --t) {
            const int s = t - lo;
            if (chunk_end(t, T)) {   // G here is dL/dS_t from the steps after t
                const int ci = t / C;
                const float *ck = ckpt + ((size_t)chain * NC + ci) * K * Vt;
                float y[KR];
#pragma unroll
                for (int i = 0; i < KR; ++i) {
                    float2 sv[4];
                    cols_global(ck + (size_t)(r0 + i) * Vt + cg, sv);
                    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                    for (int p = 0; p < 4; ++p) acc = __ffma2_rn(G[i][p], sv[p], acc);
                    y[i] = acc.x + acc.y;
                }
                st_red<KR>(rbnd, 0, NW, K, warp, r0, y);
                __syncthreads();
                for (int c = tid; c < K; c += NT) {
                    float *d = bnd + ((size_t)chain * NC + ci) * K + c;
                    if (ns > 1) atomicAdd(d, red_sum<K, NW>(rbnd, 0, c));
                    else *d = red_sum<K, NW>(rbnd, 0, c);
                }
                __syncthreads();
            }
            float al[KR], kk[KR], bk[KR], qq[KR];
            rows_of<KR>(at<float>(sb, L::al) + s * K + r0, al);
            rows_of<KR>(at<Tok>(sb, L::kk) + s * K + r0, kk);
            rows_of<KR>(at<Tok>(sb, L::bk) + s * K + r0, bk);
            rows_of<KR>(at<Tok>(sb, L::qq) + s * K + r0, qq);
            float2 g[4], dl[4];
            cols_of(at<Tok>(sb, L::go) + s * V + c0, g);
            cols_of(at<float>(sb, L::dl) + s * V + c0, dl);
            // o_t = S_t^T q_t: G_t += q_t dO_t^T; ddelta = G_t^T k_t (column sums)
            float2 pr[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                const float2 q2 = splat(qq[i]), k2 = splat(kk[i]);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    G[i][p] = __ffma2_rn(q2, g[p], G[i][p]);
                    pr[p] = __ffma2_rn(G[i][p], k2, pr[p]);
                }
            }
            const float ddm = warp_colsum8(pr, lane);
            if ((lane & 3) == 0) {
                const size_t e = (((size_t)bb * T + t) * H + h) * Vt + cg + jm;
                ddelta[e] = ddm;
                dv[e] = ddm * to_f32(at<Tok>(sb, L::ww)[s * V + c0 + jm]);
                dw[e] = ddm * to_f32(at<Tok>(sb, L::vv)[s * V + c0 + jm]);
            }
            float2 dd[4];
            broadcast8(ddm, dd);
            // row sums of G_t delta_t; G_{t-1} = Diag(alpha_t)(G_t - e_t ddelta_t^T)
            float x[KR];
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                const float2 a2 = splat(al[i]), ne2 = splat(-bk[i] * kk[i]);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    acc = __ffma2_rn(G[i][p], dl[p], acc);
                    G[i][p] = __fmul2_rn(a2, __ffma2_rn(ne2, dd[p], G[i][p]));
                }
                x[i] = acc.x + acc.y;
            }
            st_red<KR>(red, hi - t, NW, K, warp, r0, x);
        }
        __syncthreads();
        for (int idx = tid; idx < (hi - lo + 1) * K; idx += NT) {
            const int s = idx / K, c = idx - s * K;   // slot s holds step hi - s
            float *d = dk + (((size_t)bb * T + hi - s) * H + h) * K + c;
            if (ns > 1) atomicAdd(d, red_sum<K, NW>(red, s, c));
            else *d = red_sum<K, NW>(red, s, c);
        }
        stage(r + 2);
        cp_commit();
        cp_wait_prev();
        __syncthreads();
    }
    if (dS0) {
#pragma unroll
        for (int i = 0; i < KR; ++i) store_cols(dS0 + ((size_t)chain * K + r0 + i) * Vt + cg, G[i]);
    }
}

// ------------------------------------------------------------------------------------ pass 3
// Forward over S with the kept delta: S_{t-1} ddelta_t gives de = -alpha ⊙ (S_{t-1} ddelta);
// then db, the complete dk, and per chunk the log-decay sums -> dalpha.
template <int KR, int NW, typename Tok, bool SPLIT>
__global__ void __launch_bounds__(NW * 32, 1)
pass_gates(const Tok *__restrict__ q, const Tok *__restrict__ k, const float *__restrict__ alpha,
           const Tok *__restrict__ b, const float *__restrict__ S0, const float *__restrict__ delta,
           const float *__restrict__ ddelta, const float *__restrict__ bnd, const float *__restrict__ dq,
           float *__restrict__ dk, float *__restrict__ db, float *__restrict__ dalpha, float *__restrict__ X, int H,
           int T, int NC, int Vt_arg, int ns_arg) {
    constexpr int K = 32 * KR, V = 8 * NW, NT = NW * 32;
    const int Vt = SPLIT ? Vt_arg : V, ns = SPLIT ? ns_arg : 1;
    using L = Stage3<K, V, Tok>;
    extern __shared__ __align__(16) unsigned char smem[];
    float *red = reinterpret_cast<float *>(smem);           // [NB][NW][K]
    float *hbuf = red + NB * NW * K;                         // [C][K] dL/dg of the chunk's steps
    float *abuf = hbuf + C * K;                              // [C][K] alpha of the chunk's steps
    unsigned char *stg = reinterpret_cast<unsigned char *>(abuf + C * K);   // [2][L::bytes]
    const int chain = blockIdx.x / ns, bb = chain / H, h = chain % H, cb = (blockIdx.x % ns) * V;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = KR * lane, c0 = 8 * warp, cg = cb + c0;
    const int nblk = (T + NB - 1) / NB;

    auto stage = [&](int blk) {
        const int t0 = blk * NB, n = min(NB, T - t0);
        if (n <= 0) return;
        unsigned char *sb = stg + (blk & 1) * L::bytes;
        const size_t row0 = ((size_t)bb * T + t0) * H + h;
        stage_rows<K>(at<float>(sb, L::al), alpha, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::kk), k, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::bk), b, row0, H, n, tid, NT, K);
        stage_rows<K>(at<Tok>(sb, L::qq), q, row0, H, n, tid, NT, K);
        if (ns == 1) {   // the complete row sums are formed here only when the block holds every column
            stage_rows<K>(at<float>(sb, L::dq), dq, row0, H, n, tid, NT, K);
            stage_rows<K>(at<float>(sb, L::dk), static_cast<const float *>(dk), row0, H, n, tid, NT, K);
        }
        stage_rows<V>(at<float>(sb, L::dl), delta + cb, row0, H, n, tid, NT, Vt);
        stage_rows<V>(at<float>(sb, L::dd), ddelta + cb, row0, H, n, tid, NT, Vt);
    };
    Mat<KR> S;
    load_mat<KR>(S, S0 ? S0 + (size_t)chain * K * Vt : nullptr, r0, cg, Vt);
    stage(0);
    cp_commit();
    stage(1);
    cp_commit();
    cp_wait_prev();
    __syncthreads();
    for (int blk = 0; blk < nblk; ++blk) {
        const int t0 = blk * NB, n = min(NB, T - t0);
        unsigned char *sb = stg + (blk & 1) * L::bytes;
        for (int s = 0; s < n; ++s) {
            float al[KR], kk[KR];
            rows_of<KR>(at<float>(sb, L::al) + s * K + r0, al);
            rows_of<KR>(at<Tok>(sb, L::kk) + s * K + r0, kk);
            float2 dl[4], dd[4];
            cols_of(at<float>(sb, L::dl) + s * V + c0, dl);
            cols_of(at<float>(sb, L::dd) + s * V + c0, dd);
            float x[KR];
#pragma unroll
            for (int i = 0; i < KR; ++i) {
                const float2 a2 = splat(al[i]), k2 = splat(kk[i]);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    acc = __ffma2_rn(S[i][p], dd[p], acc);                       // S_{t-1} ddelta_t
                    S[i][p] = __ffma2_rn(k2, dl[p], __fmul2_rn(a2, S[i][p]));   // S_t
                }
                x[i] = acc.x + acc.y;
            }
            st_red<KR>(red, s, NW, K, warp, r0, x);
        }
        __syncthreads();
        if (ns > 1) {   // partial row sums S_{t-1} ddelta over this slice's columns; gates_finalize completes
            for (int idx = tid; idx < n * K; idx += NT) {
                const int s = idx / K, c = idx - s * K;
                atomicAdd(X + (((size_t)bb * T + t0 + s) * H + h) * K + c, red_sum<K, NW>(red, s, c));
            }
            __syncthreads();
            stage(blk + 2);
            cp_commit();
            cp_wait_prev();
            __syncthreads();
            continue;
        }
        for (int idx = tid; idx < n * K; idx += NT) {
            const int s = idx / K, c = idx - s * K;
            const size_t e = (((size_t)bb * T + t0 + s) * H + h) * K + c;
            const float a = at<float>(sb, L::al)[s * K + c];
            const float kc = to_f32(at<Tok>(sb, L::kk)[s * K + c]), bc = to_f32(at<Tok>(sb, L::bk)[s * K + c]);
            const float qc = to_f32(at<Tok>(sb, L::qq)[s * K + c]);
            const float de = -a * red_sum<K, NW>(red, s, c);
            const float dkt = at<float>(sb, L::dk)[s * K + c] + bc * de;
            dk[e] = dkt;
            db[e] = kc * de;
            // dL/dg_t = q dq + e de - k (dk - b de)
            const int pos = (t0 + s) % C;
            hbuf[pos * K + c] = qc * at<float>(sb, L::dq)[s * K + c] + 2.f * bc * kc * de - kc * dkt;
            abuf[pos * K + c] = a;
        }
        __syncthreads();   // the staged rows of this block were read above: the buffer is free
        stage(blk + 2);
        cp_commit();
        cp_wait_prev();
        __syncthreads();
        const int t = t0 + n - 1;
        if (chunk_end(t, T)) {   // d log alpha summed back from the chunk end; its buffers are
            const int ci = t / C, cs = ci * C;   // next written after the next block's first barrier
            for (int c = tid; c < K; c += NT) {
                float acc = bnd[((size_t)chain * NC + ci) * K + c];
                for (int s = t - cs; s >= 0; --s) {
                    acc += hbuf[s * K + c];
                    dalpha[(((size_t)bb * T + cs + s) * H + h) * K + c] = acc / fmaxf(abuf[s * K + c], FLT_MIN);
                }
            }
        }
    }
}

// Column-sliced chains: completes pass 3 from the summed partial row sums X = S_{t-1} ddelta.
// One block per (chain, chunk), one thread per key channel, walking the chunk backwards.
template <typename Tok>
__global__ void __launch_bounds__(128)
gates_finalize(const Tok *__restrict__ q, const Tok *__restrict__ k, const float *__restrict__ alpha,
               const Tok *__restrict__ b, const float *__restrict__ X, const float *__restrict__ bnd,
               const float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ db,
               float *__restrict__ dalpha, int H, int T, int NC, int K) {
    const int chain = blockIdx.x, ci = blockIdx.y, bb = chain / H, h = chain % H;
    const int cs = ci * C, ce = min(cs + C, T);
    for (int c = threadIdx.x; c < K; c += blockDim.x) {
        float acc = bnd[((size_t)chain * NC + ci) * K + c];
        for (int t = ce - 1; t >= cs; --t) {
            const size_t e = (((size_t)bb * T + t) * H + h) * K + c;
            const float a = alpha[e], kc = to_f32(k[e]), bc = to_f32(b[e]), qc = to_f32(q[e]);
            const float de = -a * X[e];
            const float dkt = dk[e] + bc * de;
            dk[e] = dkt;
            db[e] = kc * de;
            acc += qc * dq[e] + 2.f * bc * kc * de - kc * dkt;   // dL/dg_t, summed back from the chunk end
            dalpha[e] = acc / fmaxf(a, FLT_MIN);
        }
    }
}

template <int K, int V, typename Tok>
constexpr size_t smem1() { return (size_t)NB * (V / 8) * K * 4 + 2 * Stage1<K, V, Tok>::bytes; }
template <int K, int V, typename Tok>
constexpr size_t smem2() { return (size_t)(NB + 1) * (V / 8) * K * 4 + 2 * Stage2<K, V, Tok>::bytes; }
template <int K, int V, typename Tok>
constexpr size_t smem3() { return (size_t)NB * (V / 8) * K * 4 + 2 * (size_t)C * K * 4 + 2 * Stage3<K, V, Tok>::bytes; }

template <int KR, int NW, typename Tok, bool SPLIT>
int launch_all(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
               const float *S0, const void *dO, const float *dST, float *dq, float *dk, float *dv, float *dalpha,
               float *db, float *dw, float *dS0, int B, int H, int T, int Vt, int ns, float *delta, float *ddelta,
               float *ckpt, float *bnd, float *X, cudaStream_t st) {
    constexpr int K = 32 * KR, V = 8 * NW;   // V: the columns of one block (Vt / ns)
    constexpr size_t sm1 = smem1<K, V, Tok>(), sm2 = smem2<K, V, Tok>(), sm3 = smem3<K, V, Tok>();
    static_assert(sm1 <= 227 * 1024 && sm2 <= 227 * 1024 && sm3 <= 227 * 1024, "shared memory");
    const int NC = (T + C - 1) / C, NT = NW * 32, grid = B * H * ns;
    if (ns > 1) {   // row sums accumulate over the slices
        const size_t tokk = sizeof(float) * (size_t)B * T * H * K;
        if (cudaMemsetAsync(dq, 0, tokk, st) != cudaSuccess || cudaMemsetAsync(dk, 0, tokk, st) != cudaSuccess ||
            cudaMemsetAsync(X, 0, tokk, st) != cudaSuccess ||
            cudaMemsetAsync(bnd, 0, sizeof(float) * (size_t)B * H * NC * K, st) != cudaSuccess)
            return -6;
    }
    auto f1 = pass_forward<KR, NW, Tok, SPLIT>;
    auto f2 = pass_reverse<KR, NW, Tok, SPLIT>;
    auto f3 = pass_gates<KR, NW, Tok, SPLIT>;
    if (cudaFuncSetAttribute(f1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1) != cudaSuccess ||
        cudaFuncSetAttribute(f2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2) != cudaSuccess ||
        cudaFuncSetAttribute(f3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3) != cudaSuccess)
        return -6;
    const Tok *tq = static_cast<const Tok *>(q), *tk = static_cast<const Tok *>(k), *tv = static_cast<const Tok *>(v);
    const Tok *tb = static_cast<const Tok *>(b), *tw = static_cast<const Tok *>(w), *tdo = static_cast<const Tok *>(dO);
    f1<<<grid, NT, sm1, st>>>(tk, tv, alpha, tb, tw, S0, tdo, dq, delta, ckpt, H, T, NC, Vt, ns);
    f2<<<grid, NT, sm2, st>>>(tq, tk, tv, alpha, tb, tw, tdo, dST, delta, ckpt, ddelta, bnd, dk, dv, dw, dS0, H, T,
                              NC, Vt, ns);
    f3<<<grid, NT, sm3, st>>>(tq, tk, alpha, tb, S0, delta, ddelta, bnd, dq, dk, db, dalpha, X, H, T, NC, Vt, ns);
    if (ns > 1)
        gates_finalize<Tok><<<dim3(B * H, NC), 128, 0, st>>>(tq, tk, alpha, tb, X, bnd, dq, dk, db, dalpha, H, T, NC,
                                                              K);
    return launch_status();
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Column slices per chain: few chains would leave most of the 148 SMs idle, and the value columns
// of every pass are independent, so a chain's columns are split over up to 4 blocks (at least 32
// columns, four warps, each: faster than 8 blocks of two warps) while the blocks fit on the SMs.
inline int slices(int chains, int V) {
    int ns = 1;
    while (ns * 2 * chains <= 148 && V / (8 * ns * 2) >= 4) ns *= 2;
    return ns;
}

}  // namespace bwd


size_t bwd_workspace_bytes(int B, int H, int T, int K, int V) {
    const size_t ntok = (size_t)B * T * H, NC = (size_t)(T + bwd::C - 1) / bwd::C;
    const bool split = bwd::slices(B * H, V) > 1;   // + the partial row sums of pass 3
    return 2 * bwd::align256(sizeof(float) * ntok * V) + bwd::align256(sizeof(float) * B * H * NC * K * V) +
           bwd::align256(sizeof(float) * B * H * NC * K) + (split ? bwd::align256(sizeof(float) * ntok * K) : 0);
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
    p += bwd::align256(sizeof(float) * B * H * NC * K);
    float *X = reinterpret_cast<float *>(p);
    const int ns = bwd::slices(B * H, V), nw = V / 8 / ns;   // warps per block
#define GDN2_BWD(KR, NW, TOK, SPLIT)                                                                            \
    return bwd::launch_all<KR, NW, TOK, SPLIT>(q, k, v, alpha, b, w, S0, dO, dST, dq, dk, dv, dalpha, db, dw, dS0, \
                                               B, H, T, V, ns, delta, ddelta, ckpt, bnd, X, st)
#define GDN2_BWD_NW(KR, TOK)                              \
    if (ns == 1 && nw == 16) GDN2_BWD(KR, 16, TOK, false); \
    if (ns == 1 && nw == 8) GDN2_BWD(KR, 8, TOK, false);   \
    if (ns > 1 && nw == 8) GDN2_BWD(KR, 8, TOK, true);     \
    if (ns > 1 && nw == 4) GDN2_BWD(KR, 4, TOK, true);
    if (bf16) {
        if (K == 128) { GDN2_BWD_NW(4, __nv_bfloat16) }
        if (K == 64) { GDN2_BWD_NW(2, __nv_bfloat16) }
    } else {
        if (K == 128) { GDN2_BWD_NW(4, float) }
        if (K == 64) { GDN2_BWD_NW(2, float) }
    }
#undef GDN2_BWD_NW
#undef GDN2_BWD
    return -4;
}

}  // namespace gdn2
