// Single-token decode step of the GDN-2 recurrence (page "NVIDIA представила
// Gated DeltaNet-2 ...", section "Техническая схема", the state-update equation),
// one read and one write of the fp32 state.
//
// Per (b, h), with S̄ = Diag(alpha) S the decayed state:
//   r = S̄^T (b ⊙ k)      s = S̄^T q      delta = w ⊙ v - r
//   S <- S̄ + k delta^T    o = S^T q = s + (k·q) delta
//
// The kernel is HBM-bound (~1 flop per byte of state).  One CTA of 256 threads
// owns one (b, h) state: each lane holds a float4 column slice of 16 (or 8) rows
// in registers, loaded once with streaming loads; the d_k-reductions are
// in-thread over rows, across lanes by shuffle where lanes share columns, and
// across warps through shared memory; the updated rows are written back from
// the same registers.
#include "gdn2_common.cuh"
#include "gdn2_internal.h"

namespace gdn2 {

template <typename Tok, int K, int V>
__global__ void __launch_bounds__(256) decode_kernel(const Tok *__restrict__ q, const Tok *__restrict__ k,
                                                     const Tok *__restrict__ v, const float *__restrict__ alpha,
                                                     const Tok *__restrict__ b, const Tok *__restrict__ w,
                                                     float *__restrict__ S, Tok *__restrict__ o) {
    constexpr int NT = 256, NW = NT / 32;
    constexpr int LPR = V / 4;             // lanes covering one row (float4 each)
    constexpr int RPS = 32 / LPR;          // rows one warp instruction covers
    constexpr int ROWS_PER_WARP = K / NW;  // rows owned by one warp
    constexpr int STEPS = ROWS_PER_WARP / RPS;
    static_assert(STEPS * RPS * NW == K, "row split");

    __shared__ float s_a[K], s_ae[K], s_aq[K], s_k[K], s_q[K], s_u[V], s_delta[V];
    __shared__ float s_red[2][NW][V];
    __shared__ float s_kq;

    const int bh = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int col4 = (lane % LPR) * 4;
    const int rsub = lane / LPR;
    float *Sbh = S + (size_t)bh * K * V;

    // 1. issue the state loads first (independent of the token)
    float4 reg[STEPS];
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int row = warp * ROWS_PER_WARP + s * RPS + rsub;
        reg[s] = ld_stream(reinterpret_cast<const float4 *>(Sbh + (size_t)row * V + col4));
    }
    // 2. token vectors to shared memory
    for (int i = tid; i < K; i += NT) {
        const float a = alpha[(size_t)bh * K + i];
        const float kk = ld_tok(k + (size_t)bh * K + i);
        const float bb = ld_tok(b + (size_t)bh * K + i);
        const float qq = ld_tok(q + (size_t)bh * K + i);
        s_a[i] = a;
        s_ae[i] = a * bb * kk;
        s_aq[i] = a * qq;
        s_k[i] = kk;
        s_q[i] = qq;
    }
    for (int i = tid; i < V; i += NT) s_u[i] = ld_tok(w + (size_t)bh * V + i) * ld_tok(v + (size_t)bh * V + i);
    __syncthreads();
    if (warp == 0) {
        float t = 0.f;
        for (int i = lane; i < K; i += 32) t += s_k[i] * s_q[i];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) t += __shfl_xor_sync(0xffffffffu, t, m);
        if (lane == 0) s_kq = t;
    }
    // 3. partial r and s over this thread's rows
    float pr[4] = {0.f, 0.f, 0.f, 0.f}, ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int row = warp * ROWS_PER_WARP + s * RPS + rsub;
        const float ae = s_ae[row], aq = s_aq[row];
        pr[0] += ae * reg[s].x; pr[1] += ae * reg[s].y; pr[2] += ae * reg[s].z; pr[3] += ae * reg[s].w;
        ps[0] += aq * reg[s].x; ps[1] += aq * reg[s].y; ps[2] += aq * reg[s].z; ps[3] += aq * reg[s].w;
    }
    if (RPS > 1) {
#pragma unroll
        for (int m = LPR; m < 32; m <<= 1)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                pr[j] += __shfl_xor_sync(0xffffffffu, pr[j], m);
                ps[j] += __shfl_xor_sync(0xffffffffu, ps[j], m);
            }
    }
    if (rsub == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s_red[0][warp][col4 + j] = pr[j];
            s_red[1][warp][col4 + j] = ps[j];
        }
    }
    __syncthreads();
    // 4. per column: delta and the output
    for (int j = tid; j < V; j += NT) {
        float r = 0.f, sq = 0.f;
#pragma unroll
        for (int wi = 0; wi < NW; ++wi) {
            r += s_red[0][wi][j];
            sq += s_red[1][wi][j];
        }
        const float delta = s_u[j] - r;
        s_delta[j] = delta;
        store_tok(o + (size_t)bh * V + j, sq + s_kq * delta);
    }
    __syncthreads();
    // 5. S <- Diag(alpha) S + k delta^T, from the registers
    const float d0 = s_delta[col4], d1 = s_delta[col4 + 1], d2 = s_delta[col4 + 2], d3 = s_delta[col4 + 3];
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int row = warp * ROWS_PER_WARP + s * RPS + rsub;
        const float a = s_a[row], kk = s_k[row];
        float4 n;
        n.x = a * reg[s].x + kk * d0;
        n.y = a * reg[s].y + kk * d1;
        n.z = a * reg[s].z + kk * d2;
        n.w = a * reg[s].w + kk * d3;
        st_stream(reinterpret_cast<float4 *>(Sbh + (size_t)row * V + col4), n);
    }
}

template <typename Tok>
static int launch_decode_t(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                           const void *w, float *S, void *o, int B, int H, int K, int V, cudaStream_t st) {
    const int n = B * H;
    if (n == 0) return 0;
    const Tok *Q = (const Tok *)q, *Kp = (const Tok *)k, *Vp = (const Tok *)v, *Bp = (const Tok *)b,
              *Wp = (const Tok *)w;
    Tok *O = (Tok *)o;
    if (K == 128 && V == 128)
        decode_kernel<Tok, 128, 128><<<n, 256, 0, st>>>(Q, Kp, Vp, alpha, Bp, Wp, S, O);
    else if (K == 128 && V == 64)
        decode_kernel<Tok, 128, 64><<<n, 256, 0, st>>>(Q, Kp, Vp, alpha, Bp, Wp, S, O);
    else if (K == 64 && V == 128)
        decode_kernel<Tok, 64, 128><<<n, 256, 0, st>>>(Q, Kp, Vp, alpha, Bp, Wp, S, O);
    else if (K == 64 && V == 64)
        decode_kernel<Tok, 64, 64><<<n, 256, 0, st>>>(Q, Kp, Vp, alpha, Bp, Wp, S, O);
    else
        return -4;
    return launch_status();
}

int launch_decode(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                  const void *w, float *S, void *o, int B, int H, int K, int V, int bf16, cudaStream_t st) {
    if (bf16) return launch_decode_t<__nv_bfloat16>(q, k, v, alpha, b, w, S, o, B, H, K, V, st);
    return launch_decode_t<float>(q, k, v, alpha, b, w, S, o, B, H, K, V, st);
}

}  // namespace gdn2
