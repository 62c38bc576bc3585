// Chunkwise prefill on CUDA cores (fp32 FMA throughout): the general path for
// fp32 tokens, d_k/d_v = 64, and any shape the tensor-core path does not take.
//
// Algorithm (page "NVIDIA представила Gated DeltaNet-2 ...": the update equation of
// section "Техническая схема" evaluated chunk by chunk in the WY/UT form that the
// page's implementation paragraph names, chunk size C = 64).  Writing one token as
// S_t = D_t S_{t-1} + k_t delta_t^T with delta_t = u_t - S_{t-1}^T (alpha_t ⊙ e_t),
// e = b ⊙ k, u = w ⊙ v, a chunk with incoming state S gives, for r, i < C and the
// per-channel log-decay prefix g_r = sum_{j<=r} log alpha_j:
//
//   A_ri = sum_c e_rc k_ic exp(g_rc - g_ic)  (i < r)     T = (I + A)^-1
//   P_ri = sum_c q_rc k_ic exp(g_rc - g_ic)  (i <= r)
//   W = T (exp(g) ⊙ E)    U~ = T U    Q+ = exp(g) ⊙ Q    K^ = exp(g_C - g) ⊙ K
//   Delta = U~ - W S      O = Q+ S + P Delta      S' = Diag(exp(g_C)) S + K^T Delta
//
// Stage 1 (intra_kernel) is parallel over all chunks and writes W, U~, Q+, K^, P
// and exp(g_C) to the workspace; stage 2 (inter_kernel) walks the chunks of one
// (b, h, d_v-slice) in order with S resident in shared memory.  The decay factors
// are formed as exp(g_r - g_i) <= 1 for every pair, so no factor over- or
// underflows for any alpha in (0, 1].
#include "gdn2_common.cuh"
#include "gdn2_internal.h"

namespace gdn2 {

namespace simt {

constexpr int C = 64;
constexpr int VT = 16;  // d_v columns per stage-2 CTA

// workspace layout per chunk-head, in floats
template <int K, int V>
struct WsLayout {
    static constexpr size_t W = 0;
    static constexpr size_t QP = W + (size_t)C * K;
    static constexpr size_t KH = QP + (size_t)C * K;
    static constexpr size_t UT = KH + (size_t)C * K;
    static constexpr size_t P = UT + (size_t)C * V;
    static constexpr size_t GC = P + (size_t)C * C;
    static constexpr size_t SIZE = GC + K;
};

inline size_t ws_floats_per_chunk(int K, int V) { return (size_t)3 * C * K + (size_t)C * V + (size_t)C * C + K; }

// ---------------------------------------------------------------- stage 1
template <typename Tok, int K, int V>
__global__ void __launch_bounds__(256) intra_kernel(const Tok *__restrict__ q, const Tok *__restrict__ k,
                                                    const Tok *__restrict__ v, const float *__restrict__ alpha,
                                                    const Tok *__restrict__ b, const Tok *__restrict__ w, int H,
                                                    int T, int NC, float *__restrict__ ws) {
    constexpr int KP = K + 1;  // padded row stride (conflict-free column walks)
    extern __shared__ float sm[];
    float *sq = sm;                 // [C][KP]  q
    float *sk = sq + C * KP;        // [C][KP]  k
    float *se = sk + C * KP;        // [C][KP]  e = b ⊙ k, later exp(g) ⊙ e
    float *sg = se + C * KP;        // [C][KP]  g
    float *su = sg + C * KP;        // [C][V]   u = w ⊙ v
    float *sA = su + C * V;         // [C][C+1] A
    float *sT = sA + C * (C + 1);   // [C][C+1] T

    const int n = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int tid = threadIdx.x;
    const int t0 = n * C;
    const int L = min(C, T - t0);
    float *out = ws + ((size_t)(bb * H + h) * NC + n) * WsLayout<K, V>::SIZE;

    // load the chunk (rows >= L: zero tokens, alpha = 1)
    for (int idx = tid; idx < C * K; idx += 256) {
        const int r = idx / K, c = idx % K;
        float qq = 0.f, kk = 0.f, bv = 0.f, a = 1.f;
        if (r < L) {
            const size_t off = (((size_t)bb * T + t0 + r) * H + h) * K + c;
            qq = ld_tok(q + off);
            kk = ld_tok(k + off);
            bv = ld_tok(b + off);
            a = alpha[off];
        }
        sq[r * KP + c] = qq;
        sk[r * KP + c] = kk;
        se[r * KP + c] = bv * kk;
        sg[r * KP + c] = logf(a);
    }
    for (int idx = tid; idx < C * V; idx += 256) {
        const int r = idx / V, c = idx % V;
        float u = 0.f;
        if (r < L) {
            const size_t off = (((size_t)bb * T + t0 + r) * H + h) * V + c;
            u = ld_tok(w + off) * ld_tok(v + off);
        }
        su[r * V + c] = u;
    }
    __syncthreads();
    // g = prefix sum of log alpha along the chunk, one thread per channel
    for (int c = tid; c < K; c += 256) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += sg[r * KP + c];
            sg[r * KP + c] = acc;
        }
    }
    __syncthreads();
    // A (strictly lower) and P (lower with diagonal), exp(g_r - g_i) per channel
    {
        const int i = tid & (C - 1);
        const int rg = tid >> 6;  // 4 row groups
        for (int r = rg; r < C; r += 4) {
            float a_acc = 0.f, p_acc = 0.f;
            if (i <= r) {
                for (int c = 0; c < K; ++c) {
                    const float d = expf(sg[r * KP + c] - sg[i * KP + c]);
                    const float kd = sk[i * KP + c] * d;
                    a_acc += se[r * KP + c] * kd;
                    p_acc += sq[r * KP + c] * kd;
                }
            }
            sA[r * (C + 1) + i] = (i < r) ? a_acc : 0.f;
            out[WsLayout<K, V>::P + r * C + i] = (i <= r) ? p_acc : 0.f;
        }
    }
    __syncthreads();
    // T = (I + A)^-1 by forward substitution, one column per thread:
    // T[r][j] = delta_rj - sum_{i<r} A[r][i] T[i][j]
    if (tid < C) {
        const int j = tid;
        float col[C];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            float acc = (r == j) ? 1.f : 0.f;
            if (r > j) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int i = 0; i < r; i += 2) {
                    a0 += sA[r * (C + 1) + i] * col[i];
                    if (i + 1 < r) a1 += sA[r * (C + 1) + i + 1] * col[i + 1];
                }
                acc = -(a0 + a1);
            }
            col[r] = acc;
        }
#pragma unroll
        for (int r = 0; r < C; ++r) sT[r * (C + 1) + j] = col[r];
    }
    // exp(g) ⊙ e in place; Q+ and K^ straight to the workspace; exp(g_C)
    for (int idx = tid; idx < C * K; idx += 256) {
        const int r = idx / K, c = idx % K;
        const float g = sg[r * KP + c];
        const float gam = expf(g);
        se[r * KP + c] *= gam;
        out[WsLayout<K, V>::QP + idx] = gam * sq[r * KP + c];
        out[WsLayout<K, V>::KH + idx] = expf(sg[(C - 1) * KP + c] - g) * sk[r * KP + c];
    }
    for (int c = tid; c < K; c += 256) out[WsLayout<K, V>::GC + c] = expf(sg[(C - 1) * KP + c]);
    __syncthreads();
    // W = T (exp(g) ⊙ E): thread owns a channel and a half of the rows
    for (int job = tid; job < 2 * K; job += 256) {
        const int c = job % K, rh = job / K;
        float acc[C / 2];
#pragma unroll
        for (int r = 0; r < C / 2; ++r) acc[r] = 0.f;
        for (int i = 0; i < C; ++i) {
            const float x = se[i * KP + c];
#pragma unroll
            for (int r = 0; r < C / 2; ++r) acc[r] += sT[(rh * (C / 2) + r) * (C + 1) + i] * x;
        }
#pragma unroll
        for (int r = 0; r < C / 2; ++r) out[WsLayout<K, V>::W + (rh * (C / 2) + r) * K + c] = acc[r];
    }
    // U~ = T U
    for (int job = tid; job < 2 * V; job += 256) {
        const int c = job % V, rh = job / V;
        float acc[C / 2];
#pragma unroll
        for (int r = 0; r < C / 2; ++r) acc[r] = 0.f;
        for (int i = 0; i < C; ++i) {
            const float x = su[i * V + c];
#pragma unroll
            for (int r = 0; r < C / 2; ++r) acc[r] += sT[(rh * (C / 2) + r) * (C + 1) + i] * x;
        }
#pragma unroll
        for (int r = 0; r < C / 2; ++r) out[WsLayout<K, V>::UT + (rh * (C / 2) + r) * V + c] = acc[r];
    }
}

// ---------------------------------------------------------------- stage 2
template <typename Tok, int K, int V>
__global__ void __launch_bounds__(128) inter_kernel(const float *__restrict__ ws, const float *S0,
                                                    Tok *__restrict__ o, float *ST, int H, int T,
                                                    int NC) {
    extern __shared__ float sm[];
    float *sS = sm;                  // [K][VT]
    float *sW = sS + K * VT;         // [C][K]
    float *sQ = sW + C * K;          // [C][K]
    float *sKh = sQ + C * K;         // [C][K]
    float *sP = sKh + C * K;         // [C][C]
    float *sU = sP + C * C;          // [C][VT]
    float *sD = sU + C * VT;         // [C][VT] Delta
    float *sG = sD + C * VT;         // [K]

    const int vs = blockIdx.x, h = blockIdx.y, bb = blockIdx.z;
    const int tid = threadIdx.x;
    const int v0 = vs * VT;
    const size_t chain = (size_t)bb * H + h;

    for (int idx = tid; idx < K * VT; idx += 128) {
        const int c = idx / VT, j = idx % VT;
        sS[idx] = S0 ? S0[(chain * K + c) * V + v0 + j] : 0.f;
    }
    for (int n = 0; n < NC; ++n) {
        const float *src = ws + (chain * NC + n) * WsLayout<K, V>::SIZE;
        const int t0 = n * C, L = min(C, T - t0);
        __syncthreads();  // previous chunk done with the tiles
        for (int idx = tid; idx < C * K / 4; idx += 128) {
            reinterpret_cast<float4 *>(sW)[idx] = reinterpret_cast<const float4 *>(src + WsLayout<K, V>::W)[idx];
            reinterpret_cast<float4 *>(sQ)[idx] = reinterpret_cast<const float4 *>(src + WsLayout<K, V>::QP)[idx];
            reinterpret_cast<float4 *>(sKh)[idx] = reinterpret_cast<const float4 *>(src + WsLayout<K, V>::KH)[idx];
        }
        for (int idx = tid; idx < C * C / 4; idx += 128)
            reinterpret_cast<float4 *>(sP)[idx] = reinterpret_cast<const float4 *>(src + WsLayout<K, V>::P)[idx];
        for (int idx = tid; idx < C * VT; idx += 128) {
            const int r = idx / VT, j = idx % VT;
            sU[idx] = src[WsLayout<K, V>::UT + r * V + v0 + j];
        }
        for (int c = tid; c < K; c += 128) sG[c] = src[WsLayout<K, V>::GC + c];
        __syncthreads();
        // Delta = U~ - W S
        const int j = tid % VT, r0 = tid / VT;  // 8 row lanes
        for (int r = r0; r < C; r += 128 / VT) {
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < K; ++c) acc += sW[r * K + c] * sS[c * VT + j];
            sD[r * VT + j] = sU[r * VT + j] - acc;
        }
        __syncthreads();
        // O = Q+ S + P Delta  (old S)
        for (int r = r0; r < C; r += 128 / VT) {
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < K; ++c) acc += sQ[r * K + c] * sS[c * VT + j];
            for (int i = 0; i <= r; ++i) acc += sP[r * C + i] * sD[i * VT + j];
            if (r < L) store_tok(o + (((size_t)bb * T + t0 + r) * H + h) * V + v0 + j, acc);
        }
        __syncthreads();
        // S = Diag(exp(g_C)) S + K^T Delta
        for (int c = r0; c < K; c += 128 / VT) {
            float acc = sG[c] * sS[c * VT + j];
#pragma unroll 8
            for (int i = 0; i < C; ++i) acc += sKh[i * K + c] * sD[i * VT + j];
            sS[c * VT + j] = acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < K * VT; idx += 128) {
        const int c = idx / VT, jj = idx % VT;
        ST[(chain * K + c) * V + v0 + jj] = sS[idx];
    }
}

template <int K, int V>
constexpr size_t intra_smem() {
    return sizeof(float) * ((size_t)4 * C * (K + 1) + (size_t)C * V + (size_t)2 * C * (C + 1));
}
template <int K, int V>
constexpr size_t inter_smem() {
    return sizeof(float) * ((size_t)K * VT + (size_t)3 * C * K + (size_t)C * C + (size_t)2 * C * VT + K);
}

template <typename Tok, int K, int V>
static int launch_t(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                    const float *S0, void *o, float *ST, int B, int H, int T, void *ws_base, cudaStream_t st) {
    const int NC = (T + C - 1) / C;
    float *ws = reinterpret_cast<float *>(reinterpret_cast<char *>(ws_base) + kStatusBytes);
    constexpr size_t s1 = intra_smem<K, V>(), s2 = inter_smem<K, V>();
    // set on every call (cheap, idempotent, and per device): the library keeps no state
    if (cudaFuncSetAttribute(intra_kernel<Tok, K, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1) !=
            cudaSuccess ||
        cudaFuncSetAttribute(inter_kernel<Tok, K, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2) !=
            cudaSuccess)
        return -6;
    intra_kernel<Tok, K, V><<<dim3(NC, H, B), 256, s1, st>>>((const Tok *)q, (const Tok *)k, (const Tok *)v, alpha,
                                                             (const Tok *)b, (const Tok *)w, H, T, NC, ws);
    if (int e = launch_status()) return e;
    inter_kernel<Tok, K, V><<<dim3(V / VT, H, B), 128, s2, st>>>(ws, S0, (Tok *)o, ST, H, T, NC);
    return launch_status();
}

}  // namespace simt

size_t simt_workspace_bytes(int B, int H, int T, int K, int V, int C) {
    (void)C;
    const size_t NC = (size_t)(T + simt::C - 1) / simt::C;
    return kStatusBytes + sizeof(float) * (size_t)B * H * NC * simt::ws_floats_per_chunk(K, V);
}

template <typename Tok>
static int dispatch_simt(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                         const void *w, const float *S0, void *o, float *ST, int B, int H, int T, int K, int V,
                         void *ws, cudaStream_t st) {
    if (K == 128 && V == 128) return simt::launch_t<Tok, 128, 128>(q, k, v, alpha, b, w, S0, o, ST, B, H, T, ws, st);
    if (K == 128 && V == 64) return simt::launch_t<Tok, 128, 64>(q, k, v, alpha, b, w, S0, o, ST, B, H, T, ws, st);
    if (K == 64 && V == 128) return simt::launch_t<Tok, 64, 128>(q, k, v, alpha, b, w, S0, o, ST, B, H, T, ws, st);
    if (K == 64 && V == 64) return simt::launch_t<Tok, 64, 64>(q, k, v, alpha, b, w, S0, o, ST, B, H, T, ws, st);
    return -4;
}

int launch_chunk_simt(const void *q, const void *k, const void *v, const float *alpha, const void *b,
                      const void *w, const float *S0, void *o, float *ST, int B, int H, int T, int K, int V,
                      int C, int bf16, void *ws, cudaStream_t st) {
    (void)C;
    if (bf16) return dispatch_simt<__nv_bfloat16>(q, k, v, alpha, b, w, S0, o, ST, B, H, T, K, V, ws, st);
    return dispatch_simt<float>(q, k, v, alpha, b, w, S0, o, ST, B, H, T, K, V, ws, st);
}

}  // namespace gdn2
