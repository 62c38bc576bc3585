// Fused chunkwise prefill on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
// bf16 tokens, d_k = d_v = 128, chunk C = 64.  One CTA of 256 threads owns one (b, h)
// chain: it walks the chunks in order with the fp32 state S resident on chip (fp32 in
// registers, a bf16 copy in TMEM as an MMA operand) and never writes an intermediate
// to global memory.
//
// Per chunk (page "NVIDIA представила Gated DeltaNet-2 ...": the update equation of
// section "Техническая схема" in the chunkwise WY form with C = 64 of the same page;
// g = per-channel prefix of log alpha inside the chunk, e = b ⊙ k, u = w ⊙ v):
//
//   build   Ê = e ⊙ exp(g - m), Q̂ = q ⊙ exp(g - m), K̃ = k ⊙ exp(m - g), U = u,
//           Q+ = q ⊙ exp(g), K^ = k ⊙ exp(g_C - g)          (CUDA cores -> smem bf16)
//   G1      [A; P] = [Ê; Q̂] K̃^T                  (tensor core, M=128 N=64 K=128)
//   solve   T = (I + A)^-1 (unit lower triangular, fp32, 16x16 blocks + doubling)
//   G2      W'^T = Ê^T T^T,  U~^T = U^T T^T       (tensor core, two M=128 N=64 K=64)
//   W       -W = -exp(m) ⊙ W'                       (the cumulative decay that was
//           absorbed into the rank-1 factors is put back per channel)
//   G3      Delta^T = U~^T + S^T (-W)^T,  O^T = S^T Q+^T    (A = S^T from TMEM)
//   G4/G5   O^T += Delta^T P^T,  D5 = Delta^T K^             (A = Delta^T from TMEM)
//   state   S <- Diag(exp(g_C)) S + D5^T ;  o <- O
//
// m = g_C / 2 per channel is the reference point of the decay absorbed into the rank-1
// factors: every factor exp(±(g - m)) then lies in [e^-60, e^60] as long as the chunk's
// log-decay span -g_C stays <= 120 in every channel, and each product exp(g_r - g_i)
// that A and P need is formed by the tensor core from two representable factors.  A
// chunk with a larger span takes a CUDA-core path for A and P with exp(g_r - g_i) <= 1
// per element (every other step unchanged), so any alpha in (0, 1] is handled.
#include "gdn2_common.cuh"
#include "gdn2_internal.h"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace tcfwd {

using namespace gdn2::tc;

constexpr int C = 64, KD = 128, VD = 128, NT = 256;
constexpr float SPAN_MAX = 120.f;
constexpr uint32_t WAIT_LIMIT = 1u << 22;

// TMEM columns (512 allocated)
constexpr uint32_t TM_D1 = 0;     // [A; P] (64), later W'^T (64)
constexpr uint32_t TM_D3A = 64;   // U~^T, accumulated into Delta^T (64)
constexpr uint32_t TM_D3B = 192;  // O^T (64)
constexpr uint32_t TM_D5 = 256;   // (K^T Delta)^T (128)
constexpr uint32_t TM_SA = 384;   // S^T as bf16 A operand (64)
constexpr uint32_t TM_DA = 448;   // Delta^T as bf16 A operand (32)
constexpr uint32_t TM_COLS = 512;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t SM_EQ = 0;                     // [Ê; Q̂] 128 x 128 bf16
constexpr uint32_t SM_KT = 32768;                 // K̃ 64 x 128
constexpr uint32_t SM_U = 49152;                  // U 64 x 128
constexpr uint32_t SM_QP = 65536;                 // Q+ 64 x 128
constexpr uint32_t SM_KH = 81920;                 // K^ 64 x 128
constexpr uint32_t SM_NW = 98304;                 // -W^T 128 x 64
constexpr uint32_t SM_P = 114688;                 // P 64 x 64
constexpr uint32_t SM_T = 122880;                 // T 64 x 64 (SM_NW .. +32 KB: g fp32 on the CUDA-core path)
constexpr uint32_t SM_AP = 131072;                // fp32 [128][65]: rows 0-63 A, 64-127 P
constexpr uint32_t SM_TF = SM_AP + 128 * 65 * 4;  // fp32 [64][65]: T
constexpr uint32_t SM_RQ = SM_TF + 64 * 65 * 4;   // raw q bf16 [64][128] (CUDA-core path)
constexpr uint32_t SM_VEC = SM_RQ + 16384;        // exp(m)[128], exp(g_C)[128]
constexpr uint32_t SM_WT = SM_VEC + 1024;         // fp32 [8][128] warp totals / solve scratch
constexpr uint32_t SM_MISC = SM_WT + 4096;        // mbarrier, TMEM slot
constexpr uint32_t SM_BYTES = SM_MISC + 64 + 1024;  // + alignment slack

constexpr uint32_t ID_G1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G2 = idesc_bf16(128, 64, 1, 0);
constexpr uint32_t ID_G3A = idesc_bf16(128, 64, 0, 1);
constexpr uint32_t ID_G3B = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G4 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G5 = idesc_bf16(128, 128, 0, 1);

struct Bf4 {
    float x[4];
};
__device__ __forceinline__ Bf4 unpack4(uint2 u) {
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&u.x), b = *reinterpret_cast<__nv_bfloat162 *>(&u.y);
    Bf4 r;
    r.x[0] = __low2float(a);
    r.x[1] = __high2float(a);
    r.x[2] = __low2float(b);
    r.x[3] = __high2float(b);
    return r;
}
__device__ __forceinline__ void st_bf16x4(unsigned char *base, uint32_t off, float a, float b, float c, float d) {
    uint2 u;
    u.x = pack_bf16(a, b);
    u.y = pack_bf16(c, d);
    *reinterpret_cast<uint2 *>(base + off) = u;
}
__device__ __forceinline__ float bf(const unsigned char *base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}

__global__ void __launch_bounds__(NT, 1)
    chunk_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const float *__restrict__ alpha,
                    const __nv_bfloat16 *__restrict__ b, const __nv_bfloat16 *__restrict__ w,
                    const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ ST, int H,
                    int T, unsigned int *__restrict__ status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float *AP = reinterpret_cast<float *>(sm + SM_AP);
    float *TF = reinterpret_cast<float *>(sm + SM_TF);
    float *vec_em = reinterpret_cast<float *>(sm + SM_VEC);
    float *vec_gc = vec_em + 128;
    float *WT = reinterpret_cast<float *>(sm + SM_WT);
    float *G32 = reinterpret_cast<float *>(sm + SM_NW);  // CUDA-core path only
    uint64_t *mbar = reinterpret_cast<uint64_t *>(sm + SM_MISC);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + SM_MISC + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int chain = blockIdx.x, bb = chain / H, h = chain % H;
    const int NC = (T + C - 1) / C;
    const uint32_t mb = smem_u32(mbar);

    if (warp == 0) tmem_alloc(smem_u32(tslot), TM_COLS);
    if (tid == 0) {
        mbar_init(mb, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;  // this warp's TMEM lane base
    uint32_t phase = 0;
    bool failed = false;

    // state column v of S, rows c in [64*half, 64*half + 64), fp32 in registers
    const int vcol = quarter * 32 + lane;
    float s[64];
#pragma unroll
    for (int j = 0; j < 64; ++j)
        s[j] = S0 ? S0[((size_t)chain * KD + 64 * half + j) * VD + vcol] : 0.f;
    {
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(s[32 * u + 2 * i], s[32 * u + 2 * i + 1]);
            tmem_st16(tmem + lrow + TM_SA + 32 * half + 16 * u, pk);
        }
        wait_st();
    }

    const int c4 = lane * 4;     // build: channels c4..c4+3
    const int p0 = warp * 8;     // build: positions p0..p0+7

    for (int n = 0; n < NC && !failed; ++n) {
        const int t0 = n * C, L = min(C, T - t0);
        // ---------------------------------------------------------------- prefetch next chunk into L2
        if (n + 1 < NC) {
            const int t1 = t0 + C, L1 = min(C, T - t1);
            for (int line = tid; line < 896; line += NT) {
                const int tensor = line >> 7;   // 0..4 bf16 tensors, 5..6 alpha
                int r, off;
                const char *base;
                if (tensor < 5) {
                    r = (line & 127) >> 1;
                    off = (line & 1) * 128;
                    const __nv_bfloat16 *ptrs[5] = {q, k, b, v, w};
                    base = reinterpret_cast<const char *>(ptrs[tensor]);
                    if (r < L1)
                        prefetch_l2(base + ((((size_t)bb * T + t1 + r) * H + h) * KD) * 2 + off);
                } else {
                    const int l2 = line - 640;
                    r = l2 >> 2;
                    off = (l2 & 3) * 128;
                    if (r < L1)
                        prefetch_l2(reinterpret_cast<const char *>(alpha) +
                                    ((((size_t)bb * T + t1 + r) * H + h) * KD) * 4 + off);
                }
            }
        }
        // ---------------------------------------------------------------- build
        float g[8][4];
        uint2 rq[8], rk[8], rb[8], rv[8], rw[8];   // raw bf16 x4 per position
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int t = p0 + p;
            if (t < L) {
                const size_t row = ((size_t)bb * T + t0 + t) * H + h;
                const float4 a4 = *reinterpret_cast<const float4 *>(alpha + row * KD + c4);
                g[p][0] = a4.x; g[p][1] = a4.y; g[p][2] = a4.z; g[p][3] = a4.w;
                rq[p] = *reinterpret_cast<const uint2 *>(q + row * KD + c4);
                rk[p] = *reinterpret_cast<const uint2 *>(k + row * KD + c4);
                rb[p] = *reinterpret_cast<const uint2 *>(b + row * KD + c4);
                rv[p] = *reinterpret_cast<const uint2 *>(v + row * VD + c4);
                rw[p] = *reinterpret_cast<const uint2 *>(w + row * VD + c4);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) g[p][j] = 1.f;
                rq[p] = rk[p] = rb[p] = rv[p] = rw[p] = make_uint2(0u, 0u);
            }
        }
        float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < 8; ++p)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                run[j] += __logf(g[p][j]);
                g[p][j] = run[j];
            }
        *reinterpret_cast<float4 *>(WT + warp * 128 + c4) = make_float4(run[0], run[1], run[2], run[3]);
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
#pragma unroll
        for (int p = 0; p < 8; ++p)
#pragma unroll
            for (int j = 0; j < 4; ++j) g[p][j] += pre[j];
        int wide = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) wide |= (-gC[j] > SPAN_MAX);
        const bool slow = __syncthreads_or(wide) != 0;   // also: everyone is done reading WT

        float m[4], em[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            m[j] = slow ? 0.f : 0.5f * gC[j];
            em[j] = slow ? 1.f : __expf(m[j]);
        }
        if (warp == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                vec_em[c4 + j] = em[j];
                vec_gc[c4 + j] = __expf(gC[j]);
            }
        }
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int r = p0 + p;
            const Bf4 qv = unpack4(rq[p]), kv = unpack4(rk[p]), bv = unpack4(rb[p]), vv = unpack4(rv[p]),
                      wv = unpack4(rw[p]);
            float E[4], Qh[4], Kt[4], U[4], Qp[4], Kh[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float e = bv.x[j] * kv.x[j];
                U[j] = wv.x[j] * vv.x[j];
                if (!slow) {
                    const float f1 = __expf(g[p][j] - m[j]);
                    const float f2 = __expf(m[j] - g[p][j]);
                    E[j] = e * f1;
                    Qh[j] = qv.x[j] * f1;
                    Kt[j] = kv.x[j] * f2;
                    Qp[j] = Qh[j] * em[j];
                    Kh[j] = Kt[j] * em[j];
                } else {
                    const float gam = __expf(g[p][j]);
                    E[j] = e * gam;                 // exp(g) ⊙ e, used by G2 directly
                    Qh[j] = e;                      // raw e for the CUDA-core A/P
                    Kt[j] = kv.x[j];             // raw k
                    Qp[j] = qv.x[j] * gam;
                    Kh[j] = kv.x[j] * __expf(gC[j] - g[p][j]);
                }
            }
            st_bf16x4(sm + SM_EQ, sw_off(r, c4, 128), E[0], E[1], E[2], E[3]);
            st_bf16x4(sm + SM_EQ, sw_off(64 + r, c4, 128), Qh[0], Qh[1], Qh[2], Qh[3]);
            st_bf16x4(sm + SM_KT, sw_off(r, c4, 64), Kt[0], Kt[1], Kt[2], Kt[3]);
            st_bf16x4(sm + SM_U, sw_off(r, c4, 64), U[0], U[1], U[2], U[3]);
            st_bf16x4(sm + SM_QP, sw_off(r, c4, 64), Qp[0], Qp[1], Qp[2], Qp[3]);
            st_bf16x4(sm + SM_KH, sw_off(r, c4, 64), Kh[0], Kh[1], Kh[2], Kh[3]);
            if (slow) {
                *reinterpret_cast<float4 *>(G32 + r * 128 + c4) = make_float4(g[p][0], g[p][1], g[p][2], g[p][3]);
                st_bf16x4(sm + SM_RQ, (uint32_t)(r * 256 + c4 * 2), qv.x[0], qv.x[1], qv.x[2], qv.x[3]);
            }
        }
        fence_async_smem();
        fence_before();
        __syncthreads();

        // ---------------------------------------------------------------- A and P
        if (!slow) {
            if (tid == 0) {
                fence_after();
                const uint32_t aEQ = smem_u32(sm + SM_EQ), aKT = smem_u32(sm + SM_KT);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    mma_ss(tmem + TM_D1, desc_kmajor(aEQ, 128, j), desc_kmajor(aKT, 64, j), ID_G1, j > 0);
                mma_commit(mb);
            }
            const bool ok = mbar_wait(mb, phase, WAIT_LIMIT);
            phase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
            fence_after();
            uint32_t r32[32];
            tmem_ld32(tmem + lrow + TM_D1 + 32 * half, r32);
            wait_ld();
            const int row = quarter * 32 + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int col = 32 * half + i;
                const float val = __uint_as_float(r32[i]);
                const bool keep = row < 64 ? (col < row) : (col <= row - 64);
                AP[row * 65 + col] = keep ? val : 0.f;
            }
        } else {
            // A_ri = sum_c e_rc k_ic exp(g_rc - g_ic) (i < r), P_ri = sum_c q_rc k_ic exp(..) (i <= r)
            for (int pair = warp; pair < 64 * 64; pair += 8) {
                const int r = pair >> 6, i = pair & 63;
                float a = 0.f, pp = 0.f;
                if (i <= r) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c = lane + 32 * u;
                        const float d = __expf(G32[r * 128 + c] - G32[i * 128 + c]);
                        const float kd = bf(sm + SM_KT, sw_off(i, c, 64)) * d;
                        a += bf(sm + SM_EQ, sw_off(64 + r, c, 128)) * kd;
                        pp += bf(sm + SM_RQ, (uint32_t)(r * 256 + c * 2)) * kd;
                    }
#pragma unroll
                    for (int msk = 16; msk > 0; msk >>= 1) {
                        a += __shfl_xor_sync(0xffffffffu, a, msk);
                        pp += __shfl_xor_sync(0xffffffffu, pp, msk);
                    }
                }
                if (lane == 0) {
                    AP[r * 65 + i] = (i < r) ? a : 0.f;
                    AP[(64 + r) * 65 + i] = (i <= r) ? pp : 0.f;
                }
            }
        }
        __syncthreads();

        // ---------------------------------------------------------------- T = (I + A)^-1
        {   // P rows -> bf16 P tile (all threads); diagonal 16x16 blocks of T (threads 0..63)
            const int r = tid >> 2, i0 = 16 * (tid & 3);
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(AP[(64 + r) * 65 + i0 + 2 * i], AP[(64 + r) * 65 + i0 + 2 * i + 1]);
            *reinterpret_cast<uint4 *>(sm + SM_P + sw_off(r, i0, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4 *>(sm + SM_P + sw_off(r, i0 + 8, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        if (tid < 64) {
            const int J = tid >> 4, j = tid & 15, o16 = 16 * J;
            float col[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == j) ? 1.f : 0.f;
                if (r > j) {
                    float s0 = 0.f, s1 = 0.f;
#pragma unroll
                    for (int i = 0; i < r; i += 2) {
                        if (i >= j) s0 += AP[(o16 + r) * 65 + o16 + i] * col[i];
                        if (i + 1 < r && i + 1 >= j) s1 += AP[(o16 + r) * 65 + o16 + i + 1] * col[i + 1];
                    }
                    acc = -(s0 + s1);
                }
                col[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) TF[(o16 + r) * 65 + o16 + j] = col[r];
        }
        __syncthreads();
        {   // blocks (1,0) and (3,2): T_RI = -T_RR A_RI T_II
            const int J = tid >> 7, idx = tid & 127, r = idx >> 3, c2 = (idx & 7) * 2;
            const int R = 16 * (2 * J + 1), I = 16 * (2 * J);
            float x0 = 0.f, x1 = 0.f;
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                const float a = AP[(R + r) * 65 + I + kk];
                x0 += a * TF[(I + kk) * 65 + I + c2];
                x1 += a * TF[(I + kk) * 65 + I + c2 + 1];
            }
            WT[J * 256 + r * 16 + c2] = x0;
            WT[J * 256 + r * 16 + c2 + 1] = x1;
            __syncthreads();
            float y0 = 0.f, y1 = 0.f;
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                const float t = TF[(R + r) * 65 + R + kk];
                y0 += t * WT[J * 256 + kk * 16 + c2];
                y1 += t * WT[J * 256 + kk * 16 + c2 + 1];
            }
            TF[(R + r) * 65 + I + c2] = -y0;
            TF[(R + r) * 65 + I + c2 + 1] = -y1;
        }
        __syncthreads();
        {   // rows 32..63 x cols 0..31: T = -T_hi A_hi,lo T_lo
            const int r = tid >> 3, cq = (tid & 7) * 4;
            const int k0 = cq >= 16 ? 16 : 0;
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            for (int kk = k0; kk < 32; ++kk) {
                const float a = AP[(32 + r) * 65 + kk];
#pragma unroll
                for (int u = 0; u < 4; ++u) x[u] += a * TF[kk * 65 + cq + u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) WT[r * 32 + cq + u] = x[u];
            __syncthreads();
            const int k1 = r < 16 ? 16 : 32;
            float y[4] = {0.f, 0.f, 0.f, 0.f};
            for (int kk = 0; kk < k1; ++kk) {
                const float t = TF[(32 + r) * 65 + 32 + kk];
#pragma unroll
                for (int u = 0; u < 4; ++u) y[u] += t * WT[kk * 32 + cq + u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) TF[(32 + r) * 65 + cq + u] = -y[u];
        }
        __syncthreads();
        {   // T -> bf16 tile (zero above the diagonal, one on it)
            const int r = tid >> 2, i0 = 16 * (tid & 3);
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c0 = i0 + 2 * i, c1 = c0 + 1;
                const float v0 = c0 < r ? TF[r * 65 + c0] : (c0 == r ? 1.f : 0.f);
                const float v1 = c1 < r ? TF[r * 65 + c1] : (c1 == r ? 1.f : 0.f);
                pk[i] = pack_bf16(v0, v1);
            }
            *reinterpret_cast<uint4 *>(sm + SM_T + sw_off(r, i0, 64)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4 *>(sm + SM_T + sw_off(r, i0 + 8, 64)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        fence_async_smem();
        fence_before();
        __syncthreads();

        // ---------------------------------------------------------------- G2: W'^T, U~^T
        if (tid == 0) {
            fence_after();
            const uint32_t aEQ = smem_u32(sm + SM_EQ), aU = smem_u32(sm + SM_U), aT = smem_u32(sm + SM_T);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + TM_D1, desc_mnmajor(aEQ, 128, j), desc_kmajor(aT, 64, j), ID_G2, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + TM_D3A, desc_mnmajor(aU, 64, j), desc_kmajor(aT, 64, j), ID_G2, j > 0);
            mma_commit(mb);
        }
        {
            const bool ok = mbar_wait(mb, phase, WAIT_LIMIT);
            phase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        fence_after();
        {   // -W^T[c][r] = -exp(m_c) W'^T[c][r]  -> bf16 tile NW (row c, MN-major B of G3)
            const int c = quarter * 32 + lane;
            uint32_t r32[32];
            tmem_ld32(tmem + lrow + TM_D1 + 32 * half, r32);
            wait_ld();
            const float sc = -vec_em[c];
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16(sc * __uint_as_float(r32[2 * i]), sc * __uint_as_float(r32[2 * i + 1]));
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4 *>(sm + SM_NW + sw_off(c, 32 * half + 8 * u, 128)) =
                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        fence_async_smem();
        fence_before();
        __syncthreads();

        // ---------------------------------------------------------------- G3: Delta^T, O^T
        if (tid == 0) {
            fence_after();
            const uint32_t aNW = smem_u32(sm + SM_NW), aQP = smem_u32(sm + SM_QP);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ts(tmem + TM_D3A, tmem + TM_SA + 8 * j, desc_mnmajor(aNW, 128, j), ID_G3A, 1);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ts(tmem + TM_D3B, tmem + TM_SA + 8 * j, desc_kmajor(aQP, 64, j), ID_G3B, j > 0);
            mma_commit(mb);
        }
        {
            const bool ok = mbar_wait(mb, phase, WAIT_LIMIT);
            phase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        fence_after();
        {   // Delta^T -> bf16 A operand in TMEM
            uint32_t r32[32];
            tmem_ld32(tmem + lrow + TM_D3A + 32 * half, r32);
            wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(r32[2 * i]), __uint_as_float(r32[2 * i + 1]));
            tmem_st16(tmem + lrow + TM_DA + 16 * half, pk);
            wait_st();
        }
        fence_before();
        __syncthreads();

        // ---------------------------------------------------------------- G4, G5
        if (tid == 0) {
            fence_after();
            const uint32_t aP = smem_u32(sm + SM_P), aKH = smem_u32(sm + SM_KH);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ts(tmem + TM_D3B, tmem + TM_DA + 8 * j, desc_kmajor(aP, 64, j), ID_G4, 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ts(tmem + TM_D5, tmem + TM_DA + 8 * j, desc_mnmajor(aKH, 64, j), ID_G5, j > 0);
            mma_commit(mb);
        }
        {
            const bool ok = mbar_wait(mb, phase, WAIT_LIMIT);
            phase ^= 1;
            if (__syncthreads_or(!ok)) { failed = true; break; }
        }
        fence_after();
        {   // S <- Diag(exp(g_C)) S + D5^T ; bf16 copy back to TMEM
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                uint32_t r32[32];
                tmem_ld32(tmem + lrow + TM_D5 + 64 * half + 32 * u, r32);
                wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int j = 32 * u + i;
                    s[j] = vec_gc[64 * half + j] * s[j] + __uint_as_float(r32[i]);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(s[32 * u + 2 * i], s[32 * u + 2 * i + 1]);
                tmem_st16(tmem + lrow + TM_SA + 32 * half + 16 * u, pk);
            }
            // o[t0 + r, v] for r in [32*half, 32*half + 32)
            uint32_t r32[32];
            tmem_ld32(tmem + lrow + TM_D3B + 32 * half, r32);
            wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int r = 32 * half + i;
                if (r < L)
                    o[(((size_t)bb * T + t0 + r) * H + h) * VD + vcol] = __float2bfloat16_rn(__uint_as_float(r32[i]));
            }
            wait_st();
        }
        fence_before();
        __syncthreads();
    }

    if (failed) {
        if (tid == 0) atomicOr(status, 1u);
    } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) ST[((size_t)chain * KD + 64 * half + j) * VD + vcol] = s[j];
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
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
