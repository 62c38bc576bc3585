// Backward pass of the recurrence on the tensor cores (tcgen05 + TMEM, bulk and TMA copies), sm_100a.
// bf16 tokens, d_k = d_v = 128, chunk C = 64.
//
// Page "NVIDIA представила Gated DeltaNet-2 ...": the state-update equation (section "Техническая
// схема") in the chunkwise WY form with C = 64 (the paragraph on the chunkwise kernels, which also asks
// for a backward whose gradients account for the per-channel gates).  The forward chunk in the framed
// variables of the two-stage prefill (e = b ⊙ k, u = w ⊙ v, g = per-channel log2-decay prefix):
//   Ê = e ⊙ 2^(g - ae), Q̂ = q ⊙ 2^(g - ae), K̃ = k ⊙ 2^(ak - g)     (ae, ak: the chunk's frame exponents)
//   A = strict(Ê K̃^T), P = lower(Q̂ K̃^T), T = (I + A)^-1, Z̃ = Diag(sS) S (bf16)
//   Delta = T (U - Ê Z̃),  O = Q̂ Z̃ + P Delta,  S' = Diag(sPost) (Diag(sZ) S + K̃^T Delta)
// is differentiated as the transpose of each product.  Given dO and dS' (the gradient at the chunk's
// outgoing state):
//   G̃ = Diag(sPost) dS'
//   dDelta = P^T dO + K̃ G̃,        dR = T^T dDelta                      (dU = dR)
//   dA = -strict(dR Delta^T),     dP = lower(dO Delta^T)
//   dÊ = -dR Z̃^T + dA K̃,         dQ̂ = dO Z̃^T + dP K̃,    dK̃ = dA^T Ê + dP^T Q̂ + Delta G̃^T
//   dS = Diag(sS) (Q̂^T dO - W'^T dDelta) + Diag(sZ sPost) dS'          (W' = T Ê)
// and the token gradients follow elementwise: de = 2^(g - ae) ⊙ dÊ, dq = 2^(g - ae) ⊙ dQ̂, the key's own
// part dk' = 2^(ak - g) ⊙ dK̃, dk = dk' + b ⊙ de, db = k ⊙ de, dv = w ⊙ dR, dw = v ⊙ dR; the decay
// through d(ln alpha_r) = sum_{s >= r} (q ⊙ dq + e ⊙ de - k ⊙ dk')_s + rowsum(dS' ⊙ S'), the last term
// because S' scales with the chunk's whole decay.
//
// Three stages, after a forward replay by the two-stage prefill's kernels that keeps, per chunk-head,
// the record and a side record (Ê, T, Z̃, Delta and the frame exponents):
//   rwalk_kernel: one CTA per (batch, head) chain walks the chunks backwards with the state gradient
//     resident in TMEM as dY (dS = Diag(sS) dY): per chunk
//       W1  dS' = Diag(sS_next) dY, G̃ = Diag(sPost) dS' (bf16 image), dY <- Diag(sZ / sS) G̃;
//           rho = rowsum(dS' ⊙ S') in fp32 from the next chunk's saved state operand
//       B1  dDelta^T = dO^T P + G̃^T K̃^T                           (tcgen05, M128 N64)
//       B2  dY += [-W'; Q̂]^T [dDelta; dO]                         (tcgen05, M128 N128 K128)
//     and stores G̃, dDelta and rho in the side record.
//   grad_kernel: every chunk-head in parallel (one CTA per SM):
//       D1  dR = T^T dDelta;  D2  [dA; dP] = [-dR; dO] Delta^T;
//       D3  [dÊ; dQ̂] = [-dR; dO] Z̃^T + [dA; dP] K̃;  D4  dK̃ = Delta G̃^T + dA^T Ê + dP^T Q̂
//     then the elementwise gradients and the decay's reverse sums over the chunk.
// Every wait is bounded; on expiry a kernel sets the workspace status word and stops.
#include <cuda.h>
#include <float.h>

#include <algorithm>

#include "gdn2_common.cuh"
#include "gdn2_internal.h"
#include "split_layout.cuh"
#include "tc_chunk.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace bwdtc {

using namespace gdn2::tc;
using namespace gdn2::tcc;
using namespace gdn2::split;

constexpr uint32_t WAIT_LIMIT = 1u << 22;
constexpr uint32_t STATUS_RWALK = 16u, STATUS_GRAD = 32u;

__device__ __forceinline__ bool group_wait(uint32_t mb, uint32_t parity, uint32_t bar, uint32_t n,
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
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// ============================================================================ reverse walk
// Warps 0-7: TMEM lane quarter w % 4 (state row c), value-column half w / 4.  Warp 8 issues the copies
// of each chunk's record parts (-W', Q̂, K̃, P, the frame factors) and dO tile into a double-buffered slot.
constexpr int RW_NT = 288;
constexpr uint32_t RS_A3 = 0, RS_KT = 32768, RS_P = 49152, RS_VEC = 57344, RS_DO = 59392, RS_BYTES = 75776;
constexpr uint32_t RS_LOAD = (R_U - R_A3) + (R_COPY - R_P) + 16384;   // bytes landing in a slot
constexpr uint32_t RW_G = 2 * RS_BYTES;      // G̃ [c x v] (MN-major A of B1)
constexpr uint32_t RW_DD = RW_G + 32768;     // dDelta as [v x i] (K-major B of B2)
constexpr uint32_t RW_MISC = RW_DD + 16384;
constexpr uint32_t RW_RHO = RW_MISC + 256;   // rho partials [2][128]
constexpr uint32_t RW_BYTES = RW_RHO + 1024 + 1024;
enum : uint32_t { MR_FULL = 0, MR_B2 = 16, MR_B1 = 32, MR_TSLOT = 48, MR_ABORT = 52 };
constexpr uint32_t RW_TM_Y = 0, RW_TM_D = 128, RW_TM_COLS = 256;
constexpr uint32_t RBAR = 1;
constexpr uint32_t ID_B1A = idesc_bf16(128, 64, 1, 1);    // dO^T P
constexpr uint32_t ID_B1B = idesc_bf16(128, 64, 1, 0);    // G̃^T K̃^T
constexpr uint32_t ID_B2A = idesc_bf16(128, 128, 1, 0);   // (-W')^T dDelta
constexpr uint32_t ID_B2B = idesc_bf16(128, 128, 1, 1);   // Q̂^T dO

__global__ void __launch_bounds__(RW_NT, 1)
    rwalk_kernel(const __grid_constant__ CUtensorMap map_do, const unsigned char *records, unsigned char *aux,
                 const float *dST, const float *STf, float *dS0, int H, int NC, unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int chain = blockIdx.x, bb = chain / H, h = chain % H;
    const uint32_t misc = smem_u32(sm + RW_MISC);
    volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sm + RW_MISC + MR_ABORT);

    if (warp == 0) tmem_alloc(misc + MR_TSLOT, RW_TM_COLS);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(misc + MR_FULL + 8 * s, 1);
            mbar_init(misc + MR_B2 + 8 * s, 1);
        }
        mbar_init(misc + MR_B1, 1);
        *abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&map_do);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + RW_MISC + MR_TSLOT);
    auto idx = [&](int n) { return ((size_t)bb * NC + n) * H + h; };   // chunk-head number of chunk n
    auto slot_addr = [&](int nl) { return (uint32_t)(nl & 1) * RS_BYTES; };

    if (warp < 8) {
        const int q4 = warp & 3, half = warp >> 2, cb = 64 * half;
        const int crow = 32 * q4 + lane;
        const uint32_t lq = (uint32_t)(32 * q4) << 16;
        const uint32_t aG = smem_u32(sm + RW_G), aDD = smem_u32(sm + RW_DD);
        float *rho_part = reinterpret_cast<float *>(sm + RW_RHO);
        float ss_next = 1.f;   // sS of the chunk after the current one (dS' = dS_T at the last chunk)
        bool ok = true;
        for (int nl = 0; nl < NC; ++nl) {
            const int n = NC - 1 - nl;
            const uint32_t slot = slot_addr(nl);
            // the state at the end of chunk n, for rho: chunk n+1's saved bf16 operand (its row crow, the
            // columns cb..cb+63, 16-byte units read in logical order out of the swizzle), or S_T itself
            uint4 zt[8];
            if (nl > 0) {
                const unsigned char *zr = aux + idx(n + 1) * X_BYTES + X_Z + half * 16384 + crow * 128;
#pragma unroll
                for (int u = 0; u < 8; ++u) zt[u] = *reinterpret_cast<const uint4 *>(zr + 16 * (u ^ (crow & 7)));
            }
            {
                if (tid == 0) bulk_wait_read_all();   // the previous chunk's G̃ and dDelta copies have read them
                bool w_ok = mbar_wait(misc + MR_FULL + 8 * (nl & 1), (uint32_t)((nl >> 1) & 1), WAIT_LIMIT);
                if (nl > 0)
                    w_ok = w_ok && mbar_wait(misc + MR_B2 + 8 * ((nl - 1) & 1), (uint32_t)(((nl - 1) >> 1) & 1), WAIT_LIMIT);
                w_ok = w_ok && !*abort;
                const bool fail = group_or(RBAR, 256, !w_ok);
                fence_after();
                if (fail) { *abort = 1u; ok = false; break; }
            }
            const uint32_t aDO = smem_u32(sm + slot + RS_DO);
            if (tid == 0) {   // B1, first part: dDelta^T = dO^T P (needs no state gradient)
                const uint32_t aP = smem_u32(sm + slot + RS_P);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ss(tmem + RW_TM_D, desc_mnmajor(aDO, 64, j), desc_mnmajor(aP, 64, j), ID_B1A, j > 0);
            }
            // ---------------------------------------------------------------- W1
            const float *vec = reinterpret_cast<const float *>(sm + slot + RS_VEC);
            // sZ / sS is 1 on a tensor-core chunk (sZ = sS, even when 2^m has flushed to zero) and sZ on a
            // wide-span chunk (sS = 1)
            const float ssn = vec[crow], zsc = vec[128 + crow], zr = zsc == ssn ? 1.f : zsc / ssn, post = vec[256 + crow];
            float rho = 0.f;
            uint32_t x0[32], x1[32];
            __syncwarp();
            if (nl > 0) {
                tmem_ld32(tmem + lq + RW_TM_Y + cb, x0);
                tmem_ld32(tmem + lq + RW_TM_Y + cb + 32, x1);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 8; ++u) {   // rho = sum_v dY Z̃ of the next chunk: its frame factors cancel
                    const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
                    const uint32_t zw[4] = {zt[u].x, zt[u].y, zt[u].z, zt[u].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        rho += __uint_as_float(x[2 * i]) * bf_lo(zw[i]) + __uint_as_float(x[2 * i + 1]) * bf_hi(zw[i]);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x0[i] = __float_as_uint(ss_next * __uint_as_float(x0[i]));
                    x1[i] = __float_as_uint(ss_next * __uint_as_float(x1[i]));
                }
            } else {   // dS' = dS_T (or 0), S' = S_T
                const float *gp = dST ? dST + ((size_t)chain * KD + crow) * VD + cb : nullptr;
                const float *sp = STf + ((size_t)chain * KD + crow) * VD + cb;
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 a = gp ? *reinterpret_cast<const float4 *>(gp + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 c = gp ? *reinterpret_cast<const float4 *>(gp + 32 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 s4 = *reinterpret_cast<const float4 *>(sp + i);
                    const float4 t4 = *reinterpret_cast<const float4 *>(sp + 32 + i);
                    rho += a.x * s4.x + a.y * s4.y + a.z * s4.z + a.w * s4.w;
                    rho += c.x * t4.x + c.y * t4.y + c.z * t4.z + c.w * t4.w;
                    x0[i] = __float_as_uint(a.x); x0[i + 1] = __float_as_uint(a.y);
                    x0[i + 2] = __float_as_uint(a.z); x0[i + 3] = __float_as_uint(a.w);
                    x1[i] = __float_as_uint(c.x); x1[i + 1] = __float_as_uint(c.y);
                    x1[i + 2] = __float_as_uint(c.z); x1[i + 3] = __float_as_uint(c.w);
                }
            }
            // G̃ = Diag(sPost) dS' -> bf16 image; dY <- Diag(sZ / sS) G̃ (the factors one after the other)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x0[i] = __float_as_uint(post * __uint_as_float(x0[i]));
                x1[i] = __float_as_uint(post * __uint_as_float(x1[i]));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
                const uint4 pk = make_uint4(pack_bf16(__uint_as_float(x[0]), __uint_as_float(x[1])),
                                            pack_bf16(__uint_as_float(x[2]), __uint_as_float(x[3])),
                                            pack_bf16(__uint_as_float(x[4]), __uint_as_float(x[5])),
                                            pack_bf16(__uint_as_float(x[6]), __uint_as_float(x[7])));
                *reinterpret_cast<uint4 *>(sm + RW_G + sw_off(crow, cb + 8 * u, 128)) = pk;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                x0[i] = __float_as_uint(zr * __uint_as_float(x0[i]));
                x1[i] = __float_as_uint(zr * __uint_as_float(x1[i]));
            }
            tmem_st32(tmem + lq + RW_TM_Y + cb, x0);
            tmem_st32(tmem + lq + RW_TM_Y + cb + 32, x1);
            wait_st();
            ss_next = ssn;
            rho_part[half * 128 + crow] = rho;
            fence_async_smem();
            fence_before();
            group_sync(RBAR, 256);
            if (tid == 0) {   // B1, second part: dDelta^T += G̃^T K̃^T; G̃ out to the side record
                fence_after();
                const uint32_t aKT = smem_u32(sm + slot + RS_KT);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    mma_ss(tmem + RW_TM_D, desc_mnmajor(aG, 128, j), desc_kmajor(aKT, 64, j), ID_B1B, 1);
                mma_commit(misc + MR_B1);
                bulk_s2g(aux + idx(n) * X_BYTES + X_G, aG, 32768);
                bulk_commit();
            }
            if (half == 0)
                reinterpret_cast<float *>(aux + idx(n) * X_BYTES + X_RHO)[crow] = rho_part[crow] + rho_part[128 + crow];
            // ---------------------------------------------------------------- dDelta^T (lane v, column i) -> bf16 [v x i]
            if (!group_wait(misc + MR_B1, (uint32_t)(nl & 1), RBAR, 256, abort)) { ok = false; break; }
            __syncwarp();
            {
                uint32_t y[32];
                tmem_ld32(tmem + lq + RW_TM_D + 32 * half, y);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t *x = y + 8 * u;
                    const uint4 pk = make_uint4(pack_bf16(__uint_as_float(x[0]), __uint_as_float(x[1])),
                                                pack_bf16(__uint_as_float(x[2]), __uint_as_float(x[3])),
                                                pack_bf16(__uint_as_float(x[4]), __uint_as_float(x[5])),
                                                pack_bf16(__uint_as_float(x[6]), __uint_as_float(x[7])));
                    *reinterpret_cast<uint4 *>(sm + RW_DD + sw_off(crow, 32 * half + 8 * u, 128)) = pk;
                }
            }
            fence_async_smem();
            fence_before();
            group_sync(RBAR, 256);
            if (tid == 0) {   // B2: dY += (-W')^T dDelta + Q̂^T dO; dDelta out to the side record
                fence_after();
                const uint32_t aA3 = smem_u32(sm + slot + RS_A3);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ss(tmem + RW_TM_Y, desc_mnmajor(aA3, 128, j), desc_kmajor(aDD, 128, j), ID_B2A, 1);
#pragma unroll
                for (int j = 4; j < 8; ++j)
                    mma_ss(tmem + RW_TM_Y, desc_mnmajor(aA3, 128, j), desc_mnmajor(aDO, 64, j - 4), ID_B2B, 1);
                mma_commit(misc + MR_B2 + 8 * (nl & 1));
                bulk_s2g(aux + idx(n) * X_BYTES + X_DD, aDD, 16384);
                bulk_commit();
            }
        }
        // dS0 = Diag(sS_0) dY once the first chunk's B2 is complete
        ok = ok && NC > 0 &&
             group_wait(misc + MR_B2 + 8 * ((NC - 1) & 1), (uint32_t)(((NC - 1) >> 1) & 1), RBAR, 256, abort);
        __syncwarp();
        if (ok && dS0) {
            float *dst = dS0 + ((size_t)chain * KD + crow) * VD + cb;
            uint32_t x0[32], x1[32];
            tmem_ld32(tmem + lq + RW_TM_Y + cb, x0);
            tmem_ld32(tmem + lq + RW_TM_Y + cb + 32, x1);
            wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                *reinterpret_cast<float4 *>(dst + i) =
                    make_float4(ss_next * __uint_as_float(x0[i]), ss_next * __uint_as_float(x0[i + 1]),
                                ss_next * __uint_as_float(x0[i + 2]), ss_next * __uint_as_float(x0[i + 3]));
                *reinterpret_cast<float4 *>(dst + 32 + i) =
                    make_float4(ss_next * __uint_as_float(x1[i]), ss_next * __uint_as_float(x1[i + 1]),
                                ss_next * __uint_as_float(x1[i + 2]), ss_next * __uint_as_float(x1[i + 3]));
            }
        }
        if (tid == 0) bulk_wait_all();   // the side-record copies complete before the block exits
    } else if (lane == 0) {
        // ------------------------------------------------------------------ producer
        int last0 = -1, last1 = -1;   // the last step that loaded slot 0 / slot 1
        for (int nl = 0; nl < NC; ++nl) {
            const int n = NC - 1 - nl;
            if (nl >= 2 && !thread_wait(misc + MR_B2 + 8 * (nl & 1), (uint32_t)(((nl - 2) >> 1) & 1), abort)) break;
            const uint32_t fb = misc + MR_FULL + 8 * (nl & 1), dst = smem_u32(sm + slot_addr(nl));
            const unsigned char *rec = records + idx(n) * R_BYTES;
            mbar_arrive_expect_tx(fb, RS_LOAD);
            bulk_g2s(dst + RS_A3, rec + R_A3, R_U - R_A3, fb);       // [-W'; Q̂] and K̃
            bulk_g2s(dst + RS_P, rec + R_P, R_COPY - R_P, fb);       // P and the frame factors
            tma_load_4d(dst + RS_DO, &map_do, 0, h, n * C, bb, fb);
            tma_load_4d(dst + RS_DO + 8192, &map_do, 64, h, n * C, bb, fb);
            if (nl & 1) last1 = nl; else last0 = nl;
        }
        // no copy may be left in flight when the block exits
        if (last0 >= 0) mbar_wait(misc + MR_FULL, (uint32_t)((last0 >> 1) & 1), WAIT_LIMIT);
        if (last1 >= 0) mbar_wait(misc + MR_FULL + 8, (uint32_t)((last1 >> 1) & 1), WAIT_LIMIT);
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0 && *abort) atomicOr(status, STATUS_RWALK);
    if (warp == 0) tmem_dealloc(tmem, RW_TM_COLS);
}

// ============================================================================ gradient kernel
// One CTA per chunk-head (one resident per SM), 8 warps: TMEM lane quarter w % 4, column half w / 4.
// Shared memory: the operand images, each placed so that the 128-row reads of a 64-row operand (the
// upper lanes of D1 and D4, never read back) stay inside the allocation.
constexpr int GK_NT = 256;
constexpr uint32_t G_T = 0;          // T [r x i]              (MN-major A of D1; its upper lanes read G_DD)
constexpr uint32_t G_DD = 8192;      // dDelta [v x i]         (K-major B of D1)
constexpr uint32_t G_RO = 24576;     // [-dR; dO] [r' x v]     (K-major A of D2, D3)
constexpr uint32_t G_Z = 57344;      // Z̃ [c x v]              (K-major B of D3)
constexpr uint32_t G_DL = 90112;     // Delta [i x v]          (K-major B of D2, A of D4)
constexpr uint32_t G_A2 = 106496;    // [dA; dP] [r' x i]      (K-major A of D3, MN-major A of D4)
constexpr uint32_t G_KT = 122880;    // K̃ [i x c]              (MN-major B of D3)
constexpr uint32_t G_E = 139264;     // Ê [r x c]              (MN-major B of D4)
constexpr uint32_t G_Q = 155648;     // Q̂ [r x c]              (MN-major B of D4)
constexpr uint32_t G_G = 172032;     // G̃ [c x v]              (K-major B of D4)
constexpr uint32_t G_MISC = 204800;
constexpr uint32_t G_VEC = G_MISC + 256;   // ae, ak, rho, then two [128] hand-over sums: 5 x 128 fp32
constexpr uint32_t G_BYTES = G_VEC + 2560 + 1024;
// fp32 [64][GLD] arrays of the epilogue, over operand images that are dead by then ([dA; dP] stays: a
// wide-span chunk reads it once more)
constexpr int GLD = 132;
constexpr uint32_t G_PRE = 0, G_H1 = G_PRE + 64 * GLD * 4, G_HQ = G_KT;
static_assert(G_H1 + 64 * GLD * 4 <= G_A2 && G_HQ + 64 * GLD * 4 <= G_MISC, "epilogue arrays overlap");
enum : uint32_t { MG_L1 = 0, MG_L2 = 8, MG_L3 = 16, MG_M1 = 24, MG_M2 = 32, MG_M4 = 40, MG_TSLOT = 48, MG_ABORT = 52 };
constexpr uint32_t GT_D1 = 0, GT_D2 = 128, GT_D3 = 192, GT_D4 = 320, GT_COLS = 512;
constexpr uint32_t GBAR = 1;
constexpr uint32_t ID_D1 = idesc_bf16(128, 128, 1, 0);
constexpr uint32_t ID_D2 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_D3A = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t ID_D3B = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_D4A = idesc_bf16(128, 128, 0, 0);
constexpr uint32_t ID_D4B = idesc_bf16(128, 128, 1, 1);

__device__ __forceinline__ float bf_at(const unsigned char *p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p)); }

// Wide-span chunk: A and P were formed exactly, outside the factored frame, so the terms of dÊ, dQ̂ and
// dK̃ that pass through them are summed here on CUDA cores with the exact factor 2^(g_j - g_i) <= 1
// (j >= i) of each element (a rare correctness path, kept out of line).  M is the bf16 [dA; dP] tile,
// tokens are read from global memory (row0: the chunk's first token row, stride: rows per step), pre
// is the log2-decay prefix [64][GLD].
//   sum_{i < iend} M[arow][i] x_i[c] 2^(g_r[c] - g_i[c])                 (dA k -> dÊ, dP k -> dQ̂)
__device__ __noinline__ float wide_row_sum(const unsigned char *M, int arow, int r, int iend, const __nv_bfloat16 *x,
                                           size_t row0, size_t stride, const float *pre, int c) {
    float s = 0.f;
    const float gr = pre[r * GLD + c];
    for (int i = 0; i < iend; ++i) {
        const float m = bf_at(M + sw_off(arow, i, 128));
        if (m != 0.f) s += m * __bfloat162float(x[(row0 + (size_t)i * stride) * KD + c]) * exp2f(gr - pre[i * GLD + c]);
    }
    return s;
}
//   sum_{jbeg <= j < jend} M[moff + j][i] x_j[c] (y_j[c]) 2^(g_j[c] - g_i[c])   (dA^T e, dP^T q -> dK̃)
__device__ __noinline__ float wide_col_sum(const unsigned char *M, int moff, int i, int jbeg, int jend,
                                           const __nv_bfloat16 *x, const __nv_bfloat16 *y, size_t row0, size_t stride,
                                           const float *pre, int c) {
    float s = 0.f;
    const float gi = pre[i * GLD + c];
    for (int j = jbeg; j < jend; ++j) {
        const float m = bf_at(M + sw_off(moff + j, i, 128));
        if (m != 0.f) {
            const size_t o = (row0 + (size_t)j * stride) * KD + c;
            float t = __bfloat162float(x[o]);
            if (y) t *= __bfloat162float(y[o]);
            s += m * t * exp2f(pre[j * GLD + c] - gi);
        }
    }
    return s;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x); f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
    f[4] = bf_lo(u.z); f[5] = bf_hi(u.z); f[6] = bf_lo(u.w); f[7] = bf_hi(u.w);
}

__global__ void __launch_bounds__(GK_NT, 1)
    grad_kernel(const __grid_constant__ CUtensorMap map_do, const __nv_bfloat16 *__restrict__ q,
                const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                const __nv_bfloat16 *__restrict__ b, const __nv_bfloat16 *__restrict__ w,
                const float *__restrict__ alpha, const unsigned char *records, const unsigned char *aux,
                float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dalpha,
                float *__restrict__ db, float *__restrict__ dw, int H, int T, int NC, unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ch = blockIdx.x, h = ch % H, n = (ch / H) % NC, bb = ch / (H * NC);
    const int t0 = n * C, L = min(C, T - t0);
    const unsigned char *rec = records + (size_t)ch * R_BYTES, *ax = aux + (size_t)ch * X_BYTES;
    const uint32_t misc = smem_u32(sm + G_MISC);
    volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(sm + G_MISC + MG_ABORT);
    const uint32_t base = smem_u32(sm);

    if (warp == 0) tmem_alloc(misc + MG_TSLOT, GT_COLS);
    if (tid == 0) {
        for (uint32_t m = MG_L1; m <= MG_M4; m += 8) mbar_init(misc + m, 1);
        *abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        prefetch_tmap(&map_do);
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + G_MISC + MG_TSLOT);
    if (tid == 0) {   // every operand in flight at once, in the order the products need them
        mbar_arrive_expect_tx(misc + MG_L1, 8192 + 16384);
        bulk_g2s(base + G_T, ax + X_T, 8192, misc + MG_L1);
        bulk_g2s(base + G_DD, ax + X_DD, 16384, misc + MG_L1);
        mbar_arrive_expect_tx(misc + MG_L2, 16384 + 49152 + 32768);
        tma_load_4d(base + G_RO + 8192, &map_do, 0, h, t0, bb, misc + MG_L2);
        tma_load_4d(base + G_RO + 16384 + 8192, &map_do, 64, h, t0, bb, misc + MG_L2);
        bulk_g2s(base + G_Z, ax + X_Z, 49152, misc + MG_L2);   // Z̃ and Delta (adjacent in both)
        bulk_g2s(base + G_G, ax + X_G, 32768, misc + MG_L2);
        mbar_arrive_expect_tx(misc + MG_L3, 16384 + 16384 + 8192 + 8192);
        bulk_g2s(base + G_KT, rec + R_KT, 16384, misc + MG_L3);
        bulk_g2s(base + G_E, ax + X_E, 16384, misc + MG_L3);
        bulk_g2s(base + G_Q, rec + R_A3 + 8192, 8192, misc + MG_L3);    // Q̂: rows 64-127 of both halves
        bulk_g2s(base + G_Q + 8192, rec + R_A3 + 24576, 8192, misc + MG_L3);
    }
    float *vecs = reinterpret_cast<float *>(sm + G_VEC);
    bool wide_l = false;
    if (tid < 128) {
        const float ae = reinterpret_cast<const float *>(ax + X_AE)[tid], ak = reinterpret_cast<const float *>(ax + X_AK)[tid];
        vecs[tid] = ae;
        vecs[128 + tid] = ak;
        vecs[256 + tid] = reinterpret_cast<const float *>(ax + X_RHO)[tid];
        wide_l = ae != ak;   // a wide-span chunk: unscaled factors (ae = 0, ak = g_C); otherwise both are m
    }
    const bool wide = group_or(GBAR, 256, wide_l);
    const int q4 = warp & 3, half = warp >> 2, cb = 64 * half;
    const uint32_t lq = (uint32_t)(32 * q4) << 16;
    const int r = 32 * (q4 & 1) + lane;             // chunk row of this thread's TMEM lane (mod 64)
    const size_t row = ((size_t)bb * T + t0 + r) * H + h;   // its token row (valid when r < L)
    // loads read row min(r, L - 1), always inside the tensor: a load under a condition on the row
    // cannot be issued ahead of the branch, and each would then wait out its own memory latency
    const size_t lrow = ((size_t)bb * T + t0 + min(r, L - 1)) * H + h;
    bool ok = true;
    uint32_t committed = 0;   // tid 0: the last MMA barrier committed (for the exit)

    // ---------------------------------------------------------------- D1: dR = T^T dDelta
    if (tid == 0) {
        ok = thread_wait(misc + MG_L1, 0, abort);
        if (ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + GT_D1, desc_mnmajor(base + G_T, 64, j), desc_kmajor(base + G_DD, 128, j), ID_D1, j > 0);
            mma_commit(misc + MG_M1);
            committed = MG_M1;
            ok = thread_wait(misc + MG_L2, 0, abort);
        }
        if (ok) {   // D4, first part: Delta G̃^T (needs no gradient of this chunk)
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ss(tmem + GT_D4, desc_kmajor(base + G_DL, 64, j), desc_kmajor(base + G_G, 128, j), ID_D4A, j > 0);
        }
    }
    // ---------------------------------------------------------------- R1: -dR -> [-dR; dO]; dv, dw
    if (q4 < 2) {
        uint4 vv[8], ww[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            vv[u] = *reinterpret_cast<const uint4 *>(v + lrow * VD + cb + 8 * u);
            ww[u] = *reinterpret_cast<const uint4 *>(w + lrow * VD + cb + 8 * u);
        }
        ok = mbar_wait(misc + MG_M1, 0, WAIT_LIMIT) && !*abort;
        if (!ok) *abort = 1u;
        __syncwarp();
        fence_after();
        uint32_t x0[32], x1[32];
        tmem_ld32(tmem + lq + GT_D1 + cb, x0);
        tmem_ld32(tmem + lq + GT_D1 + cb + 32, x1);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t *x = (u < 4 ? x0 : x1) + 8 * (u & 3);
            float d8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) d8[i] = __uint_as_float(x[i]);
            *reinterpret_cast<uint4 *>(sm + G_RO + sw_off(r, cb + 8 * u, 128)) =
                make_uint4(pack_bf16(-d8[0], -d8[1]), pack_bf16(-d8[2], -d8[3]), pack_bf16(-d8[4], -d8[5]),
                           pack_bf16(-d8[6], -d8[7]));
            if (r < L) {
                float vf[8], wf[8];
                unpack8(vv[u], vf);
                unpack8(ww[u], wf);
                float *pv = dv + row * VD + cb + 8 * u, *pw = dw + row * VD + cb + 8 * u;
                *reinterpret_cast<float4 *>(pv) = make_float4(wf[0] * d8[0], wf[1] * d8[1], wf[2] * d8[2], wf[3] * d8[3]);
                *reinterpret_cast<float4 *>(pv + 4) = make_float4(wf[4] * d8[4], wf[5] * d8[5], wf[6] * d8[6], wf[7] * d8[7]);
                *reinterpret_cast<float4 *>(pw) = make_float4(vf[0] * d8[0], vf[1] * d8[1], vf[2] * d8[2], vf[3] * d8[3]);
                *reinterpret_cast<float4 *>(pw + 4) = make_float4(vf[4] * d8[4], vf[5] * d8[5], vf[6] * d8[6], vf[7] * d8[7]);
            }
        }
    }
    fence_async_smem();
    fence_before();
    if (group_or(GBAR, 256, *abort != 0u)) ok = false;
    // ---------------------------------------------------------------- D2: [dA; dP] = [-dR; dO] Delta^T; D3, first part
    if (tid == 0 && ok) {
        fence_after();
#pragma unroll
        for (int j = 0; j < 8; ++j)
            mma_ss(tmem + GT_D2, desc_kmajor(base + G_RO, 128, j), desc_kmajor(base + G_DL, 64, j), ID_D2, j > 0);
        mma_commit(misc + MG_M2);
        committed = MG_M2;
#pragma unroll
        for (int j = 0; j < 8; ++j)   // [-dR; dO] Z̃^T
            mma_ss(tmem + GT_D3, desc_kmajor(base + G_RO, 128, j), desc_kmajor(base + G_Z, 128, j), ID_D3A, j > 0);
    }
    // ---------------------------------------------------------------- R2: masks, bf16 -> [dA; dP]
    if (ok) ok = group_wait(misc + MG_M2, 0, GBAR, 256, abort);
    if (ok) {
        const int rr = 32 * q4 + lane;   // lanes 0-63: dA row rr (strictly lower), 64-127: dP row rr - 64 (lower)
        const int lim = rr < 64 ? rr : rr - 64 + 1;   // columns i < lim are kept
        __syncwarp();
        uint32_t y[32];
        tmem_ld32(tmem + lq + GT_D2 + 32 * half, y);
        wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = 32 * half + 8 * u + i < lim ? __uint_as_float(y[8 * u + i]) : 0.f;
            *reinterpret_cast<uint4 *>(sm + G_A2 + sw_off(rr, 32 * half + 8 * u, 128)) =
                make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
        }
        fence_async_smem();
        fence_before();
        group_sync(GBAR, 256);
        // -------------------------------------------------------------- D3: += [dA; dP] K̃;  D4: += dA^T Ê + dP^T Q̂
        if (tid == 0) {
            fence_after();
            if (thread_wait(misc + MG_L3, 0, abort)) {
                if (!wide) {   // (a wide-span chunk takes these terms on CUDA cores)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ss(tmem + GT_D3, desc_kmajor(base + G_A2, 128, j), desc_mnmajor(base + G_KT, 64, j), ID_D3B, 1);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ss(tmem + GT_D4, desc_mnmajor(base + G_A2, 128, j), desc_mnmajor(base + G_E, 64, j), ID_D4B, 1);
#pragma unroll
                for (int j = 4; j < 8; ++j)
                    mma_ss(tmem + GT_D4, desc_mnmajor(base + G_A2, 128, j), desc_mnmajor(base + G_Q, 64, j - 4), ID_D4B, 1);
                }
                mma_commit(misc + MG_M4);
                committed = MG_M4;
            }
        }
    }
    // ---------------------------------------------------------------- the log2-decay prefix, while the products run
    // Thread tid: channel cc, rows 32 hh .. 32 hh + 31.  Every alpha of the thread is loaded before the
    // first is used; the upper half adds the lower half's total (handed over in shared memory).
    const int cc = tid & 127, hh = tid >> 7;
    auto alpha_at = [&](int rr) { return alpha[(((size_t)bb * T + t0 + min(rr, L - 1)) * H + h) * KD + cc]; };
    float gpre[32];
    if (ok) {
        float al[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) al[i] = alpha_at(32 * hh + i);
        float g = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            g += fast_log2(32 * hh + i < L ? fmaxf(al[i], FLT_MIN) : 1.f);
            gpre[i] = g;
        }
        if (hh == 0) vecs[384 + cc] = g;
    }
    if (ok) ok = group_wait(misc + MG_M4, 0, GBAR, 256, abort);
    if (ok) {
        float *pre = reinterpret_cast<float *>(sm + G_PRE);
        const float base = hh ? vecs[384 + cc] : 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) pre[(32 * hh + i) * GLD + cc] = base + gpre[i];
        group_sync(GBAR, 256);
        // -------------------------------------------------------------- row phase
        const float *ae = vecs, *ak = vecs + 128;
        float *H1 = reinterpret_cast<float *>(sm + G_H1), *HQ = reinterpret_cast<float *>(sm + G_HQ);
        const bool rows_ek = q4 < 2;   // lanes 0-63: dÊ and dK̃ of row r; lanes 64-127: dQ̂ of row r
        __syncwarp();
#pragma unroll 1
        for (int s = 0; s < 2; ++s) {
            const int c0 = cb + 32 * s;
            uint32_t x[32], y[32];
            tmem_ld32(tmem + lq + GT_D3 + c0, x);
            if (rows_ek) tmem_ld32(tmem + lq + GT_D4 + c0, y);
            uint4 t1[4], t2[4];
            {
                const __nv_bfloat16 *x1 = rows_ek ? b : q;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    t1[u] = *reinterpret_cast<const uint4 *>(x1 + lrow * KD + c0 + 8 * u);
                    if (rows_ek) t2[u] = *reinterpret_cast<const uint4 *>(k + lrow * KD + c0 + 8 * u);
                }
            }
            wait_ld();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + 8 * u;
                float g8[8], fe[8];
                *reinterpret_cast<float4 *>(g8) = *reinterpret_cast<const float4 *>(pre + r * GLD + c);
                *reinterpret_cast<float4 *>(g8 + 4) = *reinterpret_cast<const float4 *>(pre + r * GLD + c + 4);
#pragma unroll
                for (int i = 0; i < 8; ++i) fe[i] = fast_exp2(g8[i] - ae[c + i]);
                float hv[8];
                if (rows_ek) {
                    float bf[8], kf[8], de[8], dko[8], dbv[8], dkv[8];
                    if (r < L) {
                        unpack8(t1[u], bf);
                        unpack8(t2[u], kf);
                    }
                    float xa[8], xb[8];   // the A and P terms of a wide-span chunk
#pragma unroll
                    for (int i = 0; i < 8; ++i) { xa[i] = 0.f; xb[i] = 0.f; }
                    if (wide && r < L) {
                        const size_t row0 = ((size_t)bb * T + t0) * H + h;
                        for (int i = 0; i < 8; ++i) {
                            xa[i] = wide_row_sum(sm + G_A2, r, r, r, k, row0, H, pre, c + i);
                            xb[i] = wide_col_sum(sm + G_A2, 0, r, r + 1, L, b, k, row0, H, pre, c + i) +
                                    wide_col_sum(sm + G_A2, 64, r, r, L, q, nullptr, row0, H, pre, c + i);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (r >= L) { bf[i] = 0.f; kf[i] = 0.f; }
                        de[i] = fe[i] * __uint_as_float(x[8 * u + i]) + xa[i];
                        dko[i] = fast_exp2(ak[c + i] - g8[i]) * __uint_as_float(y[8 * u + i]) + xb[i];
                        dbv[i] = kf[i] * de[i];
                        dkv[i] = dko[i] + bf[i] * de[i];
                        hv[i] = bf[i] * kf[i] * de[i] - kf[i] * dko[i];
                    }
                    if (r < L) {
                        float *pb = db + row * KD + c, *pk = dk + row * KD + c;
                        *reinterpret_cast<float4 *>(pb) = make_float4(dbv[0], dbv[1], dbv[2], dbv[3]);
                        *reinterpret_cast<float4 *>(pb + 4) = make_float4(dbv[4], dbv[5], dbv[6], dbv[7]);
                        *reinterpret_cast<float4 *>(pk) = make_float4(dkv[0], dkv[1], dkv[2], dkv[3]);
                        *reinterpret_cast<float4 *>(pk + 4) = make_float4(dkv[4], dkv[5], dkv[6], dkv[7]);
                    }
                    *reinterpret_cast<float4 *>(H1 + r * GLD + c) = make_float4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<float4 *>(H1 + r * GLD + c + 4) = make_float4(hv[4], hv[5], hv[6], hv[7]);
                } else {
                    float qf[8], dqv[8], xa[8];
                    if (r < L) unpack8(t1[u], qf);
#pragma unroll
                    for (int i = 0; i < 8; ++i) xa[i] = 0.f;
                    if (wide && r < L) {
                        const size_t row0 = ((size_t)bb * T + t0) * H + h;
                        for (int i = 0; i < 8; ++i) xa[i] = wide_row_sum(sm + G_A2, 64 + r, r, r + 1, k, row0, H, pre, c + i);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (r >= L) qf[i] = 0.f;
                        dqv[i] = fe[i] * __uint_as_float(x[8 * u + i]) + xa[i];
                        hv[i] = qf[i] * dqv[i];
                    }
                    if (r < L) {
                        float *pq = dq + row * KD + c;
                        *reinterpret_cast<float4 *>(pq) = make_float4(dqv[0], dqv[1], dqv[2], dqv[3]);
                        *reinterpret_cast<float4 *>(pq + 4) = make_float4(dqv[4], dqv[5], dqv[6], dqv[7]);
                    }
                    *reinterpret_cast<float4 *>(HQ + r * GLD + c) = make_float4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<float4 *>(HQ + r * GLD + c + 4) = make_float4(hv[4], hv[5], hv[6], hv[7]);
                }
            }
        }
        group_sync(GBAR, 256);
        // -------------------------------------------------------------- decay: reverse sums over the chunk
        {   // thread tid: channel cc, rows 32 hh .. 32 hh + 31; the lower half starts from the upper
            // half's total (handed over in shared memory)
            const float rho = vecs[256 + cc];
            float al[32], hs[32], tot = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) al[i] = alpha_at(32 * hh + i);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int rr = 32 * hh + i;
                hs[i] = H1[rr * GLD + cc] + HQ[rr * GLD + cc];
                tot += hs[i];
            }
            if (hh == 1) vecs[512 + cc] = tot;
            group_sync(GBAR, 256);
            float acc = hh ? 0.f : vecs[512 + cc];
#pragma unroll
            for (int i = 31; i >= 0; --i) {
                const int rr = 32 * hh + i;
                acc += hs[i];
                if (rr < L) dalpha[(((size_t)bb * T + t0 + rr) * H + h) * KD + cc] = (acc + rho) / fmaxf(al[i], FLT_MIN);
            }
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0) {   // nothing in flight when the block exits (after an abort)
        mbar_wait(misc + MG_L1, 0, WAIT_LIMIT);
        mbar_wait(misc + MG_L2, 0, WAIT_LIMIT);
        mbar_wait(misc + MG_L3, 0, WAIT_LIMIT);
        if (committed) mbar_wait(misc + committed, 0, WAIT_LIMIT);
        if (*abort) atomicOr(status, STATUS_GRAD);
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0) tmem_dealloc(tmem, GT_COLS);
}

}  // namespace bwdtc

size_t chunk_bwd_tc_workspace_bytes(int B, int H, int T) {
    if (T == 0) return kStatusBytes;
    const size_t chains = (size_t)B * H, nch = chains * (size_t)((T + split::C - 1) / split::C);
    return kStatusBytes + nch * (split::R_BYTES + split::X_BYTES) + chains * sizeof(float) * 128 * 128 +
           replay_segment_bytes(B, H, T);
}

int launch_chunk_bwd_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                        const float *S0, const void *dO, const float *dST, float *dq, float *dk, float *dv,
                        float *dalpha, float *db, float *dw, float *dS0, int B, int H, int T, void *ws,
                        cudaStream_t st) {
    CUtensorMap map_do;
    if (!token_map(&map_do, dO, B, T, H)) return -6;
    const int chains = B * H, NC = (T + split::C - 1) / split::C, nch = chains * NC;
    unsigned int *status = reinterpret_cast<unsigned int *>(ws);
    unsigned char *records = static_cast<unsigned char *>(ws) + kStatusBytes;
    unsigned char *aux = records + (size_t)nch * split::R_BYTES;
    float *STf = reinterpret_cast<float *>(aux + (size_t)nch * split::X_BYTES);
    float *seg = STf + (size_t)chains * 128 * 128;
    int rc = launch_split_replay(q, k, v, alpha, b, w, S0, STf, B, H, T, records, aux, seg, map_do, status, st);
    if (rc != 0) return rc;
    const int smem_r = (int)bwdtc::RW_BYTES, smem_g = (int)bwdtc::G_BYTES;
    if (cudaFuncSetAttribute(bwdtc::rwalk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_r) != cudaSuccess ||
        cudaFuncSetAttribute(bwdtc::grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_g) != cudaSuccess)
        return -6;
    bwdtc::rwalk_kernel<<<chains, bwdtc::RW_NT, smem_r, st>>>(map_do, records, aux, dST, STf, dS0, H, NC, status);
    using bf = __nv_bfloat16;
    bwdtc::grad_kernel<<<nch, bwdtc::GK_NT, smem_g, st>>>(map_do, (const bf *)q, (const bf *)k, (const bf *)v,
                                                          (const bf *)b, (const bf *)w, alpha, records, aux, dq, dk,
                                                          dv, dalpha, db, dw, H, T, NC, status);
    return launch_status();
}

}  // namespace gdn2
