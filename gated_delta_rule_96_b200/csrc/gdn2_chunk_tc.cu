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
// wider span forms A and P on CUDA cores from exp(g_r - g_i) <= 1 per element (written
// straight into the TMEM accumulator G1 would have produced) and uses unscaled factors
// elsewhere (m = 0), so any alpha in (0, 1] is handled.
//
// Only the state update (G3 -> Delta -> G4/G5 -> rescale) is serial from chunk to chunk;
// everything before it depends on the tokens alone.  The block therefore runs three
// CUDA-core stages as a pipeline over chunks, each in its own warpgroup:
//   warps 0-3   state group: rescales Z and writes its bf16 copy, Delta epilogue of chunk n
//   warps 4-7   build group: loads, log-decay prefix and the bf16 operands of chunk n+1
//               (double-buffered [Ê; Q̂] and K̃)
//   warps 8-11  solve group: A/P readout, triangular solve, [T; P] tile and the -W'
//               epilogue of chunk n
//   warps 12-13 u group: U = w ⊙ v of the next chunk
//   warps 14-15 o group: o epilogue of chunk n
// Each GEMM is issued by thread 0 of the group that wrote its last operand (G1 build, G2
// solve, G3 and G4/G5 state), so no thread polls for work.
// Registers are rebalanced per warpgroup with setmaxnreg (the build group holds a whole
// chunk's loads in flight).
// Every event that a waiter may see two chunks late has one mbarrier per buffer slot.
// Every wait is bounded; on expiry the block sets the workspace status word and exits.
//
// The layer-edge instance (chunk_tc_kernel<true>) takes the layer's raw inputs: the o warps
// also map the decay logits of chunk n + 4 into a four-slot ring in the workspace
// (alpha = exp(-softplus(a))), the build group folds the inverse norms of q and k into its
// decay factors and applies the sigmoid to b, the u group to w, and the o group applies
// RMSNorm to o when given a weight.
#include <algorithm>

#include "gdn2_common.cuh"
#include "gdn2_internal.h"
#include "tc_chunk.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace tcfwd {

using namespace gdn2::tc;
using namespace gdn2::tcc;

constexpr int C = 64, KD = 128, VD = 128;
constexpr int NT = 512;                       // 16 warps
constexpr int GROUP = 128;                    // threads of the state, build and solve groups
constexpr uint32_t BAR_STATE = 1, BAR_BUILD = 2, BAR_SOLVE = 3;   // named barrier ids
constexpr float SPAN_MAX_LOG2 = 173.123f;     // 120 nats in log2 units
constexpr uint32_t WAIT_LIMIT = 1u << 22;

// TMEM columns (512 allocated)
constexpr uint32_t TM_D1 = 0;                 // [A; P] fp32 (64)
constexpr uint32_t TM_D2 = 64;                // [W'; *] (128)
constexpr uint32_t TM_D3 = 192;               // [U~ -> Delta; O] (128)
constexpr uint32_t TM_Z = 320;                // Z fp32 (128)
constexpr uint32_t TM_COLS = 512;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t SM_S = 0;                      // Z in bf16 [c x v], B of G3 (MN-major)
constexpr uint32_t SM_EQ = 32768;                 // 2 slots of [Ê -> -W'; Q̂] 128 x 128 (K-major A of G1 / G3)
constexpr uint32_t EQ_BYTES = 32768;
constexpr uint32_t SM_KT = 98304;                 // 2 slots of K̃ [i x c] 64 x 128
constexpr uint32_t KT_BYTES = 16384;
constexpr uint32_t SM_U = 131072;                 // 2 slots of U [i x v] 64 x 128
constexpr uint32_t U_BYTES = 16384;
constexpr uint32_t SM_DL = 163840;                // Delta [i x v] 64 x 128
constexpr uint32_t SM_T = 180224;                 // T [r x i] 64 x 64, followed by
constexpr uint32_t SM_P = 188416;                 // P [r x i]: [T; P] is one K-major 128-row operand
constexpr uint32_t SM_AS = 196608;                // fp32 [64][LDA]: A below the diagonal, T^T on and above it
constexpr uint32_t SM_VEC = SM_AS + 64 * LDA * 4; // [2 slots][sS, sZ, sPost] (6 x 128 fp32)
constexpr uint32_t SM_WT = SM_VEC + 3072;         // build group: [4][128] warp totals + g_0 [128]
constexpr uint32_t SM_X = SM_WT + 2560;           // solve group: per-warp mma scratch (4 KB)
constexpr uint32_t SM_MISC = SM_X + 4096;         // mbarriers, TMEM slot, flags
constexpr uint32_t SM_OST = SM_MISC + 256;         // o group: 2 warps x 32 rows x 80 B staging
constexpr uint32_t SM_BYTES = SM_OST + 5120 + 1024;

// mbarriers (byte offsets inside SM_MISC); the first five are pairs indexed by chunk & 1
enum : uint32_t {
    MB_VEC = 0, MB_G3 = 16, MB_G45 = 32, MB_U = 48, MB_G2 = 64,
    MB_G1 = 80, MB_READOUT = 88, MB_S1DONE = 96, MB_D3FREE = 104, MB_END = 112
};
constexpr uint32_t MISC_TSLOT = 160, MISC_ABORT = 164;
// layer-edge ring: RING_SLOTS full / free barrier pairs, slot m % RING_SLOTS for chunk m
constexpr uint32_t MB_RFULL = 168, MB_RFREE = 200;

// Layer-edge ring (per block, in the workspace): the o warps write the decay rows of chunk m,
// alpha = exp(-softplus(a)) in fp32, into slot m % RING_SLOTS, RING_SLOTS chunks ahead of the
// build group, which reads them as it reads plain alpha.  q, k and b stay raw: the build group
// folds the inverse norms of q and k into its decay factors and applies the sigmoid to b where
// it uses it.
constexpr int RING_SLOTS = 4;
constexpr uint32_t RING_BYTES = C * KD * 4;   // 32 KB

// Launch flags of the segmented (parallel-in-time) prefill.  A block owns segment
// blockIdx.x % nseg of chain blockIdx.x / nseg; S0 and S_T are indexed by block.
enum : uint32_t {
    SEG_ZERO_WRITES = 1,   // U = 0: the run propagates the state only (the homogeneous part)
    SEG_SKIP_O = 2,        // o is not stored
    SEG_IDENTITY_S0 = 4,   // the segment starts from S = I (d_k = d_v)
    SEG_ST_LAST = 8,       // only the chain's last segment stores S_T, at S_T[chain]
};

constexpr uint32_t ID_G1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_G2 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G3 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G4 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G5 = idesc_bf16(128, 128, 1, 1);

// load of data that other warps of the block wrote earlier in this kernel (the layer-edge
// ring): a plain global load, not the read-only path
__device__ __forceinline__ float4 ld_f4(const float *p) {
    float4 v;
    asm volatile("ld.global.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p) : "memory");
    return v;
}

struct Ctx {
    unsigned char *sm;
    uint32_t tmem, misc;
    const __nv_bfloat16 *q, *k, *v, *b, *w;
    const float *alpha;
    __nv_bfloat16 *o;
    int T, H, bb, h, NC;
    int tb, te;        // token range of this block's segment: [tb, te)
    const float *onorm;   // RMSNorm weight of o (layer-edge variant; null: none)
    unsigned char *ring;  // this block's layer-edge ring (layer-edge variant)
    uint32_t flags;    // SEG_* below
};

__device__ __forceinline__ uint32_t mbar(const Ctx &c, uint32_t off) { return c.misc + off; }
// slot barrier of chunk n and the parity of chunk n's phase on it
__device__ __forceinline__ uint32_t mbar_slot(const Ctx &c, uint32_t off, int n) { return c.misc + off + 8u * (n & 1); }
__device__ __forceinline__ uint32_t slot_par(int n) { return (uint32_t)((n >> 1) & 1); }
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

// ============================================================================ MMA issue
// Every GEMM is issued by thread 0 of the group that produced its last operand, right after
// the group's barrier (the operand writes are fenced to the async proxy before it); the
// thread first waits, bounded, for the other inputs and for its accumulator to be free.
// A failed wait sets the abort flag and skips the GEMM; the waiting consumers then give up.
__device__ __forceinline__ bool issue_wait(const Ctx &c, uint32_t mb, uint32_t parity) {
    if (!mbar_wait(mb, parity, WAIT_LIMIT) || *abort_flag(c)) {
        *abort_flag(c) = 1u;
        return false;
    }
    fence_after();
    return true;
}
// G1(n) = [Ê; Q̂] K̃^T -> D1, once chunk n-1's A and P were read out of D1
__device__ __forceinline__ void issue_g1(const Ctx &c, int n, bool slow) {
    fence_after();
    if (n > 0 && !issue_wait(c, mbar(c, MB_READOUT), (uint32_t)((n - 1) & 1))) return;
    if (slow) {   // A and P were written into D1 directly
        mbar_arrive(mbar(c, MB_G1));
        return;
    }
    const uint32_t aEQ = smem_u32(c.sm + SM_EQ) + (n & 1) * EQ_BYTES, aKT = smem_u32(c.sm + SM_KT) + (n & 1) * KT_BYTES;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        mma_ss(c.tmem + TM_D1, desc_kmajor(aEQ, 128, j), desc_kmajor(aKT, 64, j), ID_G1, j > 0);
    mma_commit(mbar(c, MB_G1));
}
// G2(n): [W'; *] = [T; P] Ê -> D2 and [U~; *] = [T; P] U -> D3, once U (slot n & 1) is written
// and the o rows of chunk n-1 have left D3
__device__ __forceinline__ void issue_g2(const Ctx &c, int n) {
    fence_after();
    if (!issue_wait(c, mbar_slot(c, MB_U, n), slot_par(n))) return;
    if (n > 0 && !issue_wait(c, mbar(c, MB_D3FREE), (uint32_t)((n - 1) & 1))) return;
    const uint32_t aEQ = smem_u32(c.sm + SM_EQ) + (n & 1) * EQ_BYTES, aU = smem_u32(c.sm + SM_U) + (n & 1) * U_BYTES,
                   aTP = smem_u32(c.sm + SM_T);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        mma_ss(c.tmem + TM_D2, desc_kmajor(aTP, 128, j), desc_mnmajor(aEQ, 128, j), ID_G2, j > 0);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        mma_ss(c.tmem + TM_D3, desc_kmajor(aTP, 128, j), desc_mnmajor(aU, 64, j), ID_G2, j > 0);
    mma_commit(mbar_slot(c, MB_G2, n));
}
// G3(n): [Delta; O] += [-W'; Q̂] S~, once -W' is written
__device__ __forceinline__ void issue_g3(const Ctx &c, int n) {
    fence_after();
    if (!issue_wait(c, mbar(c, MB_S1DONE), (uint32_t)(n & 1))) return;
    const uint32_t aEQ = smem_u32(c.sm + SM_EQ) + (n & 1) * EQ_BYTES, aS = smem_u32(c.sm + SM_S);
#pragma unroll
    for (int j = 0; j < 8; ++j)
        mma_ss(c.tmem + TM_D3, desc_kmajor(aEQ, 128, j), desc_mnmajor(aS, 128, j), ID_G3, 1);
    mma_commit(mbar_slot(c, MB_G3, n));
}
// G4/G5(n): O += P Delta, Z += K̃^T Delta
__device__ __forceinline__ void issue_g45(const Ctx &c, int n) {
    fence_after();
    const uint32_t aKT = smem_u32(c.sm + SM_KT) + (n & 1) * KT_BYTES, aDL = smem_u32(c.sm + SM_DL),
                   aTP = smem_u32(c.sm + SM_T);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        mma_ss(c.tmem + TM_D3, desc_kmajor(aTP, 128, j), desc_mnmajor(aDL, 64, j), ID_G4, 1);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        mma_ss(c.tmem + TM_Z, desc_mnmajor(aKT, 64, j), desc_mnmajor(aDL, 64, j), ID_G5, 1);
    mma_commit(mbar_slot(c, MB_G45, n));
}

// ============================================================================ build group
// Rows of one chunk's q, k, b (bf16) and alpha (fp32): row t of the chunk is at element
// (base + t * stride) * KD.  Plain inputs: the token tensors; layer-edge variant: the ring slot.
struct Src {
    const __nv_bfloat16 *q, *k, *b;
    const float *a;
    size_t base, stride;       // rows of q and k
    size_t base_ba, stride_ba; // rows of b and alpha
    __device__ __forceinline__ size_t row(int t) const { return base + (size_t)t * stride; }
    __device__ __forceinline__ size_t row_ba(int t) const { return base_ba + (size_t)t * stride_ba; }
};

// Wide-span chunk: A_ri = sum_c e_rc k_ic exp2(g_rc - g_ic) for i < r and P_ri likewise with
// q for i <= r, one row per thread (rows of A on threads 0-63, of P on 64-127: the TMEM lane
// of D1 that G1 would have written).  For each channel the exponent g_rc - g_ic is summed from
// log2 alpha while i walks down from r, so it never leaves [-inf, 0]; rows are re-read from
// global memory (resident in L2).
template <bool EDGES>
__device__ __forceinline__ void wide_span_ap(const Ctx &c, const Src &src, int tid1, int L) {
    const int r = tid1 & 63;
    const bool isP = tid1 >= 64;
    const uint32_t lane_base = c.tmem + ((uint32_t)((tid1 >> 5) * 32) << 16) + TM_D1;
    const int rc = min(r, L - 1);
    const size_t rowr = src.row(rc), rowr_ba = src.row_ba(rc);
    auto log2a = [&](int t, int cc) { return fast_log2(fmaxf(src.a[src.row_ba(t) * KD + cc], 1.17549435e-38f)); };
    auto inv_norm = [&](const __nv_bfloat16 *x, size_t row) {   // layer edges: 1 / max(|x_row|, eps)
        float ss = 0.f;
        for (int cc = 0; cc < KD; ++cc) {
            const float v = __bfloat162float(x[row * KD + cc]);
            ss += v * v;
        }
        return rsqrtf(fmaxf(ss, EDGE_NORM_EPS * EDGE_NORM_EPS));
    };
    const float sr = EDGES ? inv_norm(isP ? src.q : src.k, rowr) : 1.f;
#pragma unroll 1
    for (int i0 = 0; i0 < 64; i0 += 16) {
        float acc[16], sk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            acc[i] = 0.f;
            sk[i] = EDGES ? inv_norm(src.k, src.row(min(i0 + i, L - 1))) : 1.f;
        }
        if (r < L && i0 <= r) {
#pragma unroll 1
            for (int cc = 0; cc < KD; ++cc) {
                const float bg = EDGES ? sigmoid_f(__bfloat162float(src.b[rowr * KD + cc]))
                                       : __bfloat162float(src.b[rowr * KD + cc]);
                const float x = sr * (isP ? __bfloat162float(src.q[rowr * KD + cc]) : bg * __bfloat162float(src.k[rowr * KD + cc]));
                // exponent at i = i0 + 15 (or r): log2 of alpha over positions i+1 .. r
                const int itop = min(i0 + 15, r);
                float d = 0.f;
#pragma unroll 1
                for (int jj = r; jj > itop; --jj) d += log2a(jj, cc);
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    if (i0 + i <= itop) {
                        acc[i] += x * sk[i] * __bfloat162float(src.k[src.row(i0 + i) * KD + cc]) * exp2f(d);
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

// Builds the bf16 operands of every chunk into slot n & 1 as soon as the slot is free
// (G3 and G4/G5 of chunk n-2 complete).  Warp w1 owns positions 16 w1 .. 16 w1 + 15, lane l
// the channels 4l .. 4l+3; the positions are processed as two halves of 8.
template <bool EDGES>
__device__ __forceinline__ void build_group(const Ctx &c, int tid1) {
    unsigned char *sm = c.sm;
    float *vec = reinterpret_cast<float *>(sm + SM_VEC);
    float *WT = reinterpret_cast<float *>(sm + SM_WT);
    float *v_g0 = WT + 512;
    const int w1 = tid1 >> 5, lane = tid1 & 31;
    const int c4 = lane * 4, p0 = w1 * 16;
    const int T = c.T, H = c.H, bb = c.bb, h = c.h;

    for (int n = 0; n < c.NC; ++n) {
        const int t0 = c.tb + n * C, L = min(C, c.te - t0);
        unsigned char *EQ = sm + SM_EQ + (n & 1) * EQ_BYTES;
        unsigned char *KT = sm + SM_KT + (n & 1) * KT_BYTES;
        // ---------------------------------------------------------------- loads and log-decay prefix
        // Layer-edge variant: b and alpha come mapped from the ring slot the o warps filled; q and k
        // are raw, their inverse norms folded into the decay factors below.
        const size_t row0 = ((size_t)bb * T + t0) * H + h;
        Src src{c.q, c.k, c.b, c.alpha, row0, (size_t)H, row0, (size_t)H};
        if (EDGES) {
            src.a = reinterpret_cast<const float *>(c.ring + (n % RING_SLOTS) * RING_BYTES);
            src.base_ba = 0;
            src.stride_ba = 1;
        }
        float al[16][4];   // alpha (1 past the end of the sequence)
        uint2 rq[16], rk[16], rb[16];
        if (!EDGES) {
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const size_t row = src.row(min(p0 + p, L - 1));
                const float4 a4 = __ldg(reinterpret_cast<const float4 *>(src.a + row * KD + c4));
                al[p][0] = a4.x; al[p][1] = a4.y; al[p][2] = a4.z; al[p][3] = a4.w;
                rq[p] = __ldg(reinterpret_cast<const uint2 *>(src.q + row * KD + c4));
                rk[p] = __ldg(reinterpret_cast<const uint2 *>(src.k + row * KD + c4));
                rb[p] = __ldg(reinterpret_cast<const uint2 *>(src.b + row * KD + c4));
            }
        } else {   // raw q, k, b first; the decay rows once the producer has filled the ring slot
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const size_t row = src.row(min(p0 + p, L - 1));
                rq[p] = __ldg(reinterpret_cast<const uint2 *>(src.q + row * KD + c4));
                rk[p] = __ldg(reinterpret_cast<const uint2 *>(src.k + row * KD + c4));
                rb[p] = __ldg(reinterpret_cast<const uint2 *>(src.b + row * KD + c4));
            }
            if (!group_wait(c, mbar(c, MB_RFULL + 8 * (n % RING_SLOTS)), (uint32_t)((n / RING_SLOTS) & 1), BAR_BUILD,
                            GROUP))
                return;
#pragma unroll
            for (int p = 0; p < 16; ++p) {   // the ring is written in this kernel: coherent loads
                const float4 a4 = ld_f4(src.a + src.row_ba(min(p0 + p, L - 1)) * KD + c4);
                al[p][0] = a4.x; al[p][1] = a4.y; al[p][2] = a4.z; al[p][3] = a4.w;
            }
        }
        // layer edges: q and k are divided by their norms over the 128 channels (4 per lane: a warp
        // holds a row) where they are used; lane l keeps the inverse norms of the warp's position l / 2
        float iq_l = 1.f, ik_l = 1.f;
        if (EDGES) {
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const float2 qa = unpack2(rq[p].x), qb = unpack2(rq[p].y), ka = unpack2(rk[p].x), kb = unpack2(rk[p].y);
                float sq = qa.x * qa.x + qa.y * qa.y + qb.x * qb.x + qb.y * qb.y;
                float sk = ka.x * ka.x + ka.y * ka.y + kb.x * kb.x + kb.y * kb.y;
#pragma unroll
                for (int msk = 16; msk > 0; msk >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, msk);
                    sk += __shfl_xor_sync(0xffffffffu, sk, msk);
                }
                if ((lane >> 1) == p) { iq_l = sq; ik_l = sk; }
            }
            iq_l = rsqrtf(fmaxf(iq_l, EDGE_NORM_EPS * EDGE_NORM_EPS));
            ik_l = rsqrtf(fmaxf(ik_l, EDGE_NORM_EPS * EDGE_NORM_EPS));
        }
        if (n + 1 < c.NC) {   // next chunk's rows of q, k, b, alpha into L2 (one 128-B line per request)
            const int r = tid1 & 63, half = tid1 >> 6;
            const int t = min(r, c.te - t0 - C - 1);
            const size_t row = ((size_t)bb * T + t0 + C + t) * H + h;
            prefetch_l2((const char *)(c.q + row * KD) + 128 * half);
            prefetch_l2((const char *)(c.k + row * KD) + 128 * half);
            prefetch_l2((const char *)(c.b + row * KD) + 128 * half);
            if (!EDGES) {   // the producer reads the raw alpha rows of the layer-edge variant
                prefetch_l2((const char *)(c.alpha + row * KD) + 256 * half);
                prefetch_l2((const char *)(c.alpha + row * KD) + 256 * half + 128);
            }
        }
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            if (p0 + p >= L) rq[p] = rk[p] = rb[p] = make_uint2(0u, 0u);
#pragma unroll
            for (int j = 0; j < 4; ++j)   // past the end: alpha = 1; subnormal alpha: smallest normal
                al[p][j] = p0 + p >= L ? 1.f : fmaxf(al[p][j], 1.17549435e-38f);
        }
        // log2 of the product of each half's 8 alphas per channel: sum of the exponent fields plus
        // log2 of the product of the mantissas (in [1, 256): cannot under- or overflow)
        float lw[2][4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int ex = 0;
                float mp = 1.f;
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const uint32_t u = __float_as_uint(al[8 * hf + p][j]);
                    ex += (int)(u >> 23) - 127;
                    mp *= __uint_as_float((u & 0x7FFFFFu) | 0x3F800000u);
                }
                lw[hf][j] = (float)ex + fast_log2(mp);
            }
        *reinterpret_cast<float4 *>(WT + w1 * 128 + c4) =
            make_float4(lw[0][0] + lw[1][0], lw[0][1] + lw[1][1], lw[0][2] + lw[1][2], lw[0][3] + lw[1][3]);
        if (w1 == 0)
            *reinterpret_cast<float4 *>(v_g0 + c4) = make_float4(fast_log2(al[0][0]), fast_log2(al[0][1]),
                                                                 fast_log2(al[0][2]), fast_log2(al[0][3]));
        group_sync(BAR_BUILD, GROUP);
        float pre[4] = {0.f, 0.f, 0.f, 0.f}, gC[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) {
            const float4 t4 = *reinterpret_cast<const float4 *>(WT + w2 * 128 + c4);
            const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                gC[j] += tv[j];
                if (w2 < w1) pre[j] += tv[j];
            }
        }
        const float4 g04 = *reinterpret_cast<const float4 *>(v_g0 + c4);
        const float g0[4] = {g04.x, g04.y, g04.z, g04.w};
        int wide = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) wide |= (g0[j] - gC[j] > SPAN_MAX_LOG2);
        const bool slow = group_or(BAR_BUILD, GROUP, wide != 0);   // WT and v_g0 reads done
        float m2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) m2[j] = slow ? 0.f : 0.5f * (g0[j] + gC[j]);

        // ---------------------------------------------------------------- wait for the slot
        // [Ê; Q̂], K̃ and the vector slot of chunk n-2 are free once its G3 and G4/G5 completed.
        if (n >= 2) {
            if (!group_wait(c, mbar_slot(c, MB_G3, n), slot_par(n - 2), BAR_BUILD, GROUP)) return;
            if (!group_wait(c, mbar_slot(c, MB_G45, n), slot_par(n - 2), BAR_BUILD, GROUP)) return;
        }
        if (w1 == 0) {   // per-channel factors of this chunk for the state group
            // sS: scale of the bf16 state operand of G3 (exp(m)); sZ: scale of the TMEM state that
            // G5 accumulates into; sPost: factor that turns the accumulated Z into the next state.
            // Tensor-core chunk: sS = sZ = exp(m), sPost = exp(g_C - m) (G5 uses K̃).
            // Wide-span chunk:   sS = 1, sZ = exp(g_C), sPost = 1 (G5 uses K^ = exp(g_C - g) ⊙ K).
            float *vs = vec + (n & 1) * 384;
            float sS[4], sZ[4], sP[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sS[j] = slow ? 1.f : fast_exp2(m2[j]);
                sZ[j] = slow ? fast_exp2(gC[j]) : sS[j];
                sP[j] = slow ? 1.f : fast_exp2(gC[j] - m2[j]);
            }
            *reinterpret_cast<float4 *>(vs + c4) = make_float4(sS[0], sS[1], sS[2], sS[3]);
            *reinterpret_cast<float4 *>(vs + 128 + c4) = make_float4(sZ[0], sZ[1], sZ[2], sZ[3]);
            *reinterpret_cast<float4 *>(vs + 256 + c4) = make_float4(sP[0], sP[1], sP[2], sP[3]);
            mbar_arrive(mbar_slot(c, MB_VEC, n));   // 32 arrivals
        }
        // ---------------------------------------------------------------- build
        if (!slow) {
            // exp(g - m) at each position from one exponential at the thread's first position and
            // running products of alpha after it; exp(m - g) backwards from one exponential at the
            // last position of each half.  Both start inside the chunk, where every factor lies
            // within exp(+-span/2): a start before the first position (exp(-m) itself) can leave
            // fp32's range when the chunk's first alpha is tiny.
            float f1[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) f1[j] = fast_exp2(pre[j] + fast_log2(al[0][j]) - m2[j]);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                // packed bf16 arithmetic: each factor is rounded to bf16 once, each product once
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int r = p0 + 8 * hf + p, pp = 8 * hf + p;
                    if (pp > 0)
#pragma unroll
                        for (int j = 0; j < 4; ++j) f1[j] *= al[pp][j];
                    if (EDGES) {   // the inverse norms join the decay factors before their one rounding
                        const float iq = __shfl_sync(0xffffffffu, iq_l, 2 * pp), ik = __shfl_sync(0xffffffffu, ik_l, 2 * pp);
                        const uint32_t b01 = bsigmoid2(rb[pp].x), b23 = bsigmoid2(rb[pp].y);
                        *reinterpret_cast<uint2 *>(EQ + sw_off(r, c4, 128)) =
                            make_uint2(bmul2(bmul2(b01, rk[pp].x), pack_bf16(f1[0] * ik, f1[1] * ik)),
                                       bmul2(bmul2(b23, rk[pp].y), pack_bf16(f1[2] * ik, f1[3] * ik)));
                        *reinterpret_cast<uint2 *>(EQ + sw_off(64 + r, c4, 128)) =
                            make_uint2(bmul2(rq[pp].x, pack_bf16(f1[0] * iq, f1[1] * iq)),
                                       bmul2(rq[pp].y, pack_bf16(f1[2] * iq, f1[3] * iq)));
                    } else {
                        const uint32_t F01 = pack_bf16(f1[0], f1[1]), F23 = pack_bf16(f1[2], f1[3]);
                        *reinterpret_cast<uint2 *>(EQ + sw_off(r, c4, 128)) =
                            make_uint2(bmul2(bmul2(rb[pp].x, rk[pp].x), F01), bmul2(bmul2(rb[pp].y, rk[pp].y), F23));
                        *reinterpret_cast<uint2 *>(EQ + sw_off(64 + r, c4, 128)) =
                            make_uint2(bmul2(rq[pp].x, F01), bmul2(rq[pp].y, F23));
                    }
                }
                float f2[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    f2[j] = fast_exp2(m2[j] - (pre[j] + lw[0][j] + (hf ? lw[1][j] : 0.f)));
#pragma unroll
                for (int p = 7; p >= 0; --p) {
                    const int r = p0 + 8 * hf + p, pp = 8 * hf + p;
                    const float ik = EDGES ? __shfl_sync(0xffffffffu, ik_l, 2 * pp) : 1.f;
                    *reinterpret_cast<uint2 *>(KT + sw_off(r, c4, 64)) =
                        make_uint2(bmul2(rk[pp].x, pack_bf16(EDGES ? f2[0] * ik : f2[0], EDGES ? f2[1] * ik : f2[1])),
                                   bmul2(rk[pp].y, pack_bf16(EDGES ? f2[2] * ik : f2[2], EDGES ? f2[3] * ik : f2[3])));
#pragma unroll
                    for (int j = 0; j < 4; ++j) f2[j] *= al[pp][j];
                }
            }
        } else {
            // D1 is free once chunk n-1's A and P were read out of it
            if (n > 0 && !group_wait(c, mbar(c, MB_READOUT), (uint32_t)((n - 1) & 1), BAR_BUILD, GROUP)) return;
            float run[4] = {pre[0], pre[1], pre[2], pre[3]};
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const int r = p0 + 8 * hf + p;
                    const float2 q01 = unpack2(rq[8 * hf + p].x), q23 = unpack2(rq[8 * hf + p].y);
                    const float2 k01 = unpack2(rk[8 * hf + p].x), k23 = unpack2(rk[8 * hf + p].y);
                    const float2 b01 = unpack2(rb[8 * hf + p].x), b23 = unpack2(rb[8 * hf + p].y);
                    float qq[4] = {q01.x, q01.y, q23.x, q23.y}, kk[4] = {k01.x, k01.y, k23.x, k23.y};
                    float bv[4] = {b01.x, b01.y, b23.x, b23.y};
                    if (EDGES) {
                        const float iq = __shfl_sync(0xffffffffu, iq_l, 2 * (8 * hf + p));
                        const float ik = __shfl_sync(0xffffffffu, ik_l, 2 * (8 * hf + p));
#pragma unroll
                        for (int j = 0; j < 4; ++j) { qq[j] *= iq; kk[j] *= ik; bv[j] = sigmoid_f(bv[j]); }
                    }
                    float E[4], Qh[4], Kt[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        run[j] += fast_log2(al[8 * hf + p][j]);
                        const float gam = exp2f(run[j]);
                        E[j] = bv[j] * kk[j] * gam;
                        Qh[j] = qq[j] * gam;
                        Kt[j] = kk[j] * exp2f(gC[j] - run[j]);
                    }
                    *reinterpret_cast<uint2 *>(EQ + sw_off(r, c4, 128)) =
                        make_uint2(pack_bf16(E[0], E[1]), pack_bf16(E[2], E[3]));
                    *reinterpret_cast<uint2 *>(EQ + sw_off(64 + r, c4, 128)) =
                        make_uint2(pack_bf16(Qh[0], Qh[1]), pack_bf16(Qh[2], Qh[3]));
                    *reinterpret_cast<uint2 *>(KT + sw_off(r, c4, 64)) =
                        make_uint2(pack_bf16(Kt[0], Kt[1]), pack_bf16(Kt[2], Kt[3]));
                }
            }
            wide_span_ap<EDGES>(c, src, tid1, L);
        }
        fence_async_smem();
        fence_before();
        group_sync(BAR_BUILD, GROUP);
        if (EDGES && tid1 == 0) mbar_arrive(mbar(c, MB_RFREE + 8 * (n % RING_SLOTS)));   // ring slot read
        if (tid1 == 0) issue_g1(c, n, slow);
    }
}

// ============================================================================ solve group
// Per chunk: A and P out of TMEM, T = (I + A)^-1, the [T; P] operand tile, then -W' over
// Ê once G2 has run.  Warp pw of the group reads TMEM lanes 32 pw .. 32 pw + 31 (rows of
// A for pw < 2, of P for pw >= 2).
__device__ __forceinline__ void solve_group(const Ctx &c, int tid2) {
    unsigned char *sm = c.sm;
    float *AS = reinterpret_cast<float *>(sm + SM_AS);
    float *XS = reinterpret_cast<float *>(sm + SM_X);
    const int pw = tid2 >> 5, lane = tid2 & 31;
    const uint32_t lrow = (uint32_t)(pw * 32) << 16;

    for (int i = tid2; i < 512; i += GROUP)   // T tile: blocks above the diagonal stay zero
        reinterpret_cast<uint4 *>(sm + SM_T)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int n = 0; n < c.NC; ++n) {
        unsigned char *EQ = sm + SM_EQ + (n & 1) * EQ_BYTES;
        // ---------------------------------------------------------------- A (fp32 smem) and P (registers)
        if (!group_wait(c, mbar(c, MB_G1), (uint32_t)(n & 1), BAR_SOLVE, GROUP)) return;
        uint32_t ra[32], rb[32];
        tmem_ld32(c.tmem + lrow + TM_D1, ra);
        tmem_ld32(c.tmem + lrow + TM_D1 + 32, rb);
        wait_ld();
        fence_before();
        group_sync(BAR_SOLVE, GROUP);
        if (tid2 == 0) mbar_arrive(mbar(c, MB_READOUT));   // D1 may be overwritten
        uint32_t pk[32];
        if (pw < 2) {   // rows 0..63: A, strictly lower
            const int r = pw * 32 + lane;
#pragma unroll
            for (int i = 0; i < 64; i += 4) {
                const uint32_t *src = i < 32 ? ra + i : rb + (i - 32);
                float4 x;
                x.x = i < r ? __uint_as_float(src[0]) : 0.f;
                x.y = i + 1 < r ? __uint_as_float(src[1]) : 0.f;
                x.z = i + 2 < r ? __uint_as_float(src[2]) : 0.f;
                x.w = i + 3 < r ? __uint_as_float(src[3]) : 0.f;
                *reinterpret_cast<float4 *>(AS + r * LDA + i) = x;
            }
        } else {        // rows 64..127: P, lower with the diagonal, kept packed until its tile is free
            const int r = (pw - 2) * 32 + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int c0 = 2 * i;
                const uint32_t *src = c0 < 32 ? ra + c0 : rb + (c0 - 32);
                pk[i] = pack_bf16(c0 <= r ? __uint_as_float(src[0]) : 0.f, c0 + 1 <= r ? __uint_as_float(src[1]) : 0.f);
            }
        }
        group_sync(BAR_SOLVE, GROUP);

        // ---------------------------------------------------------------- T = (I + A)^-1
        // The bf16 T tile is written block by block as T is formed (G2 of the previous chunk,
        // its reader, has completed); its blocks above the diagonal stay zero.
        solve_unit_lower(AS, XS, sm + SM_T, tid2, BAR_SOLVE);
        // ---------------------------------------------------------------- P tile (after G4 of chunk n-1)
        if (n > 0 && !group_wait(c, mbar_slot(c, MB_G45, n - 1), slot_par(n - 1), BAR_SOLVE, GROUP)) return;
        if (pw >= 2) {
            const int r = (pw - 2) * 32 + lane;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4 *>(sm + SM_P + sw_off(r, 8 * u, 64)) =
                    make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
        fence_async_smem();
        group_sync(BAR_SOLVE, GROUP);
        if (tid2 == 0) issue_g2(c, n);

        // ---------------------------------------------------------------- -W' over Ê; zero the O rows of D3
        if (!group_wait(c, mbar_slot(c, MB_G2, n), slot_par(n), BAR_SOLVE, GROUP)) return;
        if (pw < 2) {
            const int r = pw * 32 + lane;
#pragma unroll
            for (int u2 = 0; u2 < 4; u2 += 2) {
                uint32_t r32[2][32];
                tmem_ld32(c.tmem + lrow + TM_D2 + 32 * u2, r32[0]);
                tmem_ld32(c.tmem + lrow + TM_D2 + 32 * u2 + 32, r32[1]);
                wait_ld();
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int cc = 32 * u2 + 8 * u;
                    const uint32_t *x = r32[u >> 2] + 8 * (u & 3);
                    uint32_t q4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        q4[i] = pack_bf16(-__uint_as_float(x[2 * i]), -__uint_as_float(x[2 * i + 1]));
                    *reinterpret_cast<uint4 *>(EQ + sw_off(r, cc, 128)) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
                }
            }
        } else {
            uint32_t z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) tmem_st32(c.tmem + lrow + TM_D3 + 32 * u2, z);
            wait_st();
        }
        fence_async_smem();
        fence_before();
        group_sync(BAR_SOLVE, GROUP);
        if (tid2 == 0) mbar_arrive(mbar(c, MB_S1DONE));
    }
}

// ============================================================================ state group
__device__ __forceinline__ void state_group(const Ctx &c, int tid, float *ST) {
    unsigned char *sm = c.sm;
    const float *vec = reinterpret_cast<const float *>(sm + SM_VEC);
    const int warp = tid >> 5;
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const int crow = tid;   // TMEM lane = row c of Z (and row r of D3)
    float egm_prev = 1.f;

    for (int n = 0; n < c.NC; ++n) {
        // ---------------------------------------------------------------- S_n = sPost_n-1 Z; Z <- sZ_n S_n; bf16(sS_n S_n)
        if (!group_wait(c, mbar_slot(c, MB_VEC, n), slot_par(n), BAR_STATE, GROUP)) return;
        if (n > 0 && !group_wait(c, mbar_slot(c, MB_G45, n - 1), slot_par(n - 1), BAR_STATE, GROUP)) return;
        const float *vs = vec + (n & 1) * 384;
        // The factors are applied one after the other: first sPost of chunk n-1, which turns Z into the
        // true state S_n, then this chunk's sS / sZ.  Their product alone can lie far below fp32's
        // range (both are about 2^(-span/2) for a chunk of log-decay span 'span') even though every
        // scaled value is representable.
        const float post = egm_prev;             // sPost of chunk n-1
        const float ssc = vs[crow];              // scale of the bf16 operand
        const float zsc = vs[128 + crow];        // scale of the TMEM state
        egm_prev = vs[256 + crow];
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
            uint32_t r32[32];
            tmem_ld32(c.tmem + lrow + TM_Z + 32 * u2, r32);
            wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(post * __uint_as_float(r32[i]));   // S_n
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
        group_sync(BAR_STATE, GROUP);
        if (tid == 0) issue_g3(c, n);

        // ---------------------------------------------------------------- Delta rows -> bf16 tile
        if (!group_wait(c, mbar_slot(c, MB_G3, n), slot_par(n), BAR_STATE, GROUP)) return;
        if (warp < 2) {
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(c.tmem + lrow + TM_D3 + 32 * u2, r32);
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
        group_sync(BAR_STATE, GROUP);
        if (tid == 0) issue_g45(c, n);
    }
    // the last chunk's G4/G5 must be complete before Z is read
    if (!group_wait(c, mbar_slot(c, MB_G45, c.NC - 1), slot_par(c.NC - 1), BAR_STATE, GROUP)) return;
    // S_T = Diag(sPost) Z of the last chunk
    if (!ST) return;
    float *dst = ST + crow * VD;
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

// ============================================================================ value and o groups
// u group (warps 12-13): U = w ⊙ v of chunk n into slot n & 1, written once G2 of chunk n-2
// (the slot's last reader) has completed; signals MB_U of the slot (64 arrivals).  Lane l
// holds channels 4l..4l+3, the warp picks 32 positions; rows past the end are zero.
// o group (warps 14-15, TMEM lanes 64-127 = the O rows of D3): the o rows of chunk n once
// its G4 has completed, transposed through shared memory so that each store instruction
// writes 8 rows x 64 B; signals MB_D3FREE (64 arrivals).
__device__ __forceinline__ bool warp_wait(const Ctx &c, uint32_t mb, uint32_t parity) {
    const bool ok = mbar_wait(mb, parity, WAIT_LIMIT) && !*abort_flag(c);
    if (!__all_sync(0xffffffffu, ok)) {
        *abort_flag(c) = 1u;
        return false;
    }
    fence_after();
    return true;
}

// Layer-edge producer (o warps, 64 threads): the raw decay-logit rows of chunk m mapped into ring
// slot m % RING_SLOTS, alpha = 1 / (1 + e^a) = exp(-softplus(a)).  Loads are issued eight at a
// time before any is used.
__device__ __forceinline__ void produce_a(const Ctx &c, int m, int tid2) {
    const int t0 = c.tb + m * C, L = min(C, c.te - t0);
    float *slot = reinterpret_cast<float *>(c.ring + (m % RING_SLOTS) * RING_BYTES);
    const size_t base = ((size_t)c.bb * c.T + t0) * c.H + c.h;
#pragma unroll 1
    for (int j0 = 0; j0 < 32; j0 += 8) {   // 64 rows x 32 pieces of 4 fp32
        float4 av[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int p = tid2 + 64 * (j0 + j), r = min(p >> 5, L - 1);
            av[j] = __ldg(reinterpret_cast<const float4 *>(c.alpha + (base + (size_t)r * c.H) * KD) + (p & 31));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int p = tid2 + 64 * (j0 + j), r = p >> 5;
            if (r < L)
                reinterpret_cast<float4 *>(slot + (size_t)r * KD)[p & 31] =
                    make_float4(alpha_of_logit(av[j].x), alpha_of_logit(av[j].y), alpha_of_logit(av[j].z),
                                alpha_of_logit(av[j].w));
        }
    }
}
// raw decay-logit rows of chunk m into L2 ahead of their mapping
__device__ __forceinline__ void prefetch_edges(const Ctx &c, int m, int tid2) {
    if (m >= c.NC) return;
    const int t0 = c.tb + m * C, L = min(C, c.te - t0);
    const int r = tid2 & 63;
    if (r >= L) return;
    const size_t row = ((size_t)c.bb * c.T + t0 + r) * c.H + c.h;
    const char *a = (const char *)(c.alpha + row * KD);
    prefetch_l2(a); prefetch_l2(a + 128); prefetch_l2(a + 256); prefetch_l2(a + 384);
}
// chunk m's decay rows in its ring slot, once the build group has read the slot's previous chunk;
// each of the 64 producer threads arrives on the slot's full barrier
__device__ __forceinline__ bool fill_ring(const Ctx &c, int m, int tid2) {
    if (m >= c.NC) return true;
    if (m >= RING_SLOTS &&
        !warp_wait(c, mbar(c, MB_RFREE + 8 * (m % RING_SLOTS)), (uint32_t)(((m - RING_SLOTS) / RING_SLOTS) & 1)))
        return false;
    produce_a(c, m, tid2);
    mbar_arrive(mbar(c, MB_RFULL + 8 * (m % RING_SLOTS)));   // release: the rows above are visible
    return true;
}

template <bool EDGES>
__device__ __forceinline__ void u_group(const Ctx &c, int tid2) {
    const int vw = tid2 >> 5, lane = tid2 & 31, c4 = lane * 4;
    const int T = c.T, H = c.H, bb = c.bb, h = c.h;
    for (int n = 0; n < c.NC; ++n) {
        const int t0 = c.tb + n * C, L = min(C, c.te - t0);
        unsigned char *U = c.sm + SM_U + (n & 1) * U_BYTES;
        if (n + 1 < c.NC) {   // next chunk's rows of v and w into L2
            const int t = min(tid2, c.te - t0 - C - 1);
            const size_t row = ((size_t)bb * T + t0 + C + t) * H + h;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                prefetch_l2((const char *)(c.v + row * VD) + 128 * i);
                prefetch_l2((const char *)(c.w + row * VD) + 128 * i);
            }
        }
        if (n >= 2 && !warp_wait(c, mbar_slot(c, MB_G2, n), slot_par(n - 2))) return;
#pragma unroll 1
        for (int p0 = 32 * vw; p0 < 32 * vw + 32; p0 += 8) {
            uint2 rv[8], rw[8];
            const int Lw = (c.flags & SEG_ZERO_WRITES) ? 0 : L;   // no writes: U = 0
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int t = min(p0 + p, max(Lw, 1) - 1);
                const size_t row = ((size_t)bb * T + t0 + t) * H + h;
                rv[p] = __ldg(reinterpret_cast<const uint2 *>(c.v + row * VD + c4));
                rw[p] = __ldg(reinterpret_cast<const uint2 *>(c.w + row * VD + c4));
            }
#pragma unroll
            for (int p = 0; p < 8; ++p)
                *reinterpret_cast<uint2 *>(U + sw_off(p0 + p, c4, 64)) =
                    p0 + p < Lw ? (EDGES ? make_uint2(bmul2(bsigmoid2(rw[p].x), rv[p].x), bmul2(bsigmoid2(rw[p].y), rv[p].y))
                                         : make_uint2(bmul2(rw[p].x, rv[p].x), bmul2(rw[p].y, rv[p].y)))
                                : make_uint2(0u, 0u);
        }
        fence_async_smem();
        mbar_arrive(mbar_slot(c, MB_U, n));
    }
}

template <bool EDGES>
__device__ __forceinline__ void o_group(const Ctx &c, int tid2) {
    const int ow = tid2 >> 5, lane = tid2 & 31;   // this thread's row of O: TMEM lane 64 + tid2
    const uint32_t lrow = (uint32_t)(64 + ow * 32) << 16;
    unsigned char *stg = c.sm + SM_OST + ow * 2560;   // 32 rows x 80 B (64 B of data + 16 B pad)
    const bool store = !(c.flags & SEG_SKIP_O);
    if (EDGES) {   // alpha of the first RING_SLOTS chunks, then each chunk's after the output of the one 4 earlier
        for (int m = 0; m <= RING_SLOTS; ++m) prefetch_edges(c, m, tid2);
        for (int m = 0; m < RING_SLOTS; ++m)
            if (!fill_ring(c, m, tid2)) return;
    }
    for (int n = 0; n < c.NC; ++n) {
        const int t0 = c.tb + n * C, L = store ? min(C, c.te - t0) : 0;
        if (!warp_wait(c, mbar_slot(c, MB_G45, n), slot_par(n))) return;
        float rms_scale = 1.f;   // RMSNorm of the row (layer-edge variant): a first pass for mean(o^2)
        if (EDGES && c.onorm) {
            float ss = 0.f;
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
                uint32_t r32[32];
                tmem_ld32(c.tmem + lrow + TM_D3 + 32 * u2, r32);
                wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) ss += __uint_as_float(r32[i]) * __uint_as_float(r32[i]);
            }
            rms_scale = rsqrtf(ss * (1.f / VD) + EDGE_RMS_EPS);
        }
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
            uint32_t r32[32];
            tmem_ld32(c.tmem + lrow + TM_D3 + 32 * u2, r32);
            wait_ld();
            if (EDGES && c.onorm)
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    r32[i] = __float_as_uint(__uint_as_float(r32[i]) * rms_scale * __ldg(c.onorm + 32 * u2 + i));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uint4 pk;
                pk.x = pack_bf16(__uint_as_float(r32[8 * u]), __uint_as_float(r32[8 * u + 1]));
                pk.y = pack_bf16(__uint_as_float(r32[8 * u + 2]), __uint_as_float(r32[8 * u + 3]));
                pk.z = pack_bf16(__uint_as_float(r32[8 * u + 4]), __uint_as_float(r32[8 * u + 5]));
                pk.w = pack_bf16(__uint_as_float(r32[8 * u + 6]), __uint_as_float(r32[8 * u + 7]));
                *reinterpret_cast<uint4 *>(stg + lane * 80 + 16 * u) = pk;
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {   // 8 rows x 64 B per store instruction
                const int rr = 8 * i + (lane >> 2), pc = lane & 3, orow = ow * 32 + rr;
                const uint4 val = *reinterpret_cast<const uint4 *>(stg + rr * 80 + 16 * pc);
                if (orow < L)
                    *reinterpret_cast<uint4 *>(c.o + (((size_t)c.bb * c.T + t0 + orow) * c.H + c.h) * VD + 32 * u2 + 8 * pc) = val;
            }
            __syncwarp();
        }
        fence_before();
        mbar_arrive(mbar(c, MB_D3FREE));
        if (EDGES) {
            if (!fill_ring(c, n + RING_SLOTS, tid2)) return;
            prefetch_edges(c, n + RING_SLOTS + 1, tid2);
        }
    }
}

template <bool EDGES>
__global__ void __launch_bounds__(NT, 1)
    chunk_tc_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                    const __nv_bfloat16 *__restrict__ v, const float *__restrict__ alpha,
                    const __nv_bfloat16 *__restrict__ b, const __nv_bfloat16 *__restrict__ w,
                    const float *S0, __nv_bfloat16 *__restrict__ o, float *ST, int H,
                    int T, int seg_len, int nseg, uint32_t flags, const float *__restrict__ onorm,
                    unsigned char *ring, unsigned int *__restrict__ status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int chain = blockIdx.x / nseg, seg = blockIdx.x % nseg;
    Ctx c;
    c.sm = sm;
    c.misc = smem_u32(sm + SM_MISC);
    c.q = q; c.k = k; c.v = v; c.b = b; c.w = w; c.alpha = alpha; c.o = o;
    c.T = T; c.H = H; c.bb = chain / H; c.h = chain % H;
    c.tb = seg * seg_len; c.te = min(T, c.tb + seg_len); c.NC = (c.te - c.tb + C - 1) / C;
    c.flags = flags;
    c.onorm = onorm;
    c.ring = EDGES ? ring + (size_t)blockIdx.x * RING_SLOTS * RING_BYTES : nullptr;
    float *st_dst = (flags & SEG_ST_LAST) ? (seg == nseg - 1 ? ST + (size_t)chain * KD * VD : nullptr)
                                          : ST + (size_t)blockIdx.x * KD * VD;

    if (warp == 12) tmem_alloc(c.misc + MISC_TSLOT, TM_COLS);
    if (tid == 0) {
        for (uint32_t off = 0; off < MB_END; off += 8)
            mbar_init(c.misc + off, (off == MB_VEC || off == MB_VEC + 8) ? 32u
                                     : (off == MB_U || off == MB_U + 8 || off == MB_D3FREE) ? 64u : 1u);
        if (EDGES)
            for (int i = 0; i < RING_SLOTS; ++i) {
                mbar_init(c.misc + MB_RFULL + 8 * i, 64u);   // the 64 producer threads
                mbar_init(c.misc + MB_RFREE + 8 * i, 1u);    // the build group's thread 0
            }
        *reinterpret_cast<volatile uint32_t *>(sm + SM_MISC + MISC_ABORT) = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    c.tmem = *reinterpret_cast<volatile uint32_t *>(sm + SM_MISC + MISC_TSLOT);

    if (warp < 4) {   // Z <- S0 (the first rescale multiplies by exp(m) of chunk 0)
        regs_dec<104>();
        const int crow = tid;
        const uint32_t lrow = (uint32_t)(warp * 32) << 16;
        const float *src = S0 ? S0 + ((size_t)blockIdx.x * KD + crow) * VD : nullptr;
        const bool ident = (flags & SEG_IDENTITY_S0) != 0;
#pragma unroll
        for (int u2 = 0; u2 < 4; ++u2) {
            uint32_t r32[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 x = src ? *reinterpret_cast<const float4 *>(src + 32 * u2 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                r32[i] = __float_as_uint(x.x); r32[i + 1] = __float_as_uint(x.y);
                r32[i + 2] = __float_as_uint(x.z); r32[i + 3] = __float_as_uint(x.w);
            }
            if (ident)
#pragma unroll
                for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(32 * u2 + i == crow ? 1.f : 0.f);
            tmem_st32(c.tmem + lrow + TM_Z + 32 * u2, r32);
        }
        wait_st();
        fence_before();
        group_sync(BAR_STATE, GROUP);
        fence_after();
        state_group(c, tid, st_dst);
        regs_inc<128>();   // every warpgroup leaves its role with the launch budget
    } else if (warp < 8) {
        regs_inc<208>();
        build_group<EDGES>(c, tid - 128);
        regs_dec<128>();
    } else if (warp < 12) {
        regs_inc<128>();
        solve_group(c, tid - 256);
        regs_dec<128>();
    } else {
        regs_dec<72>();
        if (warp < 14)
            u_group<EDGES>(c, tid - 384);
        else
            o_group<EDGES>(c, tid - 448);
        regs_inc<128>();
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (tid == 0 && *reinterpret_cast<volatile uint32_t *>(sm + SM_MISC + MISC_ABORT)) atomicOr(status, 1u);
    if (warp == 12) tmem_dealloc(c.tmem, TM_COLS);
}


// ============================================================================ segment scan
// S_g = M_(g-1) S_(g-1) + N_(g-1) along the segments of each chain (g = 1 .. nseg-1), S_0 = S0.
// One block per (chain, 16-column slice of S); fp32.  Each step stages M_(g-1) (64 KB) in shared
// memory, rows padded to SCAN_LD floats so that the two rows a warp reads fall in different banks;
// the next step's M is loaded into registers while this step computes.  Thread (r0, col) keeps rows
// r0, r0 + 16, ..., r0 + 112 of its column and reads M four k at a time.
constexpr int SCAN_LD = KD + 4;
constexpr int SCAN_SMEM = (KD * SCAN_LD + KD * 16) * 4;   // M, then the previous state's column slice
__global__ void __launch_bounds__(256) segment_scan_kernel(const float *__restrict__ M, const float *__restrict__ N,
                                                           const float *S0, float *__restrict__ Sg, int nseg) {
    extern __shared__ float scan_sm[];
    float *Ms = scan_sm, *sprev = scan_sm + KD * SCAN_LD;   // Ms [KD][SCAN_LD], sprev [KD][16]
    const int chain = blockIdx.x, c0 = 16 * blockIdx.y, tid = threadIdx.x;
    const size_t KV = (size_t)KD * VD;
    const int col = tid & 15, r0 = tid >> 4;   // rows r0, r0 + 16, ..., r0 + 112
    for (int r = r0; r < KD; r += 16) {
        const float v = S0 ? S0[chain * KV + (size_t)r * VD + c0 + col] : 0.f;
        sprev[r * 16 + col] = v;
        Sg[((size_t)chain * nseg) * KV + (size_t)r * VD + c0 + col] = v;
    }
    constexpr int NV = KD * KD / 4 / 256;   // float4 of M per thread
    float4 mreg[NV];
    auto load_m = [&](int g) {
        const float4 *Mg = reinterpret_cast<const float4 *>(M + ((size_t)chain * nseg + g - 1) * KV);
#pragma unroll
        for (int u = 0; u < NV; ++u) mreg[u] = __ldg(Mg + tid + 256 * u);
    };
    if (nseg > 1) load_m(1);
    for (int g = 1; g < nseg; ++g) {
        const float *Ng = N + ((size_t)chain * nseg + g - 1) * KV;
        __syncthreads();   // the previous step's reads of Ms are done
#pragma unroll
        for (int u = 0; u < NV; ++u) {
            const int i = tid + 256 * u;   // float4 i of M: row i / 32, columns 4 (i % 32) ..
            *reinterpret_cast<float4 *>(Ms + (i >> 5) * SCAN_LD + 4 * (i & 31)) = mreg[u];
        }
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = Ng[(size_t)(r0 + 16 * i) * VD + c0 + col];
        __syncthreads();
        if (g + 1 < nseg) load_m(g + 1);
#pragma unroll 2
        for (int kk = 0; kk < KD; kk += 4) {
            const float s0 = sprev[kk * 16 + col], s1 = sprev[(kk + 1) * 16 + col], s2 = sprev[(kk + 2) * 16 + col],
                        s3 = sprev[(kk + 3) * 16 + col];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 m = *reinterpret_cast<const float4 *>(Ms + (r0 + 16 * i) * SCAN_LD + kk);
                acc[i] = fmaf(m.x, s0, acc[i]);
                acc[i] = fmaf(m.y, s1, acc[i]);
                acc[i] = fmaf(m.z, s2, acc[i]);
                acc[i] = fmaf(m.w, s3, acc[i]);
            }
        }
        __syncthreads();   // every thread has read sprev
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sprev[(r0 + 16 * i) * 16 + col] = acc[i];
            Sg[((size_t)chain * nseg + g) * KV + (size_t)(r0 + 16 * i) * VD + c0 + col] = acc[i];
        }
    }
}

}  // namespace tcfwd

bool tc_supported(int B, int H, int T, int K, int V, int C, int bf16) {
    (void)B; (void)H; (void)T;
    return bf16 && K == 128 && V == 128 && C == 64;
}

namespace {

// Parallel-in-time plan for few, long chains: the sequence of each chain is cut into nseg
// segments of whole chunks so that about 128 blocks run at once.  Every segment's state map
// S_out = M S_in + N is found in parallel (N from S_in = 0, M from S_in = I with the writes
// switched off), the maps are composed along the chain, and the segments run again from their
// true start states.  Three passes over 1/nseg of the sequence instead of one over all of it.
struct SegPlan {
    int nseg, seg_len;
};
SegPlan seg_plan(int B, int H, int T) {
    const int chains = B * H, NC = (T + tcfwd::C - 1) / tcfwd::C;
    int nseg = 1;
    if (chains > 0 && chains <= 64 && NC >= 32) nseg = std::min(128 / chains, NC / 8);
    if (nseg < 2) return {1, NC * tcfwd::C};
    const int per = (NC + nseg - 1) / nseg;   // chunks per segment
    return {(NC + per - 1) / per, per * tcfwd::C};
}

}  // namespace

size_t tc_workspace_bytes(int B, int H, int T, int, int, int, int edges) {
    const SegPlan sp = seg_plan(B, H, T);
    const size_t seg = sp.nseg == 1 ? 0 : 3 * sizeof(float) * (size_t)B * H * sp.nseg * tcfwd::KD * tcfwd::VD;
    const size_t ring = edges ? (size_t)B * H * sp.nseg * tcfwd::RING_SLOTS * tcfwd::RING_BYTES : 0;
    return kStatusBytes + seg + ring;
}

int launch_segment_scan(const float *M, const float *N, const float *S0, float *Sg, int chains, int nseg,
                        cudaStream_t st) {
    if (cudaFuncSetAttribute(tcfwd::segment_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tcfwd::SCAN_SMEM) != cudaSuccess)
        return -6;
    tcfwd::segment_scan_kernel<<<dim3(chains, tcfwd::VD / 16), 256, tcfwd::SCAN_SMEM, st>>>(M, N, S0, Sg, nseg);
    return launch_status();
}

int launch_chunk_tc(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                    const float *S0, void *o, float *ST, int B, int H, int T, int K, int V, int C, void *ws,
                    cudaStream_t st, int edges, const float *onorm) {
    if (!tc_supported(B, H, T, K, V, C, 1)) return -4;
    const int smem = (int)tcfwd::SM_BYTES;
    auto kern = edges ? tcfwd::chunk_tc_kernel<true> : tcfwd::chunk_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -6;
    const SegPlan sp = seg_plan(B, H, T);
    const size_t seg_bytes = sp.nseg == 1 ? 0 : 3 * sizeof(float) * (size_t)B * H * sp.nseg * tcfwd::KD * tcfwd::VD;
    unsigned char *ring = edges ? static_cast<unsigned char *>(ws) + kStatusBytes + seg_bytes : nullptr;
    auto run = [&](int nseg, int seg_len, uint32_t flags, const float *s0, float *st_out) {
        kern<<<B * H * nseg, tcfwd::NT, smem, st>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, alpha,
            (const __nv_bfloat16 *)b, (const __nv_bfloat16 *)w, s0, (__nv_bfloat16 *)o, st_out, H, T, seg_len, nseg,
            flags, onorm, ring, reinterpret_cast<unsigned int *>(ws));
    };
    if (sp.nseg == 1) {
        run(1, sp.seg_len, 0u, S0, ST);
        return launch_status();
    }
    const size_t KV = (size_t)tcfwd::KD * tcfwd::VD, per_pass = (size_t)B * H * sp.nseg * KV;
    float *Nm = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + kStatusBytes);
    float *Mm = Nm + per_pass, *Sg = Mm + per_pass;
    run(sp.nseg, sp.seg_len, tcfwd::SEG_SKIP_O, nullptr, Nm);
    run(sp.nseg, sp.seg_len, tcfwd::SEG_SKIP_O | tcfwd::SEG_ZERO_WRITES | tcfwd::SEG_IDENTITY_S0, nullptr, Mm);
    const int rc = launch_segment_scan(Mm, Nm, S0, Sg, B * H, sp.nseg, st);
    if (rc != 0) return rc;
    run(sp.nseg, sp.seg_len, tcfwd::SEG_ST_LAST, Sg, ST);
    return launch_status();
}

}  // namespace gdn2
