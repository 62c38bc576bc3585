// Memory layouts shared by the two-stage prefill (gdn2_chunk_split.cu) and the tensor-core backward
// (gdn2_chunk_bwd_tc.cu): the per-chunk-head record the first stage writes and the second reads, the
// backward's per-chunk-head side record, and the tensor maps of the token tensors.
//
// Every operand image is a bf16 tile in the swizzled layout of sw_off (tc_ptx.cuh): 64-column halves
// of R rows x 128 bytes, so one image serves either operand major of tcgen05.mma.  Chunk-heads are
// numbered (batch, chunk, head) with the head fastest, the order in which the first stage writes them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn2 {
namespace split {

constexpr int C = 64, KD = 128, VD = 128;

// ---------------------------------------------------------------------------- record (bytes)
constexpr uint32_t R_A3 = 0;        // [-W'; Q̂]: 128 x 128 K-major (A of G3), 128-row halves
constexpr uint32_t R_KT = 32768;    // K̃ [i x c]: 64 x 128 (MN-major A of G5), 64-row halves
constexpr uint32_t R_U = 49152;     // Ũ [i x v]: 64 x 128
constexpr uint32_t R_P = 65536;     // P [r x i]: 64 x 64, lower with the diagonal
constexpr uint32_t R_VEC = 73728;   // sS, sZ, sPost: 3 x 128 fp32
constexpr uint32_t R_COPY = R_VEC + 3 * 128 * 4;   // bytes moved per record
constexpr uint32_t R_BYTES = 75776;                // record stride (1024-aligned)
// a walk that stores no o copies K̃ and Ũ as one range
static_assert(R_U == R_KT + 16384 && R_COPY <= R_BYTES, "record layout");

// ---------------------------------------------------------------------------- backward side record
// Written by the forward replay (first stage: Ê, T and the frame exponents; second stage: Z̃, Delta)
// and by the reverse walk (G̃, dDelta, rho); read by the gradient kernel.
constexpr uint32_t X_E = 0;          // Ê [r x c], 64-row halves (16 KB)
constexpr uint32_t X_T = 16384;      // T = (I + A)^-1 [r x i], 64 x 64 (8 KB)
constexpr uint32_t X_Z = 24576;      // Z̃ [c x v]: the bf16 state operand of the chunk, 128-row halves (32 KB)
constexpr uint32_t X_DL = 57344;     // Delta [i x v], 64-row halves (16 KB)
constexpr uint32_t X_G = 73728;      // G̃ = Diag(sPost) dS' [c x v], 128-row halves (32 KB)
constexpr uint32_t X_DD = 106496;    // dDelta stored as [v x i]: 128 rows x 64 (16 KB)
constexpr uint32_t X_RHO = 122880;   // rho = rowsum(dS' ⊙ S') fp32 [128]
constexpr uint32_t X_AE = 123392;    // frame exponents fp32 [128]: Ê = e ⊙ 2^(g - ae), K̃ = k ⊙ 2^(ak - g)
constexpr uint32_t X_AK = 123904;
constexpr uint32_t X_BYTES = 124928;

// Walk launch flags.  Segmented walk (few long chains): block blockIdx.x walks segment blockIdx.x % nseg
// (chunks [seg * seg_len, (seg + 1) * seg_len) of the window) of chain blockIdx.x / nseg; S0 and S_T are
// then indexed by block.
enum : uint32_t {
    WALK_ZERO_WRITES = 1,   // Ũ = 0: the walk propagates the state only (the segment's homogeneous map)
    WALK_SKIP_O = 2,        // o is not stored
    WALK_IDENTITY_S0 = 4,   // the segment starts from S = I (d_k = d_v)
    WALK_ST_LAST = 8,       // only the chain's last segment stores S_T, at S_T[chain]
};

struct TokMaps {   // [B, T, H, 128] token tensors as 4-D maps (d, H, T, B): bf16 with a 64 x 1 x 64 x 1 box
    CUtensorMap q, k, b, v, w, alpha;   // in the 128-byte swizzle; alpha fp32 with a 128 x 1 x 64 x 1 box
};

}  // namespace split

// A [B, T, H, 128] token tensor as the 4-D map (d, H, T, B).  bf16: a 64 x 1 x 64 x 1 box in the 128-byte
// swizzle, one box being the 64 x 64 half-tile of the operand layout; fp32: a 128 x 1 x 64 x 1 box, rows of
// 512 bytes.  Rows past T read as zero.
bool token_map(CUtensorMap *m, const void *base, int B, int T, int H, bool fp32 = false);
int sm_count();

// Forward replay of the backward (gdn2_chunk_split.cu): both stages of the prefill over the whole
// sequence, o not stored, S_T written, every chunk-head's record and side record filled.  `seg` holds
// replay_segment_bytes(B, H, T) bytes of scratch for the segmented walk of few long chains; any_map is
// any valid token map (the walk's o map, never written through).
size_t replay_segment_bytes(int B, int H, int T);
int launch_split_replay(const void *q, const void *k, const void *v, const float *alpha, const void *b, const void *w,
                        const float *S0, float *ST, int B, int H, int T, unsigned char *records, unsigned char *aux,
                        float *seg, const CUtensorMap &any_map, unsigned int *status, cudaStream_t st);

}  // namespace gdn2
