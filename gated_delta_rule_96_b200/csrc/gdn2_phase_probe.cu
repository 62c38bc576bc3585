// Measurement kernel for the tensor-core phases of the chunkwise prefill (sm_100a).
//
// The chunkwise WY form with C = 64 (page "NVIDIA представила Gated DeltaNet-2 ...", the paragraph
// on the chunkwise kernels) turns each 64-token chunk of a 128 x 128 head into five groups of
// tcgen05 products, issued by the prefill kernels with these shapes and operand layouts:
//   G1  [A; P]   = [Ê; Q̂] K̃^T        M128 N64  K128   (A K-major, B K-major)
//   G2  [W'; .]  = [T; P] Ê,  [Ũ; .] = [T; P] U   2 x M128 N128 K64 (A K-major, B MN-major)
//   G3  [Δ; O]   = [-W'; Q̂] Z̃        M128 N128 K128   (A K-major, B MN-major)
//   G4  O       += [.; P] Δ           M128 N128 K64    (A K-major, B MN-major)
//   G5  Z       += K̃^T Δ              M128 N128 K64    (A MN-major, B MN-major)
// This kernel issues exactly those instructions, `reps` chunks in a row per CTA, on operands that
// stay in shared memory, so the tensor pipe's rate on the prefill's GEMM phases can be measured
// without the CUDA-core stages around them:
//   mode 0: every chunk's products back to back (the pipe's throughput on these shapes);
//   mode 1: each group waits for the completion of the one before it, as the prefill's data flow
//           requires (G1 -> G2 -> G3 -> G4/G5 -> next chunk), with a single issuing thread.
// The operand values are a fixed small pattern; the accumulators are discarded.
#include "gdn2_common.cuh"
#include "gdn2_internal.h"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace probe {

using namespace gdn2::tc;

constexpr uint32_t S_EQ = 0, S_KT = 32768, S_U = 49152, S_TP = 65536, S_S = 81920, S_DL = 114688,
                   S_MISC = 131072, S_BYTES = S_MISC + 64 + 1024;
constexpr uint32_t ID_G1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_N128 = idesc_bf16(128, 128, 0, 1);
constexpr uint32_t ID_G5 = idesc_bf16(128, 128, 1, 1);
constexpr uint32_t TM_D1 = 0, TM_D2 = 64, TM_D3 = 192, TM_Z = 320, TM_COLS = 512;
constexpr uint32_t WAIT_LIMIT = 1u << 24;

__global__ void __launch_bounds__(128, 1) phase_kernel(int mode, int reps, unsigned int *status) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x;
    const uint32_t misc = smem_u32(sm + S_MISC);
    // a fixed pattern of small bf16 values (exact products, no overflow in any accumulator)
    for (uint32_t i = tid; i < S_MISC / 4; i += 128) {
        const float a = 0.0078125f * (float)((i * 2654435761u >> 27) & 7), b = -0.0078125f * (float)((i >> 3) & 3);
        reinterpret_cast<uint32_t *>(sm)[i] = pack_bf16(a, b);
    }
    if (tid == 0) {
        mbar_init(misc, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid < 32) tmem_alloc(misc + 16, TM_COLS);
    fence_async_smem();
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + S_MISC + 16);
    if (tid == 0) {
        const uint32_t aEQ = smem_u32(sm + S_EQ), aKT = smem_u32(sm + S_KT), aU = smem_u32(sm + S_U),
                       aTP = smem_u32(sm + S_TP), aS = smem_u32(sm + S_S), aDL = smem_u32(sm + S_DL);
        uint32_t phase = 0;
        bool ok = true;
        auto sync_group = [&]() {   // mode 1: the next group waits for this one to complete
            if (mode != 1 || !ok) return;
            mma_commit(misc);
            ok = mbar_wait(misc, phase, WAIT_LIMIT);
            phase ^= 1u;
            fence_after();
        };
        for (int r = 0; r < reps && ok; ++r) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ss(tmem + TM_D1, desc_kmajor(aEQ, 128, j), desc_kmajor(aKT, 64, j), ID_G1, j > 0);
            sync_group();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + TM_D2, desc_kmajor(aTP, 128, j), desc_mnmajor(aEQ, 128, j), ID_N128, j > 0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + TM_D3, desc_kmajor(aTP, 128, j), desc_mnmajor(aU, 64, j), ID_N128, j > 0);
            sync_group();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                mma_ss(tmem + TM_D3, desc_kmajor(aEQ, 128, j), desc_mnmajor(aS, 128, j), ID_N128, 1);
            sync_group();
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + TM_D3, desc_kmajor(aTP, 128, j), desc_mnmajor(aDL, 64, j), ID_N128, 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_ss(tmem + TM_Z, desc_mnmajor(aKT, 64, j), desc_mnmajor(aDL, 64, j), ID_G5, r > 0 || j > 0);
            sync_group();
        }
        if (ok) {   // every product complete before the accumulators are freed
            mma_commit(misc);
            ok = mbar_wait(misc, phase, WAIT_LIMIT);
        }
        if (!ok) atomicOr(status, 8u);
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (tid < 32) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace probe

int launch_phase_probe(int mode, int reps, int nctas, unsigned int *status, cudaStream_t st) {
    const int smem = (int)probe::S_BYTES;
    if (cudaFuncSetAttribute(probe::phase_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return -6;
    probe::phase_kernel<<<nctas, 128, smem, st>>>(mode, reps, status);
    return launch_status();
}

}  // namespace gdn2
