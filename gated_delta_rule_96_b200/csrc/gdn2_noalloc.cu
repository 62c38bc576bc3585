// gdn2_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory.
//
// Some hosts own every byte of device memory (a framework's pool allocator, a fixed
// per-process memory budget) and do not let a plugin allocate on its own, and some
// latency-sensitive callers forbid cudaMalloc on their hot path because it can
// synchronise the whole device.  Such callers cannot provide the workspace that
// gdn2_chunk_fwd needs.  This entry point runs the CUDA-core chunkwise path with its
// scratch in a fixed array that lives in the library's own device memory instead.
//
// Cost of that choice: every GPU that loads the library reserves
// GDN2_NOALLOC_SCRATCH_BYTES for the array until the process exits, and all calls
// share the one array, so calls that overlap on the GPU (other streams, other host
// threads) race on it and corrupt each other's results.
#include <cuda.h>

#include <mutex>

#include "gdn2.h"
#include "gdn2_internal.h"

namespace {

// The scratch itself.  In host code this name is only a host-side stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the array's address and the id of the context it was looked up in.  A device
// reset (cudaDeviceReset) replaces the context and reloads the module, so an address from
// the old context is never reused: a new context id triggers a new lookup.
struct Cached {
    unsigned long long ctx_id;
    void *addr;
};
Cached g_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Id of the calling thread's current context (driver entry points fetched through the
// runtime, so the library does not link libcuda).  False when no context is current yet.
bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void *f1 = nullptr, *f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault) != cudaSuccess || !f1) return false;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault) != cudaSuccess || !f2) return false;
        get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the array on the current device: looked up with that device current,
// once per device and context (cudaGetSymbolAddress allocates nothing).
int scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long id = 0;
    const bool known = current_context_id(&id);
    if (!known || !g_cache[dev].addr || g_cache[dev].ctx_id != id) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDN2_ERR_CUDA;
        if (!current_context_id(&id)) return GDN2_ERR_CUDA;   // the lookup made the context current
        g_cache[dev] = {id, p};
    }
    *out = g_cache[dev].addr;
    return GDN2_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dim_ok(int d) { return d == 64 || d == 128; }

}  // namespace

extern "C" int gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *alpha,
                                      const void *b, const void *w, const float *S0, void *o, float *S_T, int B,
                                      int H, int T, int d_k, int d_v, int C, int dtype, void *stream) {
    if (B < 0 || H < 0 || T < 0) return GDN2_ERR_SHAPE;
    if (dtype != GDN2_F32 && dtype != GDN2_BF16) return GDN2_ERR_DTYPE;
    if (!dim_ok(d_k) || !dim_ok(d_v) || C != 64) return GDN2_ERR_UNSUPPORTED;
    if (!S_T) return GDN2_ERR_NULL;
    if (T > 0 && (!q || !k || !v || !alpha || !b || !w || !o)) return GDN2_ERR_NULL;
    if (!aligned16(S_T) || (S0 && !aligned16(S0))) return GDN2_ERR_ALIGN;
    if (T > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(alpha) || !aligned16(b) ||
                  !aligned16(w) || !aligned16(o)))
        return GDN2_ERR_ALIGN;
    const size_t need = gdn2::simt_workspace_bytes(B, H, T, d_k, d_v, C);
    if (need > (size_t)GDN2_NOALLOC_SCRATCH_BYTES) return GDN2_ERR_NOALLOC_LIMIT;
    if (B == 0 || H == 0) return GDN2_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
        const size_t state_bytes = sizeof(float) * (size_t)B * H * d_k * d_v;
        cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess
                                        : cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, st))
                           : cudaMemsetAsync(S_T, 0, state_bytes, st);
        return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
    }
    void *scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != GDN2_OK) return rc;
    // Nothing in the scratch has to start at zero: within one call stage 1 writes every
    // element stage 2 reads, so the previous call's leftovers are never read.
    return gdn2::launch_chunk_simt(q, k, v, alpha, b, w, S0, o, S_T, B, H, T, d_k, d_v, C,
                                   dtype == GDN2_BF16 ? 1 : 0, scratch, st);
}
