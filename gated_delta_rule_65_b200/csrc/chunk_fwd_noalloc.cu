// chunk_fwd_noalloc.cu -- gdr2_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers only ever receive input and output buffers: plugins inside a host framework that
// owns every byte of device memory through its own pool, and latency-critical loops where a
// cudaMalloc (which may synchronise the device) is not allowed. They cannot provide the workspace
// that gdr2_chunk_fwd asks for. This entry point runs the same chunkwise forward (the plain fp32-FMA
// kernels of chunk_simt.cu, unchanged) with its scratch in a fixed array compiled into the library.
//
// The array below lives in every GPU that loads this library until the process exits. In host code its name
// is only a host-side stand-in: every call looks up the array's device address with cudaGetSymbolAddress, with
// the caller's device current, and passes that address to the kernels. The lookup is cheap once the module is
// loaded, and repeating it keeps the address right after the caller resets the device or rebuilds its primary
// context (the module, and with it the array, may then sit elsewhere).
#include <stdint.h>

#include "gdr2.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current device's context.
int scratch_for_current_device(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GDR2_ERR_CUDA;
    *out = p;
    return GDR2_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" GDR2_API int gdr2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                                               const void *b, const void *w, const float *initial_state, void *o,
                                               float *final_state, int B, int T, int H, int dk, int dv, int dtype,
                                               void *stream) {
    if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_F32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GDR2_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return GDR2_ERR_UNSUPPORTED;
    const void *req[] = {q, k, v, log_alpha, b, w, o};
    for (const void *p : req)
        if (p == nullptr || !aligned16(p)) return GDR2_ERR_INVALID_ARG;
    if (!aligned16(initial_state) || !aligned16(final_state)) return GDR2_ERR_INVALID_ARG;
    // chunk count first, so that no product of the sizes can wrap around before the comparison
    const size_t chunks = (size_t)B * (size_t)H * (size_t)((T + 63) / 64);
    if (chunks > kNoAllocScratchBytes) return GDR2_ERR_WORKSPACE;
    const size_t need = gdr2::simt_workspace_bytes(B, T, H, dk, dv, 0);
    if (need == 0 || need > kNoAllocScratchBytes) return GDR2_ERR_WORKSPACE;  // larger than the fixed scratch

    void *scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != GDR2_OK) return st;
    gdr2::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.b = b; a.w = w; a.initial_state = initial_state;
    a.o = o; a.final_state = final_state;
    a.B = B; a.T = T; a.H = H; a.dk_ = dk; a.dv_ = dv; a.dtype = dtype;
    a.workspace = scratch; a.workspace_bytes = kNoAllocScratchBytes;
    return gdr2::launch_simt_fwd(a, (cudaStream_t)stream) == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}
