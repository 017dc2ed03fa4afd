// tma_host.h -- host-side creation of TMA tensor maps (cuTensorMapEncodeTiled obtained through the
// runtime's driver entry-point query, so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr2 {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Tiled tensor map. dims[0] is the contiguous dimension; strides_bytes has rank-1 entries (dims 1..).
inline bool make_tensor_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *gaddr, const uint64_t *dims,
                            const uint64_t *strides_bytes, const uint32_t *box, CUtensorMapSwizzle sw) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    uint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, dt, (cuuint32_t)rank, const_cast<void *>(gaddr), (const cuuint64_t *)dims,
                     (const cuuint64_t *)strides_bytes, (const cuuint32_t *)box, (const cuuint32_t *)estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace gdr2
