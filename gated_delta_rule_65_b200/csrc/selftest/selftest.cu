// selftest.cu -- checks of the sm_100a building blocks in tc.cuh, built as libgdr2_selftest.so and
// used only by the test suite: one tcgen05 GEMM (M = 128) in every K-major / MN-major operand
// combination (bf16 and fp16 operands, and fp16 with the A operand in TMEM), the shared-memory image of a 128-byte-swizzled TMA load, and the bounded mbarrier wait
// (it gives up and reports through the status word when nothing arrives), and the index checks of the debug
// build (this file is compiled with them on).
#define GDR2_DEBUG 1
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "../tc.cuh"
#include "../tma_host.h"

using namespace gdr2;
using namespace gdr2::tc;

namespace {

// D[m][n] = sum_k opA[m][k] * opB[n][k], M = 128.
// a_mn = 0: A is [M][K] (K contiguous); 1: A is [K][M].  b_mn = 0: B is [N][K]; 1: B is [K][N].
__global__ void __launch_bounds__(128) gemm_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int N,
                                                   int K, int a_mn, int b_mn) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ta = base;              // up to 128 x 128 bf16 = 32 KB
    uint8_t *tb = base + 32768;      // up to 128 x 128 bf16
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int M = 128;
    const int ra = a_mn ? K : M, ca = a_mn ? M : K;
    const int rb = b_mn ? K : N, cb = b_mn ? N : K;
    for (int i = tid; i < ra * ca; i += 128) rt_put(ta, ra, i / ca, i % ca, __bfloat162float(A[i]));
    for (int i = tid; i < rb * cb; i += 128) rt_put(tb, rb, i / cb, i % cb, __bfloat162float(B[i]));
    fence_async_smem();
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, a_mn != 0, b_mn != 0);
        for (int k0 = 0; k0 < K; k0 += 16) {
            const uint64_t ad = a_mn ? desc_mnmajor(ta, ra, k0) : desc_kmajor(ta, ra, k0);
            const uint64_t bd = b_mn ? desc_mnmajor(tb, rb, k0) : desc_kmajor(tb, rb, k0);
            mma_bf16(tmem, ad, bd, id, k0 > 0);
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    fence_after_sync();
    if (ok) {
        const int row = warp * 32 + lane;
        for (int c = 0; c < N; c += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tmem, warp, c), v);
            for (int i = 0; i < 16; ++i) D[row * N + c + i] = v[i];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// fp16 variants. mode 0: A and B from shared memory (a_mn / b_mn select the majors), fp16 operands.
// mode 1: A from TMEM (K-major by construction: thread m writes row m, two fp16 per 32-bit column) and B from
// shared memory (b_mn selects its major). D[m][n] = sum_k opA[m][k] * opB[n][k], M = 128, fp32 accumulate.
__device__ __forceinline__ void h_put(uint8_t *tile, int R, int r, int c, float v) {
    *reinterpret_cast<__half *>(tile + rt_off(R, r, c)) = __float2half_rn(v);
}

__global__ void __launch_bounds__(128) gemm_f16_kernel(const __half *A, const __half *B, float *D, int N, int K,
                                                       int a_mn, int b_mn, int mode) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ta = base;
    uint8_t *tb = base + 32768;
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int M = 128;
    const int rb = b_mn ? K : N, cb = b_mn ? N : K;
    if (mode == 0) {
        const int ra = a_mn ? K : M, ca = a_mn ? M : K;
        for (int i = tid; i < ra * ca; i += 128) h_put(ta, ra, i / ca, i % ca, __half2float(A[i]));
    }
    for (int i = tid; i < rb * cb; i += 128) h_put(tb, rb, i / cb, i % cb, __half2float(B[i]));
    fence_async_smem();
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t tA = tmem + 128;  // A operand columns (mode 1): K / 2 of them
    if (mode == 1) {  // thread = row m = lane of this warp's quadrant; A is stored [M][K]
        const int m = warp * 32 + lane;
        for (int c = 0; c < K / 2; c += 16) {
            uint32_t r[16];
            for (int e = 0; e < 16; ++e)
                r[e] = pack_f16x2(__half2float(A[m * K + 2 * (c + e)]), __half2float(A[m * K + 2 * (c + e) + 1]));
            tmem_st16_raw(tmem_lane_addr(tA, warp, c), r);
        }
        tmem_st_wait();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid == 0) {
        const uint32_t id = idesc_f16(M, N, a_mn != 0 && mode == 0, b_mn != 0);
        for (int k0 = 0; k0 < K; k0 += 16) {
            const uint64_t bd = b_mn ? desc_mnmajor(tb, rb, k0) : desc_kmajor(tb, rb, k0);
            if (mode == 0) {
                const int ra = a_mn ? K : M;
                const uint64_t ad = a_mn ? desc_mnmajor(ta, ra, k0) : desc_kmajor(ta, ra, k0);
                mma_bf16(tmem, ad, bd, id, k0 > 0);
            } else {
                mma_ts(tmem, tA + (uint32_t)(k0 / 2), bd, id, k0 > 0);
            }
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    fence_after_sync();
    if (ok) {
        const int row = warp * 32 + lane;
        for (int c = 0; c < N; c += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tmem, warp, c), v);
            for (int i = 0; i < 16; ++i) D[row * N + c + i] = v[i];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// TMEM image of an M = 64 product: all 128 lanes x N columns (sentinel NaN where nothing was written).
// A is [64][K] and B is [N][K], both K-major.
__global__ void __launch_bounds__(128) gemm_m64_dump_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B,
                                                            float *dump, int N, int K) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ta = base;
    uint8_t *tb = base + 32768;
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 64 * K; i += 128) rt_put(ta, 64, i / K, i % K, __bfloat162float(A[i]));
    for (int i = tid; i < N * K; i += 128) rt_put(tb, N, i / K, i % K, __bfloat162float(B[i]));
    fence_async_smem();
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    {
        float nan16[16];
        for (int e = 0; e < 16; ++e) nan16[e] = __int_as_float(0x7fc00000);
        for (int c = 0; c < N; c += 16) tmem_st16(tmem_lane_addr(tmem, warp, c), nan16);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid == 0) {
        const uint32_t id = idesc_bf16(64, N, false, false);
        for (int k0 = 0; k0 < K; k0 += 16) mma_bf16(tmem, desc_kmajor(ta, 64, k0), desc_kmajor(tb, N, k0), id, k0 > 0);
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    fence_after_sync();
    if (ok) {
        const int lane_id = warp * 32 + lane;
        for (int c = 0; c < N; c += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tmem, warp, c), v);
            for (int i = 0; i < 16; ++i) dump[lane_id * N + c + i] = v[i];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// Raw shared-memory bytes of a [rows x 128] bf16 tile loaded as two 64-column boxes (SWIZZLE_128B).
__global__ void __launch_bounds__(128) tma_layout_kernel(const __grid_constant__ CUtensorMap map, uint8_t *out,
                                                         int rows) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *tile = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_expect_tx(&bar, (uint32_t)rows * 256u);
        tma_load_2d(tile, &map, 0, 0, &bar);
        tma_load_2d(tile + rows * 128, &map, 64, 0, &bar);
    }
    if (!mbar_wait(&bar, 0)) return;
    for (int i = threadIdx.x; i < rows * 256; i += blockDim.x) out[i] = tile[i];
}

int sync_status(cudaError_t e) {
    if (e != cudaSuccess) return 4;
    return cudaDeviceSynchronize() == cudaSuccess ? 0 : 4;
}

// One warp waits, with a bounded wait of `limit` polls, for phase 0 of an mbarrier with one expected
// arrival. With publish = 0 nothing ever arrives, so every poll fails and the wait must give up and set
// kStatusTimeout rather than spin on; with publish = 1 thread 0 arrives first and the wait succeeds.
// done = 1 (the phase completed) or 2 (the wait gave up).
__global__ void __launch_bounds__(32) wait_kernel(uint32_t limit, int publish, int *done) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (publish && threadIdx.x == 0) mbar_expect_tx(&bar, 0u);  // an arrival with no bytes to wait for
    const bool ok = mbar_wait(&bar, 0u, limit);
    if (threadIdx.x == 0) *done = ok ? 1 : 2;
}

// The debug build's tile-index check: the byte offset of element (r, 0) of an RT tile with R rows is computed
// (no memory is touched); r outside [0, R) sets the bounds bit of the status word.
__global__ void index_check_kernel(int R, int r, uint32_t *off) {
    if (threadIdx.x == 0) *off = rt_off(R, r, 0);
}

}  // namespace

extern "C" {

__attribute__((visibility("default"))) int gdr2st_gemm(const void *A, const void *B, float *D, int N, int K,
                                                       int a_mn, int b_mn) {
    if ((N != 64 && N != 128) || (K != 64 && K != 128)) return 1;
    const int smem = 65536 + 1024;
    if (cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 4;
    gemm_kernel<<<1, 128, smem>>>((const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, D, N, K, a_mn, b_mn);
    return sync_status(cudaGetLastError());
}

__attribute__((visibility("default"))) int gdr2st_gemm_f16(const void *A, const void *B, float *D, int N, int K,
                                                           int a_mn, int b_mn, int mode) {
    if ((N != 64 && N != 128) || (K != 64 && K != 128) || (mode != 0 && mode != 1)) return 1;
    const int smem = 65536 + 1024;
    if (cudaFuncSetAttribute(gemm_f16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 4;
    gemm_f16_kernel<<<1, 128, smem>>>((const __half *)A, (const __half *)B, D, N, K, a_mn, b_mn, mode);
    return sync_status(cudaGetLastError());
}

__attribute__((visibility("default"))) int gdr2st_gemm_m64_dump(const void *A, const void *B, float *dump, int N,
                                                                int K) {
    if ((N != 64 && N != 128) || (K != 64 && K != 128)) return 1;
    const int smem = 65536 + 1024;
    if (cudaFuncSetAttribute(gemm_m64_dump_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 4;
    gemm_m64_dump_kernel<<<1, 128, smem>>>((const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, dump, N, K);
    return sync_status(cudaGetLastError());
}

__attribute__((visibility("default"))) int gdr2st_tma_layout(const void *src, void *out, int rows) {
    if (rows < 8 || rows > 256 || rows % 8) return 1;
    CUtensorMap map;
    uint64_t dims[2] = {128, (uint64_t)rows};
    uint64_t strides[1] = {256};
    uint32_t box[2] = {64, (uint32_t)rows};
    if (!make_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, src, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B))
        return 4;
    const int smem = rows * 256 + 1024;
    if (cudaFuncSetAttribute(tma_layout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 4;
    tma_layout_kernel<<<1, 128, smem>>>(map, (uint8_t *)out, rows);
    return sync_status(cudaGetLastError());
}

// Status bits of this library's kernels since the last call (cleared on read), -1 if unreadable.
__attribute__((visibility("default"))) int gdr2st_wait_error(void) { return take_status(); }

// Runs index_check_kernel and returns the status bits it left (kStatusBounds = 4 for r outside [0, R)), or -2
// on a CUDA error.
__attribute__((visibility("default"))) int gdr2st_index_check(int R, int r, uint32_t *off) {
    if (take_status() < 0) return -2;
    index_check_kernel<<<1, 32>>>(R, r, off);
    if (sync_status(cudaGetLastError()) != 0) return -2;
    return take_status();
}

// Runs wait_kernel (limit polls, publish 0 / 1) and returns the status bits it left, or -2 on a CUDA error.
__attribute__((visibility("default"))) int gdr2st_bounded_wait(unsigned limit, int publish, int *done) {
    if (take_status() < 0) return -2;  // start from a clean word
    wait_kernel<<<1, 32>>>(limit, publish, done);
    if (sync_status(cudaGetLastError()) != 0) return -2;
    return take_status();
}

}  // extern "C"
