// status.cuh -- the device status word of a translation unit. Kernels never trap: a bounded wait that gives
// up, or an input outside the range the chunk form represents in fp32, sets a bit here and the kernel
// finishes uniformly. The host reads and clears the word with take_status(), which gdr2_check() calls for
// every translation unit that can set it.
#pragma once

#include <cuda_runtime.h>

namespace gdr2 {

constexpr int kStatusTimeout = 1;  // a bounded mbarrier wait expired
constexpr int kStatusRange = 2;    // a chunk's cumulative log-decay left the range of its path (below)
constexpr int kStatusBounds = 4;   // an index check of a debug build (GDR2_DEBUG) failed

// Bound on the in-chunk cumulative log-decay G of one channel (the sum of log_alpha over the chunk's rows)
// beyond which the chunk form's decay-scaled factors leave fp32's normal range: a factor e^{80} = 5.5e34
// (FLT_MAX 3.4e38), and e^{-80} with the 2^-9 lo part of a hi / lo pair 3.5e-38 (FLT_MIN 1.2e-38).
// The fp32 path scales keys by e^{-G} and erase keys by e^{G}, so |G_C| <= 80 (a mean log_alpha of -1.25
// per token over a full 64-token chunk); the tensor-core path takes them relative to the mid-chunk value
// G_C / 2, so |G_C| <= 160.
constexpr float kMaxChunkLogDecay = 80.f;
constexpr float kMaxChunkLogDecayTC = 160.f;

static __device__ int g_status;

__device__ __forceinline__ void flag_status(int bits) { atomicOr(&g_status, bits); }

// Index checks of the debug build (compiled with -DGDR2_DEBUG): a failed check sets kStatusBounds, which
// gdr2_check reports as GDR2_ERR_BOUNDS; the kernel carries on (it never traps). GDR2_DGUARD(cond) is the same
// check as an expression, so that a debug build can also skip the access it guards. Release builds compile both
// to nothing (GDR2_DGUARD to true).
#ifdef GDR2_DEBUG
#define GDR2_DCHECK(cond)                                                \
    do {                                                                 \
        if (!(cond)) ::gdr2::flag_status(::gdr2::kStatusBounds);         \
    } while (0)
#define GDR2_DGUARD(cond) ((cond) ? true : (::gdr2::flag_status(::gdr2::kStatusBounds), false))
#else
#define GDR2_DCHECK(cond) \
    do {                  \
    } while (0)
#define GDR2_DGUARD(cond) true
#endif

// Host: this translation unit's status bits, cleared on read; -1 when the word cannot be read.
static inline int take_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return -1;
    if (v != 0) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_status, &z, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace gdr2
