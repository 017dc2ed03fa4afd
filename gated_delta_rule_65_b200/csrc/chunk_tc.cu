// chunk_tc.cu -- tensor-core (tcgen05 + TMEM + TMA) chunkwise Gated Delta Rule-2 forward for bf16
// operands, dk = dv = 128, C = 64, fp32 state.
//
// The algorithm is the chunkwise WY form of the review's section "Chunkwise Parallel Training via WY
// Representation" (Steps 1-3, Eqs. 20-24; the T factor of Appendix C.2), in two kernels:
//
//  local  grid (NT, H, B), 128 threads (thread i = key/value channel i), one chunk per CTA.
//         Step 1 in fp32: cumulative log-decay G per channel, gamma = exp(G), and
//         Q_gamma = gamma q, Kbar = k / gamma, Ebar = gamma b k, K_tail = (gamma_C / gamma) k, Z = w v.
//         On tcgen05 (M = 64): T = Ebar Kbar^T and A_qk = Q_gamma Kbar^T; A = (I + T)^-1 by forward
//         substitution in fp32 (one column per thread); Y = A Ebar and U = A Z.
//  state  grid (B*H), 128 threads, one CTA per (batch, head): the serial pass of Eq. 23 with the state
//         kept transposed, S^T [dv x dk], fp32 in TMEM (lane j = value channel j), so all products
//         have M = dv = 128:
//             R^T = U^T - S^T Y^T,   O^T = S^T Q_gamma^T + R^T A_qk^T,
//             S^T <- S^T Diag(gamma_C) + R^T K_tail.
//
// Precision: every operand derived from the inputs carries decay factors, and rounding it to bf16
// costs ~2^-9 relative per use; over the ~10 roundings of the chunk algebra that exceeds the target
// error bound. So every derived operand is held as a pair hi = bf16(x), lo = bf16(x - hi) and every
// product is Ah Bh + Ah Bl + Al Bh on the bf16 tensor pipe (fp32 accumulation), which keeps ~16 bits;
// U stays fp32. The workspace between the kernels holds these pairs.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma_host.h"

namespace gdr2 {
namespace {

using namespace tc;

constexpr int C = kChunk;
constexpr int D = 128;

// Workspace of the tensor-core forward, per chunk (ch = (b*H + h)*NT + c).
struct WsTC {
    __nv_bfloat16 *Yh, *Yl, *Qh, *Ql, *Kh, *Kl;  // [nch][64][128]  Y, Q_gamma, K_tail (hi / lo)
    __nv_bfloat16 *Ah, *Al;                      // [nch][64][64]   tril(A_qk)      (hi / lo)
    float *U;                                    // [nch][64][128]
    float *gC;                                   // [nch][128]
};

// Backward-only workspace, fp32, per chunk. Row-major in the orientation each tensor is produced in.
struct WsBwd {
    float *Qg, *Kb, *Eb, *Z;          // [64 r][128]       forward operands of the chunk
    float *A;                         // [64 r][64 s]      (I + T)^-1
    float *S0T, *dST;                 // [128 j][128 i]    state entering the chunk / its gradient (S_C side)
    float *RT, *dRT;                  // [128 j][64 r]     R^T and dR^T
    float *dAqk, *dA, *X, *dT;        // [64][64]
    float *dQgT, *dKtT, *dYT, *dEbT, *dKbT;  // [128 i][64 r]
    float *dZT;                       // [128 j][64 s]
};

constexpr size_t kTileBytes = (size_t)C * D * 2;  // 16 KB
constexpr size_t kCCBytes = (size_t)C * C * 2;    // 8 KB

size_t tc_ws_bytes_per_chunk() { return 6 * kTileBytes + 2 * kCCBytes + (size_t)C * D * 4 + D * 4; }
size_t tc_bwd_ws_bytes_per_chunk() {
    return sizeof(float) * (4 * (size_t)C * D + (size_t)C * C + 2 * (size_t)D * D + 2 * (size_t)D * C +
                            4 * (size_t)C * C + 6 * (size_t)D * C);
}

WsBwd carve_bwd(void *base, size_t nch) {
    float *p = (float *)base;
    auto take = [&](size_t per) { float *r = p; p += per * nch; return r; };
    WsBwd w{};
    w.Qg = take((size_t)C * D); w.Kb = take((size_t)C * D); w.Eb = take((size_t)C * D); w.Z = take((size_t)C * D);
    w.A = take((size_t)C * C);
    w.S0T = take((size_t)D * D); w.dST = take((size_t)D * D);
    w.RT = take((size_t)D * C); w.dRT = take((size_t)D * C);
    w.dAqk = take((size_t)C * C); w.dA = take((size_t)C * C); w.X = take((size_t)C * C); w.dT = take((size_t)C * C);
    w.dQgT = take((size_t)D * C); w.dKtT = take((size_t)D * C); w.dYT = take((size_t)D * C);
    w.dEbT = take((size_t)D * C); w.dKbT = take((size_t)D * C); w.dZT = take((size_t)D * C);
    return w;
}

WsTC carve_tc(void *base, size_t nch) {
    uint8_t *p = (uint8_t *)base;
    auto take = [&](size_t per) { uint8_t *r = p; p += per * nch; return r; };
    WsTC w{};
    w.Yh = (__nv_bfloat16 *)take(kTileBytes);
    w.Yl = (__nv_bfloat16 *)take(kTileBytes);
    w.Qh = (__nv_bfloat16 *)take(kTileBytes);
    w.Ql = (__nv_bfloat16 *)take(kTileBytes);
    w.Kh = (__nv_bfloat16 *)take(kTileBytes);
    w.Kl = (__nv_bfloat16 *)take(kTileBytes);
    w.Ah = (__nv_bfloat16 *)take(kCCBytes);
    w.Al = (__nv_bfloat16 *)take(kCCBytes);
    w.U = (float *)take((size_t)C * D * 4);
    w.gC = (float *)take(D * 4);
    return w;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void split2(float x, __nv_bfloat16 &h, __nv_bfloat16 &l) {
    h = __float2bfloat16_rn(x);
    l = __float2bfloat16_rn(x - __bfloat162float(h));
}

// 8 fp32 values -> two rows of 8 bf16 (hi / lo) in global memory (16-byte stores).
__device__ __forceinline__ void store_split8(__nv_bfloat16 *dh, __nv_bfloat16 *dl, const float *v) {
    __nv_bfloat16 h[8], l[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split2(v[e], h[e], l[e]);
    *reinterpret_cast<uint4 *>(dh) = *reinterpret_cast<uint4 *>(h);
    *reinterpret_cast<uint4 *>(dl) = *reinterpret_cast<uint4 *>(l);
}

// =================================================================================================
// local kernel: one chunk per CTA
// =================================================================================================
constexpr int kLocalThreads = 512;
constexpr int kTsmStride = 68;                   // fp32 row stride of T and A in shared memory
constexpr size_t kLocTile = 16384;               // RT tile 64 x 128 bf16
constexpr size_t kSqBytes = 64 * kTsmStride * 4; // 17408
constexpr size_t kLocalSmem = 8 * kLocTile + 2 * kCCBytes + 2 * kSqBytes + 3 * 256 * 4 + 1024;

struct LocalMaps {
    CUtensorMap q, k, b, v, w, la;
};

// A = (I + T)^-1 for a strictly lower triangular 64 x 64 T (fp32, row stride kTsmStride), blocked in
// 16 x 16 tiles: the four diagonal blocks by forward substitution (one column per thread), then block
// row i = 1..3 from A_ij = -A_ii sum_{k=j}^{i-1} T_ik A_kj. All 128 threads take part.
__device__ void wy_inverse(const float *Tm, float *Am, float *W) {
    const int tid = threadIdx.x;
    for (int x = tid; x < 64 * kTsmStride; x += kLocalThreads) Am[x] = 0.f;
    __syncthreads();
    if (tid < 64) {
        const int d = tid >> 4, cc = tid & 15, o = 16 * d;
        float a[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s = (r == cc) ? 1.f : 0.f;
            const float *Tr = Tm + (o + r) * kTsmStride + o;
#pragma unroll
            for (int j = 0; j < r; ++j) s = fmaf(-Tr[j], a[j], s);
            a[r] = s;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Am[(o + r) * kTsmStride + o + cc] = a[r];
    }
    __syncthreads();
    for (int i = 1; i < 4; ++i) {
        // W_j = sum_{k=j}^{i-1} T_ik A_kj   for j < i
        for (int x = tid; x < i * 256; x += kLocalThreads) {
            const int j = x >> 8, r = (x >> 4) & 15, c = x & 15;
            float s = 0.f;
            const float *Tr = Tm + (16 * i + r) * kTsmStride;
            for (int kk = 16 * j; kk < 16 * i; ++kk) s = fmaf(Tr[kk], Am[kk * kTsmStride + 16 * j + c], s);
            W[x] = s;
        }
        __syncthreads();
        // A_ij = -A_ii W_j
        for (int x = tid; x < i * 256; x += kLocalThreads) {
            const int j = x >> 8, r = (x >> 4) & 15, c = x & 15;
            float s = 0.f;
            const float *Ar = Am + (16 * i + r) * kTsmStride + 16 * i;
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) s = fmaf(Ar[kk], W[(j << 8) + kk * 16 + c], s);
            Am[(16 * i + r) * kTsmStride + 16 * j + c] = -s;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kLocalThreads, 1)
    local_kernel(const __grid_constant__ LocalMaps maps, WsTC ws, WsBwd bw, int T, int H, int NT) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tQh = base, *tQl = base + kLocTile;                     // Q_gamma   (raw q arrives in tQl)
    uint8_t *tKh = base + 2 * kLocTile, *tKl = base + 3 * kLocTile;  // Kbar      (raw k arrives in tKl)
    uint8_t *tEh = base + 4 * kLocTile, *tEl = base + 5 * kLocTile;  // Ebar      (raw b arrives in tEl)
    uint8_t *tZh = base + 6 * kLocTile, *tZl = base + 7 * kLocTile;  // Z         (raw w in tZh, v in tZl)
    uint8_t *tAh = base + 8 * kLocTile, *tAl = tAh + kCCBytes;       // A = (I + T)^-1
    float *Tsm = reinterpret_cast<float *>(tAl + kCCBytes);          // [64][kTsmStride]
    float *Asm = Tsm + 64 * kTsmStride;                              // [64][kTsmStride]
    float *Wsm = Asm + 64 * kTsmStride;                              // [3][16][16]
    float *la_s = Tsm;  // raw log-decay [64][128] fp32, consumed before T is written
    __shared__ uint64_t bar_in, bar1, bar2;
    __shared__ uint32_t tslot;
    __shared__ float seg_sum[4][128];

    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t ch = ((size_t)bi * H + h) * NT + c;
    const int t0 = c * C;
    const int i = tid & 127;     // channel
    const int sg = tid >> 7;     // row segment: rows [16 sg, 16 sg + 16)

    if (tid == 0) {
        mbar_init(&bar_in, 1);
        mbar_init(&bar1, 1);
        mbar_init(&bar2, 1);
        mbar_fence_init();
        mbar_expect_tx(&bar_in, 5u * (uint32_t)kLocTile + 64u * 128u * 4u);
        const CUtensorMap *mp[5] = {&maps.q, &maps.k, &maps.b, &maps.w, &maps.v};
        uint8_t *dst[5] = {tQl, tKl, tEl, tZh, tZl};
        for (int x = 0; x < 5; ++x) {
            tma_load_4d(dst[x], mp[x], 0, h, t0, bi, &bar_in);
            tma_load_4d(dst[x] + 8192, mp[x], 64, h, t0, bi, &bar_in);
        }
        tma_load_4d(la_s, &maps.la, 0, h, t0, bi, &bar_in);
    }
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t tT = tmem, tAqk = tmem + 64, tY = tmem, tU = tmem + 128;

    bool ok = mbar_wait(&bar_in, 0);
    // Step 1: cumulative log-decay of channel i (fp32): 16-row segment sums, then segment offsets.
    float G[16];
    {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            acc += la_s[(16 * sg + r) * D + i];
            G[r] = acc;
        }
        seg_sum[sg][i] = acc;
    }
    __syncthreads();
    float off = 0.f, GC = 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const float v = seg_sum[x][i];
        if (x < sg) off += v;
        GC += v;
    }
    if (sg == 0) ws.gC[ch * D + i] = expf(GC);
    if (ok) {
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const int r = 16 * sg + rr;
            const float kk = rt_get(tKl, 64, r, i), bb = rt_get(tEl, 64, r, i), qq = rt_get(tQl, 64, r, i);
            const float vv = rt_get(tZl, 64, r, i), wv = rt_get(tZh, 64, r, i);
            const float g = off + G[rr];
            const float gam = expf(g), ginv = expf(-g), gt = expf(GC - g);
            const float qg = qq * gam, kt = kk * gt, kb = kk * ginv, eb = bb * kk * gam, z = wv * vv;
            split_put(tQh, tQl, 64, r, i, qg);
            split_put(tKh, tKl, 64, r, i, kb);
            split_put(tEh, tEl, 64, r, i, eb);
            split_put(tZh, tZl, 64, r, i, z);
            const size_t wo = (ch * C + r) * D + i;
            split2(qg, ws.Qh[wo], ws.Ql[wo]);
            split2(kt, ws.Kh[wo], ws.Kl[wo]);
            if (bw.Qg) {
                bw.Qg[wo] = qg;
                bw.Kb[wo] = kb;
                bw.Eb[wo] = eb;
                bw.Z[wo] = z;
            }
        }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // T = Ebar Kbar^T, A_qk = Q_gamma Kbar^T (M = 64, N = 64, K = 128)
    if (ok && tid == 0) {
        const uint32_t id = idesc_bf16(64, 64, false, false);
        for (int k0 = 0; k0 < 128; k0 += 16)
            mma3(tT, desc_kmajor(tEh, 64, k0), desc_kmajor(tEl, 64, k0), desc_kmajor(tKh, 64, k0),
                 desc_kmajor(tKl, 64, k0), id, k0 > 0);
        for (int k0 = 0; k0 < 128; k0 += 16)
            mma3(tAqk, desc_kmajor(tQh, 64, k0), desc_kmajor(tQl, 64, k0), desc_kmajor(tKh, 64, k0),
                 desc_kmajor(tKl, 64, k0), id, k0 > 0);
        mma_commit(&bar1);
    }
    ok = ok && mbar_wait(&bar1, 0);
    fence_after_sync();
    // M = 64 accumulator layout: row m sits in TMEM lane 32 * (m / 16) + m % 16. Warp w reads lane
    // quadrant w % 4; its task (w / 4) picks 32 columns of T (tasks 0, 1) or of A_qk (tasks 2, 3).
    const int quad = warp & 3, task = warp >> 2;
    const int m = 16 * quad + (lane & 15);
    const bool holds_row = lane < 16;
    if (ok) {
        const int cbase = (task & 1) * 32;
        for (int c0 = cbase; c0 < cbase + 32; c0 += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(task < 2 ? tT : tAqk, quad, c0), v);
            if (holds_row) {
                if (task < 2) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(Tsm + m * kTsmStride + c0 + e) =
                            make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (c0 + e > m) v[e] = 0.f;
                    const size_t wo = (ch * C + m) * C + c0;
                    store_split8(ws.Ah + wo, ws.Al + wo, v);
                    store_split8(ws.Ah + wo + 8, ws.Al + wo + 8, v + 8);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // Step 2: A = (I + T)^-1 (fp32), then the hi / lo operand tiles.
    wy_inverse(Tsm, Asm, Wsm);
    for (int x = tid; x < 64 * 8; x += kLocalThreads) {
        const int r = x >> 3, c8 = (x & 7) * 8;
        const float *src = Asm + r * kTsmStride + c8;
        float v8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v8[e] = src[e];
        split_store8(tAh, tAl, 64, r, c8, v8);
        if (bw.A) {
            float *dst = bw.A + (ch * C + r) * C + c8;
            *reinterpret_cast<float4 *>(dst) = make_float4(v8[0], v8[1], v8[2], v8[3]);
            *reinterpret_cast<float4 *>(dst + 4) = make_float4(v8[4], v8[5], v8[6], v8[7]);
        }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // Y = A Ebar, U = A Z (M = 64, N = 128, K = 64; Ebar and Z used MN-major)
    if (ok && tid == 0) {
        const uint32_t id = idesc_bf16(64, 128, false, true);
        for (int k0 = 0; k0 < 64; k0 += 16)
            mma3(tY, desc_kmajor(tAh, 64, k0), desc_kmajor(tAl, 64, k0), desc_mnmajor(tEh, 64, k0),
                 desc_mnmajor(tEl, 64, k0), id, k0 > 0);
        for (int k0 = 0; k0 < 64; k0 += 16)
            mma3(tU, desc_kmajor(tAh, 64, k0), desc_kmajor(tAl, 64, k0), desc_mnmajor(tZh, 64, k0),
                 desc_mnmajor(tZl, 64, k0), id, k0 > 0);
        mma_commit(&bar2);
    }
    ok = ok && mbar_wait(&bar2, 0);
    fence_after_sync();
    if (ok) {  // tasks 0, 1: Y columns [0,64) / [64,128); tasks 2, 3: U columns
        const int cbase = (task & 1) * 64;
        for (int c0 = cbase; c0 < cbase + 64; c0 += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(task < 2 ? tY : tU, quad, c0), v);
            if (holds_row) {
                const size_t wo = (ch * C + m) * D + c0;
                if (task < 2) {
                    store_split8(ws.Yh + wo, ws.Yl + wo, v);
                    store_split8(ws.Yh + wo + 8, ws.Yl + wo + 8, v + 8);
                } else {
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(ws.U + wo + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// =================================================================================================
// state kernel: one (batch, head) per CTA, serial over chunks
// =================================================================================================
constexpr int kStateThreads = 128;
constexpr size_t kGroupA = 4 * kTileBytes;                 // Yh, Yl, Qh, Ql
constexpr size_t kGroupB = 2 * kTileBytes + 2 * kCCBytes + 1024;  // Kh, Kl, Ah, Al, gamma_C
constexpr size_t kStateSmem = 2 * 32768 + 2 * 16384 + kGroupA + kGroupB + 1024;

struct StateMaps {
    CUtensorMap Yh, Yl, Qh, Ql, Kh, Kl, Ah, Al, gC;
};

__device__ __forceinline__ void load_group_a(const StateMaps &m, uint8_t *g, uint64_t *bar, int row0, bool with_q) {
    const int nt = with_q ? 4 : 2;
    mbar_expect_tx(bar, (uint32_t)nt * (uint32_t)kTileBytes);
    const CUtensorMap *maps[4] = {&m.Yh, &m.Yl, &m.Qh, &m.Ql};
    for (int x = 0; x < nt; ++x) {
        tma_load_2d(g + x * kTileBytes, maps[x], 0, row0, bar);
        tma_load_2d(g + x * kTileBytes + 8192, maps[x], 64, row0, bar);
    }
}

__device__ __forceinline__ void load_group_b(const StateMaps &m, uint8_t *g, uint64_t *bar, int row0, int chunk,
                                             bool with_aqk) {
    mbar_expect_tx(bar, 2u * (uint32_t)kTileBytes + (with_aqk ? 2u * (uint32_t)kCCBytes : 0u) + 512u);
    tma_load_2d(g, &m.Kh, 0, row0, bar);
    tma_load_2d(g + 8192, &m.Kh, 64, row0, bar);
    tma_load_2d(g + kTileBytes, &m.Kl, 0, row0, bar);
    tma_load_2d(g + kTileBytes + 8192, &m.Kl, 64, row0, bar);
    if (with_aqk) {
        tma_load_2d(g + 2 * kTileBytes, &m.Ah, 0, row0, bar);
        tma_load_2d(g + 2 * kTileBytes + kCCBytes, &m.Al, 0, row0, bar);
    }
    tma_load_2d(g + 2 * kTileBytes + 2 * kCCBytes, &m.gC, 0, chunk, bar);
}

__global__ void __launch_bounds__(kStateThreads, 1)
    state_kernel(const __grid_constant__ StateMaps maps, const float *__restrict__ S0, __nv_bfloat16 *o, float *ST,
                 WsTC ws, WsBwd bw, int T, int H, int NT) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tSh = base, *tSl = base + 32768;              // S^T hi / lo  [128 j x 128 i]
    uint8_t *tRh = base + 65536, *tRl = base + 81920;      // R^T hi / lo  [128 j x 64 r]
    uint8_t *gA = base + 98304;                            // Yh, Yl, Qh, Ql   [64 r x 128 i]
    uint8_t *gB = gA + kGroupA;                            // Kh, Kl [64 r x 128 i], Ah, Al [64 x 64], gamma_C
    uint8_t *tYh = gA, *tYl = gA + kTileBytes, *tQh = gA + 2 * kTileBytes, *tQl = gA + 3 * kTileBytes;
    uint8_t *tKh = gB, *tKl = gB + kTileBytes, *tAh = gB + 2 * kTileBytes, *tAl = tAh + kCCBytes;
    const float *gC = reinterpret_cast<const float *>(tAl + kCCBytes);
    __shared__ uint64_t barA, barB, bar_a, bar_b;
    __shared__ uint32_t tslot;

    const int bhi = blockIdx.x, h = bhi % H, bi = bhi / H;
    const size_t bh = (size_t)bhi;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int j = tid;

    if (tid == 0) {
        mbar_init(&barA, 1);
        mbar_init(&barB, 1);
        mbar_init(&bar_a, 1);
        mbar_init(&bar_b, 1);
        mbar_fence_init();
        load_group_a(maps, gA, &barA, (int)(bh * NT) * C, o != nullptr);
        load_group_b(maps, gB, &barB, (int)(bh * NT) * C, (int)(bh * NT), o != nullptr);
    }
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t tS = tmem, tR = tmem + 128, tO = tmem + 192;

    for (int i0 = 0; i0 < D; i0 += 16) {  // S^T row j = column j of S0
        float vs[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) vs[e] = S0 ? S0[(bh * D + i0 + e) * D + j] : 0.f;
        tmem_st16(tmem_lane_addr(tS, warp, i0), vs);
        split_store8(tSh, tSl, 128, j, i0, vs);
        split_store8(tSh, tSl, 128, j, i0 + 8, vs + 8);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    const uint32_t id64 = idesc_bf16(128, 64, false, false);
    const uint32_t id128mn = idesc_bf16(128, 128, false, true);
    bool ok = true;
    for (int c = 0; c < NT; ++c) {
        const size_t ch = bh * NT + c;
        const uint32_t par = (uint32_t)(c & 1);
        const int n = min(C, T - c * C);
        float u[64];  // U^T row j of this chunk, fetched early (fp32)
#pragma unroll
        for (int r = 0; r < 64; ++r) u[r] = ws.U[(ch * C + r) * D + j];
        if (bw.S0T && ok) {  // state entering this chunk, S^T row j (fp32)
            for (int i0 = 0; i0 < D; i0 += 16) {
                float vs[16];
                tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4 *>(bw.S0T + (ch * D + j) * D + i0 + e) =
                        make_float4(vs[e], vs[e + 1], vs[e + 2], vs[e + 3]);
            }
        }

        ok = ok && mbar_wait(&barA, par);
        fence_after_sync();
        if (ok && tid == 0) {  // R_acc = S^T Y^T, O_acc = S^T Q_gamma^T
            for (int k0 = 0; k0 < 128; k0 += 16)
                mma3(tR, desc_kmajor(tSh, 128, k0), desc_kmajor(tSl, 128, k0), desc_kmajor(tYh, 64, k0),
                     desc_kmajor(tYl, 64, k0), id64, k0 > 0);
            if (o)
                for (int k0 = 0; k0 < 128; k0 += 16)
                    mma3(tO, desc_kmajor(tSh, 128, k0), desc_kmajor(tSl, 128, k0), desc_kmajor(tQh, 64, k0),
                         desc_kmajor(tQl, 64, k0), id64, k0 > 0);
            mma_commit(&bar_a);
        }
        ok = ok && mbar_wait(&barB, par);
        if (ok) {  // S^T <- S^T Diag(gamma_C)
            for (int i0 = 0; i0 < D; i0 += 16) {
                float vs[16];
                const uint32_t a = tmem_lane_addr(tS, warp, i0);
                tmem_ld16(a, vs);
#pragma unroll
                for (int e = 0; e < 16; ++e) vs[e] *= gC[i0 + e];
                tmem_st16(a, vs);
            }
        }
        ok = ok && mbar_wait(&bar_a, par);
        fence_after_sync();
        if (ok && tid == 0 && c + 1 < NT) load_group_a(maps, gA, &barA, (int)(ch + 1) * C, o != nullptr);
        if (ok) {  // R^T = U^T - S^T Y^T  (hi / lo into shared memory)
            for (int r0 = 0; r0 < C; r0 += 16) {
                float vr[16];
                tmem_ld16(tmem_lane_addr(tR, warp, r0), vr);
#pragma unroll
                for (int e = 0; e < 16; ++e) vr[e] = u[r0 + e] - vr[e];
                split_store8(tRh, tRl, 128, j, r0, vr);
                split_store8(tRh, tRl, 128, j, r0 + 8, vr + 8);
                if (bw.RT) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(bw.RT + (ch * D + j) * C + r0 + e) =
                            make_float4(vr[e], vr[e + 1], vr[e + 2], vr[e + 3]);
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (ok && tid == 0) {  // O_acc += R^T A_qk^T, S^T += R^T K_tail
            if (o)
                for (int k0 = 0; k0 < 64; k0 += 16)
                    mma3(tO, desc_kmajor(tRh, 128, k0), desc_kmajor(tRl, 128, k0), desc_kmajor(tAh, 64, k0),
                         desc_kmajor(tAl, 64, k0), id64, true);
            for (int k0 = 0; k0 < 64; k0 += 16)
                mma3(tS, desc_kmajor(tRh, 128, k0), desc_kmajor(tRl, 128, k0), desc_mnmajor(tKh, 64, k0),
                     desc_mnmajor(tKl, 64, k0), id128mn, true);
            mma_commit(&bar_b);
        }
        ok = ok && mbar_wait(&bar_b, par);
        fence_after_sync();
        if (ok && tid == 0 && c + 1 < NT)
            load_group_b(maps, gB, &barB, (int)(ch + 1) * C, (int)(ch + 1), o != nullptr);
        if (ok && o) {
            for (int r0 = 0; r0 < C; r0 += 16) {  // O^T row j -> o[:, j]
                float vo[16];
                tmem_ld16(tmem_lane_addr(tO, warp, r0), vo);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (r0 + e < n) o[(((size_t)bi * T + c * C + r0 + e) * H + h) * D + j] = __float2bfloat16_rn(vo[e]);
            }
        }
        if (ok) {
            for (int i0 = 0; i0 < D; i0 += 16) {  // S^T hi / lo for the next chunk
                float vs[16];
                tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
                split_store8(tSh, tSl, 128, j, i0, vs);
                split_store8(tSh, tSl, 128, j, i0 + 8, vs + 8);
            }
        }
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok) != 0;  // every thread leaves the loop together
        fence_after_sync();
        if (!ok) break;
    }
    if (ok && ST) {
        for (int i0 = 0; i0 < D; i0 += 16) {
            float vs[16];
            tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
#pragma unroll
            for (int e = 0; e < 16; ++e) ST[(bh * D + i0 + e) * D + j] = vs[e];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}


// =================================================================================================
// backward: reverse serial pass, one (batch, head) per CTA (transposed, TMEM lane j = value channel)
//     dR^T = dO^T A_qk + dS_C^T K_tail^T
//     dS_0^T = dS_C^T Diag(gamma_C) + dO^T Q_gamma - dR^T Y
// dS_C^T (fp32) and dR^T (fp32) of every chunk go to the workspace; the last dS_0 is dS0.
// =================================================================================================
constexpr size_t kRevLoad = kTileBytes /*dO*/ + 2 * kCCBytes /*A_qk*/ + 2 * kTileBytes /*K_tail*/ +
                            2 * kTileBytes /*Q*/ + 2 * kTileBytes /*Y*/ + 1024 /*gamma_C*/;
constexpr size_t kRevSmem = 2 * 32768 /*dS^T*/ + 2 * 16384 /*-dR^T*/ + kRevLoad + 1024;

struct RevMaps {
    CUtensorMap dO, Ah, Al, Kh, Kl, Qh, Ql, Yh, Yl, gC;
};

__global__ void __launch_bounds__(kStateThreads, 1)
    rev_kernel(const __grid_constant__ RevMaps maps, int has_dO, const float *__restrict__ dST_in, float *dS0,
               WsBwd bw, int T, int H, int NT) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tDh = base, *tDl = base + 32768;            // dS^T hi / lo   [128 j x 128 i]
    uint8_t *tNh = base + 65536, *tNl = base + 81920;    // -dR^T hi / lo  [128 j x 64 r]
    uint8_t *L = base + 98304;
    uint8_t *tdO = L;                                    // dO [64 r x 128 j] (bf16, exact)
    uint8_t *tAh = tdO + kTileBytes, *tAl = tAh + kCCBytes;              // A_qk [64 s x 64 r]
    uint8_t *tKh = tAl + kCCBytes, *tKl = tKh + kTileBytes;              // K_tail [64 r x 128 i]
    uint8_t *tQh = tKl + kTileBytes, *tQl = tQh + kTileBytes;            // Q_gamma [64 r x 128 i]
    uint8_t *tYh = tQl + kTileBytes, *tYl = tYh + kTileBytes;            // Y [64 r x 128 i]
    const float *gC = reinterpret_cast<const float *>(tYl + kTileBytes);
    __shared__ uint64_t full, bar1, bar2;
    __shared__ uint32_t tslot;

    const int bhi = blockIdx.x, h = bhi % H, bi = bhi / H;
    const size_t bh = (size_t)bhi;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int j = tid;

    auto issue = [&](int c) {
        const int row0 = (int)(bh * NT + c) * C;
        uint32_t bytes = 2u * (uint32_t)kCCBytes + 6u * (uint32_t)kTileBytes + 512u;
        if (has_dO) bytes += (uint32_t)kTileBytes;
        mbar_expect_tx(&full, bytes);
        if (has_dO) {
            tma_load_4d(tdO, &maps.dO, 0, h, c * C, bi, &full);
            tma_load_4d(tdO + 8192, &maps.dO, 64, h, c * C, bi, &full);
        }
        tma_load_2d(tAh, &maps.Ah, 0, row0, &full);
        tma_load_2d(tAl, &maps.Al, 0, row0, &full);
        const CUtensorMap *m6[6] = {&maps.Kh, &maps.Kl, &maps.Qh, &maps.Ql, &maps.Yh, &maps.Yl};
        uint8_t *d6[6] = {tKh, tKl, tQh, tQl, tYh, tYl};
        for (int x = 0; x < 6; ++x) {
            tma_load_2d(d6[x], m6[x], 0, row0, &full);
            tma_load_2d(d6[x] + 8192, m6[x], 64, row0, &full);
        }
        tma_load_2d(const_cast<float *>(gC), &maps.gC, 0, (int)(bh * NT + c), &full);
    };

    if (tid == 0) {
        mbar_init(&full, 1);
        mbar_init(&bar1, 1);
        mbar_init(&bar2, 1);
        mbar_fence_init();
    }
    if (!has_dO)
        for (int x = tid; x < (int)(kTileBytes / 16); x += kStateThreads)
            reinterpret_cast<uint4 *>(tdO)[x] = make_uint4(0, 0, 0, 0);
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid == 0) issue(NT - 1);
    const uint32_t tmem = tslot;
    const uint32_t tS = tmem, tR = tmem + 128;

    for (int i0 = 0; i0 < D; i0 += 16) {  // dS^T row j = column j of dS_T
        float vs[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) vs[e] = dST_in ? dST_in[(bh * D + i0 + e) * D + j] : 0.f;
        tmem_st16(tmem_lane_addr(tS, warp, i0), vs);
        split_store8(tDh, tDl, 128, j, i0, vs);
        split_store8(tDh, tDl, 128, j, i0 + 8, vs + 8);
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    const uint32_t id_a = idesc_bf16(128, 64, true, true);      // dO^T (MN) x A_qk (MN)
    const uint32_t id_b = idesc_bf16(128, 64, false, false);    // dS^T (K) x K_tail (K)
    const uint32_t id_c = idesc_bf16(128, 128, true, true);     // dO^T (MN) x Q_gamma (MN)
    const uint32_t id_d = idesc_bf16(128, 128, false, true);    // -dR^T (K) x Y (MN)
    bool ok = true;
    int it = 0;
    for (int c = NT - 1; c >= 0; --c, ++it) {
        const size_t ch = bh * NT + c;
        const uint32_t par = (uint32_t)(it & 1);
        for (int i0 = 0; i0 < D; i0 += 16) {  // dS_C^T row j (fp32) to the workspace
            float vs[16];
            tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<float4 *>(bw.dST + (ch * D + j) * D + i0 + e) =
                    make_float4(vs[e], vs[e + 1], vs[e + 2], vs[e + 3]);
        }
        ok = ok && mbar_wait(&full, par);
        fence_after_sync();
        if (ok && tid == 0) {
            for (int k0 = 0; k0 < 64; k0 += 16) {  // dO^T A_qk (dO exact in bf16: two terms)
                mma_bf16(tR, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tAh, 64, k0), id_a, k0 > 0);
                mma_bf16(tR, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tAl, 64, k0), id_a, true);
            }
            for (int k0 = 0; k0 < 128; k0 += 16)
                mma3(tR, desc_kmajor(tDh, 128, k0), desc_kmajor(tDl, 128, k0), desc_kmajor(tKh, 64, k0),
                     desc_kmajor(tKl, 64, k0), id_b, true);
            mma_commit(&bar1);
        }
        if (ok) {  // dS^T <- dS^T Diag(gamma_C)
            for (int i0 = 0; i0 < D; i0 += 16) {
                float vs[16];
                const uint32_t a = tmem_lane_addr(tS, warp, i0);
                tmem_ld16(a, vs);
#pragma unroll
                for (int e = 0; e < 16; ++e) vs[e] *= gC[i0 + e];
                tmem_st16(a, vs);
            }
        }
        ok = ok && mbar_wait(&bar1, par);
        fence_after_sync();
        if (ok) {  // dR^T row j -> workspace (fp32) and -dR^T (hi / lo) for the next product
            for (int r0 = 0; r0 < C; r0 += 16) {
                float vr[16];
                tmem_ld16(tmem_lane_addr(tR, warp, r0), vr);
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4 *>(bw.dRT + (ch * D + j) * C + r0 + e) =
                        make_float4(vr[e], vr[e + 1], vr[e + 2], vr[e + 3]);
#pragma unroll
                for (int e = 0; e < 16; ++e) vr[e] = -vr[e];
                split_store8(tNh, tNl, 128, j, r0, vr);
                split_store8(tNh, tNl, 128, j, r0 + 8, vr + 8);
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (ok && tid == 0) {
            for (int k0 = 0; k0 < 64; k0 += 16) {  // + dO^T Q_gamma
                mma_bf16(tS, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tQh, 64, k0), id_c, true);
                mma_bf16(tS, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tQl, 64, k0), id_c, true);
            }
            for (int k0 = 0; k0 < 64; k0 += 16)  // - dR^T Y
                mma3(tS, desc_kmajor(tNh, 128, k0), desc_kmajor(tNl, 128, k0), desc_mnmajor(tYh, 64, k0),
                     desc_mnmajor(tYl, 64, k0), id_d, true);
            mma_commit(&bar2);
        }
        ok = ok && mbar_wait(&bar2, par);
        fence_after_sync();
        if (ok && tid == 0 && c > 0) issue(c - 1);
        if (ok) {
            for (int i0 = 0; i0 < D; i0 += 16) {
                float vs[16];
                tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
                split_store8(tDh, tDl, 128, j, i0, vs);
                split_store8(tDh, tDl, 128, j, i0 + 8, vs + 8);
            }
        }
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok) != 0;
        fence_after_sync();
        if (!ok) break;
    }
    if (ok && dS0) {
        for (int i0 = 0; i0 < D; i0 += 16) {
            float vs[16];
            tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
#pragma unroll
            for (int e = 0; e < 16; ++e) dS0[(bh * D + i0 + e) * D + j] = vs[e];
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// =================================================================================================
// backward: batched per-chunk GEMM on tcgen05 with hi / lo operands
//     D[m][n] = alpha * sum_k opA[m][k] opB[n][k]  (+ D[m][n] when accumulate), masked
// Operands are read from global memory in the orientation they are stored in: A is stored [M][K]
// (TA = false, used K-major) or [K][M] (TA = true, used MN-major); likewise B as [N][K] or [K][N].
// A "token" operand is a raw input tensor [B, T, H, 128] addressed by the chunk's tokens of head h
// (rows past T read as zero); other operands are per-chunk fp32 arrays.
// =================================================================================================
struct GOp {
    const void *p;
    int bf16;   // element type: 1 = bf16 (exact: no lo part), 0 = fp32
    int token;  // 1 = raw [B,T,H,128] input, rows = tokens of this chunk
    int ld;     // row stride (elements) for per-chunk arrays
    long long cs;  // per-chunk stride (elements) for per-chunk arrays
};

__device__ __forceinline__ void load8(const GOp &op, int r, int c8, int bi, int h, int c, size_t ch, int T, int H,
                                      float *v) {
    if (op.p == nullptr) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = 0.f;
    } else if (op.token) {
        const int t = c * C + r;
        if (t < T) {
            const __nv_bfloat16 *src = (const __nv_bfloat16 *)op.p + (((size_t)bi * T + t) * H + h) * D + c8;
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src));
            const __nv_bfloat162 *hp = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(hp[e]);
                v[2 * e] = f.x;
                v[2 * e + 1] = f.y;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
    } else {
        const float *src = (const float *)op.p + (size_t)ch * op.cs + (size_t)r * op.ld + c8;
        const float4 a = __ldg(reinterpret_cast<const float4 *>(src)), b = __ldg(reinterpret_cast<const float4 *>(src + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

// Operand -> hi / lo tiles; four 8-element groups per thread in flight at a time.
__device__ __forceinline__ void load_operand(const GOp &op, uint8_t *th, uint8_t *tl, int rows, int cols, int bi,
                                             int h, int c, size_t ch, int T, int H) {
    const int per_row = cols / 8;
    const int total = rows * per_row;
    for (int x0 = threadIdx.x; x0 < total; x0 += 4 * blockDim.x) {
        float v[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int x = x0 + u * blockDim.x;
            if (x < total) load8(op, x / per_row, (x % per_row) * 8, bi, h, c, ch, T, H, v[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int x = x0 + u * blockDim.x;
            if (x < total) split_store8(th, tl, rows, x / per_row, (x % per_row) * 8, v[u]);
        }
    }
}

template <int M, int N, int K, bool TA, bool TB>
__global__ void __launch_bounds__(256, 1) gemm_kernel(GOp A, GOp B, float *Dst, int ldd, float alpha, int accumulate,
                                                      int mask, int T, int H, int NT) {
    constexpr int RA = TA ? K : M, CA = TA ? M : K;
    constexpr int RB = TB ? K : N, CB = TB ? N : K;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tAh = base, *tAl = base + RA * CA * 2;
    uint8_t *tBh = base + 2 * RA * CA * 2, *tBl = tBh + RB * CB * 2;
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t ch = ((size_t)bi * H + h) * NT + c;

    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    load_operand(A, tAh, tAl, RA, CA, bi, h, c, ch, T, H);
    load_operand(B, tBh, tBl, RB, CB, bi, h, c, ch, T, H);
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    if (tid == 0) {
        const uint32_t id = idesc_bf16(M, N, TA, TB);
        for (int k0 = 0; k0 < K; k0 += 16) {
            const uint64_t ah = TA ? desc_mnmajor(tAh, RA, k0) : desc_kmajor(tAh, RA, k0);
            const uint64_t al = TA ? desc_mnmajor(tAl, RA, k0) : desc_kmajor(tAl, RA, k0);
            const uint64_t bh2 = TB ? desc_mnmajor(tBh, RB, k0) : desc_kmajor(tBh, RB, k0);
            const uint64_t bl = TB ? desc_mnmajor(tBl, RB, k0) : desc_kmajor(tBl, RB, k0);
            mma_bf16(tmem, ah, bh2, id, k0 > 0);
            if (!B.bf16) mma_bf16(tmem, ah, bl, id, true);
            if (!A.bf16) mma_bf16(tmem, al, bh2, id, true);
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    fence_after_sync();
    // accumulator row m: lane m (M = 128) or lane 32 * (m / 16) + m % 16 (M = 64); warps w and w + 4 share
    // a lane quadrant and split the columns.
    const int quad = warp & 3, half = warp >> 2;
    const int m = (M == 128) ? (quad * 32 + lane) : (16 * quad + (lane & 15));
    const bool holds = (M == 128) || lane < 16;
    if (ok) {
        float *drow = Dst + ch * (size_t)M * ldd + (size_t)m * ldd;
        for (int n0 = half * (N / 2); n0 < (half + 1) * (N / 2); n0 += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tmem, quad, n0), v);
            if (holds) {
#pragma unroll
                for (int e4 = 0; e4 < 16; e4 += 4) {
                    float4 prev = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (accumulate) prev = *reinterpret_cast<const float4 *>(drow + n0 + e4);
                    float x[4];
                    const float pv[4] = {prev.x, prev.y, prev.z, prev.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int n = n0 + e4 + e;
                        x[e] = alpha * v[e4 + e];
                        if ((mask == 1 && n > m) || (mask == 2 && n >= m)) x[e] = 0.f;
                        x[e] += pv[e];
                    }
                    *reinterpret_cast<float4 *>(drow + n0 + e4) = make_float4(x[0], x[1], x[2], x[3]);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// Two products into one accumulator: D = alpha (opA1 opB1^T + opA2 opB2^T), masked. Same operand
// conventions as gemm_kernel; the second term may have its own K and orientations.
template <int M, int N, int K1, bool TA1, bool TB1, int K2, bool TA2, bool TB2>
__global__ void __launch_bounds__(256, 1) gemm_dual_kernel(GOp A1, GOp B1, GOp A2, GOp B2, float *Dst, int ldd,
                                                           float alpha, int mask, int T, int H, int NT) {
    constexpr int RA1 = TA1 ? K1 : M, CA1 = TA1 ? M : K1, RB1 = TB1 ? K1 : N, CB1 = TB1 ? N : K1;
    constexpr int RA2 = TA2 ? K2 : M, CA2 = TA2 ? M : K2, RB2 = TB2 ? K2 : N, CB2 = TB2 ? N : K2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *a1h = base, *a1l = a1h + RA1 * CA1 * 2;
    uint8_t *b1h = a1l + RA1 * CA1 * 2, *b1l = b1h + RB1 * CB1 * 2;
    uint8_t *a2h = b1l + RB1 * CB1 * 2, *a2l = a2h + RA2 * CA2 * 2;
    uint8_t *b2h = a2l + RA2 * CA2 * 2, *b2l = b2h + RB2 * CB2 * 2;
    __shared__ uint64_t bar;
    __shared__ uint32_t tslot;
    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t ch = ((size_t)bi * H + h) * NT + c;
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    load_operand(A1, a1h, a1l, RA1, CA1, bi, h, c, ch, T, H);
    load_operand(B1, b1h, b1l, RB1, CB1, bi, h, c, ch, T, H);
    load_operand(A2, a2h, a2l, RA2, CA2, bi, h, c, ch, T, H);
    load_operand(B2, b2h, b2l, RB2, CB2, bi, h, c, ch, T, H);
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    if (tid == 0) {
        const uint32_t id1 = idesc_bf16(M, N, TA1, TB1), id2 = idesc_bf16(M, N, TA2, TB2);
        for (int k0 = 0; k0 < K1; k0 += 16) {
            const uint64_t ah = TA1 ? desc_mnmajor(a1h, RA1, k0) : desc_kmajor(a1h, RA1, k0);
            const uint64_t al = TA1 ? desc_mnmajor(a1l, RA1, k0) : desc_kmajor(a1l, RA1, k0);
            const uint64_t bh2 = TB1 ? desc_mnmajor(b1h, RB1, k0) : desc_kmajor(b1h, RB1, k0);
            const uint64_t bl = TB1 ? desc_mnmajor(b1l, RB1, k0) : desc_kmajor(b1l, RB1, k0);
            mma_bf16(tmem, ah, bh2, id1, k0 > 0);
            if (!B1.bf16) mma_bf16(tmem, ah, bl, id1, true);
            if (!A1.bf16) mma_bf16(tmem, al, bh2, id1, true);
        }
        for (int k0 = 0; k0 < K2; k0 += 16) {
            const uint64_t ah = TA2 ? desc_mnmajor(a2h, RA2, k0) : desc_kmajor(a2h, RA2, k0);
            const uint64_t al = TA2 ? desc_mnmajor(a2l, RA2, k0) : desc_kmajor(a2l, RA2, k0);
            const uint64_t bh2 = TB2 ? desc_mnmajor(b2h, RB2, k0) : desc_kmajor(b2h, RB2, k0);
            const uint64_t bl = TB2 ? desc_mnmajor(b2l, RB2, k0) : desc_kmajor(b2l, RB2, k0);
            mma_bf16(tmem, ah, bh2, id2, true);
            if (!B2.bf16) mma_bf16(tmem, ah, bl, id2, true);
            if (!A2.bf16) mma_bf16(tmem, al, bh2, id2, true);
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    fence_after_sync();
    const int quad = warp & 3, half = warp >> 2;
    const int m = (M == 128) ? (quad * 32 + lane) : (16 * quad + (lane & 15));
    const bool holds = (M == 128) || lane < 16;
    if (ok) {
        float *drow = Dst + ch * (size_t)M * ldd + (size_t)m * ldd;
        for (int n0 = half * (N / 2); n0 < (half + 1) * (N / 2); n0 += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tmem, quad, n0), v);
            if (holds) {
#pragma unroll
                for (int e4 = 0; e4 < 16; e4 += 4) {
                    float x[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int n = n0 + e4 + e;
                        x[e] = alpha * v[e4 + e];
                        if ((mask == 1 && n > m) || (mask == 2 && n >= m)) x[e] = 0.f;
                    }
                    *reinterpret_cast<float4 *>(drow + n0 + e4) = make_float4(x[0], x[1], x[2], x[3]);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// dT = -tril(A^T dA A^T, -1) in one kernel: X = A^T dA stays on chip (TMEM -> hi / lo tile) and the
// stored A tile serves both products (MN-major in the first, K-major in the second).
__global__ void __launch_bounds__(128, 1) xdt_kernel(const float *__restrict__ Aw, const float *__restrict__ dAw,
                                                     float *__restrict__ dTw, int H, int NT) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *aH = base, *aL = base + kCCBytes, *dH = base + 2 * kCCBytes, *dL = base + 3 * kCCBytes;
    uint8_t *xH = base + 4 * kCCBytes, *xL = base + 5 * kCCBytes;
    __shared__ uint64_t bar1, bar2;
    __shared__ uint32_t tslot;
    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t ch = ((size_t)bi * H + h) * NT + c;
    if (tid == 0) {
        mbar_init(&bar1, 1);
        mbar_init(&bar2, 1);
        mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&tslot, 128);
    const GOp ga{Aw, 0, 0, C, (long long)C * C}, gd{dAw, 0, 0, C, (long long)C * C};
    load_operand(ga, aH, aL, C, C, bi, h, c, ch, 0, H);
    load_operand(gd, dH, dL, C, C, bi, h, c, ch, 0, H);
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot, tX = tmem, tD = tmem + 64;
    if (tid == 0) {  // X[r][s] = sum_t A[t][r] dA[t][s]
        const uint32_t id = idesc_bf16(64, 64, true, true);
        for (int k0 = 0; k0 < 64; k0 += 16)
            mma3(tX, desc_mnmajor(aH, 64, k0), desc_mnmajor(aL, 64, k0), desc_mnmajor(dH, 64, k0),
                 desc_mnmajor(dL, 64, k0), id, k0 > 0);
        mma_commit(&bar1);
    }
    bool ok = mbar_wait(&bar1, 0);
    fence_after_sync();
    const int m = 16 * warp + (lane & 15);
    const bool holds = lane < 16;
    if (ok) {
        for (int n0 = 0; n0 < 64; n0 += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tX, warp, n0), v);
            if (holds) {
                split_store8(xH, xL, 64, m, n0, v);
                split_store8(xH, xL, 64, m, n0 + 8, v + 8);
            }
        }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (ok && tid == 0) {  // (X A^T)[r][s] = sum_t X[r][t] A[s][t]
        const uint32_t id = idesc_bf16(64, 64, false, false);
        for (int k0 = 0; k0 < 64; k0 += 16)
            mma3(tD, desc_kmajor(xH, 64, k0), desc_kmajor(xL, 64, k0), desc_kmajor(aH, 64, k0),
                 desc_kmajor(aL, 64, k0), id, k0 > 0);
        mma_commit(&bar2);
    }
    ok = ok && mbar_wait(&bar2, 0);
    fence_after_sync();
    if (ok) {
        float *drow = dTw + ch * (size_t)C * C + (size_t)m * C;
        for (int n0 = 0; n0 < 64; n0 += 16) {
            float v[16];
            tmem_ld16(tmem_lane_addr(tD, warp, n0), v);
            if (holds) {
#pragma unroll
                for (int e4 = 0; e4 < 16; e4 += 4) {
                    float x[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) x[e] = (n0 + e4 + e < m) ? -v[e4 + e] : 0.f;
                    *reinterpret_cast<float4 *>(drow + n0 + e4) = make_float4(x[0], x[1], x[2], x[3]);
                }
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

template <int M, int N, int K1, bool TA1, bool TB1, int K2, bool TA2, bool TB2>
cudaError_t run_gemm_dual(const char *name, GOp A1, GOp B1, GOp A2, GOp B2, float *Dst, int ldd, const ChunkArgs &a,
                          int NT, cudaStream_t st) {
    constexpr size_t smem = 2 * 2 * ((size_t)M * K1 + (size_t)N * K1 + (size_t)M * K2 + (size_t)N * K2) + 1024;
    auto kern = gemm_dual_kernel<M, N, K1, TA1, TB1, K2, TA2, TB2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH(name, st, (kern<<<dim3(NT, a.H, a.B), 256, smem, st>>>(A1, B1, A2, B2, Dst, ldd, 1.f, 0, a.T, a.H, NT)));
    return cudaGetLastError();
}

template <int M, int N, int K, bool TA, bool TB>
cudaError_t run_gemm(const char *name, GOp A, GOp B, float *Dst, int ldd, float alpha, int accumulate, int mask,
                     const ChunkArgs &a, int NT, cudaStream_t st) {
    constexpr size_t smem = 2 * (size_t)M * K * 2 + 2 * (size_t)N * K * 2 + 1024;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<M, N, K, TA, TB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH(name, st,
                (gemm_kernel<M, N, K, TA, TB><<<dim3(NT, a.H, a.B), 256, smem, st>>>(A, B, Dst, ldd, alpha,
                                                                                    accumulate, mask, a.T, a.H, NT)));
    return cudaGetLastError();
}

// =================================================================================================
// backward: gradient assembly, one chunk per CTA, thread i = key channel i (and value channel i)
//     dq = dQ_gamma gamma, db = dEbar k gamma, dk = dEbar b gamma + dKbar / gamma + dK_tail gamma_C / gamma
//     dG = dQ_gamma Q_gamma + dEbar Ebar - dKbar Kbar - dK_tail K_tail, plus at the last row
//          sum_r dK_tail K_tail + dgamma_C gamma_C;  dlog_alpha = reverse cumulative sum of dG
//     dw = dZ v, dv = dZ w
// =================================================================================================
// 512 threads: thread (sg, i) owns channel i and rows [16 sg, 16 sg + 16); the reverse cumulative sum
// adds the dG totals of the later row segments (shared memory) to a within-segment suffix sum.
template <typename TOut>
__global__ void __launch_bounds__(512, 2) assemble_kernel(const TOut *__restrict__ k, const TOut *__restrict__ b,
                                                      const TOut *__restrict__ v, const TOut *__restrict__ w,
                                                      const float *__restrict__ la, WsBwd bw, TOut *__restrict__ dq,
                                                      TOut *__restrict__ dk, TOut *__restrict__ db,
                                                      float *__restrict__ dla, TOut *__restrict__ dv,
                                                      TOut *__restrict__ dw, int T, int H, int NT) {
    __shared__ float segG[4][128], segD[4][128], segTail[4][128], segC[4][128];
    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z;
    const int i = threadIdx.x & 127, sg = threadIdx.x >> 7;
    const size_t ch = ((size_t)bi * H + h) * NT + c;
    const int t0 = c * C, r0 = 16 * sg;
    auto tok = [&](int t) { return (((size_t)bi * T + t) * H + h) * D + i; };

    // log-decay: segment-local cumulative sums, then offsets from the earlier segments
    float la_r[16], G[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int t = t0 + r0 + r;
        la_r[r] = (t < T) ? __ldg(la + tok(t)) : 0.f;
    }
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        acc += la_r[r];
        G[r] = acc;
    }
    segG[sg][i] = acc;
    // dgamma_C[i] = sum_j dS_C[i][j] S_0[i][j], j split over the four segments
    {
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int jj = 0; jj < 32; ++jj) {
            const size_t x = (ch * D + 32 * sg + jj) * D + i;
            part[jj & 3] = fmaf(__ldg(bw.dST + x), __ldg(bw.S0T + x), part[jj & 3]);
        }
        segC[sg][i] = (part[0] + part[1]) + (part[2] + part[3]);
    }
    __syncthreads();
    float off = 0.f, GC = 0.f, dgC = 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const float g = segG[x][i];
        if (x < sg) off += g;
        GC += g;
        dgC += segC[x][i];
    }
    const float gC = expf(GC);

    const float *__restrict__ dQg = bw.dQgT + (ch * D + i) * C + r0, *__restrict__ dEb = bw.dEbT + (ch * D + i) * C + r0;
    const float *__restrict__ dKb = bw.dKbT + (ch * D + i) * C + r0, *__restrict__ dKt = bw.dKtT + (ch * D + i) * C + r0;
    const float *__restrict__ dZ = bw.dZT + (ch * D + i) * C + r0;
    float dG[16];
    float tail = 0.f, dsum = 0.f;
#pragma unroll
    for (int r4 = 0; r4 < 16; r4 += 4) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(dQg + r4)), e = __ldg(reinterpret_cast<const float4 *>(dEb + r4));
        const float4 f = __ldg(reinterpret_cast<const float4 *>(dKb + r4)), g4 = __ldg(reinterpret_cast<const float4 *>(dKt + r4));
        const float4 z = __ldg(reinterpret_cast<const float4 *>(dZ + r4));
        const float dqg[4] = {a.x, a.y, a.z, a.w}, deb[4] = {e.x, e.y, e.z, e.w};
        const float dkb[4] = {f.x, f.y, f.z, f.w}, dkt[4] = {g4.x, g4.y, g4.z, g4.w}, dz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = r4 + u;
            const int t = t0 + r0 + r;
            const bool live = t < T;
            const size_t o = live ? tok(t) : 0;
            const float kk = live ? to_f(__ldg(k + o)) : 0.f, bb = live ? to_f(__ldg(b + o)) : 0.f;
            const float g = off + G[r];
            const float gam = expf(g), ginv = expf(-g), gt = expf(GC - g);
            const float qg = __ldg(bw.Qg + (ch * C + r0 + r) * D + i);
            const float kt = kk * gt;
            dG[r] = dqg[u] * qg + deb[u] * (bb * kk * gam) - dkb[u] * (kk * ginv) - dkt[u] * kt;
            dsum += dG[r];
            tail = fmaf(dkt[u], kt, tail);
            if (live) {
                dq[o] = from_f<TOut>(dqg[u] * gam);
                db[o] = from_f<TOut>(deb[u] * kk * gam);
                dk[o] = from_f<TOut>(deb[u] * bb * gam + dkb[u] * ginv + dkt[u] * gt);
                dw[o] = from_f<TOut>(dz[u] * to_f(__ldg(v + o)));
                dv[o] = from_f<TOut>(dz[u] * to_f(__ldg(w + o)));
            }
        }
    }
    segD[sg][i] = dsum;
    segTail[sg][i] = tail;
    __syncthreads();
    // dlog_alpha[r] = (dgamma_C gamma_C + sum_r dK_tail K_tail) + sum_{r' >= r} dG[r']
    float later = dgC * gC;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        later += segTail[x][i];
        if (x > sg) later += segD[x][i];
    }
    float run = later;
#pragma unroll
    for (int r = 15; r >= 0; --r) {
        run += dG[r];
        const int t = t0 + r0 + r;
        if (t < T) dla[tok(t)] = run;
    }
}

// -------------------------------------------------------------------------------------------------
bool ws_map(CUtensorMap *m, const void *p, uint64_t rows, uint64_t cols) {
    uint64_t dims[2] = {cols, rows};
    uint64_t str[1] = {cols * 2};
    uint32_t box[2] = {64, 64};
    return make_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool gc_map(CUtensorMap *m, const void *p, uint64_t nch) {
    uint64_t dims[2] = {(uint64_t)D, nch};
    uint64_t str[1] = {(uint64_t)D * 4};
    uint32_t box[2] = {(uint32_t)D, 1};
    return make_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Raw token tensor [B, T, H, 128] (bf16): boxes of 64 channels x 64 tokens of one head.
bool tok_map(CUtensorMap *m, const void *p, int B, int T, int H) {
    uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)H * D * 2, (uint64_t)T * H * D * 2};
    uint32_t box[4] = {64, 1, 64, 1};
    return make_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool state_maps(StateMaps *m, const WsTC &ws, uint64_t nch) {
    const uint64_t rows = nch * C;
    return ws_map(&m->Yh, ws.Yh, rows, D) && ws_map(&m->Yl, ws.Yl, rows, D) && ws_map(&m->Qh, ws.Qh, rows, D) &&
           ws_map(&m->Ql, ws.Ql, rows, D) && ws_map(&m->Kh, ws.Kh, rows, D) && ws_map(&m->Kl, ws.Kl, rows, D) &&
           ws_map(&m->Ah, ws.Ah, rows, C) && ws_map(&m->Al, ws.Al, rows, C) && gc_map(&m->gC, ws.gC, nch);
}

bool la_map(CUtensorMap *m, const float *p, int B, int T, int H) {
    uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    uint64_t str[3] = {(uint64_t)D * 4, (uint64_t)H * D * 4, (uint64_t)T * H * D * 4};
    uint32_t box[4] = {(uint32_t)D, 1, 64, 1};
    return make_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

cudaError_t run_local(const ChunkArgs &a, const WsTC &ws, const WsBwd &bw, int NT, cudaStream_t st) {
    LocalMaps m;
    if (!tok_map(&m.q, a.q, a.B, a.T, a.H) || !tok_map(&m.k, a.k, a.B, a.T, a.H) ||
        !tok_map(&m.b, a.b, a.B, a.T, a.H) || !tok_map(&m.v, a.v, a.B, a.T, a.H) ||
        !tok_map(&m.w, a.w, a.B, a.T, a.H) || !la_map(&m.la, a.log_alpha, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLocalSmem);
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH(bw.Qg ? "tc_local_train" : "tc_local", st,
                local_kernel<<<dim3(NT, a.H, a.B), kLocalThreads, kLocalSmem, st>>>(m, ws, bw, a.T, a.H, NT));
    return cudaGetLastError();
}

cudaError_t run_state(const ChunkArgs &a, const WsTC &ws, const WsBwd &bw, int NT, bool fwd, cudaStream_t st) {
    StateMaps m;
    if (!state_maps(&m, ws, (uint64_t)a.B * a.H * NT)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH(fwd ? (bw.S0T ? "tc_state_fwd_train" : "tc_state_fwd") : "tc_state_fwd_store", st,
                state_kernel<<<a.B * a.H, kStateThreads, kStateSmem, st>>>(
                    m, a.initial_state, fwd ? (__nv_bfloat16 *)a.o : nullptr, fwd ? a.final_state : nullptr, ws, bw,
                    a.T, a.H, NT));
    return cudaGetLastError();
}

GOp tok_op(const void *p) { return GOp{p, 1, 1, 0, 0}; }
GOp arr_op(const float *p, int ld, long long cs) { return GOp{p, 0, 0, ld, cs}; }

}  // namespace

bool tc_supported(const ChunkArgs &a) { return a.dtype == 1 && a.dk_ == 128 && a.dv_ == 128; }

size_t tc_workspace_bytes(int B, int T, int H, int for_bwd) {
    const size_t NT = (size_t)(T + C - 1) / C;
    return (tc_ws_bytes_per_chunk() + (for_bwd ? tc_bwd_ws_bytes_per_chunk() : 0)) * (size_t)B * H * NT;
}

cudaError_t launch_tc_fwd(const ChunkArgs &a, cudaStream_t st) {
    const int NT = (a.T + C - 1) / C;
    const size_t nch = (size_t)a.B * a.H * NT;
    WsTC ws = carve_tc(a.workspace, nch);
    cudaError_t e = run_local(a, ws, WsBwd{}, NT, st);
    if (e != cudaSuccess) return e;
    return run_state(a, ws, WsBwd{}, NT, true, st);
}

cudaError_t launch_tc_fwd_train(const ChunkArgs &a, cudaStream_t st) {
    const int NT = (a.T + C - 1) / C;
    const size_t nch = (size_t)a.B * a.H * NT;
    WsTC ws = carve_tc(a.workspace, nch);
    WsBwd bw = carve_bwd((uint8_t *)a.workspace + tc_ws_bytes_per_chunk() * nch, nch);
    cudaError_t e;
    if ((e = run_local(a, ws, bw, NT, st)) != cudaSuccess) return e;
    WsBwd store{};
    store.S0T = bw.S0T;
    store.RT = bw.RT;
    return run_state(a, ws, store, NT, true, st);  // o and final state, plus the per-chunk states and R^T
}

cudaError_t launch_tc_bwd(const ChunkArgs &a, cudaStream_t st, bool saved) {
    const int NT = (a.T + C - 1) / C;
    const size_t nch = (size_t)a.B * a.H * NT;
    WsTC ws = carve_tc(a.workspace, nch);
    WsBwd bw = carve_bwd((uint8_t *)a.workspace + tc_ws_bytes_per_chunk() * nch, nch);
    cudaError_t e;
    if (!saved) {
        if ((e = run_local(a, ws, bw, NT, st)) != cudaSuccess) return e;
        WsBwd store{};
        store.S0T = bw.S0T;
        store.RT = bw.RT;
        if ((e = run_state(a, ws, store, NT, false, st)) != cudaSuccess) return e;
    }

    RevMaps rm;
    StateMaps sm;
    if (!state_maps(&sm, ws, nch)) return cudaErrorInvalidValue;
    rm.Ah = sm.Ah; rm.Al = sm.Al; rm.Kh = sm.Kh; rm.Kl = sm.Kl; rm.Qh = sm.Qh; rm.Ql = sm.Ql;
    rm.Yh = sm.Yh; rm.Yl = sm.Yl; rm.gC = sm.gC;
    const int has_dO = a.d_o != nullptr;
    if (has_dO) {
        if (!tok_map(&rm.dO, a.d_o, a.B, a.T, a.H)) return cudaErrorInvalidValue;
    } else {
        rm.dO = sm.Yh;  // never read
    }
    if ((e = cudaFuncSetAttribute(rev_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRevSmem)) !=
        cudaSuccess)
        return e;
    GDR2_LAUNCH("tc_state_rev", st,
                rev_kernel<<<a.B * a.H, kStateThreads, kRevSmem, st>>>(rm, has_dO, a.d_final_state,
                                                                        a.d_initial_state, bw, a.T, a.H, NT));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const GOp dO = tok_op(a.d_o);
    const long long sCD = (long long)C * D, sCC = (long long)C * C, sDD = (long long)D * D, sDC = (long long)D * C;
#define GDR2_TRY(x) \
    if ((e = (x)) != cudaSuccess) return e;
    // dA_qk = tril(dO R)                              [r][s]
    GDR2_TRY((run_gemm<64, 64, 128, false, true>("tc_bwd_dAqk", dO, arr_op(bw.RT, C, sDC), bw.dAqk, C, 1.f, 0, 1, a,
                                                 NT, st)));
    // dQ_gamma^T = S_0 dO^T + Kbar^T dA_qk^T            [i][r]
    GDR2_TRY((run_gemm_dual<128, 64, 128, true, false, 64, true, false>(
        "tc_bwd_dQg", arr_op(bw.S0T, D, sDD), dO, arr_op(bw.Kb, D, sCD), arr_op(bw.dAqk, C, sCC), bw.dQgT, C, a, NT,
        st)));
    // dK_tail^T = dS_C R^T                             [i][r]
    GDR2_TRY((run_gemm<128, 64, 128, true, true>("tc_bwd_dKt", arr_op(bw.dST, D, sDD), arr_op(bw.RT, C, sDC),
                                                 bw.dKtT, C, 1.f, 0, 0, a, NT, st)));
    // dY^T = -S_0 dR^T                                 [i][r]
    GDR2_TRY((run_gemm<128, 64, 128, true, true>("tc_bwd_dY", arr_op(bw.S0T, D, sDD), arr_op(bw.dRT, C, sDC),
                                                 bw.dYT, C, -1.f, 0, 0, a, NT, st)));
    // dZ^T = dR^T A                                    [j][s]
    GDR2_TRY((run_gemm<128, 64, 64, false, true>("tc_bwd_dZ", arr_op(bw.dRT, C, sDC), arr_op(bw.A, C, sCC),
                                                 bw.dZT, C, 1.f, 0, 0, a, NT, st)));
    // dA = dR Z^T + dY Ebar^T  (gate-aware accumulation, Eqs. 64-65)   [r][s]
    GDR2_TRY((run_gemm_dual<64, 64, 128, true, false, 128, true, false>(
        "tc_bwd_dA", arr_op(bw.dRT, C, sDC), arr_op(bw.Z, D, sCD), arr_op(bw.dYT, C, sDC), arr_op(bw.Eb, D, sCD),
        bw.dA, C, a, NT, st)));
    // dT = -tril(A^T dA A^T, -1)
    {
        const size_t smem = 6 * kCCBytes + 1024;
        if ((e = cudaFuncSetAttribute(xdt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        GDR2_LAUNCH("tc_bwd_dT", st,
                    xdt_kernel<<<dim3(NT, a.H, a.B), 128, smem, st>>>(bw.A, bw.dA, bw.dT, a.H, NT));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // dEbar^T = dY^T A + Kbar^T dT^T                    [i][s]
    GDR2_TRY((run_gemm_dual<128, 64, 64, false, true, 64, true, false>(
        "tc_bwd_dEb", arr_op(bw.dYT, C, sDC), arr_op(bw.A, C, sCC), arr_op(bw.Kb, D, sCD), arr_op(bw.dT, C, sCC),
        bw.dEbT, C, a, NT, st)));
    // dKbar^T = Q_gamma^T dA_qk + Ebar^T dT             [i][s]
    GDR2_TRY((run_gemm_dual<128, 64, 64, true, true, 64, true, true>(
        "tc_bwd_dKb", arr_op(bw.Qg, D, sCD), arr_op(bw.dAqk, C, sCC), arr_op(bw.Eb, D, sCD), arr_op(bw.dT, C, sCC),
        bw.dKbT, C, a, NT, st)));
#undef GDR2_TRY
    GDR2_LAUNCH("tc_bwd_assemble", st,
                assemble_kernel<__nv_bfloat16><<<dim3(NT, a.H, a.B), 512, 0, st>>>(
                    (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.b, (const __nv_bfloat16 *)a.v,
                    (const __nv_bfloat16 *)a.w, a.log_alpha, bw, (__nv_bfloat16 *)a.dq, (__nv_bfloat16 *)a.dk,
                    (__nv_bfloat16 *)a.db, a.dlog_alpha, (__nv_bfloat16 *)a.dv, (__nv_bfloat16 *)a.dw, a.T, a.H, NT));
    return cudaGetLastError();
}

}  // namespace gdr2
