// chunk_tc.cu -- tensor-core (tcgen05 + TMEM + TMA) chunkwise Gated Delta Rule-2 for bf16 operands,
// dk = dv = 128, C = 64, fp32 state: forward, backward, and the training pair.
//
// The algorithm is the chunkwise WY form of the review's section "Chunkwise Parallel Training via WY
// Representation" (Steps 1-3, Eqs. 20-24; the T factor of Appendix C.2) and, for the backward, the
// chain rule through Eqs. 23-24 with the gate-aware WY terms of section "Gate-Aware Backward Pass"
// (Eqs. 64-65, dT = -tril(A^T dA A^T, -1), gate gradients, in-chunk reverse cumulative sum of the
// log-decay gradient).
//
// Forward:
//  local  persistent: min(chunks, SMs) CTAs of 512 threads, each walking chunks by a global index (one
//         chunk at a time). TMA brings q, k, b, v, w and the log-decay.
//         Step 1 in fp32 (segmented cumulative sum G, gamma = exp(G)): Q_gamma, Kbar, Ebar, K_tail, Z.
//         tcgen05 (M = 64): T = Ebar Kbar^T, A_qk = Q_gamma Kbar^T; blocked fp32 WY inverse
//         A = (I + T)^-1; Y = A Ebar, U = A Z.
//  state  grid (B*H), 128 threads, one CTA per (batch, head): the serial pass of Eq. 23 with the state
//         transposed, S^T [dv x dk] fp32 in TMEM (lane j = value channel), so all products have
//         M = dv = 128:  R^T = U^T - S^T Y^T,  O^T = S^T Q_gamma^T + R^T A_qk^T,
//         S^T <- S^T Diag(gamma_C) + R^T K_tail.
// Backward (after a forward that kept the per-chunk intermediates):
//  rev    grid (B*H), 128 threads: reverse serial pass, dR^T = dO^T A_qk + dS_C^T K_tail^T and
//         dS_0^T = dS_C^T Diag(gamma_C) + dO^T Q_gamma - dR^T Y.
//  chunk  persistent: min(chunks, SMs) CTAs of 512 threads, one chunk at a time by a global index:
//         every per-chunk product of the backward and the gradient assembly in one kernel,
//         intermediates in shared memory and TMEM.
//
// These are the chunk-parallel kernels. gdr2_set_chunk_path(2) forces them; automatic selection takes
// them for calls whose (batch, head) chain count leaves the per-chain kernels' last wave of SMs mostly
// empty (fewer than about 91 chains, 149 to 180, ...; the chunk-level scan can then split long chains) and for
// every packed-batch and grouped-value-head call; other bf16, dk = dv = 128 calls go to the per-chain kernels
// of chain_tc.cu.
//
// Precision: every operand derived from the inputs carries decay factors; rounding each to bf16
// (~2^-9, about ten times along the chunk algebra) exceeds the target error bound. So each derived
// operand is a pair hi = bf16(x), lo = bf16(x - hi), and products are Ah Bh + Ah Bl + Al Bh on the bf16
// tensor pipe with fp32 accumulation (~16 significant bits). Operands exact in bf16 (the raw dO) skip
// their lo term.
//
// Workspace format: every tensor that a later kernel uses as an MMA operand is stored as a "tile
// image": the shared-memory bytes of its hi tile followed by its lo tile (128-byte swizzle, the stored
// matrix's rows as tile rows). Producers write images from shared memory with bulk stores or from TMEM
// rows with 16-byte stores; consumers bring each image in with one bulk copy.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tma_host.h"

namespace gdr2 {
namespace {

using namespace tc;

constexpr int C = kChunk;
constexpr int D = 128;

// Tile image sizes (hi + lo), bytes.
constexpr size_t kImg64x128 = 2 * 64 * 128 * 2;    // 32 KB
constexpr size_t kImg64x64 = 2 * 64 * 64 * 2;      // 16 KB
constexpr size_t kImg128x128 = 2 * 128 * 128 * 2;  // 64 KB
constexpr size_t kImg128x64 = 2 * 128 * 64 * 2;    // 32 KB

// Forward workspace, per chunk (ch = (b*H + h)*NT + c). With grouped value heads the key-side entries (Y,
// Q_gamma, K_tail, A_qk, gamma_C, and A below) are per key-head chunk, the rest per value-head chunk.
struct WsTC {
    uint8_t *Y;           // image  [128 i][64 r]: -Y^T
    uint8_t *Q, *Kt;      // images [64 r][128]: Q_gamma, K_tail
    uint8_t *Aqk;         // image  [64 r][64 s]: tril(A_qk)
    float *U;             // fp32   [128 j][64 r]: U^T, 16-byte chunks of row j at position chunk ^ (j % 16)
    float *gC;            // fp32   [128]
    // chunk-level scan (only with more than one segment per chain; fp32 states [D][D] per (segment, chain)):
    float *scanA;         // [2][nseg][B H]: end states from 0 (offsets N, kind 0) and from I without U (M, kind 1)
    float *scanS;         // [nseg][B H]: state entering each segment
};

// Additional workspace kept for the backward, per chunk.
struct WsBwd {
    uint8_t *A;           // image [64 r][64 s]  (I + T)^-1
    uint8_t *S0T, *dST;   // images [128 j][128 i]: state entering the chunk, gradient at its end
    uint8_t *RT, *dRT;    // images [128 j][64 r]
    float *scanN;         // [nseg][B H]: gradient leaving each segment's first chunk when started from 0
    float *scanE;         // [nseg][B H]: gradient entering each segment's last chunk
};

constexpr size_t kFwdKeyPerChunk = 3 * kImg64x128 + kImg64x64 + D * 4;  // Y, Q_gamma, K_tail, A_qk, gamma_C
constexpr size_t kFwdValPerChunk = (size_t)C * D * 4;                    // U
constexpr size_t kBwdKeyPerChunk = kImg64x64;                            // A
constexpr size_t kBwdValPerChunk = 2 * kImg128x128 + 2 * kImg128x64;      // S_0, dS_C, R, dR
constexpr size_t kStateBytes = (size_t)D * D * 4;

// Segments of the chunk-level scan for BH chains of NT chunks (1: the plain serial pass). The rule minimises a
// model of the serial time of the forward and reverse passes: per chunk step about 4.4 us for a phase-A CTA
// (no output), 7.5 us for the forward's output pass and 5.2 us for the reverse's image pass (measured on
// B200 at one CTA per SM), in waves of 148 CTAs, plus 15 + 0.27 BH us per combine step in each direction
// (one 8-CTA cluster per chain: measured about 15 us per step at 16 chains and 31 us at 48 and 64). The
// count depends on the sizes only, so the workspace query and the launches agree on any device.
int scan_segments(int BH, int NT) {
    auto waves = [](long long ctas) { return (double)((ctas + 147) / 148); };
    double best_cost = waves(BH) * NT * (7.5 + 5.2);
    int best = 1;
    for (int n = 2; n <= 64 && n <= NT / 4; ++n) {
        const int L = (NT + n - 1) / n, neff = (NT + L - 1) / L;
        const double cost = waves(2LL * BH * neff) * L * 4.4 + waves((long long)BH * neff) * L * (7.5 + 4.3 + 5.2) +
                            2.0 * (15.0 + 0.27 * BH) * (neff - 1);
        if (cost < best_cost) {
            best_cost = cost;
            best = neff;
        }
    }
    return best;
}
size_t scan_fwd_bytes(int BH, int nseg) { return nseg > 1 ? 3 * (size_t)nseg * BH * kStateBytes : 0; }
size_t scan_bwd_bytes(int BH, int nseg) { return nseg > 1 ? 2 * (size_t)nseg * BH * kStateBytes : 0; }

WsTC carve_tc(void *base, size_t nchK, size_t nchV, int BH, int nseg) {
    uint8_t *p = (uint8_t *)base;
    auto take = [&](size_t per, size_t n) { uint8_t *r = p; p += per * n; return r; };
    WsTC w{};
    w.Y = take(kImg64x128, nchK);
    w.Q = take(kImg64x128, nchK);
    w.Kt = take(kImg64x128, nchK);
    w.Aqk = take(kImg64x64, nchK);
    w.U = (float *)take((size_t)C * D * 4, nchV);
    w.gC = (float *)take(D * 4, nchK);
    if (nseg > 1) {
        w.scanA = (float *)p;
        w.scanS = w.scanA + 2 * (size_t)nseg * BH * D * D;
    }
    return w;
}

WsBwd carve_bwd(void *base, size_t nchK, size_t nchV, int BH, int nseg) {
    uint8_t *p = (uint8_t *)base;
    auto take = [&](size_t per, size_t n) { uint8_t *r = p; p += per * n; return r; };
    WsBwd w{};
    w.A = take(kImg64x64, nchK);
    w.S0T = take(kImg128x128, nchV);
    w.dST = take(kImg128x128, nchV);
    w.RT = take(kImg128x64, nchV);
    w.dRT = take(kImg128x64, nchV);
    if (nseg > 1) {
        w.scanN = (float *)p;
        w.scanE = w.scanN + (size_t)nseg * BH * D * D;
    }
    return w;
}

// Packed variable-length batches (cu_seqlens): the token axis holds N sequences back to back; every
// sequence starts its own chunks and its own state. Chunk g of the packed axis and sequence n are
// described by two device tables built on the stream from cu_seqlens (varlen_index_kernel). Rows of a
// chunk past its sequence's end are treated as zero inputs (identity transitions), exactly like the
// rows past T of an unpacked batch. The outputs of a chunk that ends inside the packed axis cannot be
// clipped by a tensor store, so such chunks write a staging tile that varlen_fixup_kernel copies.
struct Varlen {
    const int4 *chunk;  // [G] x token start, y valid rows (0..64), z staging slot (-1: stored in place), w sequence
    const int4 *seq;    // [N] x first chunk, y chunk count, z first token, w length
    const int *order;   // [N] sequences by falling chunk count: the serial passes start the longest first
    int nslot;          // staging slots: N + 1 (slot N takes the empty chunk slots past the last sequence)
};

__device__ __forceinline__ int4 chunk_info(const Varlen &vl, int c) {
    return vl.chunk ? __ldg(vl.chunk + c) : make_int4(c * C, C, -1, 0);
}

// The same for kernels instantiated per layout: the unpacked instantiation has no row masks at all.
template <bool kPacked>
__device__ __forceinline__ int4 chunk_info_t(const Varlen &vl, int c) {
    if constexpr (kPacked) return __ldg(vl.chunk + c);
    else return make_int4(c * C, C, -1, 0);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 8 consecutive fp32 values of row r (column c, a multiple of 8) into a global tile image with R rows and
// `cols` columns: the hi chunk into the hi tile, the lo chunk into the lo tile (two 16-byte stores).
__device__ __forceinline__ void img_store8(uint8_t *img, int R, int cols, int r, int c, const float *v) {
    __nv_bfloat16 h[8], l[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        h[e] = __float2bfloat16_rn(v[e]);
        l[e] = __float2bfloat16_rn(v[e] - __bfloat162float(h[e]));
    }
    const uint32_t off = rt_off(R, r, c);
    *reinterpret_cast<uint4 *>(img + off) = *reinterpret_cast<const uint4 *>(h);
    *reinterpret_cast<uint4 *>(img + (size_t)R * cols * 2 + off) = *reinterpret_cast<const uint4 *>(l);
}

// =================================================================================================
// local kernel: one chunk per CTA
// =================================================================================================
constexpr int kLocalThreads = 512;
constexpr int kTsmStride = 68;                    // fp32 row stride of T and A in shared memory
constexpr size_t kLocTile = 16384;                // one 64 x 128 bf16 tile
constexpr size_t kSqBytes = 64 * kTsmStride * 4;  // 17408
constexpr size_t kLocalSmem = 10 * kLocTile + 2 * 8192 + 2 * kSqBytes + 1024 * 4 + 1024;

struct LocalMaps {
    CUtensorMap q, k, b, v, w, la;
};

// A = (I + T)^-1 for a strictly lower triangular 64 x 64 T (fp32, row stride kTsmStride) by recursive
// doubling of the block inverse [[A0, 0], [-A1 T10 A0, A1]]: the four 16 x 16 diagonal blocks by forward
// substitution (one column per thread), then the 16 x 16 off-diagonal block of each 32 x 32 half, then the
// 32 x 32 off-diagonal block. Every product is a fixed-length dot product over all 512 threads; the zeros
// above the diagonal of A are part of the sums. W holds 1024 fp32.
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
    {  // 32 x 32 halves p = 0, 1: W_p = T[2p+1][2p] A[2p][2p] (16 x 16 blocks)
        const int p = tid >> 8, r = (tid >> 4) & 15, c = tid & 15;
        const float *Tr = Tm + (32 * p + 16 + r) * kTsmStride + 32 * p;
        const float *Ac = Am + (32 * p) * kTsmStride + 32 * p + c;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s = fmaf(Tr[k], Ac[k * kTsmStride], s);
        W[tid] = s;
    }
    __syncthreads();
    {  // A[2p+1][2p] = -A[2p+1][2p+1] W_p
        const int p = tid >> 8, r = (tid >> 4) & 15, c = tid & 15;
        const float *Ar = Am + (32 * p + 16 + r) * kTsmStride + 32 * p + 16;
        const float *Wc = W + (p << 8) + c;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s = fmaf(Ar[k], Wc[16 * k], s);
        Am[(32 * p + 16 + r) * kTsmStride + 32 * p + c] = -s;
    }
    __syncthreads();
    // 32 x 32 level: threads 0..255 each form a 2 x 2 block, rows (r, r + 16) x columns (cq, cq + 1), from
    // float4 row loads and float2 column loads (four independent FMA chains).
    const int r32 = (tid >> 4) & 15, cq = (tid & 15) * 2;
    if (tid < 256) {  // W = T[1][0] A[0][0]
        const float4 *T0 = reinterpret_cast<const float4 *>(Tm + (32 + r32) * kTsmStride);
        const float4 *T1 = reinterpret_cast<const float4 *>(Tm + (48 + r32) * kTsmStride);
        float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            const float4 t0 = T0[k4], t1 = T1[k4];
            const float a0[4] = {t0.x, t0.y, t0.z, t0.w}, a1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 a = *reinterpret_cast<const float2 *>(Am + (4 * k4 + u) * kTsmStride + cq);
                s00 = fmaf(a0[u], a.x, s00);
                s01 = fmaf(a0[u], a.y, s01);
                s10 = fmaf(a1[u], a.x, s10);
                s11 = fmaf(a1[u], a.y, s11);
            }
        }
        *reinterpret_cast<float2 *>(W + r32 * 32 + cq) = make_float2(s00, s01);
        *reinterpret_cast<float2 *>(W + (r32 + 16) * 32 + cq) = make_float2(s10, s11);
    }
    __syncthreads();
    if (tid < 256) {  // A[1][0] = -A[1][1] W
        const float4 *A0 = reinterpret_cast<const float4 *>(Am + (32 + r32) * kTsmStride + 32);
        const float4 *A1 = reinterpret_cast<const float4 *>(Am + (48 + r32) * kTsmStride + 32);
        float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            const float4 t0 = A0[k4], t1 = A1[k4];
            const float a0[4] = {t0.x, t0.y, t0.z, t0.w}, a1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 w2 = *reinterpret_cast<const float2 *>(W + (4 * k4 + u) * 32 + cq);
                s00 = fmaf(a0[u], w2.x, s00);
                s01 = fmaf(a0[u], w2.y, s01);
                s10 = fmaf(a1[u], w2.x, s10);
                s11 = fmaf(a1[u], w2.y, s11);
            }
        }
        *reinterpret_cast<float2 *>(Am + (32 + r32) * kTsmStride + cq) = make_float2(-s00, -s01);
        *reinterpret_cast<float2 *>(Am + (48 + r32) * kTsmStride + cq) = make_float2(-s10, -s11);
    }
    __syncthreads();
}

// Persistent: one CTA per SM walks the chunks blockIdx.x, blockIdx.x + gridDim.x, ... The inputs of the
// next chunk are requested as soon as the current chunk's last products have read their tiles, so the
// loads overlap the output phase; TMEM and the barriers are set up once.
// Grouped value heads (G > 1, Hv = G H value heads): a CTA takes a key-head chunk; the key side (Q_gamma,
// K_tail, A_qk, A, Y) is formed once, and U = A Z for each of the group's value heads, one after another.
template <bool kPacked>
__global__ void __launch_bounds__(kLocalThreads, 1)
    local_kernel(const __grid_constant__ LocalMaps maps, Varlen vl, WsTC ws, WsBwd bw, int T, int H, int NG, int NT,
                 int nchunks) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tQh = base, *tQl = base + kLocTile;                     // Q_gamma   (raw q arrives in tQl)
    uint8_t *tKh = base + 2 * kLocTile, *tKl = base + 3 * kLocTile;  // Kbar      (raw k arrives in tKl)
    uint8_t *tEh = base + 4 * kLocTile, *tEl = base + 5 * kLocTile;  // Ebar      (raw b arrives in tEl)
    uint8_t *tZh = base + 6 * kLocTile, *tZl = base + 7 * kLocTile;  // Z         (raw w in tZh, v in tZl)
    uint8_t *tTh = base + 8 * kLocTile, *tTl = base + 9 * kLocTile;  // K_tail
    uint8_t *tAh = base + 10 * kLocTile, *tAl = tAh + 8192;          // A = (I + T)^-1
    float *Tsm = reinterpret_cast<float *>(tAl + 8192);              // [64][kTsmStride]
    float *Asm = Tsm + 64 * kTsmStride;                              // [64][kTsmStride]
    float *Wsm = Asm + 64 * kTsmStride;                              // [1024] WY scratch
    float *la_s = Tsm;  // raw log-decay [64][128] fp32, consumed before T is written
    // outputs staged after the last products: -Y^T hi / lo in tQh / tKh, U^T rows 0..63 / 64..127 in tEh / tTh
    __shared__ uint64_t bar_in, bar1, bar2, bar_g, bar_x;
    __shared__ uint32_t tslot;
    __shared__ float seg_sum[4][128];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = tid & 127;  // channel
    const int sg = tid >> 7;  // row segment: rows [16 sg, 16 sg + 16)
    const bool keep = bw.A != nullptr;

    // Inputs of chunk chn: part 0 arms the barrier and loads k, b, w, v and the log-decay; part 1 loads q,
    // whose slot is the lo tile of the Q_gamma image and so frees up last.
    auto issue_inputs = [&](int chn, int part) {
        const int c = chn % NT, h = (chn / NT) % H, bi = chn / (NT * H);
        const int t0 = chunk_info_t<kPacked>(vl, c).x;
        if (part == 0) {
            mbar_expect_tx(&bar_in, 5u * (uint32_t)kLocTile + 64u * 128u * 4u);
            const CUtensorMap *mp[4] = {&maps.k, &maps.b, &maps.w, &maps.v};
            uint8_t *dst[4] = {tKl, tEl, tZh, tZl};
            for (int x = 0; x < 4; ++x) {  // w and v: the group's first value head
                const int hx = x < 2 ? h : h * NG;
                tma_load_4d(dst[x], mp[x], 0, hx, t0, bi, &bar_in);
                tma_load_4d(dst[x] + 8192, mp[x], 64, hx, t0, bi, &bar_in);
            }
            tma_load_4d(la_s, &maps.la, 0, h, t0, bi, &bar_in);
        } else {
            tma_load_4d(tQl, &maps.q, 0, h, t0, bi, &bar_in);
            tma_load_4d(tQl + 8192, &maps.q, 64, h, t0, bi, &bar_in);
        }
    };

    if (tid == 0) {
        mbar_init(&bar_in, 1);
        mbar_init(&bar1, 1);
        mbar_init(&bar2, 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_x, 1);
        mbar_fence_init();
        if ((int)blockIdx.x < nchunks) {
            issue_inputs(blockIdx.x, 0);
            issue_inputs(blockIdx.x, 1);
        }
    }
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t tT = tmem, tAqk = tmem + 64, tYT = tmem, tUT = tmem + 64;
    const int quad = warp & 3, task = warp >> 2;

    bool ok = true;
    int it = 0;
    uint32_t gph = 0;          // phase of bar_g (value-head loop of grouped heads)
    const bool late = NG > 1;   // grouped heads: the next chunk's inputs follow the value-head loop
    for (int chn = (int)blockIdx.x; chn < nchunks; chn += (int)gridDim.x, ++it) {
        const uint32_t par = (uint32_t)(it & 1);
        const size_t ch = (size_t)chn;  // = (bi * H + h) * NT + c
        // U of value head h G + r of this chunk: entry ((bi H + h) G + r) NT + c
        const size_t chv0 = ((size_t)(chn / NT) * NG) * NT + chn % NT;
        const int len = chunk_info_t<kPacked>(vl, chn % NT).y;  // rows from len on are zero inputs (packed)
        GDR2_DCHECK(chn >= 0 && chn < nchunks && len >= 0 && len <= 64 &&
                    chunk_info_t<kPacked>(vl, chn % NT).x >= 0 && chunk_info_t<kPacked>(vl, chn % NT).x < T);
        ok = ok && mbar_wait(&bar_in, par);
        // Step 1: cumulative log-decay of channel i (fp32): 16-row segment sums, then segment offsets.
        float G[16];
        {
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                acc += (16 * sg + r < len) ? la_s[(16 * sg + r) * D + i] : 0.f;
                G[r] = acc;
            }
            seg_sum[sg][i] = acc;
        }
        if (tid == 0) bulk_wait_read<0>();  // the previous chunk's output stores have read their tiles
        __syncthreads();
        float off = 0.f, GC = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float v = seg_sum[x][i];
            if (x < sg) off += v;
            GC += v;
        }
        if (sg == 0) {
            ws.gC[ch * D + i] = expf(GC);
            if (!(fabsf(GC) <= kMaxChunkLogDecayTC)) flag_status(kStatusRange);  // (NaN included)
        }
        // Lanes 2p and 2p + 1 (channels ie, ie + 1) split the pair's 16 rows: the even lane takes rows 0..7 of
        // the segment, the odd lane rows 8..15, each for both channels (4-byte shared-memory accesses).
        const int odd = lane & 1, ie = i & ~1;
        float gme[16], gpa[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            gme[rr] = off + G[rr];
            gpa[rr] = __shfl_xor_sync(0xffffffffu, gme[rr], 1);
        }
        const float GCpa = __shfl_xor_sync(0xffffffffu, GC, 1);
        const float GC0 = odd ? GCpa : GC, GC1 = odd ? GC : GCpa;  // chunk log-decay of channels ie, ie + 1
        // The factors of the T and A_qk products are taken relative to the channel's mid-chunk log-decay
        // m = G_C / 2: Q' = q e^{G - m}, K' = k e^{m - G}, E' = b k e^{G - m}. Their products equal those of
        // Q_gamma = q e^{G}, Kbar = k e^{-G}, Ebar = b k e^{G}, but no factor exceeds e^{|G_C| / 2}, so a
        // chunk may decay by up to e^{-160} instead of e^{-80}. Y = A Ebar is A E' scaled by e^{m} at its
        // read-out, and the Q_gamma image is written absolute, straight from registers.
        const float m0 = 0.5f * GC0, m1 = 0.5f * GC1;
        const float em0 = __expf(m0), em1 = __expf(m1);  // e^{m} = e^{G_C / 2} of channels ie, ie + 1
        uint8_t *const qimg = ws.Q + ch * kImg64x128;
        if (ok) {
#pragma unroll
            for (int r8 = 0; r8 < 8; ++r8) {
                const int r = 16 * sg + 8 * odd + r8;
                const float a_lo = gme[r8], a_hi = gme[r8 + 8], b_lo = gpa[r8], b_hi = gpa[r8 + 8];
                const float gm = odd ? a_hi : a_lo, gp = odd ? b_hi : b_lo;  // own / partner channel, row r
                const float g0 = odd ? gp : gm, g1 = odd ? gm : gp;          // channel ie / ie + 1
                float2 kk = pair_get(tKl, 64, r, ie), bb = pair_get(tEl, 64, r, ie), qq = pair_get(tQl, 64, r, ie);
                float2 vv = pair_get(tZl, 64, r, ie), wv = pair_get(tZh, 64, r, ie);
                if (r >= len) kk = bb = qq = vv = wv = make_float2(0.f, 0.f);
                // gamma = e^{G - m} e^{m} (it may underflow: an absolute factor <= 1) and gamma_C / gamma =
                // e^{m} e^{m - G} <= 1, from the two relative factors
                const float t0 = g0 - m0, t1 = g1 - m1;
                const float ep0 = __expf(t0), en0 = __expf(-t0), gam0 = ep0 * em0, gt0 = em0 * en0;
                const float ep1 = __expf(t1), en1 = __expf(-t1), gam1 = ep1 * em1, gt1 = em1 * en1;
                pair_split_put(qimg, qimg + kImg64x128 / 2, 64, r, ie, qq.x * gam0, qq.y * gam1);  // the image
                pair_split_put(tQh, tQl, 64, r, ie, qq.x * ep0, qq.y * ep1);
                pair_split_put(tKh, tKl, 64, r, ie, kk.x * en0, kk.y * en1);
                pair_split_put(tEh, tEl, 64, r, ie, bb.x * kk.x * ep0, bb.y * kk.y * ep1);
                pair_split_put(tZh, tZl, 64, r, ie, wv.x * vv.x, wv.y * vv.y);
                pair_split_put(tTh, tTl, 64, r, ie, kk.x * gt0, kk.y * gt1);
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (ok && tid == 0) {
            bulk_store(ws.Kt + ch * kImg64x128, tTh, (uint32_t)kImg64x128);  // the K_tail image
            bulk_commit();
            // T = E' K'^T = Ebar Kbar^T, A_qk = Q' K'^T = Q_gamma Kbar^T (M = 64, N = 64, K = 128)
            const uint32_t id = idesc_bf16(64, 64, false, false);
            for (int k0 = 0; k0 < 128; k0 += 16)
                mma3(tT, desc_kmajor(tEh, 64, k0), desc_kmajor(tEl, 64, k0), desc_kmajor(tKh, 64, k0),
                     desc_kmajor(tKl, 64, k0), id, k0 > 0);
            for (int k0 = 0; k0 < 128; k0 += 16)
                mma3(tAqk, desc_kmajor(tQh, 64, k0), desc_kmajor(tQl, 64, k0), desc_kmajor(tKh, 64, k0),
                     desc_kmajor(tKl, 64, k0), id, k0 > 0);
            mma_commit(&bar1);
        }
        ok = ok && mbar_wait(&bar1, par);
        fence_after_sync();
        // M = 64 accumulator layout: row m sits in TMEM lane 32 * (m / 16) + m % 16. Warp w reads lane
        // quadrant w % 4; its task (w / 4) picks 32 columns of T (tasks 0, 1) or of A_qk (tasks 2, 3).
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
                        img_store8(ws.Aqk + ch * kImg64x64, 64, 64, m, c0, v);
                        img_store8(ws.Aqk + ch * kImg64x64, 64, 64, m, c0 + 8, v + 8);
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
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();

        // Y^T = Ebar^T A^T, U^T = Z^T A^T (M = 128 channels on the TMEM lanes, N = 64 tokens, K = 64;
        // Ebar and Z used MN-major, A K-major)
        if (ok && tid == 0) {
            if (keep) {
                bulk_store(bw.A + ch * kImg64x64, tAh, (uint32_t)kImg64x64);
                bulk_commit();
            }
            const uint32_t id = idesc_bf16(128, 64, true, false);
            for (int k0 = 0; k0 < 64; k0 += 16)
                mma3(tYT, desc_mnmajor(tEh, 64, k0), desc_mnmajor(tEl, 64, k0), desc_kmajor(tAh, 64, k0),
                     desc_kmajor(tAl, 64, k0), id, k0 > 0);
            for (int k0 = 0; k0 < 64; k0 += 16)
                mma3(tUT, desc_mnmajor(tZh, 64, k0), desc_mnmajor(tZl, 64, k0), desc_kmajor(tAh, 64, k0),
                     desc_kmajor(tAl, 64, k0), id, k0 > 0);
            mma_commit(&bar2);
        }
        ok = ok && mbar_wait(&bar2, par);
        fence_after_sync();
        if (tid == 0) {  // the products have released every input slot but q's (the Q_gamma image's lo tile)
            const bool more = ok && !late && chn + (int)gridDim.x < nchunks;
            if (more) issue_inputs(chn + (int)gridDim.x, 0);
            if (keep && !late)
                bulk_wait_read<1>();  // Q_gamma / K_tail images read; the A image may still be in flight
            else
                bulk_wait_read<0>();
            if (more) issue_inputs(chn + (int)gridDim.x, 1);
        }
        __syncthreads();
        if (ok) {  // lane = channel i; tasks 0, 1: Y^T columns [0,32) / [32,64); tasks 2, 3: U^T columns
            const int ich = 32 * quad + lane;  // = i, the channel whose G_C this thread holds
            const int cbase = (task & 1) * 32;
            const float ym = -__expf(0.5f * GC);  // Y = (A E') e^{m}; the image holds -Y^T
            for (int c0 = cbase; c0 < cbase + 32; c0 += 16) {
                float v[16];
                tmem_ld16(tmem_lane_addr(task < 2 ? tYT : tUT, quad, c0), v);
                if (task < 2) {  // the image holds -Y^T, so the serial passes only ever accumulate
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] *= ym;
                    split_store8(tQh, tKh, 128, ich, c0, v);
                    split_store8(tQh, tKh, 128, ich, c0 + 8, v + 8);
                } else {  // U^T row ich, 16-byte chunks swizzled by (row % 16)
                    uint8_t *row = (ich < 64 ? tEh : tTh) + (ich & 63) * 256;
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const int cidx = (c0 >> 2) + e4;
                        *reinterpret_cast<float4 *>(row + ((cidx ^ (ich & 15)) << 4)) =
                            make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
                    }
                }
            }
        }
        fence_async_smem();
        fence_before_sync();
        ok = __syncthreads_and(ok) != 0;
        fence_after_sync();
        if (ok && tid == 0) {
            uint8_t *y = ws.Y + ch * kImg128x64, *u = reinterpret_cast<uint8_t *>(ws.U + chv0 * D * C);
            bulk_store(y, tQh, 16384u);
            bulk_store(y + 16384, tKh, 16384u);
            bulk_store(u, tEh, 16384u);
            bulk_store(u + 16384, tTh, 16384u);
            bulk_commit();
        }
        if (late) {
            // The group's other value heads: raw w, v into the Z tiles, Z = w (.) v split in place, U^T = Z^T A^T,
            // staged in the U tiles once their previous store has read them.
            const int c = chn % NT, h = (chn / NT) % H, bi = chn / (NT * H);
            const int t0 = chunk_info_t<kPacked>(vl, c).x;
            for (int r = 1; r < NG && ok; ++r) {
                if (tid == 0) {
                    mbar_expect_tx(&bar_g, 2u * (uint32_t)kLocTile);
                    tma_load_4d(tZh, &maps.w, 0, h * NG + r, t0, bi, &bar_g);
                    tma_load_4d(tZh + 8192, &maps.w, 64, h * NG + r, t0, bi, &bar_g);
                    tma_load_4d(tZl, &maps.v, 0, h * NG + r, t0, bi, &bar_g);
                    tma_load_4d(tZl + 8192, &maps.v, 64, h * NG + r, t0, bi, &bar_g);
                }
                ok = ok && mbar_wait(&bar_g, gph & 1u);
                ++gph;
                fence_after_sync();
                if (ok) {
                    const int odd = lane & 1, ie = i & ~1;
#pragma unroll
                    for (int r8 = 0; r8 < 8; ++r8) {
                        const int rr = 16 * sg + 8 * odd + r8;
                        float2 vv = pair_get(tZl, 64, rr, ie), wv = pair_get(tZh, 64, rr, ie);
                        if (kPacked && rr >= len) vv = wv = make_float2(0.f, 0.f);  // past the sequence
                        pair_split_put(tZh, tZl, 64, rr, ie, wv.x * vv.x, wv.y * vv.y);
                    }
                }
                fence_async_smem();
                fence_before_sync();
                ok = __syncthreads_and(ok) != 0;
                fence_after_sync();
                if (ok && tid == 0) {
                    const uint32_t id = idesc_bf16(128, 64, true, false);
                    for (int k0 = 0; k0 < 64; k0 += 16)
                        mma3(tUT, desc_mnmajor(tZh, 64, k0), desc_mnmajor(tZl, 64, k0), desc_kmajor(tAh, 64, k0),
                             desc_kmajor(tAl, 64, k0), id, k0 > 0);
                    mma_commit(&bar_g);
                    bulk_wait_read<0>();  // the previous U store has read the U tiles
                }
                ok = ok && mbar_wait(&bar_g, gph & 1u);
                ++gph;
                fence_after_sync();
                ok = __syncthreads_and(ok) != 0;
                if (ok) {  // warp (quad, task): U^T rows 32 quad + lane, columns [16 task, 16 task + 16)
                    const int ich = 32 * quad + lane, c0 = 16 * task;
                    float v[16];
                    tmem_ld16(tmem_lane_addr(tUT, quad, c0), v);
                    uint8_t *row = (ich < 64 ? tEh : tTh) + (ich & 63) * 256;
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const int cidx = (c0 >> 2) + e4;
                        *reinterpret_cast<float4 *>(row + ((cidx ^ (ich & 15)) << 4)) =
                            make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
                    }
                }
                fence_async_smem();
                fence_before_sync();
                ok = __syncthreads_and(ok) != 0;
                fence_after_sync();
                if (ok && tid == 0) {
                    uint8_t *u = reinterpret_cast<uint8_t *>(ws.U + (chv0 + (size_t)r * NT) * D * C);
                    bulk_store(u, tEh, 16384u);
                    bulk_store(u + 16384, tTh, 16384u);
                    bulk_commit();
                }
            }
            if (tid == 0) {  // every input tile is free now; q's slot once the Q_gamma image has been read
                const bool more = ok && chn + (int)gridDim.x < nchunks;
                if (more) issue_inputs(chn + (int)gridDim.x, 0);
                bulk_wait_read<0>();
                if (more) issue_inputs(chn + (int)gridDim.x, 1);
            }
            __syncthreads();
        }
    }
    if (tid == 0 && !ok) mma_drain(&bar_x);  // a wait gave up: the products issued finish before TMEM is freed
    if (tid == 0) bulk_wait_all<0>();
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// =================================================================================================
// state kernel: one (batch, head) per CTA, serial over chunks
// =================================================================================================
// Segmentation of the serial pass of one (batch, head) chain, the chunk-level scan: Eq. 23 is affine in the
// state entering a chunk, S_C = M_c S_0 + N_c with M_c = Diag(gamma_C) - K_tail^T Y and N_c = K_tail^T U. A
// segment of L chunks composes to S_end = M S_start + N; phase A finds M (the pass started from I with U = 0)
// and N (started from 0) for every segment in parallel, a short serial combine gives every segment's start
// state, and phase C reruns the segments from those states, emitting o and the images.
struct SegArgs {
    int nseg, L;      // segments per chain, chunks per segment; nseg = 1 is the plain pass
    int phase_a;      // 1: transfer CTAs (kind 1) and offset CTAs (kind 0); no o, no images
    const float *S0;  // start states: the user's initial state (nseg = 1, nullable) or [nseg][B H][D][D]
    float *ST;        // end states: [2][nseg][B H][D][D] in phase A, else the user's final state (last segment)
};

constexpr size_t kGroupA = 2 * kImg64x128;                 // Y, Q_gamma
constexpr size_t kGroupB = kImg64x128 + kImg64x64 + 1024;  // K_tail, A_qk, gamma_C
constexpr size_t kStateSmem = kImg128x128 + kImg128x64 + kGroupA + kGroupB + 16384 + 1024;

// Per chunk: R^T = U^T - S^T Y^T (tensor cores, then fp32 in registers), S^T <- S^T Diag(gamma_C) + R^T K_tail,
// O^T = S^T Q_gamma^T + R^T A_qk^T. The R and S products are on the serial path and go first; O accumulates
// in one of two TMEM buffers and is written out during the next chunk (TMEM -> shared tile -> TMA store).
// Warps 0..3 hold S^T row j = tid (TMEM lane j) and do every conversion. Without o, the first lane of a fifth
// warp issues the products and the bulk copies, so that each product starts as soon as its operands are in
// place and the converting warps' own loads (U^T) never hold it up; with o (more products, and the o tile
// conversion beside them), thread 0 issuing between its own conversions measured faster.
// kOut: the pass writes o (and so runs the O products); passes without o (phase A of the scan, the backward's
// recompute) are a separate instantiation.
constexpr int kStateIssuer = 128;               // the issuing thread (first lane of warp 4)
constexpr int kStateBlock = kStateIssuer + 32;  // four converting warps and the issuing warp
template <bool kOut>
__global__ void __launch_bounds__(kStateBlock, 1)
    state_kernel(const __grid_constant__ CUtensorMap mo, const __grid_constant__ CUtensorMap mo_part, int has_o,
                 SegArgs sa, Varlen vl, WsTC ws, WsBwd bw, int T, int H, int NG, int NT, int BH) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tSh = base, *tSl = base + 32768;          // S^T hi / lo  [128 j x 128 i]
    uint8_t *tRh = base + 65536, *tRl = base + 81920;  // R^T hi / lo  [128 j x 64 r]
    uint8_t *tY = base + 98304;                        // image -Y^T     [128 i x 64 r]
    uint8_t *tQ = tY + kImg64x128;                     // Q_gamma hi [64 r x 128 i], two slots (chunk parity)
    uint8_t *tK = tQ + kImg64x128;                     // image K_tail   [64 r x 128 i]
    uint8_t *tA = tK + kImg64x128;                     // image A_qk     [64 r x 64 s]
    float *gC = reinterpret_cast<float *>(tA + kImg64x64);
    uint8_t *tOut = tA + kImg64x64 + 1024;             // o tile [64 r x 128 j] bf16, 128-byte swizzle
    uint8_t *tYh = tY, *tYl = tY + 16384, *tKh = tK, *tKl = tK + 16384;
    uint8_t *tAh = tA, *tAl = tA + 8192;
    __shared__ uint64_t barA, barB, bar_a, bar_b, bar_x;
    __shared__ uint32_t tslot;

    // CTA -> (kind, chain, segment); kind 1 (phase A only) runs the segment transfer: start I, no U.
    const int seg = blockIdx.x % sa.nseg, rest = blockIdx.x / sa.nseg;
    const bool packed = vl.chunk != nullptr;
    const int bhr = rest % BH, kind = rest / BH, h = bhr % H;
    const int bi = packed ? __ldg(vl.order + bhr / H) : bhr / H;  // batch, or sequence (longest first)
    const int bhi = bi * H + h;
    const size_t bh = (size_t)bhi;
    GDR2_DCHECK(bi >= 0 && bhi < BH && seg < sa.nseg);
    // This CTA's chunks [cb, ce): a segment of the chain, or (packed batch, bi = sequence) the sequence's
    // chunks, whose workspace entries are indexed by head and packed chunk.
    const int4 sq = packed ? __ldg(vl.seq + bi) : make_int4(seg * sa.L, min(sa.L, NT - seg * sa.L), 0, 0);
    const int cb = sq.x, ce = min(NT, sq.x + sq.y);
    const size_t wsb = packed ? (size_t)h * NT : bh * NT;  // workspace chunk index = wsb + c
    // grouped value heads (G per key head): the key-side images belong to key head h / NG
    const size_t wsbK = packed ? (size_t)(h / NG) * NT : ((size_t)bi * (H / NG) + h / NG) * NT;
    if (cb >= ce) {  // an empty sequence: the state passes through unchanged
        if (sa.ST)
            for (int x = threadIdx.x; x < D * D; x += blockDim.x) sa.ST[bh * D * D + x] = sa.S0 ? sa.S0[bh * D * D + x] : 0.f;
        return;
    }
    const bool transfer = sa.phase_a && kind == 1;
    constexpr bool out = kOut;                            // o, and the images below, only outside phase A
    const bool imgs = !sa.phase_a && bw.S0T != nullptr;
    const int tid = threadIdx.x, warp = tid >> 5;
    // with o, thread 0 issues (128 threads); without o, the first lane of a fifth warp (160 threads)
    const bool conv = tid < kStateIssuer, issuer = kOut ? tid == 0 : tid == kStateIssuer;
    const int j = tid;  // S^T row of a converting thread

    // -Y^T and the hi tile of Q_gamma. S^T Q_gamma^T only affects o, and two terms (S hi and lo times Q_gamma hi)
    // keep o within its bound (max error 0.008 RMS beyond bf16 storage on the training and long workloads in an
    // fp64 emulation, against 0.02), so Q_gamma's hi tile alone is loaded, into the slot of the chunk's parity:
    // the next chunk's lands in the other slot while S^T Q_gamma^T still reads this one.
    auto load_a = [&](size_t ch, uint32_t slot) {
        mbar_expect_tx(&barA, (uint32_t)kImg64x128 + (out ? 16384u : 0u));
        bulk_load(tY, ws.Y + ch * kImg64x128, (uint32_t)kImg64x128, &barA);
        if (out) bulk_load(tQ + 16384u * slot, ws.Q + ch * kImg64x128, 16384u, &barA);
    };
    auto load_b = [&](size_t ch) {
        mbar_expect_tx(&barB, (uint32_t)kImg64x128 + (out ? (uint32_t)kImg64x64 : 0u) + 512u);
        bulk_load(tK, ws.Kt + ch * kImg64x128, (uint32_t)kImg64x128, &barB);
        if (out) bulk_load(tA, ws.Aqk + ch * kImg64x64, (uint32_t)kImg64x64, &barB);
        bulk_load(gC, ws.gC + ch * D, 512u, &barB);
    };

    if (issuer) {
        mbar_init(&barA, 1);
        mbar_init(&barB, 1);
        mbar_init(&bar_a, 1);
        mbar_init(&bar_b, 1);
        mbar_init(&bar_x, 1);
        mbar_fence_init();
        load_a(wsbK + cb, 0);
        load_b(wsbK + cb);
    }
    if (warp == 0) tmem_alloc(&tslot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t tS = tmem, tR = tmem + 128, tO0 = tmem + 192;  // O buffers at 192 and 256

    // O^T of a finished chunk (TMEM lane j = value channel) -> o tile in shared memory.
    auto o_to_tile = [&](uint32_t tO) {
        for (int r0 = 0; r0 < C; r0 += 16) {
            float vo[16];
            tmem_ld16(tmem_lane_addr(tO, warp, r0), vo);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                *reinterpret_cast<__nv_bfloat16 *>(tOut + rt_off(64, r0 + e, j)) = __float2bfloat16_rn(vo[e]);
        }
    };
    auto o_store = [&](int c) {  // rows past T fall outside the tensor and are not written
        const int4 e = chunk_info(vl, c);  // e.z >= 0: the chunk ends inside a packed batch; staged in slot e.z
        const CUtensorMap *m = e.z < 0 ? &mo : &mo_part;
        const int t = e.z < 0 ? e.x : 0, b4 = e.z < 0 ? (packed ? 0 : bi) : e.z;
        tma_store_4d(m, tOut, 0, h, t, b4);
        tma_store_4d(m, tOut + 8192, 64, h, t, b4);
        bulk_commit();
    };

    const float *S0p = sa.phase_a ? nullptr
                       : sa.nseg == 1 ? (sa.S0 ? sa.S0 + bh * D * D : nullptr)
                                      : sa.S0 + ((size_t)seg * BH + bh) * D * D;
    if (conv)
        for (int i0 = 0; i0 < D; i0 += 16) {  // S^T row j = column j of the start state
            float vs[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                vs[e] = transfer ? (i0 + e == j ? 1.f : 0.f) : S0p ? S0p[(i0 + e) * D + j] : 0.f;
            tmem_st16(tmem_lane_addr(tS, warp, i0), vs);
            split_store8(tSh, tSl, 128, j, i0, vs);
            split_store8(tSh, tSl, 128, j, i0 + 8, vs + 8);
        }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    const uint32_t id64 = idesc_bf16(128, 64, false, false);
    const uint32_t id64mn = idesc_bf16(128, 64, false, true);
    const uint32_t id128mn = idesc_bf16(128, 128, false, true);
    bool ok = true;
    for (int c = cb; c < ce; ++c) {
        const size_t ch = wsb + c, chk = wsbK + c;  // value-side and key-side workspace entries
        const uint32_t par = (uint32_t)((c - cb) & 1);
        const uint32_t tO = tO0 + 64u * par;
        if constexpr (kOut) {  // thread 0 issues the products between its own conversions
            float u[64];  // U^T row j of this chunk, fetched early (fp32)
            {
                const float4 *src = reinterpret_cast<const float4 *>(ws.U + (ch * D + j) * C);
    #pragma unroll
                for (int r4 = 0; r4 < 16; ++r4) {  // 16-byte chunks of the row are swizzled by (row % 16)
                    const float4 x = transfer ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(src + (r4 ^ (j & 15)));
                    u[4 * r4] = x.x;
                    u[4 * r4 + 1] = x.y;
                    u[4 * r4 + 2] = x.z;
                    u[4 * r4 + 3] = x.w;
                }
            }

            if (issuer && imgs) {  // image of the state entering this chunk
                bulk_store(bw.S0T + ch * kImg128x128, tSh, (uint32_t)kImg128x128);
                bulk_commit();
            }
            ok = ok && mbar_wait(&barA, par);
            fence_after_sync();
            if (ok && issuer) {
                for (int k0 = 0; k0 < 128; k0 += 16)  // R_acc = S^T (-Y^T) (the -Y^T image used MN-major)
                    mma3(tR, desc_kmajor(tSh, 128, k0), desc_kmajor(tSl, 128, k0), desc_mnmajor(tYh, 128, k0),
                         desc_mnmajor(tYl, 128, k0), id64mn, k0 > 0);
                mma_commit(&bar_a);
                if (out) {
                    uint8_t *tQh = tQ + 16384u * par;
                    for (int k0 = 0; k0 < 128; k0 += 16) {  // O_acc = S^T Q_gamma^T (S hi and lo, Q_gamma hi)
                        const uint64_t bq = desc_kmajor(tQh, 64, k0);
                        mma_bf16(tO, desc_kmajor(tSh, 128, k0), bq, id64, k0 > 0);
                        mma_bf16(tO, desc_kmajor(tSl, 128, k0), bq, id64, true);
                    }
                }
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
            if (ok && out && c > cb) o_to_tile(tO0 + 64u * (par ^ 1u));  // complete since bar_b of c - 1
            ok = ok && mbar_wait(&bar_a, par);
            fence_after_sync();
            if (ok && issuer && c + 1 < ce) load_a(chk + 1, par ^ 1u);  // -Y^T read; the other Q_gamma slot free
            if (ok) {  // R^T = U^T + R_acc  (hi / lo into shared memory)
                for (int r0 = 0; r0 < C; r0 += 16) {
                    float vr[16];
                    tmem_ld16(tmem_lane_addr(tR, warp, r0), vr);
    #pragma unroll
                    for (int e = 0; e < 16; ++e) vr[e] = u[r0 + e] + vr[e];
                    split_store8(tRh, tRl, 128, j, r0, vr);
                    split_store8(tRh, tRl, 128, j, r0 + 8, vr + 8);
                }
            }
            fence_async_smem();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
            if (ok && issuer) {
                for (int k0 = 0; k0 < 64; k0 += 16)  // S^T += R^T K_tail
                    mma3(tS, desc_kmajor(tRh, 128, k0), desc_kmajor(tRl, 128, k0), desc_mnmajor(tKh, 64, k0),
                         desc_mnmajor(tKl, 64, k0), id128mn, true);
                if (out)  // O_acc += R^T A_qk^T
                    for (int k0 = 0; k0 < 64; k0 += 16)
                        mma3(tO, desc_kmajor(tRh, 128, k0), desc_kmajor(tRl, 128, k0), desc_kmajor(tAh, 64, k0),
                             desc_kmajor(tAl, 64, k0), id64, true);
                mma_commit(&bar_b);
                if (imgs) {
                    bulk_store(bw.RT + ch * kImg128x64, tRh, (uint32_t)kImg128x64);
                    bulk_commit();
                }
                if (out && c > cb) o_store(c - 1);
            }
        } else {  // the issuing warp (fifth warp) beside four converting warps
            if (issuer) {  // the R product (and S^T Q_gamma^T) as soon as -Y^T is in
                if (imgs) {  // image of the state entering this chunk
                    bulk_store(bw.S0T + ch * kImg128x128, tSh, (uint32_t)kImg128x128);
                    bulk_commit();
                }
                ok = ok && mbar_wait(&barA, par);
                fence_after_sync();
                if (ok) {
                    for (int k0 = 0; k0 < 128; k0 += 16)  // R_acc = S^T (-Y^T) (the -Y^T image used MN-major)
                        mma3(tR, desc_kmajor(tSh, 128, k0), desc_kmajor(tSl, 128, k0), desc_mnmajor(tYh, 128, k0),
                             desc_mnmajor(tYl, 128, k0), id64mn, k0 > 0);
                    mma_commit(&bar_a);
                    if (out) {
                        uint8_t *tQh = tQ + 16384u * par;
                        for (int k0 = 0; k0 < 128; k0 += 16) {  // O_acc = S^T Q_gamma^T (S hi and lo, Q_gamma hi)
                            const uint64_t bq = desc_kmajor(tQh, 64, k0);
                            mma_bf16(tO, desc_kmajor(tSh, 128, k0), bq, id64, k0 > 0);
                            mma_bf16(tO, desc_kmajor(tSl, 128, k0), bq, id64, true);
                        }
                    }
                }
                ok = ok && mbar_wait(&bar_a, par);  // the R product has read -Y^T; the other Q_gamma slot is free
                if (ok && c + 1 < ce) load_a(chk + 1, par ^ 1u);
            }
            if (conv) {
                float u[64];  // U^T row j of this chunk (fp32)
                {
                    const float4 *src = reinterpret_cast<const float4 *>(ws.U + (ch * D + j) * C);
    #pragma unroll
                    for (int r4 = 0; r4 < 16; ++r4) {  // 16-byte chunks of the row are swizzled by (row % 16)
                        const float4 x = transfer ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(src + (r4 ^ (j & 15)));
                        u[4 * r4] = x.x;
                        u[4 * r4 + 1] = x.y;
                        u[4 * r4 + 2] = x.z;
                        u[4 * r4 + 3] = x.w;
                    }
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
                if (ok && out && c > cb) o_to_tile(tO0 + 64u * (par ^ 1u));  // complete since bar_b of c - 1
                ok = ok && mbar_wait(&bar_a, par);
                fence_after_sync();
                if (ok) {  // R^T = U^T + R_acc  (hi / lo into shared memory)
                    for (int r0 = 0; r0 < C; r0 += 16) {
                        float vr[16];
                        tmem_ld16(tmem_lane_addr(tR, warp, r0), vr);
    #pragma unroll
                        for (int e = 0; e < 16; ++e) vr[e] = u[r0 + e] + vr[e];
                        split_store8(tRh, tRl, 128, j, r0, vr);
                        split_store8(tRh, tRl, 128, j, r0 + 8, vr + 8);
                    }
                }
            }
            fence_async_smem();
            fence_before_sync();
            __syncthreads();
            fence_after_sync();
            if (ok && issuer) {
                ok = mbar_wait(&barB, par);  // K_tail and A_qk (the converting warps have seen them already)
                if (ok) {
                    for (int k0 = 0; k0 < 64; k0 += 16)  // S^T += R^T K_tail
                        mma3(tS, desc_kmajor(tRh, 128, k0), desc_kmajor(tRl, 128, k0), desc_mnmajor(tKh, 64, k0),
                             desc_mnmajor(tKl, 64, k0), id128mn, true);
                    if (out)  // O_acc += R^T A_qk^T
                        for (int k0 = 0; k0 < 64; k0 += 16)
                            mma3(tO, desc_kmajor(tRh, 128, k0), desc_kmajor(tRl, 128, k0), desc_kmajor(tAh, 64, k0),
                                 desc_kmajor(tAl, 64, k0), id64, true);
                    mma_commit(&bar_b);
                    if (imgs) {
                        bulk_store(bw.RT + ch * kImg128x64, tRh, (uint32_t)kImg128x64);
                        bulk_commit();
                    }
                    if (out && c > cb) o_store(c - 1);
                }
            }
        }
        ok = ok && mbar_wait(&bar_b, par);
        fence_after_sync();
        if (ok && issuer) {
            if (c + 1 < ce) load_b(chk + 1);
            bulk_wait_read<0>();  // the S^T and R^T images and the o tile have been read before reuse
        }
        __syncthreads();
        if (ok && conv) {
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
    if (ok && out && conv) o_to_tile(tO0 + 64u * (uint32_t)((ce - 1 - cb) & 1));
    fence_async_smem();
    fence_before_sync();
    ok = __syncthreads_and(ok) != 0;
    fence_after_sync();
    if (ok && out && issuer) o_store(ce - 1);
    float *STp = sa.phase_a ? sa.ST + (((size_t)kind * sa.nseg + seg) * BH + bh) * D * D
                 : (seg == sa.nseg - 1 && sa.ST) ? sa.ST + bh * D * D
                                                   : nullptr;
    if (ok && STp && conv) {
        for (int i0 = 0; i0 < D; i0 += 16) {
            float vs[16];
            tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
#pragma unroll
            for (int e = 0; e < 16; ++e) STp[(i0 + e) * D + j] = vs[e];
        }
    }
    if (issuer && !ok) mma_drain(&bar_x);  // a wait gave up: the products issued finish before TMEM is freed
    if (issuer) bulk_wait_all<0>();
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// =================================================================================================
// backward: reverse serial pass, one (batch, head) per CTA (transposed, TMEM lane j = value channel)
//     dR^T = dO^T A_qk + dS_C^T K_tail^T
//     dS_0^T = dS_C^T Diag(gamma_C) + dO^T Q_gamma - dR^T Y
// The images of dS_C^T and dR^T of every chunk go to the workspace; the last dS_0 is dS0.
// =================================================================================================
constexpr size_t kRevSmem = kImg128x128 + kImg128x64 + 16384 /*dO*/ + kImg64x64 + 3 * kImg64x128 + 1024 + 1024;

// Warps 0..3 hold dS^T row j = tid and do the conversions; the first lane of a fifth warp issues the products
// and the bulk copies (as in the forward pass without o), so that issuing never holds up a converting warp.
__global__ void __launch_bounds__(kStateBlock, 1)
    rev_kernel(const __grid_constant__ CUtensorMap mdO, int has_dO, SegArgs sa, Varlen vl, WsTC ws, WsBwd bw, int T,
               int H, int NG, int NT, int BH) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *tDh = base, *tDl = base + 32768;          // dS^T hi / lo   [128 j x 128 i]
    uint8_t *tNh = base + 65536, *tNl = base + 81920;  // dR^T hi / lo   [128 j x 64 r]
    uint8_t *tdO = base + 98304;                       // dO [64 r x 128 j] (bf16, exact)
    uint8_t *tA = tdO + 16384;                         // image A_qk    [64 s x 64 r]
    uint8_t *tK = tA + kImg64x64;                      // image K_tail  [64 r x 128 i]
    uint8_t *tQ = tK + kImg64x128;                     // image Q_gamma [64 r x 128 i]
    uint8_t *tY = tQ + kImg64x128;                     // image -Y^T    [128 i x 64 r]
    float *gC = reinterpret_cast<float *>(tY + kImg64x128);
    uint8_t *tAh = tA, *tAl = tA + 8192, *tKh = tK, *tKl = tK + 16384, *tQh = tQ, *tQl = tQ + 16384;
    uint8_t *tYh = tY, *tYl = tY + 16384;
    __shared__ uint64_t full, bar1, bar2, bar_x;
    __shared__ uint32_t tslot;

    // CTA -> (chain, segment). Phase A runs each segment from dS = 0 (its offset); the transfer of a
    // segment is the transpose of the forward's, so it is not recomputed here.
    const bool packed = vl.chunk != nullptr;
    const int seg = blockIdx.x % sa.nseg, bhr = blockIdx.x / sa.nseg, h = bhr % H;
    const int bi = packed ? __ldg(vl.order + bhr / H) : bhr / H;  // batch, or sequence (longest first)
    const int bhi = bi * H + h;
    const size_t bh = (size_t)bhi;
    GDR2_DCHECK(bi >= 0 && bhi < BH && seg < sa.nseg);
    // chunks [cb, ce), walked backwards: a segment of the chain, or (packed batch, bi = sequence) the
    // sequence's chunks, whose workspace entries are indexed by head and packed chunk
    const int4 sq = packed ? __ldg(vl.seq + bi) : make_int4(seg * sa.L, min(sa.L, NT - seg * sa.L), 0, 0);
    const int cb = sq.x, ce = min(NT, sq.x + sq.y);
    const size_t wsb = packed ? (size_t)h * NT : bh * NT;  // workspace chunk index = wsb + c
    // grouped value heads (G per key head): the key-side images belong to key head h / NG
    const size_t wsbK = packed ? (size_t)(h / NG) * NT : ((size_t)bi * (H / NG) + h / NG) * NT;
    if (cb >= ce) {  // an empty sequence: the gradient passes through unchanged
        if (sa.ST)
            for (int x = threadIdx.x; x < D * D; x += blockDim.x) sa.ST[bh * D * D + x] = sa.S0 ? sa.S0[bh * D * D + x] : 0.f;
        return;
    }
    const bool imgs = !sa.phase_a;
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool conv = tid < kStateIssuer, issuer = tid == kStateIssuer;
    const int j = tid;  // dS^T row of a converting thread

    auto issue = [&](int c) {
        const size_t ch = wsbK + c;  // every load here is a key-side image but dO
        uint32_t bytes = (uint32_t)(kImg64x64 + 3 * kImg64x128) + 512u;
        if (has_dO) bytes += 16384u;
        mbar_expect_tx(&full, bytes);
        if (has_dO) {  // rows past a packed sequence's end meet zero rows of A_qk and Q_gamma
            const int t = chunk_info(vl, c).x, b4 = packed ? 0 : bi;
            tma_load_4d(tdO, &mdO, 0, h, t, b4, &full);
            tma_load_4d(tdO + 8192, &mdO, 64, h, t, b4, &full);
        }
        bulk_load(tA, ws.Aqk + ch * kImg64x64, (uint32_t)kImg64x64, &full);
        bulk_load(tK, ws.Kt + ch * kImg64x128, (uint32_t)kImg64x128, &full);
        bulk_load(tQ, ws.Q + ch * kImg64x128, (uint32_t)kImg64x128, &full);
        bulk_load(tY, ws.Y + ch * kImg64x128, (uint32_t)kImg64x128, &full);
        bulk_load(gC, ws.gC + ch * D, 512u, &full);
    };

    if (issuer) {
        mbar_init(&full, 1);
        mbar_init(&bar1, 1);
        mbar_init(&bar2, 1);
        mbar_init(&bar_x, 1);
        mbar_fence_init();
    }
    if (!has_dO)
        for (int x = tid; x < 16384 / 16; x += blockDim.x) reinterpret_cast<uint4 *>(tdO)[x] = make_uint4(0, 0, 0, 0);
    if (warp == 0) tmem_alloc(&tslot, 256);
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (issuer) issue(ce - 1);
    const uint32_t tmem = tslot;
    const uint32_t tS = tmem, tR = tmem + 128;

    // gradient entering the segment's last chunk: dS_T (nseg = 1), 0 (phase A) or the combined value
    const float *dSp = sa.phase_a ? nullptr
                       : sa.nseg == 1 ? (sa.S0 ? sa.S0 + bh * D * D : nullptr)
                                      : sa.S0 + ((size_t)seg * BH + bh) * D * D;
    if (conv)
        for (int i0 = 0; i0 < D; i0 += 16) {  // dS^T row j = column j of that gradient
            float vs[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) vs[e] = dSp ? dSp[(i0 + e) * D + j] : 0.f;
            tmem_st16(tmem_lane_addr(tS, warp, i0), vs);
            split_store8(tDh, tDl, 128, j, i0, vs);
            split_store8(tDh, tDl, 128, j, i0 + 8, vs + 8);
        }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    const uint32_t id_a = idesc_bf16(128, 64, true, true);    // dO^T (MN) x A_qk (MN)
    const uint32_t id_b = idesc_bf16(128, 64, false, false);  // dS^T (K) x K_tail (K)
    const uint32_t id_c = idesc_bf16(128, 128, true, true);   // dO^T (MN) x Q_gamma (MN)
    const uint32_t id_d = idesc_bf16(128, 128, false, false);  // dR^T (K) x (-Y^T) (K)
    bool ok = true;
    int it = 0;
    for (int c = ce - 1; c >= cb; --c, ++it) {
        const size_t ch = wsb + c;
        const uint32_t par = (uint32_t)(it & 1);
        if (issuer && imgs) {  // image of dS_C^T (the tiles hold it until the end of this chunk)
            bulk_store(bw.dST + ch * kImg128x128, tDh, (uint32_t)kImg128x128);
            bulk_commit();
        }
        ok = ok && mbar_wait(&full, par);  // (the converting warps need gamma_C)
        fence_after_sync();
        if (ok && issuer) {
            for (int k0 = 0; k0 < 64; k0 += 16) {  // dO^T A_qk (dO exact in bf16: two terms)
                mma_bf16(tR, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tAh, 64, k0), id_a, k0 > 0);
                mma_bf16(tR, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tAl, 64, k0), id_a, true);
            }
            for (int k0 = 0; k0 < 128; k0 += 16)
                mma3(tR, desc_kmajor(tDh, 128, k0), desc_kmajor(tDl, 128, k0), desc_kmajor(tKh, 64, k0),
                     desc_kmajor(tKl, 64, k0), id_b, true);
            mma_commit(&bar1);
        }
        if (ok && conv) {  // dS^T <- dS^T Diag(gamma_C)
            for (int i0 = 0; i0 < D; i0 += 16) {
                float vs[16];
                const uint32_t a = tmem_lane_addr(tS, warp, i0);
                tmem_ld16(a, vs);
#pragma unroll
                for (int e = 0; e < 16; ++e) vs[e] *= gC[i0 + e];
                tmem_st16(a, vs);
            }
        }
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (ok && issuer)  // + dO^T Q_gamma, queued behind the dR products (it does not depend on dR)
            for (int k0 = 0; k0 < 64; k0 += 16) {
                mma_bf16(tS, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tQh, 64, k0), id_c, true);
                mma_bf16(tS, desc_mnmajor(tdO, 64, k0), desc_mnmajor(tQl, 64, k0), id_c, true);
            }
        if (conv) {
            ok = ok && mbar_wait(&bar1, par);
            fence_after_sync();
        }
        if (ok && conv) {  // dR^T row j (hi / lo) for the next product and for the workspace image
            for (int r0 = 0; r0 < C; r0 += 16) {
                float vr[16];
                tmem_ld16(tmem_lane_addr(tR, warp, r0), vr);
                split_store8(tNh, tNl, 128, j, r0, vr);
                split_store8(tNh, tNl, 128, j, r0 + 8, vr + 8);
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (ok && issuer) {
            for (int k0 = 0; k0 < 64; k0 += 16)  // + dR^T (-Y)
                mma3(tS, desc_kmajor(tNh, 128, k0), desc_kmajor(tNl, 128, k0), desc_kmajor(tYh, 128, k0),
                     desc_kmajor(tYl, 128, k0), id_d, true);
            mma_commit(&bar2);
            if (imgs) {
                bulk_store(bw.dRT + ch * kImg128x64, tNh, (uint32_t)kImg128x64);
                bulk_commit();
            }
        }
        ok = ok && mbar_wait(&bar2, par);
        fence_after_sync();
        if (ok && issuer) {
            if (c > cb) issue(c - 1);
            bulk_wait_read<0>();  // the dS_C^T and dR^T images have been read before the tiles are rewritten
        }
        __syncthreads();
        if (ok && conv) {
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
    float *dS0p = sa.phase_a ? sa.ST + ((size_t)seg * BH + bh) * D * D
                  : (seg == 0 && sa.ST) ? sa.ST + bh * D * D
                                        : nullptr;
    if (ok && dS0p && conv) {
        for (int i0 = 0; i0 < D; i0 += 16) {
            float vs[16];
            tmem_ld16(tmem_lane_addr(tS, warp, i0), vs);
#pragma unroll
            for (int e = 0; e < 16; ++e) dS0p[(i0 + e) * D + j] = vs[e];
        }
    }
    if (issuer && !ok) mma_drain(&bar_x);  // a wait gave up: the products issued finish before TMEM is freed
    if (issuer) bulk_wait_all<0>();
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// =================================================================================================
// backward: fused chunk-local kernel, one chunk per CTA, 512 threads (thread (grp, i) = channel i, rows
// [16 grp, 16 grp + 16); warp w reads TMEM lane quadrant w % 4, columns [16 grp, 16 grp + 16)).
// With R = U - Y S_0, dR, S_0 and dS_C from the serial passes, every per-chunk product of the chain rule
// through Eqs. 23-24 runs on tcgen05 with hi / lo operands, all intermediates on chip:
//   P1  dA_qk = tril(dO R^T)                       P2  dQ_gamma = dO S_0^T + dA_qk Kbar
//   P3  dK_tail = R dS_C^T                         P4  dY = -dR S_0^T
//   P5  dZ = A^T dR                                P6  dA = dR Z^T + dY Ebar^T   (Eqs. 64-65)
//   P7  dT = -tril(A^T dA A^T, -1)                 P8  dEbar = A^T dY + dT Kbar
//   P9  dKbar = dA_qk^T Q_gamma + dT^T Ebar        dgamma_C = diag(dS_C S_0^T)
// (stored transposed where that puts the channel on the TMEM lane). The assembly then forms
//   dq = dQ_gamma gamma, db = dEbar k gamma, dk = dEbar b gamma + dKbar / gamma + dK_tail gamma_C / gamma,
//   dw = dZ v, dv = dZ w, and dlog_alpha as the in-chunk reverse cumulative sum of
//   dG = dQ_gamma Q_gamma + dEbar Ebar - dKbar Kbar - dK_tail K_tail (plus, at the last row,
//   sum_r dK_tail K_tail + dgamma_C gamma_C).
// Q_gamma, Kbar, Ebar and Z are recomputed from the raw inputs; A = (I + T)^-1 comes from the forward.
// Shared memory (224 KB) is reused across the phases (R0 32K | R1 64K | R2 64K | R3 32K | R4 16K | R5 16K):
//   phase 1   R0 dR^T, R1 S_0^T, R2 dS_C^T, R3 R^T, R4 dO, R5 A            (images, dO exact bf16)
//   phase 2   R1 Q_gamma | Kbar, R2 Ebar | Z, R3 dY^T, R4 dA_qk            (raw q, k, b, w, v land in the
//             lo / hi slots of the derived tiles and are replaced in place); later R0 dA | X, dT in Z's hi
//   assembly  raw q, k -> R3, b -> R4, v -> R0[0:16K), w -> R5 (reloaded once their regions die); the
//             gradients leave straight from registers (bf16 stores; the four warps of a row segment cover whole
//             256-byte rows), dlog_alpha as fp32 rows; every shared region is then free, and the next chunk's
//             loads are issued at once.
// TMEM columns: dQ_gamma 0, dK_tail 64, dY / dEbar 128, dA_qk / dKbar 192, dZ 256, dA 320, X 384, dT 448;
// in the first phase 384 .. 511 hold dS_C S_0^T (its diagonal is dgamma_C; grouped heads: 384 .. 387 carry
// the four row segments' shares of it) and 320 .. 323 the per-segment log-decay sums between the warps of a
// channel.
// =================================================================================================
constexpr int kBwdThreads = 512;
constexpr size_t kBwdSmem = 224 * 1024 + 1024;

struct BwdMaps {
    CUtensorMap q, k, b, v, w, dO;         // bf16 token tensors, loads
    CUtensorMap dv, dw;                    // value-side gradients, tile stores of the grouped-head loop
};

// Gradient tensors written by plain stores from the assembly's registers ([T, H, 128] rows of each batch).
struct GradPtrs {
    __nv_bfloat16 *dq, *dk, *db, *dv, *dw;
};

// Start-address step (16-byte units) of the descriptor for K elements k0 .. k0 + 15 of a tile with R rows:
// MN-major, 16 rows of 128 bytes; K-major, 32 bytes within a 64-column sub-tile, then the next sub-tile.
template <bool MN, int R>
__device__ __forceinline__ constexpr uint32_t desc_step(int k0) {
    return MN ? (uint32_t)(k0 * 8) : (uint32_t)(((k0 >> 6) * R * 128 + (k0 & 63) * 2) >> 4);
}

// Issues the MMAs of sum_k opA[m][k] opB[n][k] into tacc. TA: A stored [K][M] (MN-major use), else [M][K];
// TB: B stored [K][N], else [N][K]. Each stored matrix is a hi tile followed by its lo tile; an exact
// operand (a_exact / b_exact) contributes no lo term.
template <int M, int N, int K, bool TA, bool TB>
__device__ __forceinline__ void issue_term(uint32_t tacc, const uint8_t *ta, bool a_exact, const uint8_t *tb,
                                           bool b_exact, bool accumulate) {
    constexpr int RA = TA ? K : M, CA = TA ? M : K, RB = TB ? K : N, CB = TB ? N : K;
    const uint32_t id = idesc_bf16(M, N, TA, TB);
    const uint64_t ah0 = TA ? desc_mnmajor(ta, RA, 0) : desc_kmajor(ta, RA, 0);
    const uint64_t bh0 = TB ? desc_mnmajor(tb, RB, 0) : desc_kmajor(tb, RB, 0);
    constexpr uint64_t a_lo = (uint64_t)(RA * CA * 2) >> 4, b_lo = (uint64_t)(RB * CB * 2) >> 4;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 16) {
        const uint64_t ah = ah0 + desc_step<TA, RA>(k0), bh = bh0 + desc_step<TB, RB>(k0);
        mma_bf16(tacc, ah, bh, id, accumulate || k0 > 0);
        if (!b_exact) mma_bf16(tacc, ah, bh + b_lo, id, true);
        if (!a_exact) mma_bf16(tacc, ah + a_lo, bh, id, true);
    }
}

// TMEM accumulator with M = 64 (row m in lane 32 (m / 16) + m % 16) -> hi / lo tile [64][64] in shared
// memory. mode 0: copy; 1: keep n <= m; 2: -x for n < m, else 0.
__device__ __forceinline__ void m64_to_tile(uint32_t tacc, uint8_t *tile, int mode) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quad = warp & 3, n0 = 16 * (warp >> 2);
    float v[16];
    tmem_ld16(tmem_lane_addr(tacc, quad, n0), v);
    if (lane < 16) {
        const int m = 16 * quad + lane;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int n = n0 + e;
            if (mode == 1 && n > m) v[e] = 0.f;
            if (mode == 2) v[e] = (n < m) ? -v[e] : 0.f;
        }
        split_store8(tile, tile + 8192, 64, m, n0, v);
        split_store8(tile, tile + 8192, 64, m, n0 + 8, v + 8);
    }
}

__device__ __forceinline__ void put_bf16(uint8_t *tile, int r, int i, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(tile + rt_off(64, r, i)) = __float2bfloat16_rn(x);
}

// Grouped value heads (kGroup, G value heads per key head): a CTA takes a key-head chunk and walks the group's
// value heads; their shares of P1, P2a, P3, P4 and the dR Z^T term of P6 accumulate in TMEM, those of
// diag(dS_C S_0^T) in registers (they contract over value channels), dv and dw of each value head leave as
// soon as its P5 is done, and the key side (P2b, P6b .. P9, dq, dk, db, dlog_alpha) then runs once.
template <bool kPacked, bool kGroup>
__global__ void __launch_bounds__(kBwdThreads, 1)
    chunk_bwd_kernel(const __grid_constant__ BwdMaps maps, GradPtrs gp, int has_dO, const float *__restrict__ la,
                     Varlen vl, WsBwd bw, float *__restrict__ dla, int T, int H, int NG, int NT, int nchunks) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    uint8_t *R0 = base, *R1 = base + 32768, *R2 = base + 98304, *R3 = base + 163840, *R4 = base + 196608,
            *R5 = base + 212992;
    uint8_t *tdRT = R0, *tS0 = R1, *tdS = R2, *tRT = R3, *tdO = R4, *tA = R5;  // phase 1
    uint8_t *tQg = R1, *tKb = R1 + 32768, *tEb = R2, *tZ = R2 + 32768;        // phase 2 (hi; lo at +16K)
    uint8_t *tdY = R3, *tdAqk = R4, *tdA = R0, *tX = R0 + 16384, *tdT = R2 + 32768;
    uint8_t *rq = R3, *rk = R3 + 16384, *rb = R4, *rv = R0, *rw = R5;  // assembly inputs
    __shared__ uint64_t bar_p1, bar_p2, bar_p3, bar_m1, bar_m2, bar_m3, bar_m4, bar_m5, bar_gl, bar_gm, bar_x;
    __shared__ uint32_t tslot;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int quad = warp & 3, grp = warp >> 2;
    const int i = tid & 127;
    // value-side workspace entry of value head h G + r of key chunk chn: ((bi H + h) G + r) NT + c
    auto vchunk = [&](int chn, int r) { return ((size_t)(chn / NT) * NG + r) * NT + chn % NT; };
    auto load_vimgs = [&](size_t cv, int hv, int t, int bi, uint64_t *bar) {  // S_0^T, dS_C^T, dR^T, R^T, dO
        mbar_expect_tx(bar, (uint32_t)(2 * kImg128x128 + 2 * kImg128x64) + (has_dO ? 16384u : 0u));
        bulk_load(tS0, bw.S0T + cv * kImg128x128, (uint32_t)kImg128x128, bar);
        bulk_load(tdS, bw.dST + cv * kImg128x128, (uint32_t)kImg128x128, bar);
        bulk_load(tdRT, bw.dRT + cv * kImg128x64, (uint32_t)kImg128x64, bar);
        bulk_load(tRT, bw.RT + cv * kImg128x64, (uint32_t)kImg128x64, bar);
        if (has_dO) {
            tma_load_4d(tdO, &maps.dO, 0, hv, t, bi, bar);
            tma_load_4d(tdO + 8192, &maps.dO, 64, hv, t, bi, bar);
        }
    };

    // First-phase loads of chunk chn. Part 0 (S_0^T, dS_C^T; arms the barrier) targets R1 / R2, free once the
    // previous chunk's assembly has read its raw tiles; part 1 (dR^T, R^T, A, dO) targets the tiles that
    // carry the previous chunk's gradients and follows the output stores.
    auto load_p1 = [&](int chn, int part) {
        const int c = chn % NT, h = (chn / NT) % H, bi = chn / (NT * H);
        const size_t ch = (size_t)chn, cv = kGroup ? vchunk(chn, 0) : ch;  // A: key side; the rest: value side
        if (part == 0) {
            mbar_expect_tx(&bar_p1, (uint32_t)(kImg128x64 + 2 * kImg128x128 + kImg128x64 + kImg64x64) +
                                        (has_dO ? 16384u : 0u));
            bulk_load(tS0, bw.S0T + cv * kImg128x128, (uint32_t)kImg128x128, &bar_p1);
            bulk_load(tdS, bw.dST + cv * kImg128x128, (uint32_t)kImg128x128, &bar_p1);
        } else {
            bulk_load(tdRT, bw.dRT + cv * kImg128x64, (uint32_t)kImg128x64, &bar_p1);
            bulk_load(tRT, bw.RT + cv * kImg128x64, (uint32_t)kImg128x64, &bar_p1);
            bulk_load(tA, bw.A + ch * kImg64x64, (uint32_t)kImg64x64, &bar_p1);
            if (has_dO) {
                const int t = chunk_info_t<kPacked>(vl, c).x;
                tma_load_4d(tdO, &maps.dO, 0, kGroup ? h * NG : h, t, bi, &bar_p1);
                tma_load_4d(tdO + 8192, &maps.dO, 64, kGroup ? h * NG : h, t, bi, &bar_p1);
            }
        }
    };

    if (tid == 0) {
        mbar_init(&bar_p1, 1);
        mbar_init(&bar_p2, 1);
        mbar_init(&bar_p3, 1);
        mbar_init(&bar_m1, 1);
        mbar_init(&bar_m2, 1);
        mbar_init(&bar_m3, 1);
        mbar_init(&bar_m4, 1);
        mbar_init(&bar_m5, 1);
        mbar_init(&bar_gl, 1);
        mbar_init(&bar_gm, 1);
        mbar_init(&bar_x, 1);
        mbar_fence_init();
        if ((int)blockIdx.x < nchunks) {
            load_p1(blockIdx.x, 0);
            load_p1(blockIdx.x, 1);
        }
    }
    if (warp == 0) tmem_alloc(&tslot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t cQg = tmem, cKt = tmem + 64, cY = tmem + 128, cEb = tmem + 128, cAqk = tmem + 192,
                   cKb = tmem + 192, cZ = tmem + 256, cdA = tmem + 320, cX = tmem + 384, cdT = tmem + 448;

    bool go = true;
    int it = 0;
    uint32_t gl_ph = 0, gm_ph = 0;  // phases of bar_gl / bar_gm (value-head loop of grouped heads)
    // this thread's 16 log-decay values of a chunk (channel i, rows [16 grp, 16 grp + 16)). In the plain
    // instantiation those of the next chunk are loaded right after the current chunk's assembly, so their
    // latency hides behind its last phase; with packed chunks or grouped heads (more state live at that
    // point) loading them at the chunk start measured faster.
    constexpr bool kCarryLa = !kPacked && !kGroup;
    float la_r[16];
    auto load_la = [&](int chn_) {
        const int c_ = chn_ % NT, h_ = (chn_ / NT) % H, b_ = chn_ / (NT * H);
        const int4 ci = chunk_info_t<kPacked>(vl, c_);
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const int t = ci.x + 16 * grp + rr;
            la_r[rr] = (t < T && 16 * grp + rr < ci.y) ? __ldg(la + (((size_t)b_ * T + t) * H + h_) * D + i) : 0.f;
        }
    };
    if (kCarryLa && (int)blockIdx.x < nchunks) load_la(blockIdx.x);
    // the log-decay segment sums cross warps through TMEM: dA's columns, or (while dA accumulates over a group)
    // dZ's, free once the group's last dv, dw are out
    const uint32_t cSeg = kGroup ? cZ : cdA;
    for (int chn = (int)blockIdx.x; chn < nchunks; chn += (int)gridDim.x, ++it) {
    const uint32_t par = (uint32_t)(it & 1);
    const int c = chn % NT, h = (chn / NT) % H, bi = chn / (NT * H);
    const int4 cinfo = chunk_info_t<kPacked>(vl, c);
    const int t0 = cinfo.x, len = cinfo.y;  // rows from len on are zero inputs (packed batches)
    GDR2_DCHECK(c >= 0 && c < NT && h >= 0 && h < H && t0 >= 0 && t0 < T && len >= 0 && len <= 64);
    const int nxt = chn + (int)gridDim.x;
    if (!has_dO) {  // exact zeros stand in for the absent upstream gradient of o
        for (int x = tid; x < 16384 / 16; x += kBwdThreads) reinterpret_cast<uint4 *>(tdO)[x] = make_uint4(0, 0, 0, 0);
        fence_async_smem();
        __syncthreads();
    }

    // Cumulative log-decay of channel i over this thread's 16 rows (segment-local; the offsets of the
    // earlier segments are added once the segment sums have been exchanged).
    float G[16];
    if (!kCarryLa) load_la(chn);
    {
        float acc = 0.f;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            acc += la_r[rr];
            G[rr] = acc;
        }
    }

    // Grouped heads: dgamma_C[i] = sum_k dS_C[i][k] S_0[i][k] sums over the group's value heads, one full
    // product each on the tensor cores; instead, column i of the dS_C^T and S_0^T images (hi + lo) is summed
    // over the rows k on the CUDA cores beside each head's products. A thread takes 16 rows of its segment
    // [32 grp, 32 grp + 32) for the column pair (i & ~1, i | 1), the even lane the first 16, the odd lane the
    // last 16 (in the order r ^ 4, so that the two rows of one access use disjoint banks).
    float dgc0 = 0.f, dgc1 = 0.f;
    auto diag_part = [&](float &p0, float &p1) {
        const int odd = tid & 1, ie = i & ~1;
#pragma unroll 4
        for (int rr = 0; rr < 16; ++rr) {
            const int r = 32 * grp + (odd ? 16 + (rr ^ 4) : rr);
            const float2 dh = pair_get(tdS, 128, r, ie), dl = pair_get(tdS + 32768, 128, r, ie);
            const float2 sh = pair_get(tS0, 128, r, ie), sl = pair_get(tS0 + 32768, 128, r, ie);
            p0 = fmaf(dh.x + dl.x, sh.x + sl.x, p0);
            p1 = fmaf(dh.y + dl.y, sh.y + sl.y, p1);
        }
    };
    auto issue_p2 = [&]() {  // phase 2 loads: raw q, k, b, w, v into the lo / hi slots of the derived tiles
        constexpr int nraw = kGroup ? 3 : 5;  // grouped heads: Z's product was taken per value head
        mbar_expect_tx(&bar_p2, (uint32_t)nraw * 16384u);
        uint8_t *dst[5] = {tQg + 16384, tKb + 16384, tEb + 16384, tZ, tZ + 16384};
        const CUtensorMap *mp[5] = {&maps.q, &maps.k, &maps.b, &maps.w, &maps.v};
        for (int x = 0; x < nraw; ++x) {
            tma_load_4d(dst[x], mp[x], 0, h, t0, bi, &bar_p2);
            tma_load_4d(dst[x] + 8192, mp[x], 64, h, t0, bi, &bar_p2);
        }
    };
    if constexpr (kGroup) {
        for (int r = 0; r < NG; ++r) {
            const int hv = h * NG + r;
            if (r == 0) {
                go = go && mbar_wait(&bar_p1, par);
            } else {
                go = go && mbar_wait(&bar_gl, gl_ph & 1u);
                ++gl_ph;
            }
            fence_after_sync();
            if (go && tid == 0) {  // value head hv's share of the phase-1 products, and its own P5
                const bool acc = r > 0;
                issue_term<64, 64, 128, false, true>(cAqk, tdO, true, tRT, false, acc);    // P1  dA_qk
                issue_term<128, 64, 128, true, true>(cY, tS0, false, tdRT, false, acc);    // P4  S_0 dR^T = -dY^T
                issue_term<128, 64, 64, false, true>(cZ, tdRT, false, tA, false, false);   // P5  dZ^T of hv
                issue_term<128, 64, 128, true, true>(cKt, tdS, false, tRT, false, acc);    // P3  dK_tail^T
                issue_term<128, 64, 128, true, false>(cQg, tS0, false, tdO, true, acc);    // P2a dQ_gamma^T
                mma_commit(&bar_gm);
            }
            if (go) diag_part(dgc0, dgc1);  // (beside the products; the images are read-only until the barrier)
            go = go && mbar_wait(&bar_gm, gm_ph & 1u);
            ++gm_ph;
            fence_after_sync();
            fence_before_sync();
            go = __syncthreads_and(go) != 0;  // S_0^T, dS_C^T, R^T and dO are no longer read
            fence_after_sync();
            if (go && tid == 0) {  // raw w, v of hv into R^T's region
                mbar_expect_tx(&bar_gl, 2u * 16384u);
                tma_load_4d(R3, &maps.w, 0, hv, t0, bi, &bar_gl);
                tma_load_4d(R3 + 8192, &maps.w, 64, hv, t0, bi, &bar_gl);
                tma_load_4d(R3 + 16384, &maps.v, 0, hv, t0, bi, &bar_gl);
                tma_load_4d(R3 + 16384 + 8192, &maps.v, 64, hv, t0, bi, &bar_gl);
            }
            go = go && mbar_wait(&bar_gl, gl_ph & 1u);
            ++gl_ph;
            fence_after_sync();
            if (go) {  // Z = w (.) v (hi / lo) into S_0^T's region; lanes 2p, 2p + 1 share rows as in the forward
                const int odd = tid & 1, ie = i & ~1;
#pragma unroll
                for (int r8 = 0; r8 < 8; ++r8) {
                    const int rr = 16 * grp + 8 * odd + r8;
                    float2 wv = pair_get(R3, 64, rr, ie), vv = pair_get(R3 + 16384, 64, rr, ie);
                    if (kPacked && rr >= len) wv = vv = make_float2(0.f, 0.f);  // past the sequence
                    pair_split_put(R1, R1 + 16384, 64, rr, ie, wv.x * vv.x, wv.y * vv.y);
                }
            }
            fence_async_smem();
            fence_before_sync();
            go = __syncthreads_and(go) != 0;
            fence_after_sync();
            if (go && tid == 0) {
                issue_term<64, 64, 128, true, false>(cdA, tdRT, false, R1, false, r > 0);  // P6a dA += dR Z^T
                mma_commit(&bar_gm);
            }
            if (go) {  // dv = dZ w over w's raw tile, dw = dZ v over v's
#pragma unroll
                for (int h4 = 0; h4 < 4; ++h4) {
                    const int c0 = 16 * grp + 4 * h4;
                    float az[4];
                    tmem_ld4(tmem_lane_addr(cZ, quad, c0), az);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int rr = c0 + e;
                        const float wv = rt_get(R3, 64, rr, i), vv = rt_get(R3 + 16384, 64, rr, i);
                        if constexpr (kPacked) {  // a tile store cannot stop at the sequence's end: rows
                            if (rr < len && t0 + rr < T) {
                                const size_t gi = (((size_t)bi * T + t0 + rr) * (H * NG) + hv) * D + i;
                                gp.dv[gi] = __float2bfloat16_rn(az[e] * wv);
                                gp.dw[gi] = __float2bfloat16_rn(az[e] * vv);
                            }
                        } else {  // in place, then one tile store per tensor
                            put_bf16(R3, rr, i, az[e] * wv);
                            put_bf16(R3 + 16384, rr, i, az[e] * vv);
                        }
                    }
                }
            }
            fence_async_smem();
            fence_before_sync();
            go = __syncthreads_and(go) != 0;
            fence_after_sync();
            if (!kPacked && go && tid == 0) {  // rows past T fall outside the tensors and are not written
                tma_store_4d(&maps.dv, R3, 0, hv, t0, bi);
                tma_store_4d(&maps.dv, R3 + 8192, 64, hv, t0, bi);
                tma_store_4d(&maps.dw, R3 + 16384, 0, hv, t0, bi);
                tma_store_4d(&maps.dw, R3 + 16384 + 8192, 64, hv, t0, bi);
                bulk_commit();
            }
            go = go && mbar_wait(&bar_gm, gm_ph & 1u);  // P6a has read dR^T and Z
            ++gm_ph;
            fence_after_sync();
            if (go && tid == 0) {
                bulk_wait_read<0>();  // the dv / dw stores have read R^T's region
                if (r + 1 < NG) load_vimgs(vchunk(chn, r + 1), hv + 1, t0, bi, &bar_gl);
            }
        }
    } else {
    go = go && mbar_wait(&bar_p1, par);
    fence_after_sync();
    if (go && tid == 0) {  // phase 1: every product whose operands are all in the first load
        issue_term<64, 64, 128, false, true>(cAqk, tdO, true, tRT, false, false);    // P1  dA_qk
        issue_term<128, 64, 128, true, true>(cY, tS0, false, tdRT, false, false);    // P4  S_0 dR^T = -dY^T
        issue_term<128, 64, 64, false, true>(cZ, tdRT, false, tA, false, false);     // P5  dZ^T
        issue_term<128, 64, 128, true, true>(cKt, tdS, false, tRT, false, false);    // P3  dK_tail^T
        issue_term<128, 64, 128, true, false>(cQg, tS0, false, tdO, true, false);    // P2a dQ_gamma^T
        issue_term<128, 128, 128, true, true>(cX, tdS, false, tS0, false, false);    // dS_C S_0^T
        mma_commit(&bar_m1);
    }
    go = go && mbar_wait(&bar_m1, par);
    fence_after_sync();
    if (go && tid == 0) issue_p2();  // phase 1 has read S_0^T and dS_C^T: their regions take the raw inputs
    }
    float dgC = 0.f;  // dgamma_C[i] = (dS_C S_0^T)[i][i]
    if constexpr (kGroup) {  // lane pairs swap halves: the even lane ends with column i & ~1, the odd one with i | 1
        const int odd = tid & 1;
        const float mine = odd ? dgc1 : dgc0, other = __shfl_xor_sync(0xffffffffu, odd ? dgc0 : dgc1, 1);
        tmem_st1_nowait(tmem_lane_addr(cX + grp, quad, 0), mine + other);  // this segment's share of dgamma_C[i]
    } else {  // lane i, column i of the product
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
            float d16[16];
            tmem_ld16(tmem_lane_addr(cX, quad, 32 * quad + 16 * h16), d16);
            const int lane = tid & 31;
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (16 * h16 + e == lane) dgC = d16[e];
        }
    }
    tmem_st1_nowait(tmem_lane_addr(cSeg + grp, quad, 0), G[15]);  // segment sum of the log-decay
    tmem_st_wait();
    fence_before_sync();
    go = __syncthreads_and(go) != 0;  // S_0^T, dS_C^T, R^T and dO are no longer read
    fence_after_sync();
    if constexpr (kGroup) {
        if (go && tid == 0) issue_p2();  // (the last value head's P6a has read Z's region)
        float dp[4];  // the four segments' shares in a fixed order
        tmem_ld4(tmem_lane_addr(cX, quad, 0), dp);
        dgC = (dp[0] + dp[1]) + (dp[2] + dp[3]);
    }
    float GC;
    {
        float seg[4];
        tmem_ld4(tmem_lane_addr(cSeg, quad, 0), seg);
        float off = 0.f;
        GC = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (x < grp) off += seg[x];
            GC += seg[x];
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) G[rr] = off + G[rr];
    }
    // As in the forward, Q_gamma, Kbar and Ebar enter the products relative to the channel's mid-chunk
    // log-decay m = G_C / 2 (Q' = q e^{G - m}, K' = k e^{m - G}, E' = b k e^{G - m}). With dY and P2a's
    // share of dQ_gamma scaled by e^{m} here, every accumulator carries one known factor per channel:
    // dQ' = dQ_gamma e^{m}, dE' = dEbar e^{m}, dK' = dKbar e^{-m} (and dY' Ebar'^T = dY Ebar^T in dA), which
    // the assembly removes with e^{G - m} and e^{m - G}, both at most e^{|G_C| / 2}.
    const float em = __expf(0.5f * GC);
    m64_to_tile(cAqk, tdAqk, 1);  // dA_qk image (tril)
    {
        float vy[16];  // dY'^T = -(S_0 dR^T) e^{m}
        tmem_ld16(tmem_lane_addr(cY, quad, 16 * grp), vy);
#pragma unroll
        for (int e = 0; e < 16; ++e) vy[e] = -vy[e] * em;
        split_store8(tdY, tdY + 16384, 128, i, 16 * grp, vy);
        split_store8(tdY, tdY + 16384, 128, i, 16 * grp + 8, vy + 8);
        float vq[16];  // P2a's share of dQ' (P2b accumulates dA_qk K' onto it)
        tmem_ld16(tmem_lane_addr(cQg, quad, 16 * grp), vq);
#pragma unroll
        for (int e = 0; e < 16; ++e) vq[e] *= em;
        tmem_st16(tmem_lane_addr(cQg, quad, 16 * grp), vq);
    }
    go = go && mbar_wait(&bar_p2, par);
    {  // Q', K', E', Z (hi / lo) from the raw tiles, in place; lanes 2p, 2p + 1 share rows as in the forward
       // (the even lane takes rows 0..7 of the segment, the odd lane rows 8..15, both channels)
        const int odd = tid & 1, ie = i & ~1;
        float gpa[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) gpa[rr] = __shfl_xor_sync(0xffffffffu, G[rr], 1);
        const float GCpa = __shfl_xor_sync(0xffffffffu, GC, 1);
        const float m0 = 0.5f * (odd ? GCpa : GC), m1 = 0.5f * (odd ? GC : GCpa);  // channels ie, ie + 1
        if (go) {
#pragma unroll
            for (int r8 = 0; r8 < 8; ++r8) {
                const int r = 16 * grp + 8 * odd + r8;
                const float gm = odd ? G[r8 + 8] : G[r8], gp = odd ? gpa[r8 + 8] : gpa[r8];
                const float g0 = odd ? gp : gm, g1 = odd ? gm : gp;
                float2 qq = pair_get(tQg + 16384, 64, r, ie), kk = pair_get(tKb + 16384, 64, r, ie);
                float2 bb = pair_get(tEb + 16384, 64, r, ie), wv = pair_get(tZ, 64, r, ie);
                float2 vv = pair_get(tZ + 16384, 64, r, ie);
                if (r >= len) qq = kk = bb = wv = vv = make_float2(0.f, 0.f);
                const float t0 = g0 - m0, t1 = g1 - m1;
                const float ep0 = __expf(t0), en0 = __expf(-t0), ep1 = __expf(t1), en1 = __expf(-t1);
                pair_split_put(tQg, tQg + 16384, 64, r, ie, qq.x * ep0, qq.y * ep1);
                pair_split_put(tKb, tKb + 16384, 64, r, ie, kk.x * en0, kk.y * en1);
                pair_split_put(tEb, tEb + 16384, 64, r, ie, bb.x * kk.x * ep0, bb.y * kk.y * ep1);
                if (!kGroup) pair_split_put(tZ, tZ + 16384, 64, r, ie, wv.x * vv.x, wv.y * vv.y);
            }
        }
    }
    fence_async_smem();
    fence_before_sync();
    go = __syncthreads_and(go) != 0;
    fence_after_sync();
    if (go && tid == 0) {
        if (!kGroup)  // (grouped heads: dR Z^T already sums over the value heads in dA)
            issue_term<64, 64, 128, true, false>(cdA, tdRT, false, tZ, false, false);  // P6  dA = dR Z^T
        issue_term<64, 64, 128, true, false>(cdA, tdY, false, tEb, false, true);     //         + dY Ebar^T
        mma_commit(&bar_m2);
        issue_term<128, 64, 64, true, false>(cQg, tKb, false, tdAqk, false, true);   // P2b
        issue_term<128, 64, 64, false, true>(cEb, tdY, false, tA, false, false);     // P8a
        issue_term<128, 64, 64, true, true>(cKb, tQg, false, tdAqk, false, false);   // P9a
    }
    go = go && mbar_wait(&bar_m2, par);
    fence_after_sync();
    m64_to_tile(cdA, tdA, 0);  // dR^T is dead once P5 and P6 are done
    fence_async_smem();
    fence_before_sync();
    go = __syncthreads_and(go) != 0;
    fence_after_sync();
    if (go && tid == 0) {  // P7a  X = A^T dA
        issue_term<64, 64, 64, true, true>(cX, tA, false, tdA, false, false);
        mma_commit(&bar_m3);
    }
    go = go && mbar_wait(&bar_m3, par);
    fence_after_sync();
    if (go && tid == 0) {  // raw tiles for the assembly, into regions whose last reader has finished
        constexpr int nraw = kGroup ? 3 : 4;  // grouped heads: dv and dw have left already
        mbar_expect_tx(&bar_p3, (uint32_t)(nraw + (kGroup ? 0 : 1)) * 16384u);
        uint8_t *dst[4] = {rq, rk, rb, rv};
        const CUtensorMap *mp[4] = {&maps.q, &maps.k, &maps.b, &maps.v};
        for (int x = 0; x < nraw; ++x) {
            tma_load_4d(dst[x], mp[x], 0, h, t0, bi, &bar_p3);
            tma_load_4d(dst[x] + 8192, mp[x], 64, h, t0, bi, &bar_p3);
        }
    }
    m64_to_tile(cX, tX, 0);
    fence_async_smem();
    fence_before_sync();
    go = __syncthreads_and(go) != 0;
    fence_after_sync();
    if (go && tid == 0) {  // P7b  X A^T
        issue_term<64, 64, 64, false, false>(cdT, tX, false, tA, false, false);
        mma_commit(&bar_m4);
    }
    go = go && mbar_wait(&bar_m4, par);
    fence_after_sync();
    if (!kGroup && go && tid == 0) {  // raw w into A's tile (A's last reader, P7b, has finished)
        tma_load_4d(rw, &maps.w, 0, h, t0, bi, &bar_p3);
        tma_load_4d(rw + 8192, &maps.w, 64, h, t0, bi, &bar_p3);
    }
    m64_to_tile(cdT, tdT, 2);  // dT = -tril(X A^T, -1), into Z's hi slot (Z is dead after P6)
    fence_async_smem();
    fence_before_sync();
    go = __syncthreads_and(go) != 0;
    fence_after_sync();
    if (go && tid == 0) {
        issue_term<128, 64, 64, true, false>(cEb, tKb, false, tdT, false, true);     // P8b
        issue_term<128, 64, 64, true, true>(cKb, tEb, false, tdT, false, true);      // P9b
        mma_commit(&bar_m5);
    }
    go = go && mbar_wait(&bar_m5, par);
    go = go && mbar_wait(&bar_p3, par);
    fence_after_sync();
    go = __syncthreads_and(go) != 0;  // every tile but the raw inputs is free for the outputs

    // ---- assembly ----------------------------------------------------------------------------------
    // Gradients are written in place over the raw tile their element was read from; dG goes to TMEM
    // (lane i, columns cX + 16 grp ..) for the reverse cumulative sum.
    const float gC = expf(GC), mq = 0.5f * GC, ehalf = __expf(GC - mq);  // ehalf = e^{G_C / 2}
    float tail = 0.f, dsum = 0.f;
#pragma unroll
    for (int h4 = 0; h4 < 4; ++h4) {
        const int c0 = 16 * grp + 4 * h4;
        float aq[4], ae[4], ab[4], at[4], az[4], dg4[4];
        {  // the five accumulators of these four rows behind one wait
            uint32_t rq4[4], re4[4], rb4[4], rt4[4], rz4[4];
            tmem_ld4_issue(tmem_lane_addr(cQg, quad, c0), rq4);
            tmem_ld4_issue(tmem_lane_addr(cEb, quad, c0), re4);
            tmem_ld4_issue(tmem_lane_addr(cKb, quad, c0), rb4);
            tmem_ld4_issue(tmem_lane_addr(cKt, quad, c0), rt4);
            if (!kGroup) tmem_ld4_issue(tmem_lane_addr(cZ, quad, c0), rz4);
            tmem_ld_wait();
            tmem_ld4_take(rq4, aq);
            tmem_ld4_take(re4, ae);
            tmem_ld4_take(rb4, ab);
            tmem_ld4_take(rt4, at);
            if (!kGroup) tmem_ld4_take(rz4, az);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int rr = 4 * h4 + e, r = c0 + e;
            const float kk = rt_get(rk, 64, r, i), bb = rt_get(rb, 64, r, i), qq = rt_get(rq, 64, r, i);
            // aq = dQ_gamma e^{m}, ae = dEbar e^{m}, ab = dKbar e^{-m}: gamma = e^{G} and 1 / gamma enter as
            // ep = e^{G - m} and en = e^{m - G}; gamma_C / gamma = e^{G_C / 2} en <= 1
            const float tm = G[rr] - mq, ep = __expf(tm), en = __expf(-tm), gt = ehalf * en;
            const float kt = kk * gt;
            const bool live = r < len;  // rows past a packed sequence's end add nothing to the decay sums
            dg4[e] = live ? aq[e] * (qq * ep) + ae[e] * (bb * kk * ep) - ab[e] * (kk * en) - at[e] * kt : 0.f;
            dsum += dg4[e];
            tail = live ? fmaf(at[e], kt, tail) : tail;
            if (go && live && t0 + r < T) {  // rows past T or past a packed sequence's end are not written
                const size_t gi = (((size_t)bi * T + t0 + r) * H + h) * D + i;
                gp.dq[gi] = __float2bfloat16_rn(aq[e] * ep);
                gp.db[gi] = __float2bfloat16_rn(ae[e] * kk * ep);
                gp.dk[gi] = __float2bfloat16_rn(ae[e] * bb * ep + ab[e] * en + at[e] * gt);
                if (!kGroup) {
                    const float vv = rt_get(rv, 64, r, i), wv = rt_get(rw, 64, r, i);
                    gp.dw[gi] = __float2bfloat16_rn(az[e] * vv);
                    gp.dv[gi] = __float2bfloat16_rn(az[e] * wv);
                }
            }
        }
        tmem_st4_nowait(tmem_lane_addr(cX, quad, c0), dg4);
    }
    tmem_st1_nowait(tmem_lane_addr(cdA + grp, quad, 0), dsum);  // per-segment sums, exchanged through TMEM lane i
    tmem_st1_nowait(tmem_lane_addr(cdA + 4 + grp, quad, 0), tail);
    tmem_st_wait();
    fence_async_smem();
    fence_before_sync();
    go = __syncthreads_and(go) != 0;  // the raw tiles are read: every shared region is free for the next chunk
    fence_after_sync();
    if (go && tid == 0 && nxt < nchunks) {
        load_p1(nxt, 0);
        load_p1(nxt, 1);
    }
    if (kCarryLa && nxt < nchunks) load_la(nxt);
    // dlog_alpha[r] = (dgamma_C gamma_C + sum_r dK_tail K_tail) + sum_{r' >= r} dG[r'], stored as fp32 rows
    {
        float segD[4], segT[4], dgv[16];
        tmem_ld4(tmem_lane_addr(cdA, quad, 0), segD);
        tmem_ld4(tmem_lane_addr(cdA + 4, quad, 0), segT);
        tmem_ld16(tmem_lane_addr(cX, quad, 16 * grp), dgv);
        float run = dgC * gC;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            run += segT[x];
            if (x > grp) run += segD[x];
        }
#pragma unroll
        for (int rr = 15; rr >= 0; --rr) {
            run += dgv[rr];
            const int t = t0 + 16 * grp + rr;
            if (go && t < T && 16 * grp + rr < len) dla[(((size_t)bi * T + t) * H + h) * D + i] = run;
        }
    }
    fence_before_sync();
    __syncthreads();  // TMEM read out before the next chunk's first products overwrite it
    fence_after_sync();
    }  // chunk loop
    if (tid == 0 && !go) mma_drain(&bar_x);  // a wait gave up: the products issued finish before TMEM is freed
    if (tid == 0) bulk_wait_all<0>();
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}
// =================================================================================================
// Serial combine of the chunk-level scan, one (batch, head) chain per thread-block cluster, fp32.
//   forward  (backward = 0): S_{s+1} = M_s S_s + N_s from the initial state; Sout[s] = state entering segment s
//   backward (backward = 1): E_{s-1} = M_s^T E_s + dN_s from dS_T; Sout[s] = gradient at segment s's end
// Each of the cluster's 8 CTAs forms 16 rows of the next state from its rows of M_s (or columns, for M_s^T)
// and the whole running state, and broadcasts those rows into every CTA's copy of the state through
// distributed shared memory; the copy is double-buffered, so one cluster barrier per step suffices.
// =================================================================================================
constexpr int kCombRanks = 8;              // CTAs per chain
constexpr int kCombRows = D / kCombRanks;  // rows of the state formed by one CTA
constexpr size_t kCombineSmem = 2 * kStateBytes + (size_t)kCombRows * D * 4 + 1024;

__global__ void __cluster_dims__(kCombRanks, 1, 1) __launch_bounds__(256, 1)
    scan_combine_kernel(const float *__restrict__ Mb, const float *__restrict__ Nb, const float *__restrict__ Sinit,
                        float *__restrict__ Sout, int nseg, int BH, int backward) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    extern __shared__ uint8_t smem_raw[];
    float *Sbuf = reinterpret_cast<float *>(align1024(smem_raw));  // [2][k][j]: the running state, all rows
    float *Asm = Sbuf + 2 * D * D;                                  // [k][ii]: M[i0 + ii][k] or M[k][i0 + ii]
    const int rank = (int)cl.block_rank(), bh = blockIdx.x / kCombRanks, tid = threadIdx.x;
    const int i0 = rank * kCombRows;
    const int rq = tid >> 6, cp = tid & 63;  // this thread's outputs: rows i0 + 4 rq + {0..3}, columns 2 cp + {0, 1}
    const size_t DD = (size_t)D * D;

    // operand element e (of 8) of this thread for segment s: Asm index x = tid + 256 e, k = x / 16, ii = x % 16
    float a_next[8];
    float2 n_next[4];
    auto fetch = [&](int s) {
        const float *M = Mb + ((size_t)s * BH + bh) * DD;
        const float *N = Nb + ((size_t)s * BH + bh) * DD;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int x = tid + 256 * e, k = x >> 4, ii = x & 15;
            a_next[e] = backward ? __ldg(M + (size_t)k * D + i0 + ii) : __ldg(M + (size_t)(i0 + ii) * D + k);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
            n_next[e] = __ldg(reinterpret_cast<const float2 *>(N + (size_t)(i0 + 4 * rq + e) * D + 2 * cp));
    };

    const int s_first = backward ? nseg - 1 : 0;
    fetch(backward ? nseg - 1 : 0);
    for (int x = tid; x < D * D; x += 256) {
        const float v = Sinit ? Sinit[bh * DD + x] : 0.f;
        Sbuf[x] = v;
        if (x >= i0 * D && x < (i0 + kCombRows) * D) Sout[((size_t)s_first * BH + bh) * DD + x] = v;
    }
    cl.sync();  // every CTA of the cluster runs before any writes into another's shared memory
    for (int step = 0; step < nseg - 1; ++step) {
        const int s = backward ? nseg - 1 - step : step;  // segment whose transfer is applied
        const int so = backward ? s - 1 : s + 1;           // segment whose entry is produced
        const float *S = Sbuf + (size_t)(step & 1) * DD;
        float *Snext = Sbuf + (size_t)((step + 1) & 1) * DD;
#pragma unroll
        for (int e = 0; e < 8; ++e) Asm[tid + 256 * e] = a_next[e];
        float2 nv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) nv[e] = n_next[e];
        __syncthreads();  // Asm written; the running state is complete since the last cluster barrier
        if (step + 1 < nseg - 1) fetch(backward ? s - 1 : s + 1);
        float acc[4][2] = {};
#pragma unroll 8
        for (int k = 0; k < D; ++k) {
            const float4 a = *reinterpret_cast<const float4 *>(Asm + k * kCombRows + 4 * rq);
            const float2 b = *reinterpret_cast<const float2 *>(S + k * D + 2 * cp);
            acc[0][0] = fmaf(a.x, b.x, acc[0][0]);
            acc[0][1] = fmaf(a.x, b.y, acc[0][1]);
            acc[1][0] = fmaf(a.y, b.x, acc[1][0]);
            acc[1][1] = fmaf(a.y, b.y, acc[1][1]);
            acc[2][0] = fmaf(a.z, b.x, acc[2][0]);
            acc[2][1] = fmaf(a.z, b.y, acc[2][1]);
            acc[3][0] = fmaf(a.w, b.x, acc[3][0]);
            acc[3][1] = fmaf(a.w, b.y, acc[3][1]);
        }
        float *O = Sout + ((size_t)so * BH + bh) * DD;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int off = (i0 + 4 * rq + e) * D + 2 * cp;
            const float2 v = make_float2(acc[e][0] + nv[e].x, acc[e][1] + nv[e].y);
            *reinterpret_cast<float2 *>(O + off) = v;
#pragma unroll
            for (int q = 0; q < kCombRanks; ++q)
                *reinterpret_cast<float2 *>(cl.map_shared_rank(Snext + off, q)) = v;
        }
        cl.sync();  // every CTA holds the whole next state; nobody reads the old buffer any more
    }
}

// =================================================================================================
// Packed batches: the chunk and sequence tables from cu_seqlens, and the copy of the staged outputs.
// =================================================================================================
// One CTA. Sequence n covers tokens [B_n, B_{n+1}) with B_n the running maximum of cu_seqlens[0..n]
// clamped to [0, T]: for a valid cu_seqlens (0 = c_0 <= c_1 <= ... <= c_N = T) that is exactly
// [c_n, c_{n+1}); any other input still gives disjoint sequences inside the packed axis, so no launch
// reads or writes out of bounds. The chunks of all sequences then number at most T / 64 + N = G.
constexpr int kIndexThreads = 1024;
constexpr int kOrderMax = 4096;  // sequences sorted by length (more keep their order)

__global__ void __launch_bounds__(kIndexThreads)
    varlen_index_kernel(const int *__restrict__ cu, int N, int T, int G, int4 *__restrict__ chunk,
                        int4 *__restrict__ seq, int *__restrict__ order) {
    __shared__ int sc[kIndexThreads];
    __shared__ int cnt_s[kOrderMax];
    __shared__ int carry_tok, carry_chunk;
    const int tid = threadIdx.x;
    if (tid == 0) {
        carry_tok = min(max(cu[0], 0), T);
        carry_chunk = 0;
    }
    __syncthreads();
    for (int base = 0; base < N; base += kIndexThreads) {
        const int n = base + tid;
        sc[tid] = n < N ? min(max(cu[n + 1], 0), T) : 0;
        __syncthreads();
        for (int off = 1; off < kIndexThreads; off <<= 1) {  // inclusive running maximum over the tile
            const int v = tid >= off ? sc[tid - off] : 0;
            __syncthreads();
            sc[tid] = max(sc[tid], v);
            __syncthreads();
        }
        const int hi = max(carry_tok, sc[tid]);
        const int lo = max(carry_tok, tid > 0 ? sc[tid - 1] : 0);
        const int len = n < N ? hi - lo : 0, cnt = (len + C - 1) / C;
        __syncthreads();
        sc[tid] = cnt;
        __syncthreads();
        for (int off = 1; off < kIndexThreads; off <<= 1) {  // inclusive running sum of the chunk counts
            const int v = tid >= off ? sc[tid - off] : 0;
            __syncthreads();
            sc[tid] += v;
            __syncthreads();
        }
        const int first = carry_chunk + sc[tid] - cnt;
        if (n < N) seq[n] = make_int4(first, cnt, lo, len);
        if (n < N && n < kOrderMax) cnt_s[n] = cnt;
        __syncthreads();
        if (tid == kIndexThreads - 1) {
            carry_tok = hi;
            carry_chunk = first + cnt;
        }
        __syncthreads();
    }
    const int total = carry_chunk;
    // Longest first: sequence n goes to position #{m: cnt_m > cnt_n, or cnt_m = cnt_n and m < n}. Beyond
    // kOrderMax sequences they keep their order.
    for (int n = tid; n < N; n += kIndexThreads) {
        if (N > kOrderMax) {
            order[n] = n;
            continue;
        }
        const int cn = cnt_s[n];
        int r = 0;
        for (int m = 0; m < N; ++m) {
            const int cm = cnt_s[m];
            r += (cm > cn || (cm == cn && m < n)) ? 1 : 0;
        }
        order[r] = n;
    }
    for (int g = tid; g < G; g += kIndexThreads) {
        if (g >= total) {  // slots past the last sequence: empty chunks, outputs to the spare staging slot
            chunk[g] = make_int4(0, 0, N, -1);
            continue;
        }
        int a = 0, b = N - 1;  // the last sequence whose first chunk is <= g holds chunk g
        while (a < b) {
            const int mid = (a + b + 1) >> 1;
            if (seq[mid].x <= g) a = mid;
            else b = mid - 1;
        }
        const int4 sq = seq[a];
        const int j = g - sq.x, rows = min(C, sq.w - C * j);
        chunk[g] = make_int4(sq.z + C * j, rows, rows < C ? a : -1, a);
    }
}

struct PackedOut {
    __nv_bfloat16 *p[5];
};

// grid (N, tensors): the valid rows of sequence n's staged last chunk into the packed output. A staging
// slot [64][H][128] and the packed tensor [T][H][128] share their row layout, so this is one linear copy.
__global__ void __launch_bounds__(256)
    varlen_fixup_kernel(Varlen vl, int H, const __nv_bfloat16 *__restrict__ part, PackedOut out) {
    const int n = blockIdx.x, x = blockIdx.y;
    const int4 sq = __ldg(vl.seq + n);
    if (sq.y == 0) return;
    const int4 e = __ldg(vl.chunk + sq.x + sq.y - 1);
    if (e.z < 0) return;
    const size_t row = (size_t)H * D;  // elements per token row
    const uint4 *src = reinterpret_cast<const uint4 *>(part + (size_t)(x * vl.nslot + e.z) * C * row);
    uint4 *dst = reinterpret_cast<uint4 *>(out.p[x] + (size_t)e.x * row);
    const int n16 = (int)((size_t)e.y * row / 8);
    for (int idx = threadIdx.x; idx < n16; idx += 256) dst[idx] = src[idx];
}

// -------------------------------------------------------------------------------------------------
// Streaming multiprocessors of the current device (grid size of the persistent kernels).
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0)
        return 148;
    return n;
}

// Raw token tensor [B, T, H, 128] (bf16): boxes of 64 channels x 64 tokens of one head.
bool tok_map(CUtensorMap *m, const void *p, int B, int T, int H) {
    uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)H * D * 2, (uint64_t)T * H * D * 2};
    uint32_t box[4] = {64, 1, 64, 1};
    return make_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool la_map(CUtensorMap *m, const float *p, int B, int T, int H) {
    uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    uint64_t str[3] = {(uint64_t)D * 4, (uint64_t)H * D * 4, (uint64_t)T * H * D * 4};
    uint32_t box[4] = {(uint32_t)D, 1, 64, 1};
    return make_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Chunk geometry of a call. Unpacked: B*H chains of NT = ceil(T/64) chunks, workspace entry
// (b*H + h)*NT + c. Packed (N sequences): NT = T/64 + N chunk slots per head, entry h*NT + g, one
// chain per (sequence, value head), never segmented.
// Grouped value heads: Hv = G H value heads; chains run over value heads, the key-side workspace entries
// over key heads (nchK) and the value-side ones over value heads (nchV).
struct Geo {
    int NT, chains, nseg;
    int G, Hv;
    size_t nchK, nchV;
};

Geo geometry(const ChunkArgs &a) {
    const int Hv = a.Hv > 0 ? a.Hv : a.H, G = Hv / a.H;
    if (a.N > 0) {
        const int slots = a.T / C + a.N;
        return Geo{slots, a.N * Hv, 1, G, Hv, (size_t)slots * a.H, (size_t)slots * Hv};
    }
    const int NT = (a.T + C - 1) / C, BHv = a.B * Hv;
    return Geo{NT, BHv, scan_segments(BHv, NT), G, Hv, (size_t)a.B * a.H * NT, (size_t)BHv * NT};
}

size_t fwd_arrays(const Geo &g) { return kFwdKeyPerChunk * g.nchK + kFwdValPerChunk * g.nchV; }
size_t bwd_arrays(const Geo &g) { return kBwdKeyPerChunk * g.nchK + kBwdValPerChunk * g.nchV; }

// Packed batches: the tables and the staging tiles follow the per-chunk arrays (o's tiles in every layout,
// the five gradients' tiles in the backward layout).
constexpr size_t kPartTile = (size_t)C * D * 2;  // one head's 64 x 128 bf16 tile
size_t align1k(size_t x) { return (x + 1023) & ~(size_t)1023; }

size_t packed_bytes(int N, int H, int G, bool bwd_layout) {
    return align1k((size_t)G * 16) + align1k((size_t)N * 16) + align1k((size_t)N * 4) +
           (size_t)(N + 1) * H * kPartTile * (bwd_layout ? 6 : 1);
}

struct Packed {
    Varlen vl{};
    __nv_bfloat16 *opart = nullptr, *gpart = nullptr;
};

Packed carve_packed(uint8_t *p, int N, int H, int G) {
    Packed pk;
    pk.vl.chunk = reinterpret_cast<const int4 *>(p);
    p += align1k((size_t)G * 16);
    pk.vl.seq = reinterpret_cast<const int4 *>(p);
    p += align1k((size_t)N * 16);
    pk.vl.order = reinterpret_cast<const int *>(p);
    p += align1k((size_t)N * 4);
    pk.vl.nslot = N + 1;
    pk.opart = reinterpret_cast<__nv_bfloat16 *>(p);
    pk.gpart = pk.opart + (size_t)(N + 1) * H * C * D;
    return pk;
}

// Workspace of a call: the forward arrays, the scan states, the backward arrays (bwd_layout), the
// packed-batch tables. The index kernel is launched here for packed calls.
struct Plan {
    Geo g;
    WsTC ws;
    WsBwd bw;
    Packed pk;
};

cudaError_t plan(const ChunkArgs &a, bool bwd_layout, cudaStream_t st, Plan *pl) {
    pl->g = geometry(a);
    const Geo &g = pl->g;
    uint8_t *base = (uint8_t *)a.workspace;
    pl->ws = carve_tc(base, g.nchK, g.nchV, g.chains, g.nseg);
    size_t off = fwd_arrays(g) + scan_fwd_bytes(g.chains, g.nseg);
    pl->bw = WsBwd{};
    if (bwd_layout) {
        pl->bw = carve_bwd(base + off, g.nchK, g.nchV, g.chains, g.nseg);
        off += bwd_arrays(g) + scan_bwd_bytes(g.chains, g.nseg);
    }
    pl->pk = Packed{};
    if (a.N == 0) return cudaSuccess;
    pl->pk = carve_packed(base + off, a.N, g.Hv, g.NT);  // o's staging tiles are per value head
    GDR2_LAUNCH("tc_varlen_index", st,
                varlen_index_kernel<<<1, kIndexThreads, 0, st>>>(a.cu_seqlens, a.N, a.T, g.NT,
                                                                 const_cast<int4 *>(pl->pk.vl.chunk),
                                                                 const_cast<int4 *>(pl->pk.vl.seq),
                                                                 const_cast<int *>(pl->pk.vl.order)));
    return cudaGetLastError();
}

cudaError_t run_fixup(const ChunkArgs &a, const Packed &pk, int Hv, const __nv_bfloat16 *part, PackedOut out,
                      int ntens, cudaStream_t st) {
    GDR2_LAUNCH("tc_varlen_fixup", st,
                varlen_fixup_kernel<<<dim3(a.N, ntens), 256, 0, st>>>(pk.vl, Hv, part, out));
    return cudaGetLastError();
}

cudaError_t run_local(const ChunkArgs &a, const Plan &pl, const WsBwd &bw, cudaStream_t st) {
    LocalMaps m;
    const int Hv = pl.g.Hv;  // v and w live on the value-head axis
    if (!tok_map(&m.q, a.q, a.B, a.T, a.H) || !tok_map(&m.k, a.k, a.B, a.T, a.H) ||
        !tok_map(&m.b, a.b, a.B, a.T, a.H) || !tok_map(&m.v, a.v, a.B, a.T, Hv) ||
        !tok_map(&m.w, a.w, a.B, a.T, Hv) || !la_map(&m.la, a.log_alpha, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    auto kern = a.N > 0 ? local_kernel<true> : local_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLocalSmem);
    if (e != cudaSuccess) return e;
    const int NT = pl.g.NT;
    const int nchunks = a.B * a.H * NT;
    const int grid = std::min(nchunks, sm_count());
    GDR2_LAUNCH(bw.A ? "tc_local_train" : "tc_local", st,
                kern<<<grid, kLocalThreads, kLocalSmem, st>>>(m, pl.pk.vl, pl.ws, bw, a.T, a.H, pl.g.G, NT,
                                                              nchunks));
    return cudaGetLastError();
}

cudaError_t run_state(const ChunkArgs &a, const Plan &pl, const WsBwd &bw, bool fwd, cudaStream_t st) {
    const int NT = pl.g.NT, nseg = pl.g.nseg, BH = pl.g.chains, Hv = pl.g.Hv, G = pl.g.G;
    const WsTC &ws = pl.ws;
    CUtensorMap mo, mo_part;
    memset(&mo, 0, sizeof(mo));  // left zero when not read
    memset(&mo_part, 0, sizeof(mo_part));
    const int has_o = fwd && a.o != nullptr;
    if (has_o) {
        if (!tok_map(&mo, a.o, a.B, a.T, Hv)) return cudaErrorInvalidValue;
        if (a.N > 0 && !tok_map(&mo_part, pl.pk.opart, a.N + 1, C, Hv)) return cudaErrorInvalidValue;
    }
    auto kern = has_o ? state_kernel<true> : state_kernel<false>;  // phase A below never writes o
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(state_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kStateSmem)) != cudaSuccess)
        return e;
    const char *name = fwd ? (bw.S0T ? "tc_state_fwd_train" : "tc_state_fwd") : "tc_state_fwd_store";
    if (nseg == 1) {
        GDR2_LAUNCH(name, st,
                    kern<<<BH, has_o ? kStateIssuer : kStateBlock, kStateSmem, st>>>(
                        mo, mo_part, has_o, SegArgs{1, NT, 0, a.initial_state, fwd ? a.final_state : nullptr},
                        pl.pk.vl, ws, bw, a.T, Hv, G, NT, BH));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (has_o && a.N > 0) {
            PackedOut out{};
            out.p[0] = (__nv_bfloat16 *)a.o;
            return run_fixup(a, pl.pk, Hv, pl.pk.opart, out, 1, st);
        }
        return cudaSuccess;
    }
    const int L = (NT + nseg - 1) / nseg;
    GDR2_LAUNCH("tc_scan_fwd_transfer", st,
                state_kernel<false><<<2 * BH * nseg, kStateBlock, kStateSmem, st>>>(
                    mo, mo_part, 0, SegArgs{nseg, L, 1, nullptr, ws.scanA}, pl.pk.vl, ws, bw, a.T, Hv, G, NT, BH));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(scan_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kCombineSmem)) != cudaSuccess)
        return e;
    const size_t DD = (size_t)D * D;
    GDR2_LAUNCH("tc_scan_fwd_combine", st,
                scan_combine_kernel<<<BH * kCombRanks, 256, kCombineSmem, st>>>(
                    ws.scanA + (size_t)nseg * BH * DD, ws.scanA, a.initial_state, ws.scanS, nseg, BH, 0));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    GDR2_LAUNCH(name, st,
                kern<<<BH * nseg, has_o ? kStateIssuer : kStateBlock, kStateSmem, st>>>(
                    mo, mo_part, has_o, SegArgs{nseg, L, 0, ws.scanS, fwd ? a.final_state : nullptr}, pl.pk.vl, ws,
                    bw, a.T, Hv, G, NT, BH));
    return cudaGetLastError();
}

}  // namespace

bool tc_supported(const ChunkArgs &a) { return a.dtype == 1 && a.dk_ == 128 && a.dv_ == 128; }

size_t tc_workspace_bytes(int B, int T, int H, int for_bwd, int Hv) {
    ChunkArgs a{};
    a.B = B, a.T = T, a.H = H, a.Hv = Hv;
    const Geo g = geometry(a);
    return fwd_arrays(g) + scan_fwd_bytes(g.chains, g.nseg) +
           (for_bwd ? bwd_arrays(g) + scan_bwd_bytes(g.chains, g.nseg) : 0);
}

size_t tc_workspace_bytes_packed(int N, int T, int H, int for_bwd, int Hv) {
    ChunkArgs a{};
    a.B = 1, a.T = T, a.H = H, a.N = N, a.Hv = Hv;
    const Geo g = geometry(a);
    return fwd_arrays(g) + (for_bwd ? bwd_arrays(g) : 0) + packed_bytes(N, g.Hv, g.NT, for_bwd != 0);
}

cudaError_t launch_tc_fwd(const ChunkArgs &a, cudaStream_t st) {
    Plan pl;
    cudaError_t e = plan(a, false, st, &pl);
    if (e != cudaSuccess) return e;
    if ((e = run_local(a, pl, WsBwd{}, st)) != cudaSuccess) return e;
    return run_state(a, pl, WsBwd{}, true, st);
}

cudaError_t launch_tc_fwd_train(const ChunkArgs &a, cudaStream_t st) {
    Plan pl;
    cudaError_t e = plan(a, true, st, &pl);
    if (e != cudaSuccess) return e;
    if ((e = run_local(a, pl, pl.bw, st)) != cudaSuccess) return e;
    return run_state(a, pl, pl.bw, true, st);  // o and final state, plus the per-chunk state and R^T images
}

cudaError_t launch_tc_bwd(const ChunkArgs &a, cudaStream_t st, bool saved) {
    Plan pl;
    cudaError_t e = plan(a, true, st, &pl);
    if (e != cudaSuccess) return e;
    const int NT = pl.g.NT, nseg = pl.g.nseg, BH = pl.g.chains, Hv = pl.g.Hv, G = pl.g.G;
    const WsTC &ws = pl.ws;
    const WsBwd &bw = pl.bw;
    if (!saved) {
        if ((e = run_local(a, pl, bw, st)) != cudaSuccess) return e;
        if ((e = run_state(a, pl, bw, false, st)) != cudaSuccess) return e;
    }
    // reverse serial pass
    CUtensorMap mdO;
    const int has_dO = a.d_o != nullptr;
    if (has_dO) {
        if (!tok_map(&mdO, a.d_o, a.B, a.T, Hv)) return cudaErrorInvalidValue;
    } else {
        memset(&mdO, 0, sizeof(mdO));  // never read
    }
    if ((e = cudaFuncSetAttribute(rev_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRevSmem)) !=
        cudaSuccess)
        return e;
    if (nseg == 1) {
        GDR2_LAUNCH("tc_state_rev", st,
                    rev_kernel<<<BH, kStateBlock, kRevSmem, st>>>(
                        mdO, has_dO, SegArgs{1, NT, 0, a.d_final_state, a.d_initial_state}, pl.pk.vl, ws, bw, a.T,
                        Hv, G, NT, BH));
    } else {  // chunk-level scan: offsets, combine with the forward's segment transfers (transposed), rerun
        const int L = (NT + nseg - 1) / nseg;
        const size_t DD = (size_t)D * D;
        GDR2_LAUNCH("tc_scan_rev_offset", st,
                    rev_kernel<<<BH * nseg, kStateBlock, kRevSmem, st>>>(
                        mdO, has_dO, SegArgs{nseg, L, 1, nullptr, bw.scanN}, pl.pk.vl, ws, bw, a.T, Hv, G, NT, BH));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = cudaFuncSetAttribute(scan_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kCombineSmem)) != cudaSuccess)
            return e;
        GDR2_LAUNCH("tc_scan_rev_combine", st,
                    scan_combine_kernel<<<BH * kCombRanks, 256, kCombineSmem, st>>>(
                        ws.scanA + (size_t)nseg * BH * DD, bw.scanN, a.d_final_state, bw.scanE, nseg, BH, 1));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        GDR2_LAUNCH("tc_state_rev", st,
                    rev_kernel<<<BH * nseg, kStateBlock, kRevSmem, st>>>(
                        mdO, has_dO, SegArgs{nseg, L, 0, bw.scanE, a.d_initial_state}, pl.pk.vl, ws, bw, a.T, Hv,
                        G, NT, BH));
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    BwdMaps bm;
    if (!tok_map(&bm.q, a.q, a.B, a.T, a.H) || !tok_map(&bm.k, a.k, a.B, a.T, a.H) ||
        !tok_map(&bm.b, a.b, a.B, a.T, a.H) || !tok_map(&bm.v, a.v, a.B, a.T, Hv) ||
        !tok_map(&bm.w, a.w, a.B, a.T, Hv) || !tok_map(&bm.dv, a.dv, a.B, a.T, Hv) ||
        !tok_map(&bm.dw, a.dw, a.B, a.T, Hv))
        return cudaErrorInvalidValue;
    bm.dO = mdO;
    const GradPtrs gp{(__nv_bfloat16 *)a.dq, (__nv_bfloat16 *)a.dk, (__nv_bfloat16 *)a.db, (__nv_bfloat16 *)a.dv,
                      (__nv_bfloat16 *)a.dw};
    auto bkern = a.N > 0 ? (G > 1 ? chunk_bwd_kernel<true, true> : chunk_bwd_kernel<true, false>)
                 : G > 1 ? chunk_bwd_kernel<false, true>
                         : chunk_bwd_kernel<false, false>;
    if ((e = cudaFuncSetAttribute(bkern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBwdSmem)) != cudaSuccess)
        return e;
    const int nchunks = a.B * a.H * NT;
    GDR2_LAUNCH("tc_bwd_chunk", st,
                bkern<<<std::min(nchunks, sm_count()), kBwdThreads, kBwdSmem, st>>>(
                    bm, gp, has_dO, a.log_alpha, pl.pk.vl, bw, a.dlog_alpha, a.T, a.H, G, NT, nchunks));
    return cudaGetLastError();  // (packed batches: the gradients are written row by row, no staging needed)
}

int status_take_tc() { return take_status(); }

}  // namespace gdr2
