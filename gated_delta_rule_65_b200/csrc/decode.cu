// decode.cu -- one-token recurrent decode step of the Gated Delta Rule-2 mixer.
//
// Follows the review's Appendix C.5 ("Recurrent decoding kernel") and the five steps of section
// "The Gated Delta Rule-2 State Update": the fp32 state is decayed by exp(g_t) row by row, read along
// e = b (.) k (r = Sbar^T e), written with z = w (.) v along k, and o = S_t^T q is returned. The
// output uses the identity S_t^T q = Sbar^T q + (k.q)(z - r), exact algebra on Step 4, so the state
// is read from HBM once and written once.
//
// The step is HBM-bound (131 KB of state traffic per (sequence, head) at dk = dv = 128 against
// 7*dk*dv flops). One CTA owns a [dk x COLS] column slice of one head's state (COLS = 128 when dv is
// a multiple of 128, with 512 threads, else 64 with 256 threads). Each thread keeps dk/16 rows x 4
// columns in registers as float4: a warp touches whole 512-byte (or two 256-byte) row segments per
// load, all loads are issued before the first barrier, and the state is streamed with evict-first
// loads and stores (it is touched once per step and is larger than L2).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace gdr2 {

template <int DK, int COLS, typename T>
__global__ void __launch_bounds__(COLS * 4) decode_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                          const T *__restrict__ v, const float *__restrict__ la,
                                                          const T *__restrict__ b, const T *__restrict__ w, float *S,
                                                          T *__restrict__ o, int DV) {
    constexpr int NTHR = COLS * 4;         // 256 threads for 64 columns, 512 for 128
    constexpr int NW = NTHR / 32;
    constexpr int LPR = COLS / 4;          // lanes per row (one float4 each)
    constexpr int RPW = 32 / LPR;          // rows per warp instruction
    constexpr int RPT = DK / (NW * RPW);   // rows per thread (= DK / 16)
    const int bh = blockIdx.x;
    const int col0 = blockIdx.y * COLS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cg = lane % LPR, sub = lane / LPR;
    float *Sb = S + (size_t)bh * DK * DV + col0 + cg * 4;
    auto row_of = [&](int m) { return m * (NW * RPW) + warp * RPW + sub; };

    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldcs(reinterpret_cast<const float4 *>(Sb + (size_t)row_of(m) * DV));

    __shared__ float sh_alpha[DK], sh_e[DK], sh_k[DK], sh_q[DK];
    __shared__ float4 sh_red[NW][LPR][2];
    if (tid < DK) {
        const size_t off = (size_t)bh * DK + tid;
        const float kk = to_f(k[off]);
        sh_alpha[tid] = expf(la[off]);
        sh_e[tid] = to_f(b[off]) * kk;
        sh_k[tid] = kk;
        sh_q[tid] = to_f(q[off]);
    }
    const size_t voff = (size_t)bh * DV + col0 + cg * 4;
    const float4 vv = load4(v + voff), ww = load4(w + voff);
    __syncthreads();

    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const int row = row_of(m);
        const float a = sh_alpha[row], e = sh_e[row], qq = sh_q[row];
        s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;            // Step 1
        r.x = fmaf(s[m].x, e, r.x); r.y = fmaf(s[m].y, e, r.y);         // Step 2 (partial)
        r.z = fmaf(s[m].z, e, r.z); r.w = fmaf(s[m].w, e, r.w);
        p.x = fmaf(s[m].x, qq, p.x); p.y = fmaf(s[m].y, qq, p.y);       // Sbar^T q (partial)
        p.z = fmaf(s[m].z, qq, p.z); p.w = fmaf(s[m].w, qq, p.w);
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {  // combine the rows held by one warp
        r.x += __shfl_xor_sync(0xffffffffu, r.x, off); r.y += __shfl_xor_sync(0xffffffffu, r.y, off);
        r.z += __shfl_xor_sync(0xffffffffu, r.z, off); r.w += __shfl_xor_sync(0xffffffffu, r.w, off);
        p.x += __shfl_xor_sync(0xffffffffu, p.x, off); p.y += __shfl_xor_sync(0xffffffffu, p.y, off);
        p.z += __shfl_xor_sync(0xffffffffu, p.z, off); p.w += __shfl_xor_sync(0xffffffffu, p.w, off);
    }
    if (sub == 0) {
        sh_red[warp][cg][0] = r;
        sh_red[warp][cg][1] = p;
    }
    float qk = 0.f;
    for (int i = lane; i < DK; i += 32) qk = fmaf(sh_q[i], sh_k[i], qk);
    qk = warp_sum(qk);
    __syncthreads();

    float4 R = sh_red[0][cg][0], P = sh_red[0][cg][1];
#pragma unroll
    for (int x = 1; x < NW; ++x) {
        const float4 a = sh_red[x][cg][0], c = sh_red[x][cg][1];
        R.x += a.x; R.y += a.y; R.z += a.z; R.w += a.w;
        P.x += c.x; P.y += c.y; P.z += c.z; P.w += c.w;
    }
    float4 d;                                                          // Step 3 and residual z - r
    d.x = ww.x * vv.x - R.x; d.y = ww.y * vv.y - R.y;
    d.z = ww.z * vv.z - R.z; d.w = ww.w * vv.w - R.w;
    if (warp == 0 && sub == 0) {                                       // Step 5
        float4 ov = make_float4(fmaf(qk, d.x, P.x), fmaf(qk, d.y, P.y), fmaf(qk, d.z, P.z), fmaf(qk, d.w, P.w));
        store4(o + voff, ov);
    }
#pragma unroll
    for (int m = 0; m < RPT; ++m) {                                    // Step 4
        const int row = row_of(m);
        const float kr = sh_k[row];
        float4 t = s[m];
        t.x = fmaf(kr, d.x, t.x); t.y = fmaf(kr, d.y, t.y);
        t.z = fmaf(kr, d.z, t.z); t.w = fmaf(kr, d.w, t.w);
        __stcs(reinterpret_cast<float4 *>(Sb + (size_t)row * DV), t);
    }
}


// Persistent streaming variant for dv = 128: a head's fp32 state (dk x 128, contiguous) and its token
// vectors move between HBM and shared memory as untiled bulk copies, three stages deep, so loads of
// head n+2 and the store of head n-1 overlap the update of head n. One CTA per SM, 256 threads; thread
// (sub, cg) owns rows sub + 8 m and columns 4 cg .. 4 cg + 3.
constexpr int kDecStages = 3;

template <int DK, typename T>
struct DecStage {
    static constexpr uint32_t kState = DK * 128 * 4;
    static constexpr uint32_t kVecK = ((DK * sizeof(T) + 15) / 16) * 16;
    static constexpr uint32_t kVecV = ((128 * sizeof(T) + 15) / 16) * 16;
    static constexpr uint32_t kLa = DK * 4;
    // layout: state | q | k | b | la | v | w
    static constexpr uint32_t oQ = kState, oK = oQ + kVecK, oB = oK + kVecK, oLa = oB + kVecK, oV = oLa + kLa,
                              oW = oV + kVecV, kBytes = oW + kVecV;
    static constexpr uint32_t kStride = ((kBytes + 127) / 128) * 128;
};

template <int DK, typename T>
__global__ void __launch_bounds__(256, 1) decode_stream_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                               const T *__restrict__ v, const float *__restrict__ la,
                                                               const T *__restrict__ b, const T *__restrict__ w,
                                                               float *S, T *__restrict__ o, int BH) {
    using L = DecStage<DK, T>;
    constexpr int RPT = DK / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ uint64_t full[kDecStages];
    __shared__ float sh_alpha[DK], sh_e[DK], sh_k[DK];
    __shared__ float4 sh_red[8][32][2];
    __shared__ float sh_qk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cg = lane, sub = warp;

    auto issue = [&](int item, int st) {
        GDR2_DCHECK(item >= 0 && item < BH && st >= 0 && st < kDecStages);
        uint8_t *sb = base + st * L::kStride;
        const size_t bh = (size_t)item;
        tc::mbar_expect_tx(&full[st], L::kState + 3 * DK * sizeof(T) + L::kLa + 2 * 128 * sizeof(T));
        tc::bulk_load(sb, S + bh * DK * 128, L::kState, &full[st]);
        tc::bulk_load(sb + L::oQ, q + bh * DK, DK * sizeof(T), &full[st]);
        tc::bulk_load(sb + L::oK, k + bh * DK, DK * sizeof(T), &full[st]);
        tc::bulk_load(sb + L::oB, b + bh * DK, DK * sizeof(T), &full[st]);
        tc::bulk_load(sb + L::oLa, la + bh * DK, L::kLa, &full[st]);
        tc::bulk_load(sb + L::oV, v + bh * 128, 128 * sizeof(T), &full[st]);
        tc::bulk_load(sb + L::oW, w + bh * 128, 128 * sizeof(T), &full[st]);
    };

    if (tid == 0) {
        for (int x = 0; x < kDecStages; ++x) tc::mbar_init(&full[x], 1);
        tc::mbar_fence_init();
        for (int x = 0; x < kDecStages - 1; ++x) {
            const int item = blockIdx.x + x * gridDim.x;
            if (item < BH) issue(item, x);
        }
    }
    __syncthreads();

    int j = 0;
    for (int item = blockIdx.x; item < BH; item += gridDim.x, ++j) {
        const int st = j % kDecStages;
        uint8_t *sb = base + st * L::kStride;
        float *Ss = reinterpret_cast<float *>(sb);
        const bool arrived = tc::mbar_wait(&full[st], (uint32_t)((j / kDecStages) & 1));
        if (!__syncthreads_and(arrived)) break;  // every thread leaves together
        if (tid < DK) {
            const float kk = to_f(reinterpret_cast<const T *>(sb + L::oK)[tid]);
            sh_alpha[tid] = expf(reinterpret_cast<const float *>(sb + L::oLa)[tid]);
            sh_e[tid] = to_f(reinterpret_cast<const T *>(sb + L::oB)[tid]) * kk;
            sh_k[tid] = kk;
        }
        if (warp == 0) {
            float x = 0.f;
            for (int i = lane; i < DK; i += 32)
                x = fmaf(to_f(reinterpret_cast<const T *>(sb + L::oQ)[i]), to_f(reinterpret_cast<const T *>(sb + L::oK)[i]), x);
            x = warp_sum(x);
            if (lane == 0) sh_qk = x;
        }
        __syncthreads();
        float4 s[RPT];
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f), p = r;
#pragma unroll
        for (int m = 0; m < RPT; ++m) {
            const int row = sub + 8 * m;
            s[m] = reinterpret_cast<const float4 *>(Ss + row * 128)[cg];
            const float a = sh_alpha[row], e = sh_e[row];
            const float qq = to_f(reinterpret_cast<const T *>(sb + L::oQ)[row]);
            s[m].x *= a; s[m].y *= a; s[m].z *= a; s[m].w *= a;            // Step 1
            r.x = fmaf(s[m].x, e, r.x); r.y = fmaf(s[m].y, e, r.y);         // Step 2 (partial)
            r.z = fmaf(s[m].z, e, r.z); r.w = fmaf(s[m].w, e, r.w);
            p.x = fmaf(s[m].x, qq, p.x); p.y = fmaf(s[m].y, qq, p.y);       // Sbar^T q (partial)
            p.z = fmaf(s[m].z, qq, p.z); p.w = fmaf(s[m].w, qq, p.w);
        }
        sh_red[sub][cg][0] = r;
        sh_red[sub][cg][1] = p;
        __syncthreads();
        float4 R = sh_red[0][cg][0], P = sh_red[0][cg][1];
#pragma unroll
        for (int x = 1; x < 8; ++x) {
            const float4 a = sh_red[x][cg][0], c = sh_red[x][cg][1];
            R.x += a.x; R.y += a.y; R.z += a.z; R.w += a.w;
            P.x += c.x; P.y += c.y; P.z += c.z; P.w += c.w;
        }
        const float4 vv = load4(reinterpret_cast<const T *>(sb + L::oV) + 4 * cg);
        const float4 ww = load4(reinterpret_cast<const T *>(sb + L::oW) + 4 * cg);
        float4 d;                                                          // Step 3 and residual z - r
        d.x = ww.x * vv.x - R.x; d.y = ww.y * vv.y - R.y;
        d.z = ww.z * vv.z - R.z; d.w = ww.w * vv.w - R.w;
        if (sub == 0) {                                                    // Step 5
            const float qk = sh_qk;
            store4(o + (size_t)item * 128 + 4 * cg,
                   make_float4(fmaf(qk, d.x, P.x), fmaf(qk, d.y, P.y), fmaf(qk, d.z, P.z), fmaf(qk, d.w, P.w)));
        }
#pragma unroll
        for (int m = 0; m < RPT; ++m) {                                    // Step 4, in place
            const int row = sub + 8 * m;
            const float kr = sh_k[row];
            float4 t = s[m];
            t.x = fmaf(kr, d.x, t.x); t.y = fmaf(kr, d.y, t.y);
            t.z = fmaf(kr, d.z, t.z); t.w = fmaf(kr, d.w, t.w);
            reinterpret_cast<float4 *>(Ss + row * 128)[cg] = t;
        }
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::bulk_store(S + (size_t)item * DK * 128, Ss, L::kState);
            tc::bulk_commit();
            const int nxt = item + (kDecStages - 1) * gridDim.x;
            if (nxt < BH) {
                tc::bulk_wait_read<1>();  // the store issued from that stage one round ago has read its data
                issue(nxt, (j + kDecStages - 1) % kDecStages);
            }
        }
    }
    if (tid == 0) tc::bulk_wait_all<0>();
}

template <int DK, typename T>
static bool launch_decode_stream(const DecodeArgs &a, cudaStream_t st) {
    using L = DecStage<DK, T>;
    const int smem = (int)(kDecStages * L::kStride + 128);
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return false;
    }
    if (cudaFuncSetAttribute(decode_stream_kernel<DK, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return false;
    const int BH = a.B * a.H;
    const int grid = BH < sms ? BH : sms;
    GDR2_LAUNCH("decode", st,
                (decode_stream_kernel<DK, T><<<grid, 256, smem, st>>>((const T *)a.q, (const T *)a.k, (const T *)a.v,
                                                                      a.log_alpha, (const T *)a.b, (const T *)a.w,
                                                                      a.state, (T *)a.o, BH)));
    return true;
}

template <int DK, typename T>
static void launch_decode_dk(const DecodeArgs &a, cudaStream_t st) {
    if (a.dv == 128 && launch_decode_stream<DK, T>(a, st)) return;
    dim3 grid(a.B * a.H, a.dv / 64);
    GDR2_LAUNCH("decode", st,
                (decode_kernel<DK, 64, T><<<grid, 256, 0, st>>>((const T *)a.q, (const T *)a.k, (const T *)a.v,
                                                               a.log_alpha, (const T *)a.b, (const T *)a.w, a.state,
                                                               (T *)a.o, a.dv)));
}

template <typename T>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t st) {
    if (a.dk == 128)
        launch_decode_dk<128, T>(a, st);
    else
        launch_decode_dk<64, T>(a, st);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
    return a.dtype == 1 ? launch_decode_t<__nv_bfloat16>(a, st) : launch_decode_t<float>(a, st);
}

int status_take_decode() { return take_status(); }

}  // namespace gdr2
