// prologue.cu -- the gate and normalisation prologue of the Gated Delta Rule-2 mixer (sm_100a).
//
// Per (token, head), from the branch pre-activations ("Gated DeltaNet-2", review page, section
// "Gate Parameterization", Eqs. 11-12, and "Block Design", steps 2-3):
//   q = x_q / ||x_q||,  k = x_k / ||x_k||              L2 normalisation per head (zero stays zero)
//   g = -exp(a) (.) softplus(x_f + delta)   (fp32)      Eq. 12; a, delta per head and key channel
//   b = sigmoid(x_b), times 2 for the negative-eigenvalue variant,  w = sigmoid(x_w)      Eq. 11
// The backward is the chain rule through those maps; da and ddelta sum over every token.
//
// Both directions are one pass over HBM. In the forward a warp takes two rows at a time (16 lanes per
// row, 16-byte accesses for bf16); in the backward, which holds twice the vectors per row, one row (32
// lanes). Row norms and dot products reduce over a row's lanes by shuffles. The backward's
// sums over tokens are deterministic: per-CTA partial sums, then a fixed-order sum per (head, channel).
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {
namespace {

constexpr int kProThreads = 256;  // 8 warps x 2 rows per step
constexpr int kProRows = 128;     // rows (tokens of one head) per CTA

// N consecutive floats stored from registers (N = 4 or 8; 8 bf16 = one 16-byte access).
template <int N> __device__ __forceinline__ void stv(float *p, const float *x) {
    if constexpr (N == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) *reinterpret_cast<float4 *>(p + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    }
}
template <int N> __device__ __forceinline__ void stv(__nv_bfloat16 *p, const float *x) {
    if constexpr (N == 8) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&b2);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (N == 4) {
        store4(p, make_float4(x[0], x[1], x[2], x[3]));
    } else {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(x[0], x[1]);
        *reinterpret_cast<__nv_bfloat162 *>(p) = b2;
    }
}

// N elements held as loaded (bf16 stay packed, two to a register) until they are converted: every load of
// a row can then be in flight at once without holding N floats per tensor.
template <typename T, int N> struct Raw;
template <int N> struct Raw<float, N> {
    float v[N];
    __device__ __forceinline__ void load(const float *p) {
        if constexpr (N == 2) {
            const float2 u = *reinterpret_cast<const float2 *>(p);
            v[0] = u.x, v[1] = u.y;
        } else {
#pragma unroll
            for (int i = 0; i < N / 4; ++i) {
                const float4 u = *reinterpret_cast<const float4 *>(p + 4 * i);
                v[4 * i] = u.x, v[4 * i + 1] = u.y, v[4 * i + 2] = u.z, v[4 * i + 3] = u.w;
            }
        }
    }
    __device__ __forceinline__ void get(float *x) const {
#pragma unroll
        for (int i = 0; i < N; ++i) x[i] = v[i];
    }
};
template <int N> struct Raw<__nv_bfloat16, N> {
    uint32_t v[N / 2];
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
        if constexpr (N == 8) {
            const uint4 u = *reinterpret_cast<const uint4 *>(p);
            v[0] = u.x, v[1] = u.y, v[2] = u.z, v[3] = u.w;
        } else if constexpr (N == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(p);
            v[0] = u.x, v[1] = u.y;
        } else {
            v[0] = *reinterpret_cast<const uint32_t *>(p);
        }
    }
    __device__ __forceinline__ void get(float *x) const {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v[i]));
            x[2 * i] = f.x, x[2 * i + 1] = f.y;
        }
    }
};

template <int L> __device__ __forceinline__ float sum_lanes(float v) {  // over aligned groups of L lanes
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float softplus(float x) { return x > 20.f ? x : log1pf(expf(x)); }

// The rows of a CTA: head h = blockIdx.x % H, tokens tb * kProRows + [0, kProRows) of the flattened
// (batch, time) axis, tb = blockIdx.x / H (heads vary fastest, so the CTAs in flight cover whole token
// rows of H * d elements). Lanes on a row past the end compute on the last row and store nothing, so every
// shuffle has all 32 lanes.
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kProThreads) prologue_fwd_kernel(PrologueArgs p) {
    constexpr int L = 16, CK = DK / L, CV = DV / L;  // lanes per row, channels per lane
    const int h = blockIdx.x % p.H, tb = blockIdx.x / p.H, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int half = lane / L, ck = (lane % L) * CK, cv = (lane % L) * CV;
    float ea[CK], dl[CK];
#pragma unroll
    for (int e = 0; e < CK; ++e) {
        ea[e] = expf(p.a[h * DK + ck + e]);
        dl[e] = p.delta[h * DK + ck + e];
    }
    const long long BT = (long long)p.B * p.T;
    const float bscale = p.neg_eig ? 2.f : 1.f;
    for (int it = 0; it < kProRows / 16; ++it) {
        const long long row = (long long)tb * kProRows + it * 16 + warp * 2 + half;
        const bool valid = row < BT;
        const long long r = valid ? row : BT - 1;
        const size_t ok = ((size_t)r * p.H + h) * DK + ck, ov = ((size_t)r * p.H + h) * DV + cv;
        // every load of the row first, so that they are all in flight together
        Raw<T, CK> rq, rk, rf, rb;
        Raw<T, CV> rw;
        rq.load(static_cast<const T *>(p.xq) + ok);
        rk.load(static_cast<const T *>(p.xk) + ok);
        rf.load(static_cast<const T *>(p.xf) + ok);
        rb.load(static_cast<const T *>(p.xb) + ok);
        rw.load(static_cast<const T *>(p.xw) + ov);
        float xq[CK], xk[CK], xf[CK], xb[CK], xw[CV];
        rq.get(xq);
        rk.get(xk);
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e = 0; e < CK; ++e) {
            sq = fmaf(xq[e], xq[e], sq);
            sk = fmaf(xk[e], xk[e], sk);
        }
        sq = sum_lanes<L>(sq);
        sk = sum_lanes<L>(sk);
        const float iq = sq > 0.f ? rsqrtf(sq) : 0.f, ik = sk > 0.f ? rsqrtf(sk) : 0.f;
#pragma unroll
        for (int e = 0; e < CK; ++e) {
            xq[e] *= iq;
            xk[e] *= ik;
        }
        if (valid) {
            stv<CK>(static_cast<T *>(p.q) + ok, xq);
            stv<CK>(static_cast<T *>(p.k) + ok, xk);
        }
        rf.get(xf);
        rb.get(xb);
#pragma unroll
        for (int e = 0; e < CK; ++e) {
            xf[e] = -ea[e] * softplus(xf[e] + dl[e]);
            xb[e] = bscale * sigm(xb[e]);
        }
        rw.get(xw);
#pragma unroll
        for (int e = 0; e < CV; ++e) xw[e] = sigm(xw[e]);
        if (valid) {
            stv<CK>(p.g + ok, xf);
            stv<CK>(static_cast<T *>(p.b) + ok, xb);
            stv<CV>(static_cast<T *>(p.w) + ov, xw);
        }
    }
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kProThreads) prologue_bwd_kernel(PrologueArgs p, float *__restrict__ partial) {
    // a whole warp per row: the backward holds ten loaded vectors per row, so fewer channels per lane
    // keep it at four CTAs per SM
    constexpr int L = 32, CK = DK / L, CV = DV / L;
    __shared__ float red[2][kProThreads / 32][DK];
    const int h = blockIdx.x % p.H, tb = blockIdx.x / p.H, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ck = lane * CK, cv = lane * CV;
    float ea[CK], dl[CK], acc_a[CK], acc_d[CK];
#pragma unroll
    for (int e = 0; e < CK; ++e) {
        ea[e] = expf(p.a[h * DK + ck + e]);
        dl[e] = p.delta[h * DK + ck + e];
        acc_a[e] = acc_d[e] = 0.f;
    }
    const long long BT = (long long)p.B * p.T;
    const float bscale = p.neg_eig ? 2.f : 1.f;
    for (int it = 0; it < kProRows / 8; ++it) {
        const long long row = (long long)tb * kProRows + it * 8 + warp;
        const bool valid = row < BT;
        const long long r = valid ? row : BT - 1;
        const size_t ok = ((size_t)r * p.H + h) * DK + ck, ov = ((size_t)r * p.H + h) * DV + cv;
        // every load of the row first, so that they are all in flight together
        Raw<T, CK> rq, rdq, rk, rdk, rf, rb, rdb;
        Raw<float, CK> rdg;
        Raw<T, CV> rw, rdw;
        rq.load(static_cast<const T *>(p.xq) + ok);
        rdq.load(static_cast<const T *>(p.dq) + ok);
        rk.load(static_cast<const T *>(p.xk) + ok);
        rdk.load(static_cast<const T *>(p.dk) + ok);
        rf.load(static_cast<const T *>(p.xf) + ok);
        rdg.load(p.dg + ok);
        rb.load(static_cast<const T *>(p.xb) + ok);
        rdb.load(static_cast<const T *>(p.db) + ok);
        rw.load(static_cast<const T *>(p.xw) + ov);
        rdw.load(static_cast<const T *>(p.dw) + ov);
        // dx = (dy - n (n . dy)) / ||x||, n = x / ||x||
        float xq[CK], dq[CK], xk[CK], dk[CK];
        rq.get(xq);
        rdq.get(dq);
        rk.get(xk);
        rdk.get(dk);
        float sq = 0.f, pq = 0.f, sk = 0.f, pk = 0.f;
#pragma unroll
        for (int e = 0; e < CK; ++e) {
            sq = fmaf(xq[e], xq[e], sq);
            pq = fmaf(xq[e], dq[e], pq);
            sk = fmaf(xk[e], xk[e], sk);
            pk = fmaf(xk[e], dk[e], pk);
        }
        sq = sum_lanes<L>(sq);
        pq = sum_lanes<L>(pq);
        sk = sum_lanes<L>(sk);
        pk = sum_lanes<L>(pk);
        const float iq = sq > 0.f ? rsqrtf(sq) : 0.f, nq = pq * iq * iq;
        const float ik = sk > 0.f ? rsqrtf(sk) : 0.f, nk = pk * ik * ik;
#pragma unroll
        for (int e = 0; e < CK; ++e) {
            xq[e] = (dq[e] - xq[e] * nq) * iq;
            xk[e] = (dk[e] - xk[e] * nk) * ik;
        }
        if (valid) {
            stv<CK>(static_cast<T *>(p.dxq) + ok, xq);
            stv<CK>(static_cast<T *>(p.dxk) + ok, xk);
        }
        float xf[CK], dg[CK], xb[CK], db[CK], xw[CV], dw[CV];
        rf.get(xf);
        rdg.get(dg);
        rb.get(xb);
        rdb.get(db);
#pragma unroll
        for (int e = 0; e < CK; ++e) {
            // dg/dx_f = -exp(a) sigmoid(x_f + delta); dg/da = g
            const float z = xf[e] + dl[e];
            const float gx = -ea[e] * sigm(z) * dg[e];
            if (valid) {
                acc_a[e] = fmaf(dg[e], -ea[e] * softplus(z), acc_a[e]);
                acc_d[e] += gx;
            }
            xf[e] = gx;
            const float sb = sigm(xb[e]);
            xb[e] = db[e] * bscale * sb * (1.f - sb);
        }
        rw.get(xw);
        rdw.get(dw);
#pragma unroll
        for (int e = 0; e < CV; ++e) {
            const float sw = sigm(xw[e]);
            xw[e] = dw[e] * sw * (1.f - sw);
        }
        if (valid) {
            stv<CK>(static_cast<T *>(p.dxf) + ok, xf);
            stv<CK>(static_cast<T *>(p.dxb) + ok, xb);
            stv<CV>(static_cast<T *>(p.dxw) + ov, xw);
        }
    }
#pragma unroll
    for (int e = 0; e < CK; ++e) {
        red[0][warp][ck + e] = acc_a[e];
        red[1][warp][ck + e] = acc_d[e];
    }
    __syncthreads();
    for (int x = threadIdx.x; x < 2 * DK; x += kProThreads) {
        const int which = x / DK, c = x % DK;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kProThreads / 32; ++w) v += red[which][w][c];
        partial[(((size_t)tb * 2 + which) * p.H + h) * DK + c] = v;
    }
}

// da[h][c], ddelta[h][c]: the partial sums of every row block. Slice s of the CTA adds the blocks
// s, s + 8, ... in order; the eight slice sums are then added in slice order (a fixed order).
constexpr int kRedSlices = 8;

template <int DK>
__global__ void __launch_bounds__(DK * kRedSlices) prologue_reduce_kernel(const float *__restrict__ partial, int nblk,
                                                                           int H, float *__restrict__ da,
                                                                           float *__restrict__ ddelta) {
    __shared__ float red[2][kRedSlices][DK];
    const int h = blockIdx.x, c = threadIdx.x % DK, sl = threadIdx.x / DK;
    float sa = 0.f, sd = 0.f;
#pragma unroll 4
    for (int i = sl; i < nblk; i += kRedSlices) {
        sa += partial[(((size_t)i * 2 + 0) * H + h) * DK + c];
        sd += partial[(((size_t)i * 2 + 1) * H + h) * DK + c];
    }
    red[0][sl][c] = sa;
    red[1][sl][c] = sd;
    __syncthreads();
    if (sl == 0) {
        float ta = 0.f, td = 0.f;
#pragma unroll
        for (int x = 0; x < kRedSlices; ++x) {
            ta += red[0][x][c];
            td += red[1][x][c];
        }
        da[h * DK + c] = ta;
        ddelta[h * DK + c] = td;
    }
}

int row_blocks(int B, int T) { return (int)(((long long)B * T + kProRows - 1) / kProRows); }

template <int DK, int DV, typename T>
cudaError_t run_fwd(const PrologueArgs &p, cudaStream_t st) {
    GDR2_LAUNCH("prologue_fwd", st,
                prologue_fwd_kernel<DK, DV, T><<<row_blocks(p.B, p.T) * p.H, kProThreads, 0, st>>>(p));
    return cudaGetLastError();
}

template <int DK, int DV, typename T>
cudaError_t run_bwd(const PrologueArgs &p, cudaStream_t st) {
    const int nblk = row_blocks(p.B, p.T);
    float *partial = static_cast<float *>(p.workspace);
    GDR2_LAUNCH("prologue_bwd", st,
                prologue_bwd_kernel<DK, DV, T><<<nblk * p.H, kProThreads, 0, st>>>(p, partial));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH("prologue_reduce", st,
                prologue_reduce_kernel<DK><<<p.H, DK * kRedSlices, 0, st>>>(partial, nblk, p.H, p.da, p.ddelta));
    return cudaGetLastError();
}

template <bool kFwd, typename T>
cudaError_t dispatch_dims(const PrologueArgs &p, cudaStream_t st) {
    if (p.dk_ == 128 && p.dv_ == 128) return kFwd ? run_fwd<128, 128, T>(p, st) : run_bwd<128, 128, T>(p, st);
    if (p.dk_ == 128 && p.dv_ == 64) return kFwd ? run_fwd<128, 64, T>(p, st) : run_bwd<128, 64, T>(p, st);
    if (p.dk_ == 64 && p.dv_ == 128) return kFwd ? run_fwd<64, 128, T>(p, st) : run_bwd<64, 128, T>(p, st);
    if (p.dk_ == 64 && p.dv_ == 64) return kFwd ? run_fwd<64, 64, T>(p, st) : run_bwd<64, 64, T>(p, st);
    return cudaErrorInvalidValue;
}

}  // namespace

size_t prologue_workspace_bytes(int B, int T, int H, int dk) { return (size_t)row_blocks(B, T) * 2 * H * dk * 4; }

cudaError_t launch_prologue_fwd(const PrologueArgs &p, cudaStream_t st) {
    return p.dtype == 1 ? dispatch_dims<true, __nv_bfloat16>(p, st) : dispatch_dims<true, float>(p, st);
}

cudaError_t launch_prologue_bwd(const PrologueArgs &p, cudaStream_t st) {
    return p.dtype == 1 ? dispatch_dims<false, __nv_bfloat16>(p, st) : dispatch_dims<false, float>(p, st);
}

}  // namespace gdr2
