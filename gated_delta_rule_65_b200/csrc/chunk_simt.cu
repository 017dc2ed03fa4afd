// chunk_simt.cu -- chunkwise Gated Delta Rule-2 forward and backward with plain fp32 FMA.
//
// This is the fp32-operand path (and the path for any dtype when no tensor-core kernel applies).
// It follows the chunkwise algorithm of the review's section "Chunkwise Parallel Training via WY
// Representation" term by term, with C = 64:
//   Step 1  G = in-chunk cumulative log-decay, gamma = exp(G), Kbar = k/gamma, Ebar = gamma*b*k,
//           Q_gamma = gamma*q, K_tail = (gamma_C/gamma)*k, Z = w*v
//   Step 2  T = tril(Ebar Kbar^T, -1), A = (I + T)^-1 (forward substitution), Y = A Ebar, U = A Z
//   Step 3  R = U - Y S_0, O = Q_gamma S_0 + A_qk R, S_C = Diag(gamma_C) S_0 + K_tail^T R   (Eqs. 23-24)
// and, for the backward, the chain rule through Step 3 plus the gate-aware WY terms of section
// "Gate-Aware Backward Pass" (Eqs. 64-65, dT = -tril(A^T dA A^T, -1), dB = dEbar*gamma*K,
// dW = dZ*V, dV = dZ*W, reverse in-chunk cumulative sum for the log-decay).
//
// Kernels (one launch each, all on the caller's stream):
//   prep        grid (NT, H, B)   chunk-local Steps 1-2 and A_qk, written to the workspace
//   state_fwd   grid (dv/32, H, B) serial pass over chunks for a 32-column slice of S (value
//                                 columns of S are independent in Eq. 23): R, O, S_C
//   state_bwd   grid (dv/32, H, B) reverse serial pass: dR = A_qk^T dO + K_tail dS_C,
//                                 dS_0 = gamma_C dS_C + Q_gamma^T dO - Y^T dR
//   chunk_bwd   grid (NT, H, B)   everything else of the backward, chunk-parallel
// Intermediates live in the caller's workspace; nothing here is tuned beyond plain tiling.
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {
namespace {

constexpr int C = kChunk;
constexpr int NTHR = 256;

// Per-chunk workspace tiles (fp32). Index of a chunk: ch = (b*H + h)*NT + c.
struct WS {
    float *Kb, *Eb, *Qg, *Kt, *gam, *Z, *A, *Aqk, *Y, *U;  // forward
    float *S0c, *dSc, *dR, *R, *dQg, *dKt, *dY, *dKb, *dEb;  // backward
};

struct Sizes {
    size_t tk, tv, tcc, tss;  // floats per chunk: [C,dk], [C,dv], [C,C], [dk,dv]
};

__host__ __device__ inline Sizes sizes(int dk, int dv) {
    return Sizes{(size_t)C * dk, (size_t)C * dv, (size_t)C * C, (size_t)dk * dv};
}

WS carve(float *base, int nch, int dk, int dv, bool bwd) {
    Sizes s = sizes(dk, dv);
    WS w{};
    float *p = base;
    auto take = [&](size_t per) { float *r = p; p += per * (size_t)nch; return r; };
    w.Kb = take(s.tk); w.Eb = take(s.tk); w.Qg = take(s.tk); w.Kt = take(s.tk); w.gam = take(s.tk);
    w.Y = take(s.tk); w.Z = take(s.tv); w.U = take(s.tv); w.A = take(s.tcc); w.Aqk = take(s.tcc);
    if (bwd) {
        w.S0c = take(s.tss); w.dSc = take(s.tss); w.dR = take(s.tv); w.R = take(s.tv);
        w.dQg = take(s.tk); w.dKt = take(s.tk); w.dY = take(s.tk); w.dKb = take(s.tk); w.dEb = take(s.tk);
    }
    return w;
}

size_t ws_floats(size_t nch, int dk, int dv, bool bwd) {
    Sizes s = sizes(dk, dv);
    size_t per = 6 * s.tk + 2 * s.tv + 2 * s.tcc;
    if (bwd) per += 2 * s.tss + 2 * s.tv + 5 * s.tk;
    return per * nch;
}

// C[m][n] = alpha * sum_k opA[m][k] opB[k][n] + beta * Cin[m][n] over the whole CTA.
// opA[m][k] = TA ? A[k*lda+m] : A[m*lda+k];  opB[k][n] = TB ? B[n*ldb+k] : B[k*ldb+n].
// mask: 0 = dense, 1 = keep n <= m, 2 = keep n < m (masked entries are written as 0).
template <bool TA, bool TB>
__device__ void bgemm(int M, int N, int K, const float *A, int lda, const float *B, int ldb, float *Cm, int ldc,
                      float alpha, float beta, const float *Cin, int mask) {
    for (int idx = threadIdx.x; idx < M * N; idx += blockDim.x) {
        const int m = idx / N, n = idx % N;
        const bool keep = mask == 0 || (mask == 1 ? n <= m : n < m);
        float out = 0.f;
        if (keep) {
            float acc = 0.f;
            for (int kk = 0; kk < K; ++kk) {
                const float a = TA ? A[(size_t)kk * lda + m] : A[(size_t)m * lda + kk];
                const float b = TB ? B[(size_t)n * ldb + kk] : B[(size_t)kk * ldb + n];
                acc = fmaf(a, b, acc);
            }
            out = alpha * acc;
            if (beta != 0.f) out = fmaf(beta, Cin[(size_t)m * ldc + n], out);
        }
        Cm[(size_t)m * ldc + n] = out;
    }
}

__device__ __forceinline__ size_t tok(int bi, int t, int H, int h, int Tlen, int d) {
    return (((size_t)bi * Tlen + t) * H + h) * d;
}

// ---------------------------------------------------------------------------------------------
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(NTHR) prep_kernel(const T *q, const T *k, const T *v, const float *la, const T *b,
                                                    const T *w, int Tlen, int H, int NT, WS ws) {
    extern __shared__ float sm[];
    float *G = sm;               // [C, DK] cumulative log-decay
    float *Kb = G + C * DK;      // [C, DK]
    float *Eb = Kb + C * DK;     // [C, DK]
    float *Qg = Eb + C * DK;     // [C, DK]; later reused for A
    float *Tm = Qg + C * DK;     // [C, C]
    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
    const size_t ch = ((size_t)bi * H + h) * NT + c;
    const int t0 = c * C, n = min(C, Tlen - t0);
    const Sizes s = sizes(DK, DV);

    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int r = idx / DK, i = idx % DK;
        G[idx] = r < n ? la[tok(bi, t0 + r, H, h, Tlen, DK) + i] : 0.f;
    }
    __syncthreads();
    for (int i = tid; i < DK; i += NTHR) {  // Step 1: G_r = sum_{j<=r} g_j inside the chunk
        float acc = 0.f;
        for (int r = 0; r < C; ++r) { acc += G[r * DK + i]; G[r * DK + i] = acc; }
        if (!(fabsf(acc) <= kMaxChunkLogDecay)) flag_status(kStatusRange);  // (NaN included)
    }
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int r = idx / DK, i = idx % DK;
        const float g = G[idx], gl = G[(C - 1) * DK + i];
        float kk = 0.f, bb = 0.f, qq = 0.f;
        if (r < n) {
            const size_t o = tok(bi, t0 + r, H, h, Tlen, DK) + i;
            kk = to_f(k[o]); bb = to_f(b[o]); qq = to_f(q[o]);
        }
        const float gam = expf(g);
        const float kb = kk * expf(-g), eb = bb * kk * gam, qg = qq * gam, kt = kk * expf(gl - g);
        Kb[idx] = kb; Eb[idx] = eb; Qg[idx] = qg;
        ws.Kb[ch * s.tk + idx] = kb; ws.Eb[ch * s.tk + idx] = eb; ws.Qg[ch * s.tk + idx] = qg;
        ws.Kt[ch * s.tk + idx] = kt; ws.gam[ch * s.tk + idx] = gam;
    }
    for (int idx = tid; idx < C * DV; idx += NTHR) {
        const int r = idx / DV, j = idx % DV;
        float z = 0.f;
        if (r < n) {
            const size_t o = tok(bi, t0 + r, H, h, Tlen, DV) + j;
            z = to_f(w[o]) * to_f(v[o]);
        }
        ws.Z[ch * s.tv + idx] = z;
    }
    __syncthreads();
    bgemm<false, true>(C, C, DK, Eb, DK, Kb, DK, Tm, C, 1.f, 0.f, nullptr, 2);                   // T
    bgemm<false, true>(C, C, DK, Qg, DK, Kb, DK, ws.Aqk + ch * s.tcc, C, 1.f, 0.f, nullptr, 1);  // A_qk
    __syncthreads();
    float *Am = Qg;  // Qg is no longer needed in shared memory
    if (tid < C) {   // A = (I + T)^-1, one column per thread, forward substitution down the rows
        const int col = tid;
        for (int r = 0; r < C; ++r) {
            float val = (r == col) ? 1.f : 0.f;
            if (r > col)
                for (int j = col; j < r; ++j) val = fmaf(-Tm[r * C + j], Am[j * C + col], val);
            Am[r * C + col] = val;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NTHR) ws.A[ch * s.tcc + idx] = Am[idx];
    bgemm<false, false>(C, DK, C, Am, C, Eb, DK, ws.Y + ch * s.tk, DK, 1.f, 0.f, nullptr, 0);            // Y
    bgemm<false, false>(C, DV, C, Am, C, ws.Z + ch * s.tv, DV, ws.U + ch * s.tv, DV, 1.f, 0.f, nullptr, 0);  // U
}

// ---------------------------------------------------------------------------------------------
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(NTHR) state_fwd_kernel(const float *S0, T *o, float *ST, int Tlen, int H, int NT,
                                                         WS ws, int store_states) {
    __shared__ float S[DK * 32];
    __shared__ float R[C * 32];
    const int js = blockIdx.x * 32, h = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
    const size_t bh = (size_t)bi * H + h;
    const Sizes s = sizes(DK, DV);
    for (int idx = tid; idx < DK * 32; idx += NTHR) {
        const int i = idx / 32, j = idx % 32;
        S[idx] = S0 ? S0[bh * s.tss + (size_t)i * DV + js + j] : 0.f;
    }
    __syncthreads();
    for (int c = 0; c < NT; ++c) {
        const size_t ch = bh * NT + c;
        const int n = min(C, Tlen - c * C);
        const float *Y = ws.Y + ch * s.tk, *U = ws.U + ch * s.tv, *Qg = ws.Qg + ch * s.tk;
        const float *Aqk = ws.Aqk + ch * s.tcc, *Kt = ws.Kt + ch * s.tk, *gam = ws.gam + ch * s.tk;
        if (store_states)
            for (int idx = tid; idx < DK * 32; idx += NTHR)
                ws.S0c[ch * s.tss + (size_t)(idx / 32) * DV + js + idx % 32] = S[idx];
        for (int idx = tid; idx < C * 32; idx += NTHR) {  // R = U - Y S_0
            const int r = idx / 32, j = idx % 32;
            float acc = U[r * DV + js + j];
            for (int i = 0; i < DK; ++i) acc = fmaf(-Y[r * DK + i], S[i * 32 + j], acc);
            R[idx] = acc;
        }
        __syncthreads();
        if (o)
            for (int idx = tid; idx < C * 32; idx += NTHR) {  // O = Q_gamma S_0 + A_qk R
                const int r = idx / 32, j = idx % 32;
                float acc = 0.f;
                for (int i = 0; i < DK; ++i) acc = fmaf(Qg[r * DK + i], S[i * 32 + j], acc);
                for (int t = 0; t <= r; ++t) acc = fmaf(Aqk[r * C + t], R[t * 32 + j], acc);
                if (r < n) o[tok(bi, c * C + r, H, h, Tlen, DV) + js + j] = from_f<T>(acc);
            }
        __syncthreads();
        for (int idx = tid; idx < DK * 32; idx += NTHR) {  // S_C = Diag(gamma_C) S_0 + K_tail^T R
            const int i = idx / 32, j = idx % 32;
            float acc = gam[(C - 1) * DK + i] * S[idx];
            for (int r = 0; r < C; ++r) acc = fmaf(Kt[r * DK + i], R[r * 32 + j], acc);
            S[idx] = acc;
        }
        __syncthreads();
    }
    if (ST)
        for (int idx = tid; idx < DK * 32; idx += NTHR)
            ST[bh * s.tss + (size_t)(idx / 32) * DV + js + idx % 32] = S[idx];
}

// ---------------------------------------------------------------------------------------------
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(NTHR) state_bwd_kernel(const T *dO, const float *dST, float *dS0, int Tlen, int H,
                                                         int NT, WS ws) {
    __shared__ float dS[DK * 32];
    __shared__ float dRs[C * 32];
    __shared__ float dOs[C * 32];
    const int js = blockIdx.x * 32, h = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
    const size_t bh = (size_t)bi * H + h;
    const Sizes s = sizes(DK, DV);
    for (int idx = tid; idx < DK * 32; idx += NTHR)
        dS[idx] = dST ? dST[bh * s.tss + (size_t)(idx / 32) * DV + js + idx % 32] : 0.f;
    __syncthreads();
    for (int c = NT - 1; c >= 0; --c) {
        const size_t ch = bh * NT + c;
        const int n = min(C, Tlen - c * C);
        const float *Y = ws.Y + ch * s.tk, *Qg = ws.Qg + ch * s.tk, *Aqk = ws.Aqk + ch * s.tcc;
        const float *Kt = ws.Kt + ch * s.tk, *gam = ws.gam + ch * s.tk;
        for (int idx = tid; idx < DK * 32; idx += NTHR)
            ws.dSc[ch * s.tss + (size_t)(idx / 32) * DV + js + idx % 32] = dS[idx];
        for (int idx = tid; idx < C * 32; idx += NTHR) {
            const int r = idx / 32, j = idx % 32;
            dOs[idx] = (dO && r < n) ? to_f(dO[tok(bi, c * C + r, H, h, Tlen, DV) + js + j]) : 0.f;
        }
        __syncthreads();
        for (int idx = tid; idx < C * 32; idx += NTHR) {  // dR = A_qk^T dO + K_tail dS_C
            const int r = idx / 32, j = idx % 32;
            float acc = 0.f;
            for (int t = r; t < C; ++t) acc = fmaf(Aqk[t * C + r], dOs[t * 32 + j], acc);
            for (int i = 0; i < DK; ++i) acc = fmaf(Kt[r * DK + i], dS[i * 32 + j], acc);
            dRs[idx] = acc;
            ws.dR[ch * s.tv + (size_t)r * DV + js + j] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < DK * 32; idx += NTHR) {  // dS_0 = gamma_C dS_C + Q_gamma^T dO - Y^T dR
            const int i = idx / 32, j = idx % 32;
            float acc = gam[(C - 1) * DK + i] * dS[idx];
            for (int r = 0; r < C; ++r) {
                acc = fmaf(Qg[r * DK + i], dOs[r * 32 + j], acc);
                acc = fmaf(-Y[r * DK + i], dRs[r * 32 + j], acc);
            }
            dS[idx] = acc;
        }
        __syncthreads();
    }
    if (dS0)
        for (int idx = tid; idx < DK * 32; idx += NTHR)
            dS0[bh * s.tss + (size_t)(idx / 32) * DV + js + idx % 32] = dS[idx];
}

// ---------------------------------------------------------------------------------------------
template <int DK, int DV, typename T>
__global__ void __launch_bounds__(NTHR) chunk_bwd_kernel(const T *q, const T *k, const T *v, const T *b, const T *w,
                                                         const T *dO, T *dq, T *dk, T *dv, float *dla, T *db, T *dw,
                                                         int Tlen, int H, int NT, WS ws) {
    extern __shared__ float sm[];
    float *dAqk = sm;             // [C, C]
    float *dA = dAqk + C * C;     // [C, C], later dT
    float *X = dA + C * C;        // [C, C]
    float *dOs = X + C * C;       // [C, DV]
    float *dG = dOs + C * DV;     // [C, DK]
    float *dgC = dG + C * DK;     // [DK]
    const int c = blockIdx.x, h = blockIdx.y, bi = blockIdx.z, tid = threadIdx.x;
    const size_t ch = ((size_t)bi * H + h) * NT + c;
    const int t0 = c * C, n = min(C, Tlen - t0);
    const Sizes s = sizes(DK, DV);
    const float *Kb = ws.Kb + ch * s.tk, *Eb = ws.Eb + ch * s.tk, *Qg = ws.Qg + ch * s.tk;
    const float *Kt = ws.Kt + ch * s.tk, *gam = ws.gam + ch * s.tk, *Z = ws.Z + ch * s.tv;
    const float *A = ws.A + ch * s.tcc, *Y = ws.Y + ch * s.tk, *U = ws.U + ch * s.tv;
    const float *S0c = ws.S0c + ch * s.tss, *dSc = ws.dSc + ch * s.tss, *dR = ws.dR + ch * s.tv;
    float *R = ws.R + ch * s.tv, *dQg = ws.dQg + ch * s.tk, *dKt = ws.dKt + ch * s.tk;
    float *dY = ws.dY + ch * s.tk, *dKb = ws.dKb + ch * s.tk, *dEb = ws.dEb + ch * s.tk;

    for (int idx = tid; idx < C * DV; idx += NTHR) {
        const int r = idx / DV, j = idx % DV;
        dOs[idx] = (dO && r < n) ? to_f(dO[tok(bi, t0 + r, H, h, Tlen, DV) + j]) : 0.f;
    }
    __syncthreads();
    bgemm<false, false>(C, DV, DK, Y, DK, S0c, DV, R, DV, -1.f, 1.f, U, 0);        // R = U - Y S_0
    for (int i = tid; i < DK; i += NTHR) {                                           // dgamma_C
        float acc = 0.f;
        for (int j = 0; j < DV; ++j) acc = fmaf(dSc[i * DV + j], S0c[i * DV + j], acc);
        dgC[i] = acc;
    }
    __syncthreads();
    bgemm<false, true>(C, C, DV, dOs, DV, R, DV, dAqk, C, 1.f, 0.f, nullptr, 1);    // dA_qk = tril(dO R^T)
    bgemm<false, true>(C, DK, DV, R, DV, dSc, DV, dKt, DK, 1.f, 0.f, nullptr, 0);    // dK_tail = R dS_C^T
    bgemm<false, true>(C, DK, DV, dR, DV, S0c, DV, dY, DK, -1.f, 0.f, nullptr, 0);   // dY = -dR S_0^T
    bgemm<false, true>(C, DK, DV, dOs, DV, S0c, DV, dQg, DK, 1.f, 0.f, nullptr, 0);  // dQ_gamma = dO S_0^T ...
    bgemm<false, true>(C, C, DV, dR, DV, Z, DV, dA, C, 1.f, 0.f, nullptr, 0);        // dA = dU Z^T ...
    __syncthreads();
    bgemm<false, false>(C, DK, C, dAqk, C, Kb, DK, dQg, DK, 1.f, 1.f, dQg, 0);       // ... + dA_qk Kbar
    bgemm<true, false>(C, DK, C, dAqk, C, Qg, DK, dKb, DK, 1.f, 0.f, nullptr, 0);    // dKbar = dA_qk^T Q_gamma
    bgemm<false, true>(C, C, DK, dY, DK, Eb, DK, dA, C, 1.f, 1.f, dA, 0);            // ... + dY Ebar^T (Eqs. 64-65)
    bgemm<true, false>(C, DK, C, A, C, dY, DK, dEb, DK, 1.f, 0.f, nullptr, 0);       // dEbar = A^T dY
    for (int idx = tid; idx < C * DV; idx += NTHR) {                                 // dZ = A^T dU -> dw, dv
        const int r = idx / DV, j = idx % DV;
        float acc = 0.f;
        for (int t = r; t < C; ++t) acc = fmaf(A[t * C + r], dR[t * DV + j], acc);
        if (r < n) {
            const size_t o = tok(bi, t0 + r, H, h, Tlen, DV) + j;
            dw[o] = from_f<T>(acc * to_f(v[o]));
            dv[o] = from_f<T>(acc * to_f(w[o]));
        }
    }
    __syncthreads();
    bgemm<true, false>(C, C, C, A, C, dA, C, X, C, 1.f, 0.f, nullptr, 0);            // X = A^T dA
    __syncthreads();
    bgemm<false, true>(C, C, C, X, C, A, C, dA, C, -1.f, 0.f, nullptr, 2);           // dT = -tril(X A^T, -1)
    __syncthreads();
    float *dT = dA;
    bgemm<false, false>(C, DK, C, dT, C, Kb, DK, dEb, DK, 1.f, 1.f, dEb, 0);         // dEbar += dT Kbar
    bgemm<true, false>(C, DK, C, dT, C, Eb, DK, dKb, DK, 1.f, 1.f, dKb, 0);          // dKbar += dT^T Ebar
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NTHR) {
        const int r = idx / DK, i = idx % DK;
        const float g = gam[idx], gl = gam[(C - 1) * DK + i];
        float kk = 0.f, bb = 0.f;
        size_t o = 0;
        if (r < n) {
            o = tok(bi, t0 + r, H, h, Tlen, DK) + i;
            kk = to_f(k[o]); bb = to_f(b[o]);
        }
        const float deb = dEb[idx], dkb = dKb[idx], dkt = dKt[idx], dqg = dQg[idx];
        dG[idx] = dqg * Qg[idx] + deb * Eb[idx] - dkb * Kb[idx] - dkt * Kt[idx];
        if (r < n) {
            db[o] = from_f<T>(deb * kk * g);
            dk[o] = from_f<T>(deb * bb * g + dkb / g + dkt * (gl / g));
            dq[o] = from_f<T>(dqg * g);
        }
    }
    __syncthreads();
    for (int i = tid; i < DK; i += NTHR) {  // dlog_alpha = reverse cumulative sum of dG inside the chunk
        float extra = dgC[i] * gam[(C - 1) * DK + i];
        for (int r = 0; r < C; ++r) extra = fmaf(dKt[r * DK + i], Kt[r * DK + i], extra);
        float acc = extra;
        for (int r = C - 1; r >= 0; --r) {
            acc += dG[r * DK + i];
            if (r < n) dla[tok(bi, t0 + r, H, h, Tlen, DK) + i] = acc;
        }
    }
}

template <int DK, int DV, typename T>
cudaError_t fwd_t(const ChunkArgs &a, cudaStream_t st, bool for_bwd) {
    const int NT = (a.T + C - 1) / C;
    const int nch = a.B * a.H * NT;
    WS ws = carve((float *)a.workspace, nch, DK, DV, for_bwd);
    const size_t sm_prep = sizeof(float) * (4 * C * DK + C * C);
    cudaError_t e = cudaFuncSetAttribute(prep_kernel<DK, DV, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_prep);
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH("simt_prep", st,
                prep_kernel<DK, DV, T><<<dim3(NT, a.H, a.B), NTHR, sm_prep, st>>>(
                    (const T *)a.q, (const T *)a.k, (const T *)a.v, a.log_alpha, (const T *)a.b, (const T *)a.w, a.T,
                    a.H, NT, ws));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    GDR2_LAUNCH(for_bwd ? "simt_state_fwd_store" : "simt_state_fwd", st,
                state_fwd_kernel<DK, DV, T><<<dim3(DV / 32, a.H, a.B), NTHR, 0, st>>>(
                    a.initial_state, for_bwd ? nullptr : (T *)a.o, for_bwd ? nullptr : a.final_state, a.T, a.H, NT,
                    ws, for_bwd ? 1 : 0));
    return cudaGetLastError();
}

template <int DK, int DV, typename T>
cudaError_t bwd_t(const ChunkArgs &a, cudaStream_t st, bool saved) {
    cudaError_t e = saved ? cudaSuccess : fwd_t<DK, DV, T>(a, st, true);
    if (e != cudaSuccess) return e;
    const int NT = (a.T + C - 1) / C;
    const int nch = a.B * a.H * NT;
    WS ws = carve((float *)a.workspace, nch, DK, DV, true);
    GDR2_LAUNCH("simt_state_bwd", st,
                state_bwd_kernel<DK, DV, T><<<dim3(DV / 32, a.H, a.B), NTHR, 0, st>>>(
                    (const T *)a.d_o, a.d_final_state, a.d_initial_state, a.T, a.H, NT, ws));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t sm_bwd = sizeof(float) * (3 * C * C + C * DV + C * DK + DK);
    e = cudaFuncSetAttribute(chunk_bwd_kernel<DK, DV, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_bwd);
    if (e != cudaSuccess) return e;
    GDR2_LAUNCH("simt_chunk_bwd", st,
                chunk_bwd_kernel<DK, DV, T><<<dim3(NT, a.H, a.B), NTHR, sm_bwd, st>>>(
                    (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.b, (const T *)a.w,
                    (const T *)a.d_o, (T *)a.dq, (T *)a.dk, (T *)a.dv, a.dlog_alpha, (T *)a.db, (T *)a.dw, a.T, a.H,
                    NT, ws));
    return cudaGetLastError();
}

// mode: 0 forward, 1 backward (with recompute), 2 forward that also fills the backward workspace,
// 3 backward from a workspace filled by mode 2
template <int DK, int DV, typename T>
cudaError_t run_mode(const ChunkArgs &a, cudaStream_t st, int mode) {
    if (mode == 0) return fwd_t<DK, DV, T>(a, st, false);
    if (mode == 1) return bwd_t<DK, DV, T>(a, st, false);
    if (mode == 3) return bwd_t<DK, DV, T>(a, st, true);
    cudaError_t e = fwd_t<DK, DV, T>(a, st, false);
    return e != cudaSuccess ? e : fwd_t<DK, DV, T>(a, st, true);
}

template <typename T>
cudaError_t dispatch(const ChunkArgs &a, cudaStream_t st, int mode) {
#define GDR2_CASE(DK_, DV_) \
    if (a.dk_ == DK_ && a.dv_ == DV_) return run_mode<DK_, DV_, T>(a, st, mode);
    GDR2_CASE(64, 64)
    GDR2_CASE(64, 128)
    GDR2_CASE(128, 64)
    GDR2_CASE(128, 128)
#undef GDR2_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

size_t simt_workspace_bytes(int B, int T, int H, int dk, int dv, int for_bwd) {
    const size_t NT = (size_t)((T + C - 1) / C);
    return sizeof(float) * ws_floats((size_t)B * (size_t)H * NT, dk, dv, for_bwd != 0);
}

cudaError_t launch_simt_fwd(const ChunkArgs &a, cudaStream_t st) {
    return a.dtype == 1 ? dispatch<__nv_bfloat16>(a, st, 0) : dispatch<float>(a, st, 0);
}

cudaError_t launch_simt_bwd(const ChunkArgs &a, cudaStream_t st) {
    return a.dtype == 1 ? dispatch<__nv_bfloat16>(a, st, 1) : dispatch<float>(a, st, 1);
}

cudaError_t launch_simt_fwd_train(const ChunkArgs &a, cudaStream_t st) {
    return a.dtype == 1 ? dispatch<__nv_bfloat16>(a, st, 2) : dispatch<float>(a, st, 2);
}

cudaError_t launch_simt_bwd_saved(const ChunkArgs &a, cudaStream_t st) {
    return a.dtype == 1 ? dispatch<__nv_bfloat16>(a, st, 3) : dispatch<float>(a, st, 3);
}

int status_take_simt() { return take_status(); }

}  // namespace gdr2
