// gdr2_api.cu -- the extern "C" boundary of libgdr2.so (declared in include/gdr2.h).
//
// Every entry point validates its arguments on the host before launching anything, enqueues its
// kernels on the caller's stream, and returns a status code. Nothing here allocates, frees or
// synchronises.
#include <stdint.h>

#include "gdr2.h"
#include "kernels.h"
#include "status.cuh"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void *p) { return p == nullptr || aligned16(p); }

int check_chunk_sizes(int B, int T, int H, int dk, int dv, int dtype) {
    if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_F32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GDR2_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535) return GDR2_ERR_UNSUPPORTED;  // grid y/z limits
    return GDR2_OK;
}

bool use_tc(int dk, int dv, int dtype, int /*for_bwd*/) { return dtype == GDR2_BF16 && dk == 128 && dv == 128; }

// Chunk path of the unpacked bf16, dk = dv = 128 calls: 0 = automatic, 1 = per-chain fused kernels,
// 2 = chunk-parallel kernels with serial state passes (gdr2_set_chunk_path).
int g_chunk_path = 0;
// Automatic mode: a cost model per chunk of one chain, with the step times measured on B200 (training pair,
// T = 4096 and 16384). The per-chain kernels take about 34.3 us per chunk (forward and backward), one CTA per
// chain in waves of 148 SMs; the chunk-parallel kernels spend about 0.24 us of the whole GPU per chunk on the
// chunk-local work plus about 12.6 us per chunk of a chain on their serial passes, also in waves of 148 (less
// with the chunk-level scan, which they run for few long chains). The per-chain layout wins when
// waves x 21.7 us < 0.24 us x B H: from about 91 chains up to one wave (measured crossover between 80 and 96
// chains), then again from about 181 (between 160 and 192), and so on. The model takes 148 SMs on every
// device, so that the workspace query and the launch agree.
bool chain_wins(long long chains) {
    const long long waves = (chains + 147) / 148;
    return (double)waves * 21.7 < 0.2405 * (double)chains;
}

bool use_chain(int B, int H, int dk, int dv, int dtype, bool train) {
    if (!use_tc(dk, dv, dtype, 0)) return false;
    if (g_chunk_path == 1) return true;
    if (g_chunk_path == 2) return false;
    (void)train;  // the same choice for the forward, the backward and the training pair
    return chain_wins((long long)B * H);
}

// Grouped value heads: Hv = G H value heads (G >= 1) on the tensor-core path only.
int check_gva_sizes(int B, int T, int H, int Hv, int dk, int dv, int dtype) {
    int st = check_chunk_sizes(B, T, H, dk, dv, dtype);
    if (st != GDR2_OK) return st;
    if (Hv <= 0 || Hv % H != 0) return GDR2_ERR_INVALID_ARG;
    if (!use_tc(dk, dv, dtype, 0) || Hv > 65535) return GDR2_ERR_UNSUPPORTED;
    return GDR2_OK;
}

// Packed batches run on the tensor-core path only (bf16 operands, dk = dv = 128).
int check_varlen_sizes(int N, int T, int H, int dk, int dv, int dtype) {
    if (N <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_F32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_BF16 || dk != 128 || dv != 128) return GDR2_ERR_UNSUPPORTED;
    if ((long long)N * H > 0x7fffffffLL || H > 65535 || N > 65535) return GDR2_ERR_UNSUPPORTED;
    if ((long long)(T / 64 + N) * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;
    return GDR2_OK;
}

// Packed batches with grouped value heads: both sets of limits, on the value-head counts.
int check_varlen_gva_sizes(int N, int T, int H, int Hv, int dk, int dv, int dtype) {
    int st = check_varlen_sizes(N, T, H, dk, dv, dtype);
    if (st != GDR2_OK) return st;
    if (Hv <= 0 || Hv % H != 0) return GDR2_ERR_INVALID_ARG;
    if (Hv > 65535 || (long long)N * Hv > 0x7fffffffLL || (long long)(T / 64 + N) * Hv > 0x7fffffffLL)
        return GDR2_ERR_UNSUPPORTED;
    return GDR2_OK;
}

int check_call_sizes(int B, int N, int T, int H, int Hv, int dk, int dv, int dtype) {
    if (N > 0 && Hv > 0) return check_varlen_gva_sizes(N, T, H, Hv, dk, dv, dtype);
    if (N > 0) return check_varlen_sizes(N, T, H, dk, dv, dtype);
    if (Hv > 0) return check_gva_sizes(B, T, H, Hv, dk, dv, dtype);
    return check_chunk_sizes(B, T, H, dk, dv, dtype);
}

size_t chunk_ws_bytes(int B, int T, int H, int dk, int dv, int dtype, int for_bwd) {
    if (use_chain(B, H, dk, dv, dtype, for_bwd != 0)) return for_bwd ? gdr2::chain_record_bytes(B, T, H) : 0;
    if (use_tc(dk, dv, dtype, for_bwd)) return gdr2::tc_workspace_bytes(B, T, H, for_bwd);
    return gdr2::simt_workspace_bytes(B, T, H, dk, dv, for_bwd);
}

}  // namespace

extern "C" {

int gdr2_version(void) { return 100; }

int gdr2_check(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDR2_ERR_CUDA;
    const int a = gdr2::status_take_tc(), b = gdr2::status_take_simt(), c = gdr2::status_take_decode(),
              d = gdr2::status_take_chain();
    if (a < 0 || b < 0 || c < 0 || d < 0) return GDR2_ERR_CUDA;
    const int bits = a | b | c | d;
    if (bits & gdr2::kStatusBounds) return GDR2_ERR_BOUNDS;
    if (bits & gdr2::kStatusTimeout) return GDR2_ERR_TIMEOUT;
    if (bits & gdr2::kStatusRange) return GDR2_ERR_RANGE;
    return GDR2_OK;
}

const char *gdr2_status_string(int status) {
    switch (status) {
        case GDR2_OK: return "ok";
        case GDR2_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size or dtype)";
        case GDR2_ERR_UNSUPPORTED: return "unsupported head dimensions or sizes";
        case GDR2_ERR_WORKSPACE: return "workspace missing or too small";
        case GDR2_ERR_CUDA: return "CUDA launch or device error";
        case GDR2_ERR_TIMEOUT: return "bounded device-side wait expired";
        case GDR2_ERR_RANGE: return "a chunk's cumulative log-decay left the supported range";
        case GDR2_ERR_BOUNDS: return "an index check of the debug build failed in a kernel";
        default: return "unknown status";
    }
}

int gdr2_set_chunk_path(int path) {
    if (path < 0 || path > 2) return GDR2_ERR_INVALID_ARG;
    g_chunk_path = path;
    return GDR2_OK;
}

int gdr2_get_chunk_path(void) { return g_chunk_path; }

size_t gdr2_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype, int for_bwd) {
    if (check_chunk_sizes(B, T, H, dk, dv, dtype) != GDR2_OK) return 0;
    return chunk_ws_bytes(B, T, H, dk, dv, dtype, for_bwd);
}

size_t gdr2_workspace_bytes_gva(int B, int T, int H, int Hv, int dk, int dv, int dtype, int for_bwd) {
    if (check_gva_sizes(B, T, H, Hv, dk, dv, dtype) != GDR2_OK) return 0;
    return gdr2::tc_workspace_bytes(B, T, H, for_bwd, Hv);
}

size_t gdr2_workspace_bytes_varlen(int N, int T, int H, int dk, int dv, int dtype, int for_bwd) {
    if (check_varlen_sizes(N, T, H, dk, dv, dtype) != GDR2_OK) return 0;
    return gdr2::tc_workspace_bytes_packed(N, T, H, for_bwd);
}

size_t gdr2_workspace_bytes_varlen_gva(int N, int T, int H, int Hv, int dk, int dv, int dtype, int for_bwd) {
    if (check_varlen_gva_sizes(N, T, H, Hv, dk, dv, dtype) != GDR2_OK) return 0;
    return gdr2::tc_workspace_bytes_packed(N, T, H, for_bwd, Hv);
}

}  // extern "C"

namespace {

int chunk_fwd_impl(const void *q, const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                   const float *initial_state, void *o, float *final_state, int B, int T, int H, int dk, int dv,
                   int dtype, void *workspace, size_t workspace_bytes, void *stream, bool train,
                   const int *cu_seqlens = nullptr, int N = 0, int Hv = 0) {
    int st = check_call_sizes(B, N, T, H, Hv, dk, dv, dtype);
    if (st != GDR2_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) || !ok_ptr(o) ||
        !ok_opt(initial_state) || !ok_opt(final_state) || (N > 0 && !ok_ptr(cu_seqlens)))
        return GDR2_ERR_INVALID_ARG;
    const size_t need = N > 0    ? gdr2::tc_workspace_bytes_packed(N, T, H, train ? 1 : 0, Hv)
                        : Hv > 0 ? gdr2::tc_workspace_bytes(B, T, H, train ? 1 : 0, Hv)
                                 : chunk_ws_bytes(B, T, H, dk, dv, dtype, train ? 1 : 0);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))) return GDR2_ERR_WORKSPACE;
    gdr2::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.b = b; a.w = w; a.initial_state = initial_state;
    a.o = o; a.final_state = final_state;
    a.B = B; a.T = T; a.H = H; a.dk_ = dk; a.dv_ = dv; a.dtype = dtype;
    a.cu_seqlens = cu_seqlens; a.N = N; a.Hv = Hv;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (N == 0 && Hv == 0 && use_chain(B, H, dk, dv, dtype, train))
        e = gdr2::launch_chain_fwd(a, s, train ? workspace : nullptr);
    else if (use_tc(dk, dv, dtype, 0))
        e = train ? gdr2::launch_tc_fwd_train(a, s) : gdr2::launch_tc_fwd(a, s);
    else
        e = train ? gdr2::launch_simt_fwd_train(a, s) : gdr2::launch_simt_fwd(a, s);
    return e == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

int chunk_bwd_impl(const void *q, const void *k, const void *v, const float *log_alpha, const void *b, const void *w,
                   const float *initial_state, const void *d_o, const float *d_final_state, void *dq, void *dk,
                   void *dv, float *dlog_alpha, void *db, void *dw, float *d_initial_state, int B, int T, int H,
                   int dk_, int dv_, int dtype, void *workspace, size_t workspace_bytes, void *stream, bool saved,
                   const int *cu_seqlens = nullptr, int N = 0, int Hv = 0) {
    int st = check_call_sizes(B, N, T, H, Hv, dk_, dv_, dtype);
    if (st != GDR2_OK) return st;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) ||
        !ok_opt(initial_state) || !ok_opt(d_o) || !ok_opt(d_final_state) || !ok_ptr(dq) || !ok_ptr(dk) ||
        !ok_ptr(dv) || !ok_ptr(dlog_alpha) || !ok_ptr(db) || !ok_ptr(dw) || !ok_opt(d_initial_state) ||
        (N > 0 && !ok_ptr(cu_seqlens)))
        return GDR2_ERR_INVALID_ARG;
    const size_t need = N > 0    ? gdr2::tc_workspace_bytes_packed(N, T, H, 1, Hv)
                        : Hv > 0 ? gdr2::tc_workspace_bytes(B, T, H, 1, Hv)
                                 : chunk_ws_bytes(B, T, H, dk_, dv_, dtype, 1);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))) return GDR2_ERR_WORKSPACE;
    gdr2::ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.b = b; a.w = w; a.initial_state = initial_state;
    a.d_o = d_o; a.d_final_state = d_final_state;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dlog_alpha = dlog_alpha; a.db = db; a.dw = dw;
    a.d_initial_state = d_initial_state;
    a.B = B; a.T = T; a.H = H; a.dk_ = dk_; a.dv_ = dv_; a.dtype = dtype;
    a.cu_seqlens = cu_seqlens; a.N = N; a.Hv = Hv;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (N == 0 && Hv == 0 && use_chain(B, H, dk_, dv_, dtype, true)) {
        e = cudaSuccess;
        if (!saved) {  // the forward again, for its per-chunk record only
            gdr2::ChunkArgs f = a;
            f.o = nullptr;
            f.final_state = nullptr;
            e = gdr2::launch_chain_fwd(f, s, workspace);
        }
        if (e == cudaSuccess) e = gdr2::launch_chain_bwd(a, s, workspace);
    } else if (use_tc(dk_, dv_, dtype, 1))
        e = gdr2::launch_tc_bwd(a, s, saved);
    else
        e = saved ? gdr2::launch_simt_bwd_saved(a, s) : gdr2::launch_simt_bwd(a, s);
    return e == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

}  // namespace

extern "C" {

int gdr2_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                   const void *w, const float *initial_state, void *o, float *final_state, int B, int T, int H,
                   int dk, int dv, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, B, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, false);
}

int gdr2_chunk_fwd_train(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                         const void *w, const float *initial_state, void *o, float *final_state, int B, int T, int H,
                         int dk, int dv, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, B, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, true);
}

int gdr2_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                   const void *w, const float *initial_state, const void *d_o, const float *d_final_state, void *dq,
                   void *dk, void *dv, float *dlog_alpha, void *db, void *dw, float *d_initial_state, int B, int T,
                   int H, int dk_, int dv_, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, B, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, false);
}

int gdr2_chunk_bwd_saved(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                         const void *w, const float *initial_state, const void *d_o, const float *d_final_state,
                         void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw, float *d_initial_state,
                         int B, int T, int H, int dk_, int dv_, int dtype, void *workspace, size_t workspace_bytes,
                         void *stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, B, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, true);
}

int gdr2_chunk_fwd_gva(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                       const void *w, const float *initial_state, void *o, float *final_state, int B, int T, int H,
                       int Hv, int dk, int dv, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, B, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, false, nullptr, 0, Hv);
}

int gdr2_chunk_fwd_train_gva(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                             const void *w, const float *initial_state, void *o, float *final_state, int B, int T,
                             int H, int Hv, int dk, int dv, int dtype, void *workspace, size_t workspace_bytes,
                             void *stream) {
    if (Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, B, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, true, nullptr, 0, Hv);
}

int gdr2_chunk_bwd_gva(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                       const void *w, const float *initial_state, const void *d_o, const float *d_final_state,
                       void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw, float *d_initial_state,
                       int B, int T, int H, int Hv, int dk_, int dv_, int dtype, void *workspace,
                       size_t workspace_bytes, void *stream) {
    if (Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, B, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, false,
                          nullptr, 0, Hv);
}

int gdr2_chunk_bwd_saved_gva(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                             const void *w, const float *initial_state, const void *d_o, const float *d_final_state,
                             void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                             float *d_initial_state, int B, int T, int H, int Hv, int dk_, int dv_, int dtype,
                             void *workspace, size_t workspace_bytes, void *stream) {
    if (Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, B, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, true,
                          nullptr, 0, Hv);
}

int gdr2_chunk_fwd_varlen(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                          const void *w, const float *initial_state, void *o, float *final_state,
                          const int *cu_seqlens, int N, int T, int H, int dk, int dv, int dtype, void *workspace,
                          size_t workspace_bytes, void *stream) {
    if (N <= 0) return GDR2_ERR_INVALID_ARG;  // an unpacked call is not a packed one with N = 0
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, 1, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, false, cu_seqlens, N);
}

int gdr2_chunk_fwd_train_varlen(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                                const void *w, const float *initial_state, void *o, float *final_state,
                                const int *cu_seqlens, int N, int T, int H, int dk, int dv, int dtype,
                                void *workspace, size_t workspace_bytes, void *stream) {
    if (N <= 0) return GDR2_ERR_INVALID_ARG;  // an unpacked call is not a packed one with N = 0
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, 1, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, true, cu_seqlens, N);
}

int gdr2_chunk_bwd_varlen(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                          const void *w, const float *initial_state, const void *d_o, const float *d_final_state,
                          void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                          float *d_initial_state, const int *cu_seqlens, int N, int T, int H, int dk_, int dv_,
                          int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (N <= 0) return GDR2_ERR_INVALID_ARG;  // an unpacked call is not a packed one with N = 0
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, 1, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, false,
                          cu_seqlens, N);
}

int gdr2_chunk_bwd_saved_varlen(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                                const void *w, const float *initial_state, const void *d_o,
                                const float *d_final_state, void *dq, void *dk, void *dv, float *dlog_alpha,
                                void *db, void *dw, float *d_initial_state, const int *cu_seqlens, int N, int T,
                                int H, int dk_, int dv_, int dtype, void *workspace, size_t workspace_bytes,
                                void *stream) {
    if (N <= 0) return GDR2_ERR_INVALID_ARG;  // an unpacked call is not a packed one with N = 0
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, 1, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, true,
                          cu_seqlens, N);
}

int gdr2_chunk_fwd_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                              const void *w, const float *initial_state, void *o, float *final_state,
                              const int *cu_seqlens, int N, int T, int H, int Hv, int dk, int dv, int dtype,
                              void *workspace, size_t workspace_bytes, void *stream) {
    if (N <= 0 || Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, 1, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, false, cu_seqlens, N, Hv);
}

int gdr2_chunk_fwd_train_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                    const void *b, const void *w, const float *initial_state, void *o,
                                    float *final_state, const int *cu_seqlens, int N, int T, int H, int Hv, int dk,
                                    int dv, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (N <= 0 || Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, log_alpha, b, w, initial_state, o, final_state, 1, T, H, dk, dv, dtype, workspace,
                          workspace_bytes, stream, true, cu_seqlens, N, Hv);
}

int gdr2_chunk_bwd_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                              const void *w, const float *initial_state, const void *d_o, const float *d_final_state,
                              void *dq, void *dk, void *dv, float *dlog_alpha, void *db, void *dw,
                              float *d_initial_state, const int *cu_seqlens, int N, int T, int H, int Hv, int dk_,
                              int dv_, int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (N <= 0 || Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, 1, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, false,
                          cu_seqlens, N, Hv);
}

int gdr2_chunk_bwd_saved_varlen_gva(const void *q, const void *k, const void *v, const float *log_alpha,
                                    const void *b, const void *w, const float *initial_state, const void *d_o,
                                    const float *d_final_state, void *dq, void *dk, void *dv, float *dlog_alpha,
                                    void *db, void *dw, float *d_initial_state, const int *cu_seqlens, int N, int T,
                                    int H, int Hv, int dk_, int dv_, int dtype, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    if (N <= 0 || Hv <= 0) return GDR2_ERR_INVALID_ARG;
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state, dq, dk, dv, dlog_alpha, db, dw,
                          d_initial_state, 1, T, H, dk_, dv_, dtype, workspace, workspace_bytes, stream, true,
                          cu_seqlens, N, Hv);
}

size_t gdr2_gate_prologue_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
    if (check_chunk_sizes(B, T, H, dk, dv, dtype) != GDR2_OK) return 0;
    return gdr2::prologue_workspace_bytes(B, T, H, dk);
}

int gdr2_gate_prologue_fwd(const void *xq, const void *xk, const void *xf, const void *xb, const void *xw,
                           const float *a, const float *delta, int neg_eig, void *q, void *k, float *log_alpha,
                           void *b, void *w, int B, int T, int H, int dk, int dv, int dtype, void *stream) {
    const int st = check_chunk_sizes(B, T, H, dk, dv, dtype);
    if (st != GDR2_OK) return st;
    if (((long long)B * T + 127) / 128 * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;  // one CTA per 128 rows
    if (!ok_ptr(xq) || !ok_ptr(xk) || !ok_ptr(xf) || !ok_ptr(xb) || !ok_ptr(xw) || !ok_ptr(a) || !ok_ptr(delta) ||
        !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w))
        return GDR2_ERR_INVALID_ARG;
    gdr2::PrologueArgs p{};
    p.xq = xq; p.xk = xk; p.xf = xf; p.xb = xb; p.xw = xw; p.a = a; p.delta = delta; p.neg_eig = neg_eig != 0;
    p.q = q; p.k = k; p.g = log_alpha; p.b = b; p.w = w;
    p.B = B; p.T = T; p.H = H; p.dk_ = dk; p.dv_ = dv; p.dtype = dtype;
    return gdr2::launch_prologue_fwd(p, (cudaStream_t)stream) == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

int gdr2_gate_prologue_bwd(const void *xq, const void *xk, const void *xf, const void *xb, const void *xw,
                           const float *a, const float *delta, int neg_eig, const void *dq, const void *dk,
                           const float *dlog_alpha, const void *db, const void *dw, void *dxq, void *dxk, void *dxf,
                           void *dxb, void *dxw, float *da, float *ddelta, int B, int T, int H, int dk_, int dv,
                           int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    const int st = check_chunk_sizes(B, T, H, dk_, dv, dtype);
    if (st != GDR2_OK) return st;
    if (((long long)B * T + 127) / 128 * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;  // one CTA per 128 rows
    if (!ok_ptr(xq) || !ok_ptr(xk) || !ok_ptr(xf) || !ok_ptr(xb) || !ok_ptr(xw) || !ok_ptr(a) || !ok_ptr(delta) ||
        !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dlog_alpha) || !ok_ptr(db) || !ok_ptr(dw) || !ok_ptr(dxq) ||
        !ok_ptr(dxk) || !ok_ptr(dxf) || !ok_ptr(dxb) || !ok_ptr(dxw) || !ok_ptr(da) || !ok_ptr(ddelta))
        return GDR2_ERR_INVALID_ARG;
    if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < gdr2::prologue_workspace_bytes(B, T, H, dk_))
        return GDR2_ERR_WORKSPACE;
    gdr2::PrologueArgs p{};
    p.xq = xq; p.xk = xk; p.xf = xf; p.xb = xb; p.xw = xw; p.a = a; p.delta = delta; p.neg_eig = neg_eig != 0;
    p.dq = dq; p.dk = dk; p.dg = dlog_alpha; p.db = db; p.dw = dw;
    p.dxq = dxq; p.dxk = dxk; p.dxf = dxf; p.dxb = dxb; p.dxw = dxw; p.da = da; p.ddelta = ddelta;
    p.B = B; p.T = T; p.H = H; p.dk_ = dk_; p.dv_ = dv; p.dtype = dtype;
    p.workspace = workspace; p.workspace_bytes = workspace_bytes;
    return gdr2::launch_prologue_bwd(p, (cudaStream_t)stream) == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

int gdr2_decode_step(const void *q, const void *k, const void *v, const float *log_alpha, const void *b,
                     const void *w, float *state, void *o, int B, int H, int dk, int dv, int dtype, void *stream) {
    if (B <= 0 || H <= 0 || dk <= 0 || dv <= 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_F32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    if ((dk != 64 && dk != 128) || dv % 64 != 0 || dv > 256) return GDR2_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) || !ok_ptr(state) ||
        !ok_ptr(o))
        return GDR2_ERR_INVALID_ARG;
    gdr2::DecodeArgs a{q, k, v, log_alpha, b, w, state, o, B, H, dk, dv, dtype};
    return gdr2::launch_decode(a, (cudaStream_t)stream) == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

}  // extern "C"
