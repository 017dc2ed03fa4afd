// kernels.h -- internal launcher interface between the C ABI (gdr2_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdr2 {

struct DecodeArgs {
    const void *q, *k, *v;
    const float *log_alpha;
    const void *b, *w;
    float *state;
    void *o;
    int B, H, dk, dv, dtype;
};

struct ChunkArgs {
    const void *q, *k, *v;
    const float *log_alpha;
    const void *b, *w;
    const float *initial_state;  // may be null
    // forward outputs
    void *o;
    float *final_state;          // may be null
    // backward inputs / outputs
    const void *d_o;             // may be null
    const float *d_final_state;  // may be null
    void *dq, *dk, *dv;
    float *dlog_alpha;
    void *db, *dw;
    float *d_initial_state;      // may be null
    int B, T, H, dk_, dv_, dtype;
    // packed variable-length batch: N > 0 sequences given by cu_seqlens (device, N + 1 offsets), B = 1
    const int *cu_seqlens;
    int N;
    // grouped value heads: Hv = G H value heads (v, w, o, states and their gradients); 0 means Hv = H
    int Hv;
    void *workspace;
    size_t workspace_bytes;
};

// Opt-in kernel timing (profile.cu): events on the launch stream around each launch.
int prof_begin(const char *name, cudaStream_t st);
void prof_end(int slot, cudaStream_t st);
#define GDR2_LAUNCH(name, st, ...)                       \
    do {                                                 \
        const int gdr2_slot_ = ::gdr2::prof_begin(name, st); \
        __VA_ARGS__;                                     \
        ::gdr2::prof_end(gdr2_slot_, st);                \
    } while (0)

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);

// Gate and normalisation prologue (prologue.cu).
struct PrologueArgs {
    const void *xq, *xk, *xf, *xb, *xw;  // branch pre-activations [B,T,H,dk] (xw: [B,T,H,dv]), dtype
    const float *a, *delta;              // [H, dk] fp32
    int neg_eig;
    void *q, *k;                         // forward outputs
    float *g;
    void *b, *w;
    const void *dq, *dk;                 // backward inputs
    const float *dg;
    const void *db, *dw;
    void *dxq, *dxk, *dxf, *dxb, *dxw;   // backward outputs
    float *da, *ddelta;
    int B, T, H, dk_, dv_, dtype;
    void *workspace;
    size_t workspace_bytes;
};
size_t prologue_workspace_bytes(int B, int T, int H, int dk);
cudaError_t launch_prologue_fwd(const PrologueArgs &p, cudaStream_t st);
cudaError_t launch_prologue_bwd(const PrologueArgs &p, cudaStream_t st);

// Plain fp32-FMA chunk path (any dtype): workspace size and the two passes.
size_t simt_workspace_bytes(int B, int T, int H, int dk, int dv, int for_bwd);
cudaError_t launch_simt_fwd(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_simt_bwd(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_simt_fwd_train(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_simt_bwd_saved(const ChunkArgs &a, cudaStream_t st);

// Tensor-core chunk path (bf16 operands, dk = dv = 128).
bool tc_supported(const ChunkArgs &a);
size_t tc_workspace_bytes(int B, int T, int H, int for_bwd, int Hv = 0);
size_t tc_workspace_bytes_packed(int N, int T, int H, int for_bwd, int Hv = 0);
cudaError_t launch_tc_fwd(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_tc_fwd_train(const ChunkArgs &a, cudaStream_t st);
cudaError_t launch_tc_bwd(const ChunkArgs &a, cudaStream_t st, bool saved);

// Per-chain fused tensor-core path (bf16 operands, dk = dv = 128, unpacked, one value head per key head):
// one CTA walks a (batch, head) chain's chunks in order. The training forward leaves a per-chunk record for
// the backward (chain_record_bytes).
size_t chain_record_bytes(int B, int T, int H);
cudaError_t launch_chain_fwd(const ChunkArgs &a, cudaStream_t st, void *record);
cudaError_t launch_chain_bwd(const ChunkArgs &a, cudaStream_t st, const void *record);

// Status bits (kStatusTimeout, kStatusRange) the kernels of one source file have set since the last call,
// cleared on read; -1 when the word cannot be read.
int status_take_tc();
int status_take_simt();
int status_take_decode();
int status_take_chain();

}  // namespace gdr2
