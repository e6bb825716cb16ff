// Internal declarations shared by the C-ABI layer and the kernels of libsf.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace sf {

constexpr int kChunk = 64;   // tokens per chunk
constexpr int kMaxD = 128;   // largest dk / dv

// Everything a kernel of one call needs.  Token pointers already point at the
// first token of the piece; rows of batch b start ld_t * H * d elements apart.
struct Args {
    int B, T, H, dk, dv, ld_t, NC;   // NC = ceil(T / 64)
    int dtype;                        // SF_F32 or SF_BF16
    // inputs
    const void* q;
    const void* k;
    const void* v;
    const float* g;      // may be null
    const float* beta;   // may be null
    const float* S_in;   // may be null
    const void* dO;
    const float* dS_out; // may be null
    // outputs
    void* o;
    float* S_out;        // may be null
    void* dq;
    void* dk_;
    void* dv_;
    float* dg;
    float* dbeta;
    float* dS_in;        // may be null
    // workspace (fp32, per (b,h) contiguous, TP = NC * 64 padded tokens)
    float* G;     // [BH][TP]          chunk-local inclusive cumsum of g
    float* W;     // [BH][TP][dk]      T diag(beta*gamma) K            (delta rule)
    float* U;     // [BH][TP][dv]      T diag(beta) V                  (delta rule)
    float* Sc;    // [BH][NC][dk][dv]  state entering each chunk
    float* D;     // [BH][TP][dv]      Delta = U - W S_c (V for linear attention)
    float* dD;    // [BH][TP][dv]      dL/dDelta
    float* dSc;   // [BH][NC][dk][dv]  dL/d(state leaving each chunk)
    float* dKp;   // [BH][TP][dk]      delta-rule part of dk
    float* dGp;   // [BH][TP]          delta-rule part of dG
    int* err;     // device error word
};

// Workspace carve-up for a piece of at most T tokens.
struct WsLayout {
    size_t G, W, U, Sc, D, dD, dSc, dKp, dGp;  // byte offsets inside one slot
    size_t slot_bytes;
    size_t total;  // err header + nslots * slot_bytes
};

constexpr size_t kErrBytes = 256;

WsLayout ws_layout(int B, int T, int H, int dk, int dv, bool delta, bool bwd, int nslots);
void bind_slot(Args& a, void* ws, const WsLayout& L, int slot, bool bwd);

// Kernel launchers (SIMT fp32 arithmetic; I/O in a.dtype).  Each returns the
// cudaError_t of its launch.
cudaError_t launch_intra_fwd(const Args& a, cudaStream_t s);
cudaError_t launch_state_fwd(const Args& a, cudaStream_t s);
cudaError_t launch_output(const Args& a, cudaStream_t s);
cudaError_t launch_dd_pre(const Args& a, cudaStream_t s);
cudaError_t launch_state_bwd(const Args& a, cudaStream_t s);
cudaError_t launch_grad_delta(const Args& a, cudaStream_t s);
cudaError_t launch_grad_attn(const Args& a, cudaStream_t s);

// Per-kernel timing registry (sf_timing_*).
enum KernelKind {
    KK_INTRA_FWD = 0,
    KK_STATE_FWD,
    KK_OUTPUT,
    KK_DD_PRE,
    KK_STATE_BWD,
    KK_GRAD_DELTA,
    KK_GRAD_ATTN,
    KK_COUNT
};
const char* kernel_name(int kind);
void timing_begin(int kind, cudaStream_t s);
void timing_end(int kind, cudaStream_t s);

}  // namespace sf
