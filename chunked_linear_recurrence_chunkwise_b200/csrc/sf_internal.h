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
    // Workspace.  Intermediates have element type TW = float for fp32 I/O and
    // bf16 for bf16 I/O; chunk-transposed tiles keep the 64 tokens of a chunk
    // contiguous (TP = NC * 64 padded tokens).
    float* G;     // [BH][TP]            fp32 chunk-local inclusive cumsum of g
    float* Ed;    // [BH][NC][128]       fp32 per chunk: e^{G_C - G_r} (r < 64), then e^{G_r}
    void* Wt;     // [BH][NC][dk][64]    W^T per chunk, W = T diag(beta gamma) K   (delta rule)
    void* Ut;     // [BH][NC][dv][64]    U^T per chunk, U = T diag(beta) V (V for linear attention)
    void* Sc;     // [BH][NC][dv][dk]    S^T entering each chunk
    void* Dt;     // [BH][NC][dv][64]    Delta^T per chunk (V^T for linear attention)
    void* dDt;    // [BH][NC][dv][64]    dL/dDelta, transposed per chunk
    void* dSc;    // [BH][NC][dv][dk]    (dL/dS leaving each chunk)^T
    void* Pm;     // [BH][NC][64][64]    P = (Q K^T) .* Gamma, lower incl. (backward)
    void* Tm;     // [BH][NC][64][64]    T = (I + A)^-1, bf16 (backward, tensor-core path)
    float* dKp;   // [BH][TP][dk]        fp32 delta-rule part of dk (SIMT gradient kernels)
    float* dGp;   // [BH][TP]            fp32 delta-rule part of dG (SIMT gradient kernels)
    int* err;     // device error word
    // two work counters of the gradient kernel, zero between launches (the last CTA of a
    // launch puts them back)
    unsigned* ticket;
    // SMs the gradient kernel may hold (0: all): the sub-sequence drivers leave those of a
    // state pass that runs beside it free
    int grad_sms;
};

// Workspace carve-up for a piece of at most T tokens.
struct WsLayout {
    size_t G, Ed, Wt, Ut, Sc, Dt, dDt, dSc, Pm, Tm, dKp, dGp;  // byte offsets inside one slot
    size_t slot_bytes;
    size_t total;  // err header + nslots * slot_bytes
};

constexpr size_t kErrBytes = 256;

WsLayout ws_layout(int B, int T, int H, int dk, int dv, int dtype, bool delta, bool bwd,
                   int nslots);
// Parts of a slot: the forward's intermediates (G, Ed, W^T, U^T, chunk states,
// Delta^T), P and T (tensor-core backward), the backward-only scratch.
constexpr int kPartFwd = 1, kPartPT = 2, kPartBwd = 4;
WsLayout ws_layout_parts(int B, int T, int H, int dk, int dv, int dtype, bool delta, int parts,
                         int nslots);
void bind_slot(Args& a, void* ws, const WsLayout& L, int slot, bool bwd);
// Points the arrays of `parts` at a slot that starts at `base`.
void bind_parts(Args& a, char* base, const WsLayout& L, int parts);

// Kernel launchers (SIMT fp32 arithmetic; I/O in a.dtype).  Each returns the
// cudaError_t of its launch.
cudaError_t launch_intra_fwd(const Args& a, cudaStream_t s);
cudaError_t launch_state_fwd(const Args& a, cudaStream_t s);
cudaError_t launch_output(const Args& a, cudaStream_t s);
cudaError_t launch_dd_pre(const Args& a, cudaStream_t s);
cudaError_t launch_state_bwd(const Args& a, cudaStream_t s);
cudaError_t launch_grad_delta(const Args& a, cudaStream_t s);
cudaError_t launch_grad_attn(const Args& a, cudaStream_t s);

// Tensor-core kernels (sm_100a tcgen05/TMEM/TMA; bf16, d_k = d_v = 128).
bool tc_eligible(const Args& a);
cudaError_t launch_state_fwd_tc(const Args& a, cudaStream_t s);
// with_p: also store P (backward recompute)
cudaError_t launch_intra_tc(const Args& a, bool with_p, cudaStream_t s);
// reads P from a.Pm when it is set (the forward that keeps its intermediates)
cudaError_t launch_output_tc(const Args& a, cudaStream_t s);
// reverse dS pass; consumes P from the backward intra kernel (no dDelta pre-pass)
cudaError_t launch_state_bwd_tc(const Args& a, cudaStream_t s);
// dq, dk, dv, dg of (gated) linear attention (no beta)
cudaError_t launch_grad_attn_tc(const Args& a, cudaStream_t s);
// every per-chunk gradient of the gated delta rule in one kernel (dq, dk, dv, dg, dbeta)
cudaError_t launch_grad_fused_tc(const Args& a, cudaStream_t s);

// Per-kernel timing registry (sf_timing_*).
enum KernelKind {
    KK_INTRA_FWD = 0,
    KK_STATE_FWD,
    KK_OUTPUT,
    KK_DD_PRE,
    KK_STATE_BWD,
    KK_GRAD_DELTA,
    KK_GRAD_ATTN,
    KK_INTRA_BWD,
    KK_GRAD_FUSED,
    KK_COUNT
};
const char* kernel_name(int kind);
void timing_begin(int kind, cudaStream_t s);
void timing_end(int kind, cudaStream_t s);

}  // namespace sf
