// C-ABI entry points of libsf: argument checks, workspace carve-up, the
// single-piece forward/backward and the two-stream sub-sequence driver.
//
// The sub-sequence driver follows the Sequence Accumulation schedule
// ("Sequence Accumulation and Beyond ...", Approach): pieces run in order on
// one device, the state leaving piece i is the state entering piece i+1, and
// the backward walks the pieces in reverse over the stored entering states,
// handing dS from piece i+1 to piece i (StateFlow, Abstract: boundary states
// forward, their gradients backward).  The state-transition pass of piece i is
// overlapped with the intra-chunk work of its neighbour on a second stream
// (StateFlow, Abstract, and gptget.net summary 术语表 "状态重叠": state
// transitions overlapped with surrounding computation).

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/sf.h"
#include "sf_internal.h"

namespace sf {

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace slots of the sub-sequence drivers: up to three pieces are in flight at once
// (piece i uses slot i % 3; fewer pieces need fewer slots).
constexpr int kSeqSlots = 3;

WsLayout ws_layout(int B, int T, int H, int dk, int dv, int dtype, bool delta, bool bwd,
                   int nslots) {
    return ws_layout_parts(B, T, H, dk, dv, dtype, delta,
                           bwd ? (kPartFwd | kPartPT | kPartBwd) : kPartFwd, nslots);
}

WsLayout ws_layout_parts(int B, int T, int H, int dk, int dv, int dtype, bool delta, int parts,
                         int nslots) {
    WsLayout L{};
    const bool fwd = parts & kPartFwd, pt = parts & kPartPT, bwd = parts & kPartBwd;
    const size_t BH = (size_t)B * H;
    const size_t NC = (size_t)(T + kChunk - 1) / kChunk;
    const size_t TP = NC * kChunk;
    const size_t tw = dtype == SF_BF16 ? 2 : 4;  // intermediates follow the I/O precision
    // the tensor-core path computes every delta-rule gradient in one kernel: no dKp / dGp
    const bool split_grads = !(dtype == SF_BF16 && dk == 128 && dv == 128);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up256(bytes);
        return o;
    };
    L.G = take(fwd ? BH * TP * 4 : 0);
    L.Ed = take(fwd ? BH * NC * 128 * 4 : 0);
    L.Wt = take(fwd && delta ? BH * TP * dk * tw : 0);
    L.Ut = take(fwd ? BH * TP * dv * tw : 0);
    L.Sc = take(fwd ? BH * NC * dk * dv * tw : 0);
    L.Dt = take(fwd ? BH * TP * dv * tw : 0);
    L.dDt = take(bwd ? BH * TP * dv * tw : 0);
    L.dSc = take(bwd ? BH * NC * dk * dv * tw : 0);
    L.Pm = take(pt ? BH * NC * kChunk * kChunk * tw : 0);
    L.Tm = take(pt && delta ? BH * NC * kChunk * kChunk * tw : 0);
    L.dKp = take(bwd && delta && split_grads ? BH * TP * dk * 4 : 0);
    L.dGp = take(bwd && delta && split_grads ? BH * TP * 4 : 0);
    L.slot_bytes = off;
    L.total = kErrBytes + (size_t)nslots * L.slot_bytes;
    return L;
}

void bind_parts(Args& a, char* base, const WsLayout& L, int parts) {
    if (parts & kPartFwd) {
        a.G = (float*)(base + L.G);
        a.Ed = (float*)(base + L.Ed);
        a.Wt = base + L.Wt;
        a.Ut = base + L.Ut;
        a.Sc = base + L.Sc;
        a.Dt = base + L.Dt;
    }
    if (parts & kPartPT) {
        a.Pm = base + L.Pm;
        a.Tm = base + L.Tm;
    }
    if (parts & kPartBwd) {
        a.dDt = base + L.dDt;
        a.dSc = base + L.dSc;
        a.dKp = (float*)(base + L.dKp);
        a.dGp = (float*)(base + L.dGp);
    }
}

void bind_slot(Args& a, void* ws, const WsLayout& L, int slot, bool bwd) {
    char* base = (char*)ws + kErrBytes + (size_t)slot * L.slot_bytes;
    a.G = (float*)(base + L.G);
    a.Ed = (float*)(base + L.Ed);
    a.Wt = base + L.Wt;
    a.Ut = base + L.Ut;
    a.Sc = base + L.Sc;
    a.Dt = base + L.Dt;
    a.dDt = bwd ? (void*)(base + L.dDt) : nullptr;
    a.dSc = bwd ? (void*)(base + L.dSc) : nullptr;
    a.Pm = bwd ? (void*)(base + L.Pm) : nullptr;
    a.Tm = bwd ? (void*)(base + L.Tm) : nullptr;
    a.dKp = bwd ? (float*)(base + L.dKp) : nullptr;
    a.dGp = bwd ? (float*)(base + L.dGp) : nullptr;
    a.err = (int*)ws;
    a.ticket = (unsigned*)((char*)ws + 8);
}

// ------------------------------------------------------------------ timing
namespace {
struct TimingRec {
    int kind;
    cudaStream_t stream;
    cudaEvent_t e0, e1;
};
bool g_timing_on = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;
double g_ms[KK_COUNT];
int g_launches[KK_COUNT];

cudaEvent_t pool_get() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}
}  // namespace

const char* kernel_name(int kind) {
    static const char* names[KK_COUNT] = {"intra_fwd", "state_fwd", "output",    "dd_pre",    "state_bwd",
                                          "grad_delta", "grad_attn", "intra_bwd", "grad_fused"};
    return (kind >= 0 && kind < KK_COUNT) ? names[kind] : "?";
}

void timing_begin(int kind, cudaStream_t s) {
    if (!g_timing_on) return;
    TimingRec r{kind, s, pool_get(), pool_get()};
    cudaEventRecord(r.e0, s);
    g_recs.push_back(r);
}

void timing_end(int kind, cudaStream_t s) {
    if (!g_timing_on || g_recs.empty() || g_recs.back().kind != kind) return;
    cudaEventRecord(g_recs.back().e1, s);
}

// ------------------------------------------------------------------ checks
namespace {

bool aligned(const void* p, size_t n) { return ((uintptr_t)p % n) == 0; }

sf_status check_shape(const sf_shape* s) {
    if (!s) return SF_ERR_INVALID;
    if (s->B < 0 || s->T < 0 || s->H < 0) return SF_ERR_INVALID;
    if (s->ld_t != 0 && s->ld_t < s->T) return SF_ERR_INVALID;
    if (s->chunk != kChunk) return SF_ERR_UNSUPPORTED;
    if (s->dk < 1 || s->dk > kMaxD || s->dv < 1 || s->dv > kMaxD) return SF_ERR_UNSUPPORTED;
    if (s->dtype != SF_F32 && s->dtype != SF_BF16) return SF_ERR_UNSUPPORTED;
    return SF_OK;
}

size_t esize(const sf_shape* s) { return s->dtype == SF_BF16 ? 2 : 4; }

// Required pointers must be non-NULL; every given pointer must be aligned to its element.
sf_status check_ptrs(const sf_shape* s, std::initializer_list<const void*> required,
                     std::initializer_list<const void*> io, std::initializer_list<const void*> f32) {
    for (const void* p : required)
        if (!p) return SF_ERR_INVALID;
    for (const void* p : io)
        if (p && !aligned(p, esize(s))) return SF_ERR_INVALID;
    for (const void* p : f32)
        if (p && !aligned(p, 4)) return SF_ERR_INVALID;
    return SF_OK;
}

Args make_args(const sf_shape* s) {
    Args a{};
    a.B = s->B;
    a.T = s->T;
    a.H = s->H;
    a.dk = s->dk;
    a.dv = s->dv;
    a.ld_t = s->ld_t ? s->ld_t : s->T;
    a.NC = (s->T + kChunk - 1) / kChunk;
    a.dtype = s->dtype;
    return a;
}

sf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SF_OK : SF_ERR_CUDA; }

#define SF_TRY(expr)                                   \
    do {                                               \
        cudaError_t _e = (expr);                       \
        if (_e != cudaSuccess) return SF_ERR_CUDA;     \
    } while (0)

// state copy for empty pieces: dst = src or 0
cudaError_t copy_state(float* dst, const float* src, size_t n, cudaStream_t st) {
    if (!dst) return cudaSuccess;
    if (src) return cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, st);
    return cudaMemsetAsync(dst, 0, n * sizeof(float), st);
}

// Kernel choice: the tensor-core kernels cover bf16 with d_k = d_v = 128; the
// SIMT kernels cover everything else (and are the fp32 path).
cudaError_t state_fwd(const Args& a, cudaStream_t st) {
    return tc_eligible(a) ? launch_state_fwd_tc(a, st) : launch_state_fwd(a, st);
}

cudaError_t intra(const Args& a, bool with_p, cudaStream_t st) {
    return tc_eligible(a) ? launch_intra_tc(a, with_p, st) : launch_intra_fwd(a, st);
}
cudaError_t output(const Args& a, cudaStream_t st) {
    return tc_eligible(a) ? launch_output_tc(a, st) : launch_output(a, st);
}

// The forward pieces of one call: intra (may go on its own stream), then state + output.
cudaError_t run_intra(const Args& a, cudaStream_t st) { return intra(a, false, st); }

cudaError_t run_state_output(const Args& a, cudaStream_t st, bool with_output) {
    cudaError_t e = state_fwd(a, st);
    if (e == cudaSuccess && with_output) e = output(a, st);
    return e;
}

// Everything of the backward of one piece that does not need dS: recompute of
// the intra-chunk terms and the chunk states, and dDelta's P^T dO part.
cudaError_t run_bwd_prep(Args a, cudaStream_t st) {
    cudaError_t e = intra(a, true, st);
    if (e != cudaSuccess) return e;
    a.S_out = nullptr;
    e = state_fwd(a, st);
    if (e != cudaSuccess) return e;
    // the tensor-core reverse pass forms P^T dO itself from the stored P
    return tc_eligible(a) ? cudaSuccess : launch_dd_pre(a, st);
}

// The sequential part of one piece's backward: recompute of the chunk states
// (and, on the SIMT path, the P^T dO pre-pass), then the reverse dS pass.
cudaError_t run_bwd_state(Args a, cudaStream_t st) {
    Args f = a;
    f.S_out = nullptr;
    cudaError_t e = state_fwd(f, st);
    if (e == cudaSuccess && !tc_eligible(a)) e = launch_dd_pre(a, st);
    if (e == cudaSuccess) e = tc_eligible(a) ? launch_state_bwd_tc(a, st) : launch_state_bwd(a, st);
    return e;
}

// The sequential part of one piece's backward when the forward kept its
// intermediates: (on the SIMT path, the P^T dO pre-pass) then the reverse dS pass.
cudaError_t run_bwd_state_kept(const Args& a, cudaStream_t st) {
    cudaError_t e = tc_eligible(a) ? cudaSuccess : launch_dd_pre(a, st);
    if (e == cudaSuccess) e = tc_eligible(a) ? launch_state_bwd_tc(a, st) : launch_state_bwd(a, st);
    return e;
}

// The per-chunk gradients of one piece (after its reverse pass).
cudaError_t run_bwd_chunk_grads(const Args& a, cudaStream_t st) {
    if (tc_eligible(a)) return a.beta ? launch_grad_fused_tc(a, st) : launch_grad_attn_tc(a, st);
    cudaError_t e = cudaSuccess;
    if (a.beta) e = launch_grad_delta(a, st);
    if (e == cudaSuccess) e = launch_grad_attn(a, st);
    return e;
}

// The dS-dependent part: reverse state pass, then the per-chunk gradients.
cudaError_t run_bwd_grads(const Args& a, cudaStream_t st) {
    cudaError_t e = tc_eligible(a) ? launch_state_bwd_tc(a, st) : launch_state_bwd(a, st);
    if (e == cudaSuccess) e = run_bwd_chunk_grads(a, st);
    return e;
}

}  // namespace
}  // namespace sf

using namespace sf;

// ---------------------------------------------------------------- driver
namespace {

struct SeqPlan {
    std::vector<int> start;  // token offset of each piece
    int lmax = 0;
};

sf_status plan_seq(const sf_shape* s, int n_sub, const int* lens, SeqPlan& p) {
    if (n_sub <= 0 || !lens) return SF_ERR_INVALID;
    long long sum = 0;
    p.start.resize(n_sub);
    for (int i = 0; i < n_sub; ++i) {
        if (lens[i] <= 0) return SF_ERR_INVALID;
        p.start[i] = (int)sum;
        sum += lens[i];
        p.lmax = std::max(p.lmax, lens[i]);
    }
    return sum == s->T ? SF_OK : SF_ERR_INVALID;
}

// A view of tokens [t0, t0 + len) of a [B, ld_t, H, d] tensor.
const void* tok_ptr(const void* base, int t0, int H, int d, size_t es) {
    return base ? (const void*)((const char*)base + (size_t)t0 * H * d * es) : nullptr;
}
void* tok_ptr(void* base, int t0, int H, int d, size_t es) {
    return base ? (void*)((char*)base + (size_t)t0 * H * d * es) : nullptr;
}

struct EventSet {
    std::vector<cudaEvent_t> ev;
    ~EventSet() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
    }
    cudaError_t make(int n) {
        ev.resize(n, nullptr);
        for (int i = 0; i < n; ++i) {
            cudaError_t e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
};

// The sequential state passes of the sub-sequence drivers run on a stream of
// the device's greatest priority, created on first use (one per device, kept
// for the life of the process): whenever SMs free up, the block scheduler then
// serves the critical path before the parallel work queued on the aux stream.
cudaError_t critical_stream(cudaStream_t* out) {
    static std::mutex mu;
    static std::vector<cudaStream_t> per_dev;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)per_dev.size() <= dev) per_dev.resize(dev + 1, nullptr);
    if (!per_dev[dev]) {
        int least = 0, greatest = 0;
        e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e == cudaSuccess)
            e = cudaStreamCreateWithPriority(&per_dev[dev], cudaStreamNonBlocking, greatest);
        if (e != cudaSuccess) {
            per_dev[dev] = nullptr;
            return e;
        }
    }
    *out = per_dev[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t sf_workspace_bytes(const sf_shape* s, int op) {
    if (check_shape(s) != SF_OK || (op != SF_OP_FWD && op != SF_OP_BWD)) return 0;
    // Whether beta is given is not known here: size for the delta rule (the superset).
    return ws_layout(s->B, s->T, s->H, s->dk, s->dv, s->dtype, true, op == SF_OP_BWD, 1).total;
}

size_t sf_seq_workspace_bytes(const sf_shape* s, int n_sub, const int* lens, int op) {
    if (check_shape(s) != SF_OK || n_sub <= 0 || !lens) return 0;
    long long sum = 0;
    int lmax = 0;
    for (int i = 0; i < n_sub; ++i) {
        if (lens[i] <= 0) return 0;
        sum += lens[i];
        lmax = std::max(lmax, lens[i]);
    }
    if (sum != s->T) return 0;
    const size_t states = 2 * (size_t)s->B * s->H * s->dk * s->dv * sizeof(float);
    return ws_layout(s->B, lmax, s->H, s->dk, s->dv, s->dtype, true, op == SF_OP_BWD,
                     std::min(kSeqSlots, n_sub)).total + states;
}

sf_status sf_fwd(const sf_shape* s, const void* q, const void* k, const void* v, const float* g,
                 const float* beta, const float* S_in, void* o, float* S_out, void* ws,
                 size_t ws_bytes, void* stream) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    const size_t nstate = (size_t)s->B * s->H * s->dk * s->dv;
    const bool work = (size_t)s->B * s->H * s->T > 0;
    st = check_ptrs(s, work ? std::initializer_list<const void*>{q, k, v, o}
                            : std::initializer_list<const void*>{},
                    {q, k, v, o}, {g, beta, S_in, S_out});
    if (st != SF_OK) return st;
    if (!work) return cuda_status(copy_state(S_out, S_in, nstate, cs));
    const WsLayout L = ws_layout(s->B, s->T, s->H, s->dk, s->dv, s->dtype, beta != nullptr, false, 1);
    if (!ws || ws_bytes < L.total || !aligned(ws, 256)) return SF_ERR_WORKSPACE;
    Args a = make_args(s);
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S_in = S_in; a.o = o; a.S_out = S_out;
    bind_slot(a, ws, L, 0, false);
    SF_TRY(run_intra(a, cs));
    SF_TRY(run_state_output(a, cs, true));
    return SF_OK;
}

sf_status sf_bwd(const sf_shape* s, const void* q, const void* k, const void* v, const float* g,
                 const float* beta, const float* S_in, const void* dO, const float* dS_out,
                 void* dq, void* dk, void* dv, float* dg, float* dbeta, float* dS_in, void* ws,
                 size_t ws_bytes, void* stream) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    if ((g != nullptr) != (dg != nullptr) || (beta != nullptr) != (dbeta != nullptr))
        return SF_ERR_INVALID;
    cudaStream_t cs = (cudaStream_t)stream;
    const size_t nstate = (size_t)s->B * s->H * s->dk * s->dv;
    const bool work = (size_t)s->B * s->H * s->T > 0;
    st = check_ptrs(s, work ? std::initializer_list<const void*>{q, k, v, dO, dq, dk, dv}
                            : std::initializer_list<const void*>{},
                    {q, k, v, dO, dq, dk, dv}, {g, beta, S_in, dS_out, dg, dbeta, dS_in});
    if (st != SF_OK) return st;
    if (!work) return cuda_status(copy_state(dS_in, dS_out, nstate, cs));
    const WsLayout L = ws_layout(s->B, s->T, s->H, s->dk, s->dv, s->dtype, beta != nullptr, true, 1);
    if (!ws || ws_bytes < L.total || !aligned(ws, 256)) return SF_ERR_WORKSPACE;
    Args a = make_args(s);
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S_in = S_in; a.dO = dO;
    a.dS_out = dS_out; a.dq = dq; a.dk_ = dk; a.dv_ = dv; a.dg = dg; a.dbeta = dbeta;
    a.dS_in = dS_in;
    bind_slot(a, ws, L, 0, true);
    SF_TRY(run_bwd_prep(a, cs));
    SF_TRY(run_bwd_grads(a, cs));
    return SF_OK;
}


}  // extern "C"

namespace {

// Layout of the buffer that keeps the forward's intermediates of every piece for
// a backward without recompute: piece i's region (the forward parts of a slot for
// lens[i] tokens, plus P and T on the tensor-core path) follows piece i-1's.
struct KeepPlan {
    std::vector<size_t> off;  // byte offset of each piece's region
    std::vector<WsLayout> lay;
    size_t total = 0;
};

int keep_parts(const sf_shape* s) {
    const bool tc = s->dtype == SF_BF16 && s->dk == kMaxD && s->dv == kMaxD;
    return kPartFwd | (tc ? kPartPT : 0);
}

void plan_keep(const sf_shape* s, int n_sub, const int* lens, KeepPlan& k) {
    k.off.resize(n_sub);
    k.lay.resize(n_sub);
    size_t off = 0;
    for (int i = 0; i < n_sub; ++i) {
        k.lay[i] = ws_layout_parts(s->B, lens[i], s->H, s->dk, s->dv, s->dtype, true, keep_parts(s), 1);
        k.off[i] = off;
        off += up256(k.lay[i].slot_bytes);
    }
    k.total = off;
}

// The forward driver; keep != NULL also stores every piece's intermediates there.
sf_status fwd_seq(const sf_shape* s, int n_sub, const int* lens, const void* q, const void* k,
                  const void* v, const float* g, const float* beta, const float* S_in, void* o,
                  float* S_out, float* S_saved, void* ws, size_t ws_bytes, void* keep,
                  size_t keep_bytes, void* stream_main, void* stream_aux) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    SeqPlan p;
    st = plan_seq(s, n_sub, lens, p);
    if (st != SF_OK) return st;
    const bool work = (size_t)s->B * s->H > 0;
    st = check_ptrs(s, work ? std::initializer_list<const void*>{q, k, v, o}
                            : std::initializer_list<const void*>{},
                    {q, k, v, o}, {g, beta, S_in, S_out, S_saved});
    if (st != SF_OK) return st;
    KeepPlan kp;
    if (keep) {
        plan_keep(s, n_sub, lens, kp);
        if (keep_bytes < kp.total || !aligned(keep, 256)) return SF_ERR_WORKSPACE;
    }
    if (!work) return SF_OK;
    const size_t nstate = (size_t)s->B * s->H * s->dk * s->dv;
    const WsLayout L = ws_layout(s->B, p.lmax, s->H, s->dk, s->dv, s->dtype, beta != nullptr, false,
                                 std::min(kSeqSlots, n_sub));
    const size_t need = L.total + 2 * nstate * sizeof(float);
    if (!ws || ws_bytes < need || !aligned(ws, 256)) return SF_ERR_WORKSPACE;
    float* pingpong = (float*)((char*)ws + L.total);
    cudaStream_t sm = (cudaStream_t)stream_main;
    cudaStream_t sa = stream_aux ? (cudaStream_t)stream_aux : sm;
    const size_t es = esize(s);
    const int ld_t = s->ld_t ? s->ld_t : s->T;

    // Schedule: the critical stream carries only the sequential state passes;
    // the aux stream runs the parallel work around them (intra of pieces i+1, i+2
    // ahead, output of piece i behind), three workspace slots in flight.
    constexpr int NS = kSeqSlots;
    EventSet evs;
    SF_TRY(evs.make(2 * NS + 3));
    cudaEvent_t* ev_intra = &evs.ev[0];   // intra of the slot's piece done (aux)
    cudaEvent_t* ev_state = &evs.ev[NS];  // state pass of the slot's piece done (critical)
    cudaEvent_t ev_start = evs.ev[2 * NS], ev_aux_done = evs.ev[2 * NS + 1];
    cudaEvent_t ev_crit_done = evs.ev[2 * NS + 2];
    cudaStream_t sc = sm;  // the state passes' stream
    if (sa != sm) SF_TRY(critical_stream(&sc));
    SF_TRY(cudaEventRecord(ev_start, sm));
    SF_TRY(cudaStreamWaitEvent(sa, ev_start, 0));
    SF_TRY(cudaStreamWaitEvent(sc, ev_start, 0));

    auto piece = [&](int i) {
        Args a = make_args(s);
        a.T = lens[i];
        a.NC = (lens[i] + kChunk - 1) / kChunk;
        a.ld_t = ld_t;
        const int t0 = p.start[i];
        a.q = tok_ptr(q, t0, s->H, s->dk, es);
        a.k = tok_ptr(k, t0, s->H, s->dk, es);
        a.v = tok_ptr(v, t0, s->H, s->dv, es);
        a.o = tok_ptr(o, t0, s->H, s->dv, es);
        a.g = (const float*)tok_ptr(g, t0, s->H, 1, 4);
        a.beta = (const float*)tok_ptr(beta, t0, s->H, 1, 4);
        // state entering piece i, and where the state leaving it goes
        const float* sin = (i == 0) ? S_in : (S_saved ? S_saved + (size_t)i * nstate
                                                      : pingpong + (size_t)((i - 1) & 1) * nstate);
        float* sout = (i == n_sub - 1) ? S_out
                                       : (S_saved ? S_saved + (size_t)(i + 1) * nstate
                                                  : pingpong + (size_t)(i & 1) * nstate);
        a.S_in = sin;
        a.S_out = sout;
        bind_slot(a, ws, L, i % kSeqSlots, false);
        if (keep) bind_parts(a, (char*)keep + kp.off[i], kp.lay[i], keep_parts(s));
        return a;
    };
    // with keep, the intra kernel also stores P and T (tensor-core path) for the backward
    auto run_intra_piece = [&](const Args& a) { return intra(a, keep != nullptr, sa); };

    if (S_saved) SF_TRY(copy_state(S_saved, S_in, nstate, sc));
    for (int j = 0; j < std::min(2, n_sub); ++j) {
        SF_TRY(run_intra_piece(piece(j)));
        SF_TRY(cudaEventRecord(ev_intra[j % NS], sa));
    }
    for (int i = 0; i < n_sub; ++i) {
        const Args a = piece(i);
        SF_TRY(cudaStreamWaitEvent(sc, ev_intra[i % NS], 0));
        SF_TRY(run_state_output(a, sc, false));
        SF_TRY(cudaEventRecord(ev_state[i % NS], sc));
        if (i + 2 < n_sub) {  // its slot's previous piece (i-1) finished its output
            SF_TRY(run_intra_piece(piece(i + 2)));
            SF_TRY(cudaEventRecord(ev_intra[(i + 2) % NS], sa));
        }
        SF_TRY(cudaStreamWaitEvent(sa, ev_state[i % NS], 0));
        SF_TRY(output(a, sa));
    }
    SF_TRY(cudaEventRecord(ev_aux_done, sa));
    SF_TRY(cudaEventRecord(ev_crit_done, sc));
    SF_TRY(cudaStreamWaitEvent(sm, ev_aux_done, 0));
    SF_TRY(cudaStreamWaitEvent(sm, ev_crit_done, 0));
    return SF_OK;
}

// The backward driver; keep != NULL reads the forward's intermediates from there
// (no recompute), else every piece is recomputed from S_saved.
sf_status bwd_seq(const sf_shape* s, int n_sub, const int* lens, const void* q, const void* k,
                  const void* v, const float* g, const float* beta, const float* S_saved,
                  const void* dO, const float* dS_out, void* dq, void* dk, void* dv, float* dg,
                  float* dbeta, float* dS_in, void* ws, size_t ws_bytes, const void* keep,
                  size_t keep_bytes, void* stream_main, void* stream_aux) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    if ((g != nullptr) != (dg != nullptr) || (beta != nullptr) != (dbeta != nullptr))
        return SF_ERR_INVALID;
    SeqPlan p;
    st = plan_seq(s, n_sub, lens, p);
    if (st != SF_OK) return st;
    const bool work = (size_t)s->B * s->H > 0;
    st = check_ptrs(s, work ? (keep ? std::initializer_list<const void*>{q, k, v, dO, dq, dk, dv}
                                    : std::initializer_list<const void*>{q, k, v, dO, dq, dk, dv, S_saved})
                            : std::initializer_list<const void*>{},
                    {q, k, v, dO, dq, dk, dv}, {g, beta, S_saved, dS_out, dg, dbeta, dS_in});
    if (st != SF_OK) return st;
    KeepPlan kp;
    if (keep) {
        plan_keep(s, n_sub, lens, kp);
        if (keep_bytes < kp.total || !aligned(keep, 256)) return SF_ERR_WORKSPACE;
    }
    if (!work) return SF_OK;
    const size_t nstate = (size_t)s->B * s->H * s->dk * s->dv;
    const WsLayout L = ws_layout(s->B, p.lmax, s->H, s->dk, s->dv, s->dtype, beta != nullptr, true,
                                 std::min(kSeqSlots, n_sub));
    const size_t need = L.total + 2 * nstate * sizeof(float);
    if (!ws || ws_bytes < need || !aligned(ws, 256)) return SF_ERR_WORKSPACE;
    float* pingpong = (float*)((char*)ws + L.total);
    cudaStream_t sm = (cudaStream_t)stream_main;
    cudaStream_t sa = stream_aux ? (cudaStream_t)stream_aux : sm;
    const size_t es = esize(s);
    const int ld_t = s->ld_t ? s->ld_t : s->T;

    // Schedule (pieces in reverse): the critical stream carries the sequential
    // passes of each piece (forward-state recompute unless kept, then the reverse
    // dS pass); the aux stream runs the parallel work (intra recompute two pieces
    // ahead unless kept, per-chunk gradients one piece behind), three workspace
    // slots in flight.
    constexpr int NS = kSeqSlots;
    EventSet evs;
    SF_TRY(evs.make(2 * NS + 3));
    cudaEvent_t* ev_prep = &evs.ev[0];    // intra recompute of the slot's piece done (aux)
    cudaEvent_t* ev_state = &evs.ev[NS];  // reverse pass of the slot's piece done (critical)
    cudaEvent_t ev_start = evs.ev[2 * NS], ev_aux_done = evs.ev[2 * NS + 1];
    cudaEvent_t ev_crit_done = evs.ev[2 * NS + 2];
    cudaStream_t sc = sm;  // the state passes' stream
    if (sa != sm) SF_TRY(critical_stream(&sc));
    SF_TRY(cudaEventRecord(ev_start, sm));
    SF_TRY(cudaStreamWaitEvent(sa, ev_start, 0));
    SF_TRY(cudaStreamWaitEvent(sc, ev_start, 0));

    auto piece = [&](int i) {
        Args a = make_args(s);
        a.T = lens[i];
        a.NC = (lens[i] + kChunk - 1) / kChunk;
        a.ld_t = ld_t;
        const int t0 = p.start[i];
        a.q = tok_ptr(q, t0, s->H, s->dk, es);
        a.k = tok_ptr(k, t0, s->H, s->dk, es);
        a.v = tok_ptr(v, t0, s->H, s->dv, es);
        a.dO = tok_ptr(dO, t0, s->H, s->dv, es);
        a.dq = tok_ptr(dq, t0, s->H, s->dk, es);
        a.dk_ = tok_ptr(dk, t0, s->H, s->dk, es);
        a.dv_ = tok_ptr(dv, t0, s->H, s->dv, es);
        a.g = (const float*)tok_ptr(g, t0, s->H, 1, 4);
        a.beta = (const float*)tok_ptr(beta, t0, s->H, 1, 4);
        a.dg = (float*)tok_ptr(dg, t0, s->H, 1, 4);
        a.dbeta = (float*)tok_ptr(dbeta, t0, s->H, 1, 4);
        a.S_in = S_saved ? S_saved + (size_t)i * nstate : nullptr;
        a.S_out = nullptr;
        // dS leaving piece i (from piece i+1) and dS entering it (to piece i-1)
        a.dS_out = (i == n_sub - 1) ? dS_out : pingpong + (size_t)((n_sub - 2 - i) & 1) * nstate;
        a.dS_in = (i == 0) ? dS_in : pingpong + (size_t)((n_sub - 1 - i) & 1) * nstate;
        bind_slot(a, ws, L, i % kSeqSlots, true);
        if (keep) bind_parts(a, (char*)keep + kp.off[i], kp.lay[i], keep_parts(s));
        return a;
    };

    if (!keep) {
        for (int j = n_sub - 1; j >= std::max(0, n_sub - 2); --j) {
            SF_TRY(intra(piece(j), true, sa));
            SF_TRY(cudaEventRecord(ev_prep[j % NS], sa));
        }
    }
    // ev_prep[slot]: without keep, the intra recompute of the slot's piece is done (it
    // was issued on the aux stream after the gradients of the slot's previous piece);
    // with keep, the gradients of the slot's previous piece are done.  Either way the
    // reverse pass may then overwrite the slot's dS'^T and dDelta^T.
    for (int i = n_sub - 1; i >= 0; --i) {
        const Args a = piece(i);
        if (!keep || i + NS < n_sub) SF_TRY(cudaStreamWaitEvent(sc, ev_prep[i % NS], 0));
        SF_TRY(keep ? run_bwd_state_kept(a, sc) : run_bwd_state(a, sc));
        SF_TRY(cudaEventRecord(ev_state[i % NS], sc));
        if (!keep && i - 2 >= 0) {  // its slot's previous piece (i+1) finished its gradients on this stream
            SF_TRY(intra(piece(i - 2), true, sa));
            SF_TRY(cudaEventRecord(ev_prep[(i - 2) % NS], sa));
        }
        SF_TRY(cudaStreamWaitEvent(sa, ev_state[i % NS], 0));
        // the reverse pass of piece i-1 (one CTA per batch-head) runs beside these gradients:
        // they keep off its SMs, or their resident CTAs, which take chunk-heads until none are
        // left, would hold the SMs the next reverse pass needs
        Args ag = a;
        if (i > 0) ag.grad_sms = -(s->B * s->H);
        SF_TRY(run_bwd_chunk_grads(ag, sa));
        if (keep) SF_TRY(cudaEventRecord(ev_prep[i % NS], sa));
    }
    SF_TRY(cudaEventRecord(ev_aux_done, sa));
    SF_TRY(cudaEventRecord(ev_crit_done, sc));
    SF_TRY(cudaStreamWaitEvent(sm, ev_aux_done, 0));
    SF_TRY(cudaStreamWaitEvent(sm, ev_crit_done, 0));
    return SF_OK;
}

}  // namespace

extern "C" {

sf_status sf_fwd_seq(const sf_shape* s, int n_sub, const int* lens, const void* q, const void* k,
                     const void* v, const float* g, const float* beta, const float* S_in, void* o,
                     float* S_out, float* S_saved, void* ws, size_t ws_bytes, void* stream_main,
                     void* stream_aux) {
    return fwd_seq(s, n_sub, lens, q, k, v, g, beta, S_in, o, S_out, S_saved, ws, ws_bytes, nullptr, 0,
                   stream_main, stream_aux);
}

sf_status sf_bwd_seq(const sf_shape* s, int n_sub, const int* lens, const void* q, const void* k,
                     const void* v, const float* g, const float* beta, const float* S_saved,
                     const void* dO, const float* dS_out, void* dq, void* dk, void* dv, float* dg,
                     float* dbeta, float* dS_in, void* ws, size_t ws_bytes, void* stream_main,
                     void* stream_aux) {
    return bwd_seq(s, n_sub, lens, q, k, v, g, beta, S_saved, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in,
                   ws, ws_bytes, nullptr, 0, stream_main, stream_aux);
}

size_t sf_keep_bytes(const sf_shape* s, int n_sub, const int* lens) {
    if (check_shape(s) != SF_OK || n_sub <= 0 || !lens) return 0;
    SeqPlan p;
    if (plan_seq(s, n_sub, lens, p) != SF_OK) return 0;
    KeepPlan kp;
    plan_keep(s, n_sub, lens, kp);
    return kp.total;
}

sf_status sf_fwd_seq_keep(const sf_shape* s, int n_sub, const int* lens, const void* q,
                          const void* k, const void* v, const float* g, const float* beta,
                          const float* S_in, void* o, float* S_out, void* keep, size_t keep_bytes,
                          void* ws, size_t ws_bytes, void* stream_main, void* stream_aux) {
    if (!keep) return SF_ERR_WORKSPACE;
    return fwd_seq(s, n_sub, lens, q, k, v, g, beta, S_in, o, S_out, nullptr, ws, ws_bytes, keep,
                   keep_bytes, stream_main, stream_aux);
}

sf_status sf_bwd_seq_keep(const sf_shape* s, int n_sub, const int* lens, const void* q,
                          const void* k, const void* v, const float* g, const float* beta,
                          const void* keep, size_t keep_bytes, const void* dO, const float* dS_out,
                          void* dq, void* dk, void* dv, float* dg, float* dbeta, float* dS_in,
                          void* ws, size_t ws_bytes, void* stream_main, void* stream_aux) {
    if (!keep) return SF_ERR_WORKSPACE;
    return bwd_seq(s, n_sub, lens, q, k, v, g, beta, nullptr, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in,
                   ws, ws_bytes, keep, keep_bytes, stream_main, stream_aux);
}

sf_status sf_check(void* ws, void* stream) {
    if (!ws) return SF_ERR_INVALID;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SF_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SF_ERR_CUDA;
    if (h != 0) {
        if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return SF_ERR_CUDA;
        return SF_ERR_TIMEOUT;
    }
    return SF_OK;
}

const char* sf_status_string(sf_status s) {
    switch (s) {
        case SF_OK: return "ok";
        case SF_ERR_INVALID: return "invalid argument";
        case SF_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case SF_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case SF_ERR_CUDA: return "CUDA error";
        case SF_ERR_TIMEOUT: return "a bounded device wait timed out";
    }
    return "unknown status";
}

void sf_timing_enable(int on) { g_timing_on = on != 0; }

void sf_timing_reset(void) {
    for (const TimingRec& r : g_recs) {
        g_pool.push_back(r.e0);
        g_pool.push_back(r.e1);
    }
    g_recs.clear();
    std::fill(g_ms, g_ms + KK_COUNT, 0.0);
    std::fill(g_launches, g_launches + KK_COUNT, 0);
}

int sf_timing_read(int cap, const char** names, int* launches, double* ms) {
    cudaDeviceSynchronize();
    for (const TimingRec& r : g_recs) {
        float t = 0.f;
        if (cudaEventElapsedTime(&t, r.e0, r.e1) == cudaSuccess) {
            g_ms[r.kind] += t;
            g_launches[r.kind] += 1;
        }
        g_pool.push_back(r.e0);
        g_pool.push_back(r.e1);
    }
    g_recs.clear();
    const int n = std::min(cap, (int)KK_COUNT);
    for (int i = 0; i < n; ++i) {
        if (names) names[i] = kernel_name(i);
        if (launches) launches[i] = g_launches[i];
        if (ms) ms[i] = g_ms[i];
    }
    return n;
}

int sf_timing_trace(int cap, int* kinds, int* streams, double* start_ms, double* end_ms) {
    cudaDeviceSynchronize();
    std::vector<cudaStream_t> seen;
    int n = 0;
    for (const TimingRec& r : g_recs) {
        if (n >= cap) break;
        int si = 0;
        while (si < (int)seen.size() && seen[si] != r.stream) ++si;
        if (si == (int)seen.size()) seen.push_back(r.stream);
        float t0 = -1.f, t1 = -1.f;
        cudaEventElapsedTime(&t0, g_recs.front().e0, r.e0);
        cudaEventElapsedTime(&t1, g_recs.front().e0, r.e1);
        if (kinds) kinds[n] = r.kind;
        if (streams) streams[n] = si;
        if (start_ms) start_ms[n] = t0;
        if (end_ms) end_ms[n] = t1;
        ++n;
    }
    return n;
}

}  // extern "C"
