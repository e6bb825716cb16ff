/*
 * sf.h -- C ABI of libsf, the chunkwise linear-recurrence layer for B200 (sm_100a).
 *
 * The layer is the linear recurrence with a d_k x d_v matrix state
 *
 *     S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,     o_t = S_t^T q_t,
 *
 * a_t = exp(g_t), in three forms: causal linear attention (no gate, no delta
 * term), scalar-decay gated linear attention, and the gated delta rule of Gated
 * DeltaNet, the architecture evaluated in the StateFlow summary (gptget.net,
 * "StateFlow: Sequence Pipeline Parallelism ...", section 实验设计).  A sequence
 * is cut into sub-sequences that run in order on one GPU; the boundary state S
 * is carried forward and its gradient dS backward ("StateFlow ...", Abstract;
 * "Sequence Accumulation and Beyond ...", Approach: fixed-length sub-sequences
 * processed one after another, accumulating a d x d memory state, with a
 * backward pass over stored states).  Inside a call the sequence is processed
 * in chunks of 64 tokens: an intra-chunk kernel, a state-transition pass over
 * chunks and an output kernel (gptget.net StateFlow summary, section 方法详解:
 * a linear-recurrence kernel inside each block, blocks joined by boundary
 * states, a low-latency state-transition kernel).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned.  The library never allocates, frees or synchronises, except
 *     sf_check (which synchronises the stream it is given).
 *   - Work is enqueued asynchronously on the given stream(s) (a cudaStream_t
 *     passed as void*; NULL is the legacy default stream).
 *   - Layouts (C order):  q, k: [B, ld_t, H, dk];  v, o, dO, dv: [B, ld_t, H, dv]
 *     (the call reads tokens [0, T) of each batch row);  g, beta, dg, dbeta:
 *     [B, ld_t, H] float32;  states S_in, S_out, dS_out, dS_in: [B, H, dk, dv]
 *     float32.  q, k, v, o, dO, dq, dk, dv have dtype shape->dtype.
 *   - g == NULL means a_t = 1 (no decay).  beta == NULL means plain linear
 *     attention, S_t = a_t S_{t-1} + k_t v_t^T.  S_in == NULL means a zero
 *     initial state; dS_out == NULL a zero incoming state gradient.
 *   - No attention scale is applied (scale 1); o_t reads the state after the
 *     update of token t.
 *   - On an argument error nothing is launched and an SF_ERR_* code returns.
 *     No C++ exception crosses this boundary.
 */
#ifndef SF_H_
#define SF_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SF_OK = 0,
    SF_ERR_INVALID = 1,     /* NULL/misaligned pointer, negative size, ld_t < T, lens not summing to T */
    SF_ERR_UNSUPPORTED = 2, /* dk or dv outside [1, 128], chunk != 64, unknown dtype */
    SF_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than sf_workspace_bytes() */
    SF_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
    SF_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (read by sf_check) */
} sf_status;

typedef enum { SF_F32 = 0, SF_BF16 = 1 } sf_dtype;

typedef enum { SF_OP_FWD = 0, SF_OP_BWD = 1 } sf_op;

typedef struct {
    int B, T, H;   /* batch rows, tokens in this call, heads */
    int dk, dv;    /* key and value head dimensions */
    int chunk;     /* tokens per chunk; must be 64 */
    int dtype;     /* sf_dtype of q, k, v, o, dO, dq, dk, dv */
    int ld_t;      /* tokens per batch row in memory (>= T); 0 means T */
} sf_shape;

/* Bytes of device workspace sf_fwd (op = SF_OP_FWD) or sf_bwd (SF_OP_BWD) needs
 * for this shape.  Returns 0 for an invalid shape.  The workspace is scratch:
 * its contents need not be preserved between calls, and two calls that may run
 * at the same time must not share one.  The exception is its first 16 bytes:
 * the device error word that bounded device waits set and sf_check reads and
 * clears (bytes 0-3), and the work counters of the gradient kernel (bytes
 * 8-15), which every launch leaves at zero.  They must be zero before the
 * workspace's first call: allocate it zeroed, or zero those bytes once.  This
 * holds for every workspace the sub-sequence drivers take as well. */
size_t sf_workspace_bytes(const sf_shape* shape, int op);

/* Forward over one sequence piece of T tokens:
 *   o[t] = S_t^T q[t] for t in [0, T) starting from S_in, and S_out = S_T.
 * S_out may be NULL.  T = 0 copies S_in (or zeros) to S_out. */
sf_status sf_fwd(const sf_shape* shape, const void* q, const void* k, const void* v,
                 const float* g, const float* beta, const float* S_in, void* o, float* S_out,
                 void* ws, size_t ws_bytes, void* stream);

/* Backward of sf_fwd for a loss L(o, S_out), given dO = dL/do and
 * dS_out = dL/dS_out.  Writes dq, dk, dv, dg (iff g != NULL; must then be
 * non-NULL), dbeta (iff beta != NULL) and dS_in = dL/dS_in (may be NULL).
 * Intra-chunk quantities and the chunk states are recomputed from the inputs
 * and S_in (activation recompute), so nothing from the forward is needed. */
sf_status sf_bwd(const sf_shape* shape, const void* q, const void* k, const void* v,
                 const float* g, const float* beta, const float* S_in, const void* dO,
                 const float* dS_out, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                 float* dS_in, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace for sf_fwd_seq / sf_bwd_seq with these sub-sequence
 * lengths (lens: host array of n_sub positive ints summing to shape->T). */
size_t sf_seq_workspace_bytes(const sf_shape* shape, int n_sub, const int* lens, int op);

/* Sub-sequence driver, forward.  shape->T is the whole sequence; lens (host
 * array) cuts it into n_sub pieces run in order, the state of piece i being
 * the initial state of piece i+1 (the Sequence Accumulation schedule).
 * S_saved (device, n_sub x [B, H, dk, dv] float32, may be NULL) receives the
 * state entering each piece, which sf_bwd_seq consumes.  The intra-chunk work
 * of piece i+1 is issued on stream_aux while the state pass of piece i runs
 * on stream_main (state overlap: StateFlow Abstract and 术语表 "状态重叠");
 * events order them.  When the two streams differ, the state passes run on
 * an internal stream of the device's greatest priority, forked from and
 * joined back to stream_main by events, so that the sequential critical path
 * is scheduled ahead of the parallel work (the first such call on a device
 * creates that stream; make it before any stream capture).  On return all
 * work is ordered before later work on stream_main.  stream_aux may equal
 * stream_main (no overlap, everything on stream_main).  The drivers may be
 * captured into a CUDA graph by capturing stream_main (stream_aux and the
 * internal stream join the capture through the drivers' event waits); a
 * replay runs the same kernels on the same pointers and gives the same bits. */
sf_status sf_fwd_seq(const sf_shape* shape, int n_sub, const int* lens, const void* q,
                     const void* k, const void* v, const float* g, const float* beta,
                     const float* S_in, void* o, float* S_out, float* S_saved, void* ws,
                     size_t ws_bytes, void* stream_main, void* stream_aux);

/* Sub-sequence driver, backward: pieces in reverse order, dS_in of piece i+1
 * being dS_out of piece i.  S_saved must hold the states sf_fwd_seq saved
 * (the stored boundary states the backward pass runs over). */
sf_status sf_bwd_seq(const sf_shape* shape, int n_sub, const int* lens, const void* q,
                     const void* k, const void* v, const float* g, const float* beta,
                     const float* S_saved, const void* dO, const float* dS_out, void* dq,
                     void* dk, void* dv, float* dg, float* dbeta, float* dS_in, void* ws,
                     size_t ws_bytes, void* stream_main, void* stream_aux);

/* Sub-sequence drivers without activation recompute.  The StateFlow summary
 * (gptget.net, sections 关键结果 and 方法详解) reports its pipeline both without
 * and with activation recompute; sf_fwd_seq / sf_bwd_seq are the recompute
 * form (the backward re-runs every piece from its stored entering state), these
 * are the other: the forward keeps every piece's intermediates in `keep` and
 * the backward reads them instead of recomputing.  That skips the intra-chunk
 * kernel and the forward state pass of every piece in the backward at the cost
 * of device memory that grows with T.
 *
 * sf_keep_bytes: bytes of `keep` for this shape and cut (0 on an invalid
 * argument).  On the bf16 path with d_k = d_v = 128 that is about 97 KB per
 * 64-token chunk and head: the cumulative decay, W^T, U^T, the chunk states,
 * Delta^T, P and T; on the other paths the same minus P and T, at fp32.
 *
 * sf_fwd_seq_keep: as sf_fwd_seq, with `keep` (device, 256-byte aligned,
 * keep_bytes >= sf_keep_bytes) receiving the intermediates; ws is the same
 * workspace as sf_fwd_seq's (sf_seq_workspace_bytes(..., SF_OP_FWD)).
 * sf_bwd_seq_keep: as sf_bwd_seq, reading `keep` as the forward left it (same
 * q, k, v, g, beta, shape and lens) instead of S_saved; ws as sf_bwd_seq's.
 * `keep` NULL or too small, or misaligned: SF_ERR_WORKSPACE. */
size_t sf_keep_bytes(const sf_shape* shape, int n_sub, const int* lens);

sf_status sf_fwd_seq_keep(const sf_shape* shape, int n_sub, const int* lens, const void* q,
                          const void* k, const void* v, const float* g, const float* beta,
                          const float* S_in, void* o, float* S_out, void* keep, size_t keep_bytes,
                          void* ws, size_t ws_bytes, void* stream_main, void* stream_aux);

sf_status sf_bwd_seq_keep(const sf_shape* shape, int n_sub, const int* lens, const void* q,
                          const void* k, const void* v, const float* g, const float* beta,
                          const void* keep, size_t keep_bytes, const void* dO, const float* dS_out,
                          void* dq, void* dk, void* dv, float* dg, float* dbeta, float* dS_in,
                          void* ws, size_t ws_bytes, void* stream_main, void* stream_aux);

/* Forward without a caller workspace, for callers that cannot allocate device
 * memory (a plugin that is handed only its input and output buffers by a
 * framework that plans all memory up front, code running inside an
 * allocator's callbacks, or loops that must not call cudaMalloc because it can
 * synchronise the device).  The pages have no counterpart: this is an
 * interface convenience, not part of the method.
 *
 * Same arguments, semantics and errors as sf_fwd minus (ws, ws_bytes).  The
 * scratch is a fixed 32 MiB array compiled into the library, held in device
 * memory by every GPU that loads the library until the process exits.  A shape
 * whose sf_workspace_bytes(shape, SF_OP_FWD) exceeds 32 MiB is rejected with
 * SF_ERR_WORKSPACE before anything is launched (bf16, d_k = d_v = 128 needs
 * about 1.3 KB per token and head).  Each call looks up the array's device
 * address in the current device's context; the first lookup on a device may
 * load the library's device code, so make the first call on each device before
 * any stream capture.  All calls share the one array: calls whose work may
 * overlap on the GPU (other streams, other host threads) race on it, calls
 * ordered on one stream do not.  The array keeps the previous call's contents;
 * each call first clears the error word that bounded device waits set (it lives
 * in the array), so read it with sf_check_noalloc after a call and before the
 * next one.  Allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine is called. */
sf_status sf_fwd_noalloc(const sf_shape* shape, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* S_in, void* o,
                         float* S_out, void* stream);

/* sf_check for sf_fwd_noalloc: synchronises `stream`, then reads and clears the
 * error word of the built-in scratch array on the current device.  Returns
 * SF_ERR_TIMEOUT if a kernel of an sf_fwd_noalloc call gave up a bounded wait
 * since the word was last cleared, SF_ERR_CUDA on a CUDA error, else SF_OK. */
sf_status sf_check_noalloc(void* stream);

/* Synchronises `stream`, then reads and clears the device error word kept at
 * the head of workspace `ws`.  Returns SF_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last check, SF_ERR_CUDA on a CUDA error, else SF_OK. */
sf_status sf_check(void* ws, void* stream);

/* Static string for a status code. */
const char* sf_status_string(sf_status status);

/* Per-kernel timing (profiling aid).  While enabled, every kernel launch of the
 * library is bracketed by CUDA events recorded on the stream it is launched
 * on.  sf_timing_read synchronises the device, then for each kernel kind k
 * writes launches[k] and total milliseconds ms[k] accumulated since the last
 * reset, and names[k] a static name; it returns the number of kinds (at most
 * `cap`).  sf_timing_enable(0) stops recording; sf_timing_reset clears. */
void sf_timing_enable(int on);
void sf_timing_reset(void);
int sf_timing_read(int cap, const char** names, int* launches, double* ms);

/* Timeline of the launches recorded since the last reset or read, in launch
 * order (profiling aid): synchronises the device, then for the first `cap`
 * records writes the kernel kind (an index into sf_timing_read's names), the
 * stream as a small index in order of first appearance, and the start and end
 * in milliseconds after the start of the first record.  Records are kept (a
 * later sf_timing_read still totals them).  Returns the number written. */
int sf_timing_trace(int cap, int* kinds, int* streams, double* start_ms, double* end_ms);

/* Profile-guided cut into sub-sequences (host code; no GPU is touched).
 *
 * The StateFlow pages choose nonuniform block lengths from a profile of the
 * kernels so that the sequential state passes and the parallel per-block work
 * pipeline with fewer bubbles (StateFlow (newx.sg), Abstract; StateFlow
 * (gptget.net), 术语表 and 方法详解).  sf_chunk_costs holds a profile: the
 * microseconds one 64-token chunk of all B x H heads costs in each kernel of the
 * drivers that keep the forward's intermediates, the parallel kernels measured
 * on the whole GPU, the state passes with one CTA per batch-head, and the SM
 * count.  Every field must be >= 0 and sms > 0.  The model counts work, not the
 * tail of a launch's last wave of CTAs; min_chunks keeps the planner away from
 * pieces so short that those tails dominate. */
typedef struct {
    double intra_us;      /* intra-chunk kernel (storing P and T), whole GPU */
    double output_us;     /* output kernel, whole GPU */
    double grad_us;       /* per-chunk gradient kernel(s), whole GPU */
    double state_fwd_us;  /* forward state pass */
    double state_bwd_us;  /* reverse (dS) pass */
    int sms;              /* SMs of the GPU */
    int min_chunks;       /* shortest piece sf_plan_cut may choose, in 64-token chunks (0: one) */
} sf_chunk_costs;

/* Modelled device time (microseconds) of sf_fwd_seq_keep followed by
 * sf_bwd_seq_keep for the cut `lens` (host array of n_sub positive lengths
 * summing to shape->T): the two streams of the drivers replayed with the
 * state pass holding min(B*H, sms) SMs and the parallel kernels sharing the
 * rest.  Returns -1 for invalid arguments. */
double sf_model_seq_us(const sf_shape* shape, int n_sub, const int* lens, const sf_chunk_costs* costs);

/* Writes to lens_out (host array of n_sub ints) a cut of shape->T tokens into
 * n_sub pieces, each a multiple of 64 tokens except that a ragged last chunk
 * shortens the last piece, chosen to minimise sf_model_seq_us: the even cut, or
 * one whose last pieces ramp up geometrically from a short last piece (the
 * backward starts with the last piece's reverse pass alone).  SF_ERR_INVALID
 * for NULL pointers, invalid costs, T <= 0 or n_sub outside [1, ceil(T/64)]. */
sf_status sf_plan_cut(const sf_shape* shape, int n_sub, const sf_chunk_costs* costs, int* lens_out);

#ifdef __cplusplus
}
#endif

#endif /* SF_H_ */
