// Tensor-core state-transition passes (sm_100a, bf16 operands, fp32 state).
//
// This is the low-latency state-transition kernel of the StateFlow summary
// (gptget.net, section 方法详解: chunks joined by boundary states, a
// low-latency state-transition kernel): sequential over the chunks of one
// head, one CTA per (batch, head), the d_k x d_v state held on chip in fp32.
//
// The state is kept transposed, S^T (d_v rows = TMEM lanes, d_k columns), so
// both per-chunk products are M = 128 UMMAs:
//   X^T      = S^T W^T                    (128 x 64,  K = d_k)
//   Delta^T  = U^T - X^T                   (threads, fp32)
//   P^T      = (diag(e^{G_C - G}) Delta)^T K   (128 x 128, K = 64 tokens)
//   S^T     <- gamma_C S^T + P^T            (threads, fp32 registers)
// which is S' = gamma_C S + Ktil^T Delta with the decay moved from K onto
// Delta (Ktil^T Delta = K^T diag(e^{G_C - G}) Delta), so K feeds the tensor
// core straight from its TMA tile.  S^T is rounded to bf16 only as an MMA
// operand, which the element-wise warps write into TMEM (and for the stored
// chunk states); the carried state stays fp32 in registers.
//
// Per chunk c the forward pass stores S^T entering c and Delta^T (both bf16)
// for the output and gradient kernels; W^T, U^T, K and the decay table of the
// chunks ahead are prefetched by TMA into a 3-stage ring.  The reverse pass
// (further down) mirrors it with a 2-stage ring.

#include <cuda.h>
#include <cudaTypedefs.h>

#include "../../include/sf.h"
#include "sf_internal.h"
#include "tc_common.cuh"

namespace sf {

bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapDataType dtype,
               CUtensorMapSwizzle swz) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return false;
        fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    cuuint64_t d[5];
    cuuint64_t st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) st[i] = strides_bytes[i];
    }
    CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

using namespace tc;

constexpr int kD = 128;                 // d_k = d_v on this path
constexpr int kTile = 128 * 64 * 2;     // one 128-row x 128-byte bf16 tile (16 KB)
constexpr int kStages = 3;

// Thread layout of both passes: 16 element-wise warps; warp w reads TMEM lane
// quadrant (w & 3), i.e. d_v rows j = 32 (w & 3) + lane, and owns the column
// quarter p = w >> 2 of every per-row tile (16 of 64 token columns, 32 of 128
// state columns), so each step's elementwise work is split four ways per row.
constexpr int kThreads = 512;
// Both passes add two warps whose first threads issue: one the UMMAs of the
// dependent chain, the other the copies and stores (and, in the reverse pass,
// the products off the chain), so that neither waits on the other's issues.
constexpr int kFwdThreads = kThreads + 64;
constexpr int kFwdChain = kThreads, kFwdCopy = kThreads + 32;

// Shared-memory carve-up of the forward pass (byte offsets from a 1024-byte aligned base).
struct FwdSmem {
    static constexpr int Wt = 0;                          // [stage] W^T  [d_k][64 r]
    static constexpr int Kt = Wt + kStages * kTile;       // [stage] K    [2][64 r][64 d_k]
    static constexpr int Ut = Kt + kStages * kTile;       // [stage] U^T  [d_v][64 r]
    static constexpr int St = Ut + kStages * kTile;       // S^T staging for its store [2 kblk][d_v][64]
    static constexpr int Dst = St + 2 * kTile;            // Delta^T staging for its store
    static constexpr int Ed = Dst + kTile;                // [stage][128] fp32 decay table
    static constexpr int Bar = Ed + kStages * 512;        // barriers, see the kernel
    static constexpr int Misc = Bar + (kStages + 10) * 8;  // TMEM base, abort flag
    static constexpr int Size = Misc + 16;
};

// 32 fp32 values as four bf16 16-byte chunks q0 .. q0+3 of row `row` of a swizzled tile.
__device__ __forceinline__ void put_row32(uint8_t* tile, int row, int q0, const float* v) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 u;
        u.x = pack_bf16(v[q * 8 + 0], v[q * 8 + 1]);
        u.y = pack_bf16(v[q * 8 + 2], v[q * 8 + 3]);
        u.z = pack_bf16(v[q * 8 + 4], v[q * 8 + 5]);
        u.w = pack_bf16(v[q * 8 + 6], v[q * 8 + 7]);
        *(uint4*)(tile + sw128(row, q0 + q)) = u;
    }
}

// Forward state pass.  Both per-chunk products take their A operand from tensor
// memory, where the element-wise warps put it as bf16 pairs: S^T (entering the
// chunk) for X^T = S^T W^T, and (e^{G_C - G} Delta)^T for P^T = ... K.  The
// dependent chain of a chunk is therefore UMMA -> TMEM -> registers -> TMEM ->
// UMMA; the bf16 copies of S^T and Delta^T that go to global memory are staged
// in shared memory and stored by TMA off that chain, while the next product
// runs, by the other issuing thread.  The warps hand over through mbarriers
// (one arrival per element-wise warp):
//   bar_s    S^T of chunk c in TMEM            bar_x  X^T of chunk c done (commit)
//   bar_d    scaled Delta^T in TMEM            bar_p  P^T of chunk c done (commit)
//   bar_sst  S^T staged for its store          bar_sfree  that store has read the tile
//   bar_dst  Delta^T staged for its store      bar_dfree  that store has read the tile
// TMEM (512 columns): X^T [0, 64), P^T [64, 192), S^T operand [192, 256),
// Delta^T operand [256, 288).
template <bool kDelta>
__global__ void __launch_bounds__(kFwdThreads, 1)
    state_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_wt,
                        const __grid_constant__ CUtensorMap tm_ut,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_sc,
                        const __grid_constant__ CUtensorMap tm_dt, const Args a) {
    using L = FwdSmem;
    extern __shared__ uint8_t smem_raw[];
    // the 1024-aligned base by integer rounding: with the pointer arithmetic of the other
    // kernels the reverse pass, run right after the forward pass on the same stream, gave
    // up a bounded wait a few times in a thousand steps (the cause is not known)
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Eds = (float*)(sm + L::Ed);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);  // [kStages], count 1
    uint64_t* bar_x = bar_ld + kStages;           // count 1 (commits)
    uint64_t* bar_p = bar_x + 1;
    uint64_t* bar_s = bar_x + 2;                  // count 16 (one arrival per element-wise warp)
    uint64_t* bar_d = bar_x + 3;
    uint64_t* bar_sst = bar_x + 4;
    uint64_t* bar_dst = bar_x + 5;
    uint64_t* bar_sfree = bar_x + 6;              // count 1 (the issuer)
    uint64_t* bar_dfree = bar_x + 7;
    uint64_t* bar_fin = bar_x + 8;                // count 2 (both issuers)
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, part = warp >> 2;
    const int j = quad * 32 + lane;  // d_v row = TMEM lane
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC;

    if (tid == kFwdCopy) {
        for (int i = 0; i < kStages + 9; ++i) {
            const int k = i - kStages;  // 2..5: the element-wise hand-overs; 8: both issuers
            mbar_init(bar_ld + i, (k >= 2 && k <= 5) ? 16 : (k == 8 ? 2 : 1));
        }
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(s_tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tX = tmem, tP = tmem + 64, tS = tmem + 192, tD = tmem + 256;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

    // the issuers' waits: a wait that gives up flags the abort; later waits are skipped
    bool ok = true;
    int err = 0;
    auto iwait = [&](uint64_t* bar, uint32_t parity, int e) {
        if (ok && !mbar_wait_or_abort(bar, parity, s_abort)) {
            ok = false;
            err = e;
            *s_abort = 1;
        }
    };
    if (tid == kFwdChain) {
        // ---------------- the chain's UMMAs
        for (int c = 0; c < NC; ++c) {
            const int s = c % kStages;
            const uint32_t par = c & 1;
            iwait(&bar_ld[s], (c / kStages) & 1, kErrTimeoutTma);
            iwait(bar_s, par, kErrTimeoutMma);  // S^T entering chunk c is in TMEM
            if (ok && kDelta) {
                tc_fence_after();
                const uint32_t b0 = smem_u32(sm + L::Wt + s * kTile);
                constexpr uint32_t id = idesc_bf16(128, 64, false, true);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ts(tX, tS + 8 * ks, sdesc(b0 + ks * 2048, 8192, 1024), id, ks > 0);
            }
            mma_commit(bar_x);
            iwait(bar_d, par, kErrTimeoutMma);  // (e^{G_C - G} Delta)^T is in TMEM
            if (ok) {
                tc_fence_after();
                const uint32_t b0 = smem_u32(sm + L::Kt + s * kTile);
                constexpr uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ts(tP, tD + 8 * ks, sdesc(b0 + ks * 2048, 8192, 1024), id, ks > 0);
            }
            mma_commit(bar_p);
        }
        if (!ok) atomicExch(a.err, err);
        mma_commit(bar_fin);  // every UMMA issued has finished before the TMEM is freed
        mbar_wait(bar_fin, 0);
    } else if (tid == kFwdCopy) {
        // ---------------- copies and stores
        auto issue_load = [&](int c) {
            const int s = c % kStages;
            const uint32_t bytes = (kDelta ? kTile : 0) + 2 * kTile + 512;
            mbar_expect_tx(&bar_ld[s], bytes);
            if (kDelta) tma_load_2d(sm + L::Wt + s * kTile, &tm_wt, 0, (bh * NC + c) * kD, &bar_ld[s]);
            tma_load_2d(sm + L::Ut + s * kTile, &tm_ut, 0, (bh * NC + c) * kD, &bar_ld[s]);
            tma_load_4d(sm + L::Kt + s * kTile, &tm_k, 0, h, c * kChunk, b, &bar_ld[s]);
            tma_load_4d(sm + L::Kt + s * kTile + kTile / 2, &tm_k, 64, h, c * kChunk, b, &bar_ld[s]);
            bulk_load(Eds + s * 128, a.Ed + ((size_t)bh * NC + c) * 128, 512, &bar_ld[s]);
        };
        int issued = 0;
        for (; issued < min(kStages, NC); ++issued) issue_load(issued);
        for (int c = 0; c < NC; ++c) {
            const uint32_t par = c & 1;
            // the stage of chunk c-1 is free once S^T of chunk c is handed over: the products
            // of c-1 are done and the element-wise warps have read its tiles (waited before
            // bar_dfree below lets them reach the next hand-over of S^T)
            iwait(bar_s, par, kErrTimeoutMma);
            if (ok && c >= 1 && issued < NC) {
                issue_load(issued);
                ++issued;
            }
            // the chunk state entering c to global memory, staged while X^T is computed
            iwait(bar_sst, par, kErrTimeoutMma);
            if (ok) {
                tma_store_2d(&tm_sc, sm + L::St, 0, (bh * NC + c) * kD);
                tma_store_2d(&tm_sc, sm + L::St + kTile, 64, (bh * NC + c) * kD);
            }
            bulk_commit();
            bulk_wait_read<1>();  // the Delta^T store of chunk c-1 has read its tile
            if (c > 0) mbar_arrive(bar_dfree);
            iwait(bar_dst, par, kErrTimeoutMma);
            if (ok) tma_store_2d(&tm_dt, sm + L::Dst, 0, (bh * NC + c) * kD);
            bulk_commit();
            bulk_wait_read<1>();  // the S^T store of chunk c has read its tile
            mbar_arrive(bar_sfree);
        }
        if (!ok) atomicExch(a.err, err);
        // teardown: copies still in flight land and the stores have read shared memory
        // before the CTA exits
        if (*s_abort)
            for (int cc = 0; cc < issued; ++cc) mbar_wait(&bar_ld[cc % kStages], (cc / kStages) & 1);
        mma_commit(bar_fin);
        mbar_wait(bar_fin, 0);
        bulk_wait_read<0>();
    } else if (warp < 16) {
        // ---------------- the element-wise warps
        // `bad` stays warp-uniform (the warp-collective TMEM accesses and __syncwarp
        // below need every lane): a failed wait in any lane ends the warp's loop
        bool bad = false;
        auto wait = [&](uint64_t* bar, uint32_t parity, int e) {
            if (!bad && !mbar_wait_or_abort(bar, parity, s_abort)) {
                bad = true;
                if (!*s_abort) atomicExch(a.err, e);
                *s_abort = 1;
            }
            bad = __any_sync(0xffffffffu, bad);
        };
        auto hand_over_tmem = [&](uint64_t* bar) {  // after tcgen05.st of an operand
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        auto hand_over_smem = [&](uint64_t* bar) {  // after shared-memory writes a TMA store reads
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // S^T row j, state columns i in [32 part, 32 part + 32): S[q] = S_{i, j}
        float S[32];
#pragma unroll
        for (int q = 0; q < 32; ++q)
            S[q] = a.S_in ? a.S_in[((size_t)bh * kD + part * 32 + q) * kD + j] : 0.f;
        uint8_t* St = sm + L::St + (part >> 1) * kTile;
        const int sq0 = (part & 1) * 4;  // first 16-byte chunk of this thread's 32 state columns
        for (int c = 0; c < NC && !bad; ++c) {
            const int s = c % kStages;
            const uint32_t par = c & 1;
            // (1) S^T as bf16 pairs into TMEM: the A operand of X^T = S^T W^T
            {
                uint32_t w[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) w[q] = pack_bf16(S[2 * q], S[2 * q + 1]);
                tmem_st16u(tS + lane_base + 16 * part, w);
            }
            hand_over_tmem(bar_s);
            // (2) the same bf16 S^T staged for its store, once the last one has read the tile
            if (c > 0) wait(bar_sfree, (c - 1) & 1, kErrTimeoutTma);
            put_row32(St, j, sq0, S);
            hand_over_smem(bar_sst);
            // (3) Delta^T[j][r] = U^T[j][r] - X^T[j][r] for tokens r in [16 part, 16 part + 16);
            // e^{G_C - G_r} Delta^T into TMEM (A operand of P^T), Delta^T kept for its store
            wait(&bar_ld[s], (c / kStages) & 1, kErrTimeoutTma);
            float X[16];
            if (kDelta) {
                wait(bar_x, par, kErrTimeoutMma);
                tc_fence_after();
                tmem_ld16(tX + lane_base + part * 16, X);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) X[q] = 0.f;
            }
            const float* E = Eds + s * 128;
            const uint8_t* Ut = sm + L::Ut + s * kTile;
            uint32_t dw[8], tw[8];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const int q = part * 2 + qq;  // tokens 8q .. 8q + 7
                const uint4 u = *(const uint4*)(Ut + sw128(j, q));
                const float4 e0 = *(const float4*)(E + q * 8), e1 = *(const float4*)(E + q * 8 + 4);
                const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 uf = unpack_bf16(uw[p]);
                    const float d0 = uf.x - X[qq * 8 + 2 * p];
                    const float d1 = uf.y - X[qq * 8 + 2 * p + 1];
                    dw[qq * 4 + p] = pack_bf16(d0, d1);
                    tw[qq * 4 + p] = pack_bf16(d0 * ev[2 * p], d1 * ev[2 * p + 1]);
                }
            }
            tmem_st8u(tD + lane_base + 8 * part, tw);
            hand_over_tmem(bar_d);
            // (4) Delta^T staged for its store
            if (c > 0) wait(bar_dfree, (c - 1) & 1, kErrTimeoutTma);
#pragma unroll
            for (int qq = 0; qq < 2; ++qq)
                *(uint4*)(sm + L::Dst + sw128(j, part * 2 + qq)) =
                    make_uint4(dw[qq * 4], dw[qq * 4 + 1], dw[qq * 4 + 2], dw[qq * 4 + 3]);
            hand_over_smem(bar_dst);
            // (5) S^T <- gamma_C S^T + P^T
            wait(bar_p, par, kErrTimeoutMma);
            tc_fence_after();
            float P[32];
            tmem_ld32(tP + lane_base + part * 32, P);
            tmem_ld_wait();
            const float gam = E[64 + kChunk - 1];  // gamma_C
#pragma unroll
            for (int q = 0; q < 32; ++q) S[q] = gam * S[q] + P[q];
        }
        if (!bad && a.S_out) {
#pragma unroll
            for (int q = 0; q < 32; ++q) a.S_out[((size_t)bh * kD + part * 32 + q) * kD + j] = S[q];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Shared-memory carve-up of the reverse pass (byte offsets from a 1024-aligned base).
constexpr int kBStages = 2;
struct BwdSmem {
    static constexpr int Kt = 0;                          // [stage] K   [2][64 r][64 d_k]
    static constexpr int dO = Kt + kBStages * kTile;      // [stage] dO  [2][64 r][64 d_v]
    static constexpr int Q = dO + kBStages * kTile;       // [stage] Q   [2][64 r][64 d_k], scaled in place
    static constexpr int Wt = Q + kBStages * kTile;       // [stage] W^T [d_k][64 r]
    static constexpr int P = Wt + kBStages * kTile;       // [stage] P   [64 i][64 r]
    static constexpr int St = P + kBStages * 8192;        // dS'^T staging for its store [2 kblk][d_v][64]
    static constexpr int Dst = St + 2 * kTile;            // dDelta^T [d_v][64 r] (or dv [2][64 r][64 d_v]) staging
    static constexpr int Ed = Dst + kTile;                // [stage][128] fp32 decay table
    static constexpr int Bar = Ed + kBStages * 512;       // barriers, see the kernel
    static constexpr int Misc = Bar + 16 * 8;             // TMEM base, abort flag (13 barriers)
    static constexpr int Size = Misc + 16;
};

// Reverse pass over the chunks of one head, carrying dS^T in fp32 registers:
//   dDelta^T = diag-scaled (dS'^T K^T) + dO^T P           (UMMAs, then threads)
//   dS^T    <- gamma_C dS'^T + dO^T (diag(gamma) Q) - dDelta^T W
// (the transpose of dS = gamma_C dS' + (diag(gamma) Q)^T dO - W^T dDelta with
// dDelta = P^T dO + Ktil dS').  Stores dS'^T of every chunk and dDelta^T (or
// dv = dDelta directly for linear attention).
//
// As in the forward pass, the two products on the dependent chain take their
// A operand from TMEM (dS'^T, and -dDelta^T in bf16 pairs) and the bf16 copies
// for global memory are staged off the chain.  Two issuing threads, each the
// first of its own warp: one issues the chain's UMMAs (dS'^T K^T, then
// dO^T (diag(gamma) Q) behind it while the element-wise warps form dDelta^T,
// then - dDelta^T W); the other every copy and store, and dO^T P of the next
// chunk as soon as its tiles have landed, so that neither waits on the other's
// slow issues.  Hand-overs (one arrival per element-wise warp):
//   bar_s    dS'^T of chunk c in TMEM        bar_y   dS'^T K^T done (commit)
//   bar_q    Q of chunk c scaled by gamma     bar_y2  dO^T P done (commit)
//   bar_d    -dDelta^T in TMEM (dO^T P read)  bar_z   dS^T update product done
//   bar_sst  dS'^T staged for its store       bar_sfree / bar_dfree  stores have
//   bar_dst  dDelta^T (or dv) staged          read their tiles
// TMEM (512 columns): dS'^T K^T [0, 64), dO^T P [64, 128), the dS^T update
// [128, 256), dS'^T operand [256, 320), -dDelta^T operand [320, 352).
constexpr int kBwdThreads = kFwdThreads;
constexpr int kBwdChain = kFwdChain, kBwdCopy = kFwdCopy;
template <bool kDelta>
__global__ void __launch_bounds__(kBwdThreads, 1)
    state_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_wt,
                        const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_dsc,
                        const __grid_constant__ CUtensorMap tm_ddt, const __grid_constant__ CUtensorMap tm_dv,
                        const Args a) {
    using L = BwdSmem;
    extern __shared__ uint8_t smem_raw[];
    // the 1024-aligned base by integer rounding: with the pointer arithmetic of the other
    // kernels the reverse pass, run right after the forward pass on the same stream, gave
    // up a bounded wait a few times in a thousand steps (the cause is not known)
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Eds = (float*)(sm + L::Ed);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);  // [kBStages], count 1
    uint64_t* bar_y = bar_ld + kBStages;          // count 1 (commits and the copy thread)
    uint64_t* bar_y2 = bar_y + 1;
    uint64_t* bar_z = bar_y + 2;
    uint64_t* bar_sfree = bar_y + 3;
    uint64_t* bar_dfree = bar_y + 4;
    uint64_t* bar_fin = bar_y + 5;                // count 2 (both issuers)
    uint64_t* bar_s = bar_y + 6;                  // count 16 (one arrival per element-wise warp)
    uint64_t* bar_q = bar_y + 7;
    uint64_t* bar_d = bar_y + 8;
    uint64_t* bar_sst = bar_y + 9;
    uint64_t* bar_dst = bar_y + 10;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, part = warp >> 2;
    const int j = quad * 32 + lane;  // d_v row = TMEM lane
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC;

    if (tid == kBwdCopy) {
        for (int i = 0; i < kBStages + 11; ++i) {
            const int k = i - kBStages;
            mbar_init(bar_ld + i, k < 5 ? 1 : (k == 5 ? 2 : 16));
        }
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(s_tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tY1 = tmem, tY2 = tmem + 64, tZ = tmem + 128, tS = tmem + 256, tD = tmem + 320;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

    // the issuers' waits: a wait that gives up flags the abort; later waits are skipped
    bool ok = true;
    int err = 0;
    auto iwait = [&](uint64_t* bar, uint32_t parity, int e) {
        if (ok && !mbar_wait_or_abort(bar, parity, s_abort)) {
            ok = false;
            err = e;
            *s_abort = 1;
        }
    };
    if (tid == kBwdChain) {
        // ---------------- the chain's UMMAs; the n-th iteration is chunk NC - 1 - n, stage n % 2
        for (int n = 0; n < NC; ++n) {
            const int s = n % kBStages;
            const uint32_t par = n & 1;
            iwait(bar_s, par, kErrTimeoutMma);  // dS'^T of chunk c is in TMEM
            iwait(&bar_ld[s], (n / kBStages) & 1, kErrTimeoutTma);
            if (ok) {
                tc_fence_after();
                const uint32_t kt = smem_u32(sm + L::Kt + s * kTile);
                constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)  // dS'^T K^T
                    mma_bf16_ts(tY1, tS + 8 * ks, sdesc(kt + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id,
                                ks > 0);
            }
            mma_commit(bar_y);
            iwait(bar_q, par, kErrTimeoutMma);  // Q of chunk c scaled by gamma
            if (ok) {
                tc_fence_after();
                const uint32_t dob = smem_u32(sm + L::dO + s * kTile), qb = smem_u32(sm + L::Q + s * kTile);
                constexpr uint32_t id = idesc_bf16(128, 128, true, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // dO^T (diag(gamma) Q)
                    mma_bf16(tZ, sdesc(dob + ks * 2048, 8192, 1024), sdesc(qb + ks * 2048, 8192, 1024), id, ks > 0);
            }
            iwait(bar_d, par, kErrTimeoutMma);  // -dDelta^T in TMEM
            if (ok && kDelta) {
                tc_fence_after();
                const uint32_t wt = smem_u32(sm + L::Wt + s * kTile);
                constexpr uint32_t id = idesc_bf16(128, 128, false, false);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // - dDelta^T W
                    mma_bf16_ts(tZ, tD + 8 * ks, sdesc(wt + ks * 32, 16, 1024), id, 1);
            }
            mma_commit(bar_z);
        }
        if (!ok) atomicExch(a.err, err);
        mma_commit(bar_fin);  // every UMMA of this thread has finished before the TMEM is freed
        mbar_wait(bar_fin, 0);
    } else if (tid == kBwdCopy) {
        // ---------------- copies, stores and dO^T P
        auto issue_load = [&](int n) {
            const int c = NC - 1 - n, s = n % kBStages;
            const uint32_t bytes = 3 * kTile + 8192 + (kDelta ? kTile : 0) + 512;
            mbar_expect_tx(&bar_ld[s], bytes);
            tma_load_4d(sm + L::Kt + s * kTile, &tm_k, 0, h, c * kChunk, b, &bar_ld[s]);
            tma_load_4d(sm + L::Kt + s * kTile + 8192, &tm_k, 64, h, c * kChunk, b, &bar_ld[s]);
            tma_load_4d(sm + L::dO + s * kTile, &tm_do, 0, h, c * kChunk, b, &bar_ld[s]);
            tma_load_4d(sm + L::dO + s * kTile + 8192, &tm_do, 64, h, c * kChunk, b, &bar_ld[s]);
            tma_load_4d(sm + L::Q + s * kTile, &tm_q, 0, h, c * kChunk, b, &bar_ld[s]);
            tma_load_4d(sm + L::Q + s * kTile + 8192, &tm_q, 64, h, c * kChunk, b, &bar_ld[s]);
            if (kDelta) tma_load_2d(sm + L::Wt + s * kTile, &tm_wt, 0, (bh * NC + c) * kD, &bar_ld[s]);
            tma_load_2d(sm + L::P + s * 8192, &tm_p, 0, (bh * NC + c) * kChunk, &bar_ld[s]);
            bulk_load(Eds + s * 128, a.Ed + ((size_t)bh * NC + c) * 128, 512, &bar_ld[s]);
        };
        auto issue_y2 = [&](int n) {  // dO^T P of iteration n, once its tiles have landed
            const int s = n % kBStages;
            iwait(&bar_ld[s], (n / kBStages) & 1, kErrTimeoutTma);
            if (ok) {
                tc_fence_after();
                const uint32_t dob = smem_u32(sm + L::dO + s * kTile), pb = smem_u32(sm + L::P + s * 8192);
                constexpr uint32_t id = idesc_bf16(128, 64, true, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tY2, sdesc(dob + ks * 2048, 8192, 1024), sdesc(pb + ks * 2048, 8192, 1024), id,
                             ks > 0);
            }
            mma_commit(bar_y2);
        };
        int issued = 0;
        for (; issued < min(kBStages, NC); ++issued) issue_load(issued);
        issue_y2(0);
        for (int n = 0; n < NC; ++n) {
            const int c = NC - 1 - n;
            const uint32_t par = n & 1;
            // the stage of iteration n-1 is free once the element-wise warps have handed over
            // dS'^T of this iteration: the products of n-1 are done and its tiles read
            iwait(bar_s, par, kErrTimeoutMma);
            if (ok && n >= 1 && issued < NC) {
                issue_load(issued);
                ++issued;
            }
            // dS'^T of chunk c to global memory
            iwait(bar_sst, par, kErrTimeoutMma);
            if (ok) {
                tma_store_2d(&tm_dsc, sm + L::St, 0, (bh * NC + c) * kD);
                tma_store_2d(&tm_dsc, sm + L::St + kTile, 64, (bh * NC + c) * kD);
            }
            bulk_commit();
            bulk_wait_read<1>();  // the dDelta^T (dv) store of iteration n-1 has read its tile
            if (n > 0) mbar_arrive(bar_dfree);
            // dO^T P of the next iteration once this one's has been read
            iwait(bar_d, par, kErrTimeoutMma);
            if (n + 1 < NC) issue_y2(n + 1);
            iwait(bar_dst, par, kErrTimeoutMma);
            if (ok) {
                if (kDelta) {
                    tma_store_2d(&tm_ddt, sm + L::Dst, 0, (bh * NC + c) * kD);
                } else {
                    tma_store_4d(&tm_dv, sm + L::Dst, 0, h, c * kChunk, b);
                    tma_store_4d(&tm_dv, sm + L::Dst + 8192, 64, h, c * kChunk, b);
                }
            }
            bulk_commit();
            bulk_wait_read<1>();  // the dS'^T store of iteration n has read its tile
            mbar_arrive(bar_sfree);
        }
        if (!ok) atomicExch(a.err, err);
        // teardown: copies still in flight land, every UMMA of this thread has finished
        // and the stores have read shared memory before the CTA exits
        if (*s_abort)
            for (int m = 0; m < issued; ++m) mbar_wait(&bar_ld[m % kBStages], (m / kBStages) & 1);
        mma_commit(bar_fin);
        mbar_wait(bar_fin, 0);
        bulk_wait_read<0>();
    } else if (warp < 16) {
        // ---------------- the element-wise warps (`bad` warp-uniform, as in the forward pass)
        bool bad = false;
        auto wait = [&](uint64_t* bar, uint32_t parity, int e) {
            if (!bad && !mbar_wait_or_abort(bar, parity, s_abort)) {
                bad = true;
                if (!*s_abort) atomicExch(a.err, e);
                *s_abort = 1;
            }
            bad = __any_sync(0xffffffffu, bad);
        };
        auto hand_over_tmem = [&](uint64_t* bar) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        auto hand_over_smem = [&](uint64_t* bar) {
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // dS^T row j, state columns i in [32 part, 32 part + 32): S[q] = dS_{i, j}
        float S[32];
#pragma unroll
        for (int q = 0; q < 32; ++q)
            S[q] = a.dS_out ? a.dS_out[((size_t)bh * kD + part * 32 + q) * kD + j] : 0.f;
        uint8_t* St = sm + L::St + (part >> 1) * kTile;
        const int sq0 = (part & 1) * 4;
        for (int n = 0; n < NC && !bad; ++n) {
            const int s = n % kBStages;
            const uint32_t par = n & 1;
            // (1) dS'^T as bf16 pairs into TMEM: the A operand of dS'^T K^T
            {
                uint32_t w[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) w[q] = pack_bf16(S[2 * q], S[2 * q + 1]);
                tmem_st16u(tS + lane_base + 16 * part, w);
            }
            hand_over_tmem(bar_s);
            // (2) diag(gamma) Q in place, 32 bytes of a 128-byte line per thread
            wait(&bar_ld[s], (n / kBStages) & 1, kErrTimeoutTma);
            const float* E = Eds + s * 128;
            {
                const int line = tid >> 2, r = line & 63, blk = line >> 6;
                uint8_t* ln = sm + L::Q + s * kTile + blk * 8192 + r * 128 + (tid & 3) * 32;
                const float f = E[64 + r];
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint4 u = *(uint4*)(ln + qq * 16);
                    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 x = unpack_bf16(w[p]);
                        w[p] = pack_bf16(x.x * f, x.y * f);
                    }
                    *(uint4*)(ln + qq * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            hand_over_smem(bar_q);
            // (3) dS'^T staged for its store, once the last one has read the tile
            if (n > 0) wait(bar_sfree, (n - 1) & 1, kErrTimeoutTma);
            put_row32(St, j, sq0, S);
            hand_over_smem(bar_sst);
            // (4) dDelta^T[j][r] = e^{G_C - G_r} (dS'^T K^T)[j][r] + (dO^T P)[j][r], r in
            // [16 part, 16 part + 16); -dDelta^T into TMEM (A operand of - dDelta^T W)
            wait(bar_y, par, kErrTimeoutMma);
            wait(bar_y2, par, kErrTimeoutMma);
            tc_fence_after();
            float d[16];
            {
                float y1[16], y2[16];
                tmem_ld16(tY1 + lane_base + part * 16, y1);
                tmem_ld16(tY2 + lane_base + part * 16, y2);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 16; ++q) d[q] = E[part * 16 + q] * y1[q] + y2[q];
            }
            if (kDelta) {
                uint32_t w[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q] = pack_bf16(-d[2 * q], -d[2 * q + 1]);
                tmem_st8u(tD + lane_base + 8 * part, w);
            }
            hand_over_tmem(bar_d);
            // (5) dDelta^T (or dv = dDelta, token-major, for linear attention) staged for its store
            if (n > 0) wait(bar_dfree, (n - 1) & 1, kErrTimeoutTma);
            if (kDelta) {
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    uint4 u;
                    u.x = pack_bf16(d[qq * 8 + 0], d[qq * 8 + 1]);
                    u.y = pack_bf16(d[qq * 8 + 2], d[qq * 8 + 3]);
                    u.z = pack_bf16(d[qq * 8 + 4], d[qq * 8 + 5]);
                    u.w = pack_bf16(d[qq * 8 + 6], d[qq * 8 + 7]);
                    *(uint4*)(sm + L::Dst + sw128(j, part * 2 + qq)) = u;
                }
            } else {
                const uint32_t jb = (uint32_t)(j >> 6) * 8192, jq = (j & 63) >> 3, je = (j & 7) * 2;
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    *(__nv_bfloat16*)(sm + L::Dst + jb + sw128(part * 16 + q, jq) + je) = __float2bfloat16_rn(d[q]);
            }
            hand_over_smem(bar_dst);
            // (6) dS^T <- gamma_C dS'^T + dO^T (diag(gamma) Q) - dDelta^T W
            wait(bar_z, par, kErrTimeoutMma);
            tc_fence_after();
            float z[32];
            tmem_ld32(tZ + lane_base + part * 32, z);
            tmem_ld_wait();
            const float gam = E[64 + kChunk - 1];
#pragma unroll
            for (int q = 0; q < 32; ++q) S[q] = gam * S[q] + z[q];
        }
        if (!bad && a.dS_in) {
#pragma unroll
            for (int q = 0; q < 32; ++q) a.dS_in[((size_t)bh * kD + part * 32 + q) * kD + j] = S[q];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}
}  // namespace

bool tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    const uint64_t dims[2] = {inner, rows};
    const uint64_t strides[1] = {inner * 2};
    const uint32_t box[2] = {64, box_rows};
    return make_tmap(m, base, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

// [B, ld_t, H, d] token-major input, tiles of 64 tokens x 64 features of one head.
bool tmap_tokens(CUtensorMap* m, const void* base, const Args& a, int d) {
    const uint64_t dims[4] = {(uint64_t)d, (uint64_t)a.H, (uint64_t)a.T, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)d * 2, (uint64_t)a.H * d * 2,
                                 (uint64_t)a.ld_t * a.H * d * 2};
    const uint32_t box[4] = {64, 1, 64, 1};
    return make_tmap(m, base, 4, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

bool tc_eligible(const Args& a) {
    return a.dtype == SF_BF16 && a.dk == kD && a.dv == kD;
}

cudaError_t launch_state_fwd_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
    CUtensorMap tm_wt{}, tm_ut{}, tm_k{}, tm_sc{}, tm_dt{};
    bool ok = tmap_2d(&tm_ut, a.Ut, 64, rows, 128) && tmap_tokens(&tm_k, a.k, a, kD) &&
              tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_dt, a.Dt, 64, rows, 128);
    if (a.beta) ok = ok && tmap_2d(&tm_wt, a.Wt, 64, rows, 128);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = FwdSmem::Size + 1024;
    auto kern = a.beta ? state_fwd_tc_kernel<true> : state_fwd_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_STATE_FWD, s);
    kern<<<BH, kFwdThreads, smem, s>>>(tm_wt, tm_ut, tm_k, tm_sc, tm_dt, a);
    e = cudaGetLastError();
    timing_end(KK_STATE_FWD, s);
    return e;
}

cudaError_t launch_state_bwd_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
    CUtensorMap tm_k{}, tm_do{}, tm_q{}, tm_wt{}, tm_p{}, tm_dsc{}, tm_ddt{}, tm_dv{};
    bool ok = tmap_tokens(&tm_k, a.k, a, kD) && tmap_tokens(&tm_do, a.dO, a, kD) &&
              tmap_tokens(&tm_q, a.q, a, kD) &&
              tmap_2d(&tm_p, a.Pm, 64, (uint64_t)BH * a.NC * kChunk, 64) &&
              tmap_2d(&tm_dsc, a.dSc, kD, rows, 128);
    if (a.beta)
        ok = ok && tmap_2d(&tm_wt, a.Wt, 64, rows, 128) && tmap_2d(&tm_ddt, a.dDt, 64, rows, 128);
    else
        ok = ok && tmap_tokens(&tm_dv, a.dv_, a, kD);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = BwdSmem::Size + 1024;
    auto kern = a.beta ? state_bwd_tc_kernel<true> : state_bwd_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_STATE_BWD, s);
    kern<<<BH, kBwdThreads, smem, s>>>(tm_k, tm_do, tm_q, tm_wt, tm_p, tm_dsc, tm_ddt, tm_dv, a);
    e = cudaGetLastError();
    timing_end(KK_STATE_BWD, s);
    return e;
}

}  // namespace sf
