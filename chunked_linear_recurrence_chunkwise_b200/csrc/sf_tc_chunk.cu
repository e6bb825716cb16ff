// Tensor-core per-chunk kernels (sm_100a; bf16 operands, fp32 accumulate):
// the intra-chunk kernel and the output kernel.  Both are fully parallel over
// (chunk, batch, head), one CTA per chunk-head (8 warps for the intra kernel,
// 4 for the output kernel), several CTAs per SM.
//
// Intra-chunk kernel ("a linear-recurrence kernel inside each block", the
// StateFlow summary on gptget.net, section 方法详解), per chunk:
//   B  = (K K^T) .* Gamma (strictly lower)        UMMA, fp32 in TMEM
//   A  = diag(beta) B,   T = (I + A)^-1           16x16 diagonal blocks by fp32
//                                                 substitution, the rest by UMMAs
//   W^T = (diag(beta gamma) K)^T T^T              UMMA (A operand MN-major)
//   U^T = (diag(beta) V)^T T^T                    UMMA
// For the backward recompute the same CTA stacks [Q; K] into one M = 128
// UMMA and also emits P = (Q K^T) .* Gamma (lower incl.) for the dS pass.
// Linear attention (no beta) has T = I: U^T = V^T.
//
// Output kernel, per chunk:  O^T = gamma-scaled (S^T Q^T) + Delta^T P^T with
// P = (Q K^T) .* Gamma recomputed on chip.

#include <cuda.h>

#include "../../include/sf.h"
#include "sf_internal.h"
#include "tc_common.cuh"

namespace sf {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kTile = 16384;  // 128 rows x 128 bytes
constexpr int kHalf = 8192;   // 64 rows x 128 bytes

__device__ __forceinline__ size_t tok_index(const Args& a, int b, int t, int h) {
    return ((size_t)b * a.ld_t + t) * a.H + h;
}


// Writes 64 fp32 values as one bf16 row of a K-major 128-byte-swizzled tile.
__device__ __forceinline__ void store_row64(uint8_t* tile, int row, const float* v) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint4 u;
        u.x = pack_bf16(v[q * 8 + 0], v[q * 8 + 1]);
        u.y = pack_bf16(v[q * 8 + 2], v[q * 8 + 3]);
        u.z = pack_bf16(v[q * 8 + 4], v[q * 8 + 5]);
        u.w = pack_bf16(v[q * 8 + 6], v[q * 8 + 7]);
        *(uint4*)(tile + sw128(row, q)) = u;
    }
}


// n fp32 values as bf16 16-byte chunks q0 .. q0 + n/8 - 1 of row `row` of a
// 128-byte-swizzled tile with 128-byte rows.
__device__ __forceinline__ void put_row(uint8_t* tile, int row, int q0, const float* v, int n) {
#pragma unroll
    for (int qq = 0; qq < n / 8; ++qq) {
        uint4 u;
        u.x = pack_bf16(v[qq * 8 + 0], v[qq * 8 + 1]);
        u.y = pack_bf16(v[qq * 8 + 2], v[qq * 8 + 3]);
        u.z = pack_bf16(v[qq * 8 + 4], v[qq * 8 + 5]);
        u.w = pack_bf16(v[qq * 8 + 6], v[qq * 8 + 7]);
        *(uint4*)(tile + sw128(row, q0 + qq)) = u;
    }
}

// The 64 x 64 bf16 tiles (X1, X2, X3) are row-major with 128-byte rows, so one
// tile serves as a K-major A operand and as an MN-major B operand.
constexpr int kIntraThreads = 256;
constexpr int kDS = 17;  // row stride (floats) of the fp32 16 x 16 diagonal blocks

template <bool kP>
struct IntraSmem {
    static constexpr int QK = 0;                              // kP: [kblk][Q 0-63 | K 64-127][64]
    static constexpr int QKBytes = kP ? 2 * kTile : kTile;    // else [kblk][K 0-63][64]
    static constexpr int Kb = kP ? QK + kHalf : QK;           // K, d_k block 0
    static constexpr int Kblk = kP ? kTile : kHalf;           // distance between K's d_k blocks
    static constexpr int V = QK + QKBytes;                    // [dvblk][64][64]
    static constexpr int X1 = V + kTile;                      // A_o, then N^2, then T diag(beta gamma)
    static constexpr int X2 = X1 + kHalf;                     // D, then E, then T diag(beta) (I without beta)
    static constexpr int X3 = X2 + kHalf;                     // kP: P staging, then N, then T
    static constexpr int Pst = X3;                            // (P is stored before N is written)
    // fp32 [4][16][kDS] diagonal blocks of A and their inverses; with P they live in
    // Q's two d_k blocks (dead after [Q; K] K^T), so that three CTAs fit on an SM
    static constexpr int ADBytes = 4 * 16 * kDS * 4;
    static constexpr int Adf = kP ? QK : X3 + kHalf;
    static constexpr int Dfp = kP ? QK + kTile : Adf + ADBytes;
    static constexpr int Gs = X3 + kHalf + (kP ? 0 : 2 * ADBytes);  // G
    static constexpr int Bs = Gs + 256;                       // beta
    static constexpr int BGs = Bs + 256;                      // beta gamma
    static constexpr int Bar = BGs + 256;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

// Intra-chunk kernel.  With A = diag(beta) (K K^T .* Gamma) strictly lower, split
// into its 16 x 16 diagonal blocks A_d and the rest A_o:
//   I + A = (I + A_d)(I + N),  D = (I + A_d)^-1,  N = D A_o  (strictly block-lower,
//   N^4 = 0), so  T = (I - N + N^2 - N^3) D = E + N^2 E  with  E = D - N D.
// D comes from substitution in fp32; N, N^2, N D and N^2 E are 64 x 64 UMMAs
// (bf16 operands, fp32 accumulate), E is added in fp32 in TMEM.  Then
//   W^T = K^T (T diag(beta gamma))^T,  U^T = V^T (T diag(beta))^T.
// TMEM (128 columns): [0, 64) K K^T ([Q; K] K^T with P), then N^2 | N D, then W^T;
// [64, 128) N, then T (lane offset 16), then U^T.
template <bool kDelta, bool kP>
__global__ void __launch_bounds__(kIntraThreads)
    intra_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wt,
                    const __grid_constant__ CUtensorMap tm_ut, const __grid_constant__ CUtensorMap tm_p,
                    const __grid_constant__ CUtensorMap tm_t, const Args a) {
    using L = IntraSmem<kP>;
    constexpr bool kKK = kDelta || kP;  // a K K^T (or [Q;K] K^T) product is needed
    extern __shared__ uint8_t smem_raw[];
    // the 1024-aligned base by integer rounding: the pointer arithmetic of the other kernels
    // measured slower here (37 -> 43 us per launch without the delta rule)
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Gs = (float*)(sm + L::Gs);
    float* Bs = (float*)(sm + L::Bs);
    float* BGs = (float*)(sm + L::BGs);
    float* Adf = (float*)(sm + L::Adf);
    float* Dfp = (float*)(sm + L::Dfp);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    int c, bh;
    cta_chunk_head<kP>(c, bh);  // batch-heads fastest in the form that keeps P: measured faster
    const int b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk, Lr = min(kChunk, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wh = warp >> 2;  // TMEM lane quadrant, column half
    const bool hi = lane >= 16;
    const int r = 16 * quad + (lane & 15);      // row of this thread in the M = 64 tiles

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *s_abort = 0;
        fence_barrier_init();
        const uint32_t bytes = 2 * kHalf + (kKK ? 2 * kHalf : 0) + (kP ? 2 * kHalf : 0);
        mbar_expect_tx(bar_ld, bytes);
        if (kP) {
            tma_load_4d(sm + L::QK, &tm_q, 0, h, t0, b, bar_ld);
            tma_load_4d(sm + L::QK + kTile, &tm_q, 64, h, t0, b, bar_ld);
        }
        if (kKK) {
            tma_load_4d(sm + L::Kb, &tm_k, 0, h, t0, b, bar_ld);
            tma_load_4d(sm + L::Kb + L::Kblk, &tm_k, 64, h, t0, b, bar_ld);
        }
        tma_load_4d(sm + L::V, &tm_v, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::V + kHalf, &tm_v, 64, h, t0, b, bar_ld);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, 128);
        // in-chunk inclusive cumsum of g, two tokens per lane
        const int r0 = 2 * lane, r1 = r0 + 1;
        const float g0 = (a.g && r0 < Lr) ? a.g[tok_index(a, b, t0 + r0, h)] : 0.f;
        const float g1 = (a.g && r1 < Lr) ? a.g[tok_index(a, b, t0 + r1, h)] : 0.f;
        // beta is read here too, so that both loads are in flight together
        const float b0 = (kDelta && r0 < Lr) ? a.beta[tok_index(a, b, t0 + r0, h)] : 0.f;
        const float b1 = (kDelta && r1 < Lr) ? a.beta[tok_index(a, b, t0 + r1, h)] : 0.f;
        float incl = g0 + g1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const float excl = incl - g0 - g1;
        const float G0 = excl + g0, G1 = excl + g0 + g1;
        Gs[r0] = G0;
        Gs[r1] = G1;
        // decay table of the chunk for the state passes: e^{G_C - G_r}, then e^{G_r}
        const float gC = __shfl_sync(0xffffffffu, G1, 31);
        float* ed = a.Ed + ((size_t)bh * NC + c) * 128;
        const float e0 = __expf(G0), e1 = __expf(G1);
        ed[r0] = __expf(gC - G0);
        ed[r1] = __expf(gC - G1);
        ed[64 + r0] = e0;
        ed[64 + r1] = e1;
        Bs[r0] = b0;
        Bs[r1] = b1;
        BGs[r0] = b0 * e0;
        BGs[r1] = b1 * e1;
    }
    if (!kDelta) {  // T = I: U^T = V^T
        const int rr = tid >> 2, q0 = (tid & 3) * 2;
        float e[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) e[i] = (q0 * 8 + i == rr) ? 1.f : 0.f;
        put_row(sm + L::X2, rr, q0, e, 16);
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t c0 = tmem, c64 = tmem + 64, l16 = 16u << 16;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    if (tid < kChunk) a.G[(size_t)bh * TP + t0 + tid] = Gs[tid];

    bool ld_pending = false, mma_pending = false;
    uint32_t mph = 0;
    auto mma_wait = [&]() {  // thread 0
        mma_commit(bar_mma);
        if (!mbar_wait(bar_mma, mph)) {
            *s_abort = 1;
            mma_pending = true;
            atomicExch(a.err, kErrTimeoutMma);
        }
    };
    // A's entries of row rr, columns [g0, g0 + 16) from (K K^T) values kk: the
    // diagonal block goes to Adf in fp32, the rest to the bf16 tile A_o (X1)
    auto emit_A = [&](int rr, int g0, const float* kk) {
        const float Gr = Gs[rr], br = Bs[rr];
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = g0 + i;
            v[i] = (t < rr) ? br * __expf(Gr - Gs[t]) * kk[i] : 0.f;
        }
        if ((g0 >> 4) == (rr >> 4)) {
            float* dst = Adf + ((rr >> 4) * 16 + (rr & 15)) * kDS;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                dst[i] = v[i];
                v[i] = 0.f;
            }
        }
        put_row(sm + L::X1, rr, g0 >> 3, v, 16);
    };

    if (tid == 0 && !mbar_wait(bar_ld, 0)) {
        *s_abort = 1;
        ld_pending = true;
        atomicExch(a.err, kErrTimeoutTma);
    }
    __syncthreads();
    if (*s_abort) goto teardown;

    if (kKK) {
        if (tid == 0) {
            tc_fence_after();
            if (kP) {
                constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(c0, sdesc(smem_u32(sm + L::QK) + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024),
                             sdesc(smem_u32(sm + L::Kb) + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024),
                             id, ks > 0);
            } else {
                constexpr uint32_t id = idesc_bf16(64, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t d = sdesc(smem_u32(sm + L::Kb) + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
                    mma_bf16(c0, d, d, id, ks > 0);
                }
            }
            mma_wait();
        }
        mph ^= 1;
        __syncthreads();
        if (*s_abort) goto teardown;
        tc_fence_after();
        {
            float v[32];
            tmem_ld32(c0 + lane_base + 32 * wh, v);
            tmem_ld_wait();
            if (kP) {
                // [Q; K] K^T, M = 128: lane R holds row R (P rows 0-63, K K^T rows 64-127)
                const int R = 32 * quad + lane;
                if (R < kChunk) {
                    const float GR = Gs[R];
                    float p[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int t = 32 * wh + i;
                        p[i] = (t <= R) ? __expf(GR - Gs[t]) * v[i] : 0.f;
                    }
                    put_row(sm + L::Pst, R, 4 * wh, p, 32);
                } else if (kDelta) {
                    emit_A(R - kChunk, 32 * wh, v);
                    emit_A(R - kChunk, 32 * wh + 16, v + 16);
                }
            } else {
                // K K^T, M = 64: row r in lanes 0-15; lane l + 16 takes the upper 16 columns
                float w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float recv = __shfl_xor_sync(0xffffffffu, v[16 + i], 16);
                    w[i] = hi ? recv : v[i];
                }
                emit_A(r, 32 * wh + (hi ? 16 : 0), w);
            }
        }
        fence_async_smem();
        __syncthreads();
        if (kP && tid == 0) {
            tma_store_2d(&tm_p, sm + L::Pst, 0, (bh * NC + c) * kChunk);
            bulk_commit();
        }
    }
    if (kDelta) {
        // D = (I + A_d)^-1: thread (block, column) substitutes down one column
        if (tid < 64) {
            const int bk = tid >> 4, col = tid & 15;
            const float* ab = Adf + bk * 16 * kDS;
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = (i == col) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < 15; ++j) {
                const float x = v[j];
#pragma unroll
                for (int i = j + 1; i < 16; ++i) v[i] -= ab[i * kDS + j] * x;
            }
            float* db = Dfp + bk * 16 * kDS;
            const int cc = 16 * bk + col;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                db[i * kDS + col] = v[i];
                *(__nv_bfloat16*)(sm + L::X2 + sw128(16 * bk + i, cc >> 3) + (cc & 7) * 2) =
                    __float2bfloat16_rn(v[i]);
            }
        } else {
            // zeros outside the diagonal blocks of the D tile: 6 chunks per row
            for (int k = tid - 64; k < 64 * 6; k += kIntraThreads - 64) {
                const int row = k / 6, j = k % 6, bc = 2 * (row >> 4);
                *(uint4*)(sm + L::X2 + sw128(row, j < bc ? j : j + 2)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // N = D A_o
        if (tid == 0) {
            tc_fence_after();
            const uint32_t x1 = smem_u32(sm + L::X1), x2 = smem_u32(sm + L::X2);
            constexpr uint32_t id = idesc_bf16(64, 64, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c64, sdesc(x2 + ks * 32, 16, 1024), sdesc(x1 + ks * 2048, kHalf, 1024), id, ks > 0);
            mma_wait();
            if (kP) bulk_wait_read<0>();  // the P store has read X3, where N goes next
        }
        mph ^= 1;
        __syncthreads();
        if (*s_abort) goto teardown;
        tc_fence_after();
        {
            float v[32];
            tmem_ld32(c64 + lane_base + 32 * wh, v);
            tmem_ld_wait();
            float w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float recv = __shfl_xor_sync(0xffffffffu, v[16 + i], 16);
                w[i] = hi ? recv : v[i];
            }
            put_row(sm + L::X3, r, 4 * wh + (hi ? 2 : 0), w, 16);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // N^2 = N N (lane offset 0) and N D (lane offset 16)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t x2 = smem_u32(sm + L::X2), x3 = smem_u32(sm + L::X3);
            constexpr uint32_t id = idesc_bf16(64, 64, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(c0, sdesc(x3 + ks * 32, 16, 1024), sdesc(x3 + ks * 2048, kHalf, 1024), id, ks > 0);
                mma_bf16(c0 + l16, sdesc(x3 + ks * 32, 16, 1024), sdesc(x2 + ks * 2048, kHalf, 1024), id,
                         ks > 0);
            }
            mma_wait();
        }
        mph ^= 1;
        __syncthreads();
        if (*s_abort) goto teardown;
        tc_fence_after();
        {
            // lanes 0-15: N^2 -> bf16 tile; lanes 16-31: E = D - N D -> bf16 tile and,
            // in fp32, into T's accumulator (lane offset 16)
            float v[32];
            tmem_ld32(c0 + lane_base + 32 * wh, v);
            tmem_ld_wait();
            if (!hi) {
                put_row(sm + L::X1, r, 4 * wh, v, 32);
            } else {
                const float* drow = Dfp + ((r >> 4) * 16 + (r & 15)) * kDS;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int t = 32 * wh + i;
                    const float dv = ((t >> 4) == (r >> 4)) ? drow[t & 15] : 0.f;
                    v[i] = dv - v[i];
                }
                put_row(sm + L::X2, r, 4 * wh, v, 32);
            }
            tmem_st32(c64 + lane_base + 32 * wh, v);
        }
        tmem_st_wait();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // T = E + N^2 E
        if (tid == 0) {
            tc_fence_after();
            const uint32_t x1 = smem_u32(sm + L::X1), x2 = smem_u32(sm + L::X2);
            constexpr uint32_t id = idesc_bf16(64, 64, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c64 + l16, sdesc(x1 + ks * 32, 16, 1024), sdesc(x2 + ks * 2048, kHalf, 1024), id, 1);
            mma_wait();
        }
        mph ^= 1;
        __syncthreads();
        if (*s_abort) goto teardown;
        tc_fence_after();
        {
            // T rows in lanes 16-31; lane l takes the upper 16 of the 32 columns
            float v[32];
            tmem_ld32(c64 + lane_base + 32 * wh, v);
            tmem_ld_wait();
            float w[16], t1[16], t2[16];
            const int cb = 32 * wh + (hi ? 0 : 16);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float recv = __shfl_xor_sync(0xffffffffu, v[16 + i], 16);
                w[i] = hi ? v[i] : recv;
                t1[i] = w[i] * BGs[cb + i];
                t2[i] = w[i] * Bs[cb + i];
            }
            put_row(sm + L::X1, r, cb >> 3, t1, 16);
            put_row(sm + L::X2, r, cb >> 3, t2, 16);
            if (kP) put_row(sm + L::X3, r, cb >> 3, w, 16);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (kP && tid == 0) {
            tma_store_2d(&tm_t, sm + L::X3, 0, (bh * NC + c) * kChunk);  // for the gradients
            bulk_commit();
        }
    }
    // W^T = K^T (T diag(beta gamma))^T, U^T = V^T (T diag(beta))^T; M = 128 (d rows)
    if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 64, true, false);
        const uint32_t x1 = smem_u32(sm + L::X1), x2 = smem_u32(sm + L::X2);
        if (kDelta) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c0, sdesc(smem_u32(sm + L::Kb) + ks * 2048, L::Kblk, 1024), sdesc(x1 + ks * 32, 16, 1024),
                         id, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(c64, sdesc(smem_u32(sm + L::V) + ks * 2048, kHalf, 1024), sdesc(x2 + ks * 32, 16, 1024), id,
                     ks > 0);
        mma_wait();
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        const int d = 32 * quad + lane;  // W^T / U^T row = TMEM lane
        float v[32];
        if (kDelta) {
            tmem_ld32(c0 + lane_base + 32 * wh, v);
            tmem_ld_wait();
            put_row(sm + L::QK, d, 4 * wh, v, 32);  // W^T staging (Q/K are dead)
        }
        tmem_ld32(c64 + lane_base + 32 * wh, v);
        tmem_ld_wait();
        put_row(sm + L::V, d, 4 * wh, v, 32);  // U^T staging (V is dead)
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        if (kDelta) tma_store_2d(&tm_wt, sm + L::QK, 0, (bh * NC + c) * kD);
        tma_store_2d(&tm_ut, sm + L::V, 0, (bh * NC + c) * kD);
        bulk_commit();
    }

teardown:
    if (tid == 0) {
        if (ld_pending) mbar_wait(bar_ld, 0);
        if (mma_pending) mbar_wait(bar_mma, mph ^ 1);
        bulk_wait_read<0>();  // stores have read shared memory (their writes land before the grid completes)
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

struct OutSmem {
    static constexpr int Q = 0;                // [dkblk][64 r][64]
    static constexpr int K = Q + kTile;        // [dkblk][64 r][64]
    static constexpr int St = K + kTile;       // S^T [kblk][128 j][64]
    static constexpr int Dt = St + 2 * kTile;  // Delta^T [128 j][64 r]
    static constexpr int Pb = Dt + kTile;      // P, K-major [r][64 i]
    static constexpr int Gs = Pb + kHalf;      // G
    static constexpr int Eg = Gs + 256;        // e^{G_r}, from the chunk's decay table
    static constexpr int Bar = Eg + 256;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

__global__ void __launch_bounds__(128)
    output_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_dt,
                     const __grid_constant__ CUtensorMap tm_o, const Args a) {
    using L = OutSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-aligned, shared window
    float* Gs = (float*)(sm + L::Gs);
    const float* Eg = (const float*)(sm + L::Eg);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *s_abort = 0;
        fence_barrier_init();
        mbar_expect_tx(bar_ld, 2 * kTile + 2 * kTile + kTile + 512);
        tma_load_4d(sm + L::Q, &tm_q, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K, &tm_k, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K + kHalf, &tm_k, 64, h, t0, b, bar_ld);
        tma_load_2d(sm + L::St, &tm_sc, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::Dt, &tm_dt, 0, (bh * NC + c) * kD, bar_ld);
        bulk_load(Gs, a.G + (size_t)bh * TP + t0, 256, bar_ld);
        bulk_load(sm + L::Eg, a.Ed + ((size_t)bh * NC + c) * 128 + 64, 256, bar_ld);
    }
    if (warp == 0) tmem_alloc(s_tmem, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tD1 = tmem, tX2 = tmem + 64, tX3 = tmem + 128;
    bool ld_pending = false, mma_pending = false;
    uint32_t mph = 0;
    if (tid == 0) {
        if (!mbar_wait(bar_ld, 0)) {
            *s_abort = 1;
            ld_pending = true;
            atomicExch(a.err, kErrTimeoutTma);
        } else {
            tc_fence_after();
            const uint32_t q = smem_u32(sm + L::Q), k = smem_u32(sm + L::K), st = smem_u32(sm + L::St);
            constexpr uint32_t idA = idesc_bf16(64, 64, false, false);
            constexpr uint32_t idB = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(tD1, sdesc(q + o, 16, 1024), sdesc(k + o, 16, 1024), idA, ks > 0);
                mma_bf16(tX2, sdesc(st + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024),
                         sdesc(q + o, 16, 1024), idB, ks > 0);
            }
            mma_commit(bar_mma);
            if (!mbar_wait(bar_mma, mph)) {
                *s_abort = 1;
                mma_pending = true;
                atomicExch(a.err, kErrTimeoutMma);
            }
        }
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        float v[64];
        tmem_ld32(taddr(tD1, 32 * warp, 0), *(float(*)[32]) & v[0]);
        tmem_ld32(taddr(tD1, 32 * warp, 32), *(float(*)[32]) & v[32]);
        tmem_ld_wait();
        if (lane < 16) {  // M = 64 accumulator: row 16 w + l sits in lane 32 w + l
            const int r = 16 * warp + lane;
            const float Gr = Gs[r];
            float p[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) p[i] = (i <= r) ? __expf(Gr - Gs[i]) * v[i] : 0.f;
            store_row64(sm + L::Pb, r, p);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tc_fence_after();
        const uint32_t dt = smem_u32(sm + L::Dt), pb = smem_u32(sm + L::Pb);
        constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tX3, sdesc(dt + ks * 32, 16, 1024), sdesc(pb + ks * 32, 16, 1024), id, ks > 0);
        mma_commit(bar_mma);
        if (!mbar_wait(bar_mma, mph)) {
            *s_abort = 1;
            mma_pending = true;
            atomicExch(a.err, kErrTimeoutMma);
        }
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        const int j = tid;  // O^T row = d_v index = TMEM lane
        float x2[64], x3[64];
        tmem_ld32(taddr(tX2, 32 * warp, 0), *(float(*)[32]) & x2[0]);
        tmem_ld32(taddr(tX2, 32 * warp, 32), *(float(*)[32]) & x2[32]);
        tmem_ld32(taddr(tX3, 32 * warp, 0), *(float(*)[32]) & x3[0]);
        tmem_ld32(taddr(tX3, 32 * warp, 32), *(float(*)[32]) & x3[32]);
        tmem_ld_wait();
        uint8_t* ost = sm + L::Q;  // [jblk][64 r][64 j] staging (Q/K are dead)
        const uint32_t jb = (uint32_t)(j >> 6) * kHalf, jq = (j & 63) >> 3, je = (j & 7) * 2;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
            const float o = Eg[r] * x2[r] + x3[r];
            *(__nv_bfloat16*)(ost + jb + sw128(r, jq) + je) = __float2bfloat16_rn(o);
        }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        tma_store_4d(&tm_o, sm + L::Q, 0, h, t0, b);
        tma_store_4d(&tm_o, sm + L::Q + kHalf, 64, h, t0, b);
        bulk_commit();
    }

teardown:
    if (tid == 0) {
        if (ld_pending) mbar_wait(bar_ld, 0);
        if (mma_pending) mbar_wait(bar_mma, mph ^ 1);
        bulk_wait_read<0>();  // stores have read shared memory (their writes land before the grid completes)
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// Output kernel when the intra kernel has stored P (the forward that keeps its
// intermediates): O^T = gamma-scaled (S^T Q^T) + Delta^T P^T with P read, not
// recomputed, so both products go out at once and K is not needed.
struct OutPSmem {
    static constexpr int Q = 0;                // [dkblk][64 r][64]; later the O^T staging
    static constexpr int St = Q + kTile;       // S^T [kblk][128 j][64]
    static constexpr int Dt = St + 2 * kTile;  // Delta^T [128 j][64 r]
    static constexpr int Pb = Dt + kTile;      // P, K-major [r][64 i]
    static constexpr int Eg = Pb + kHalf;      // e^{G_r}, from the chunk's decay table
    static constexpr int Bar = Eg + 256;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

__global__ void __launch_bounds__(128)
    output_p_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_p,
                       const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_dt,
                       const __grid_constant__ CUtensorMap tm_o, const Args a) {
    using L = OutPSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-aligned, shared window
    const float* Eg = (const float*)(sm + L::Eg);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC;
    const int t0 = c * kChunk;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *s_abort = 0;
        fence_barrier_init();
        mbar_expect_tx(bar_ld, kTile + 2 * kTile + kTile + kHalf + 256);
        tma_load_4d(sm + L::Q, &tm_q, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, h, t0, b, bar_ld);
        tma_load_2d(sm + L::St, &tm_sc, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::Dt, &tm_dt, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::Pb, &tm_p, 0, (bh * NC + c) * kChunk, bar_ld);
        bulk_load(sm + L::Eg, a.Ed + ((size_t)bh * NC + c) * 128 + 64, 256, bar_ld);
    }
    if (warp == 0) tmem_alloc(s_tmem, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tX2 = tmem, tX3 = tmem + 64;
    bool ld_pending = false, mma_pending = false;
    if (tid == 0) {
        if (!mbar_wait(bar_ld, 0)) {
            *s_abort = 1;
            ld_pending = true;
            atomicExch(a.err, kErrTimeoutTma);
        } else {
            tc_fence_after();
            const uint32_t q = smem_u32(sm + L::Q), st = smem_u32(sm + L::St);
            const uint32_t dt = smem_u32(sm + L::Dt), pb = smem_u32(sm + L::Pb);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(tX2, sdesc(st + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024),
                         sdesc(q + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024), id, ks > 0);  // S^T Q^T
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tX3, sdesc(dt + ks * 32, 16, 1024), sdesc(pb + ks * 32, 16, 1024), id, ks > 0);  // Delta^T P^T
            mma_commit(bar_mma);
            if (!mbar_wait(bar_mma, 0)) {
                *s_abort = 1;
                mma_pending = true;
                atomicExch(a.err, kErrTimeoutMma);
            }
        }
    }
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        const int j = tid;  // O^T row = d_v index = TMEM lane
        float x2[64], x3[64];
        tmem_ld32(taddr(tX2, 32 * warp, 0), *(float(*)[32]) & x2[0]);
        tmem_ld32(taddr(tX2, 32 * warp, 32), *(float(*)[32]) & x2[32]);
        tmem_ld32(taddr(tX3, 32 * warp, 0), *(float(*)[32]) & x3[0]);
        tmem_ld32(taddr(tX3, 32 * warp, 32), *(float(*)[32]) & x3[32]);
        tmem_ld_wait();
        uint8_t* ost = sm + L::Q;  // [jblk][64 r][64 j] staging (Q is dead: the products are done)
        const uint32_t jb = (uint32_t)(j >> 6) * kHalf, jq = (j & 63) >> 3, je = (j & 7) * 2;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
            const float o = Eg[r] * x2[r] + x3[r];
            *(__nv_bfloat16*)(ost + jb + sw128(r, jq) + je) = __float2bfloat16_rn(o);
        }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        tma_store_4d(&tm_o, sm + L::Q, 0, h, t0, b);
        tma_store_4d(&tm_o, sm + L::Q + kHalf, 64, h, t0, b);
        bulk_commit();
    }

teardown:
    if (tid == 0) {
        if (ld_pending) mbar_wait(bar_ld, 0);
        if (mma_pending) mbar_wait(bar_mma, 0);
        bulk_wait_read<0>();  // stores have read shared memory (their writes land before the grid completes)
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

template <typename K>
cudaError_t set_smem(K kern, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // all of the SM's unified L1 / shared memory as shared memory, so that as many
    // CTAs as their shared memory allows are resident
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    return e;
}

}  // namespace

cudaError_t launch_intra_tc(const Args& a, bool with_p, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
    CUtensorMap tm_q{}, tm_k{}, tm_v{}, tm_wt{}, tm_ut{}, tm_p{}, tm_t{};
    bool ok = tmap_tokens(&tm_k, a.k, a, kD) && tmap_tokens(&tm_v, a.v, a, kD) &&
              tmap_2d(&tm_ut, a.Ut, 64, rows, 128) && tmap_2d(&tm_wt, a.Wt, 64, rows, 128);
    if (with_p)
        ok = ok && tmap_tokens(&tm_q, a.q, a, kD) &&
             tmap_2d(&tm_p, a.Pm, 64, (uint64_t)BH * a.NC * kChunk, 64);
    if (with_p && a.beta) ok = ok && tmap_2d(&tm_t, a.Tm, 64, (uint64_t)BH * a.NC * kChunk, 64);
    if (!ok) return cudaErrorInvalidValue;
    const dim3 grid(a.NC, BH);
    cudaError_t e;
    const int kind = with_p ? KK_INTRA_BWD : KK_INTRA_FWD;
    timing_begin(kind, s);
    if (with_p) {
        const size_t smem = IntraSmem<true>::Size + 1024;
        auto kern = a.beta ? intra_tc_kernel<true, true> : intra_tc_kernel<false, true>;
        e = set_smem(kern, smem);
        if (e == cudaSuccess) kern<<<grid, kIntraThreads, smem, s>>>(tm_q, tm_k, tm_v, tm_wt, tm_ut, tm_p, tm_t, a);
    } else {
        const size_t smem = IntraSmem<false>::Size + 1024;
        auto kern = a.beta ? intra_tc_kernel<true, false> : intra_tc_kernel<false, false>;
        e = set_smem(kern, smem);
        if (e == cudaSuccess) kern<<<grid, kIntraThreads, smem, s>>>(tm_q, tm_k, tm_v, tm_wt, tm_ut, tm_p, tm_t, a);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    timing_end(kind, s);
    return e;
}

cudaError_t launch_output_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
    if (a.Pm) {  // P stored by the intra kernel of this forward
        CUtensorMap tm_q{}, tm_p{}, tm_sc{}, tm_dt{}, tm_o{};
        const bool ok = tmap_tokens(&tm_q, a.q, a, kD) &&
                        tmap_2d(&tm_p, a.Pm, 64, (uint64_t)BH * a.NC * kChunk, 64) &&
                        tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_dt, a.Dt, 64, rows, 128) &&
                        tmap_tokens(&tm_o, a.o, a, kD);
        if (!ok) return cudaErrorInvalidValue;
        const size_t smem = OutPSmem::Size + 1024;
        cudaError_t e = set_smem(output_p_tc_kernel, smem);
        if (e != cudaSuccess) return e;
        timing_begin(KK_OUTPUT, s);
        output_p_tc_kernel<<<dim3(a.NC, BH), 128, smem, s>>>(tm_q, tm_p, tm_sc, tm_dt, tm_o, a);
        e = cudaGetLastError();
        timing_end(KK_OUTPUT, s);
        return e;
    }
    CUtensorMap tm_q{}, tm_k{}, tm_sc{}, tm_dt{}, tm_o{};
    const bool ok = tmap_tokens(&tm_q, a.q, a, kD) && tmap_tokens(&tm_k, a.k, a, kD) &&
                    tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_dt, a.Dt, 64, rows, 128) &&
                    tmap_tokens(&tm_o, a.o, a, kD);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = OutSmem::Size + 1024;
    cudaError_t e = set_smem(output_tc_kernel, smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_OUTPUT, s);
    output_tc_kernel<<<dim3(a.NC, BH), 128, smem, s>>>(tm_q, tm_k, tm_sc, tm_dt, tm_o, a);
    e = cudaGetLastError();
    timing_end(KK_OUTPUT, s);
    return e;
}

}  // namespace sf
