// Tensor-core per-chunk kernels (sm_100a; bf16 operands, fp32 accumulate):
// the intra-chunk kernel and the output kernel.  Both are fully parallel over
// (chunk, batch, head); one CTA of 4 warps per chunk-head, two CTAs per SM.
//
// Intra-chunk kernel ("a linear-recurrence kernel inside each block", the
// StateFlow summary on gptget.net, section 方法详解), per chunk:
//   B  = (K K^T) .* Gamma (strictly lower)        UMMA, fp32 in TMEM
//   A  = diag(beta) B,   T = (I + A)^-1           fp32, blocked 16x16 inverse
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

// T = (I + A)^-1 for a 64 x 64 strictly lower A (fp32, row stride 65), by
// inverting the four 16 x 16 diagonal blocks with substitution and filling the
// off-diagonal blocks by distance: T_ij = -T_ii sum_{i>k>=j} A_ik T_kj.
// T is written with row stride 68 (16-byte aligned rows).  Each thread of the
// off-diagonal phases computes a strip of 4 adjacent columns of one row, so
// its four multiply-add chains are independent.  Called by all 128 threads of
// the CTA; ends with a barrier.
constexpr int kTS = 68;  // row stride of T in floats (16-byte aligned rows)
constexpr int kMS = 20;  // row stride of the 16 x 16 scratch blocks (16-byte aligned)
constexpr int kMB = 16 * kMS;
__device__ void tri_inverse64(const float* Af, float* Tf, float* Mb, int tid) {
    for (int e = tid; e < 64 * kTS; e += 128) Tf[e] = 0.f;
    __syncthreads();
    if (tid < 64) {
        // column `col` of the inverse of diagonal block `o`: right-looking substitution
        const int o = (tid >> 4) * 16, col = tid & 15;
        float v[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) v[r] = (r == col) ? 1.f : 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const float x = (r < col) ? 0.f : v[r];
            v[r] = x;
#pragma unroll
            for (int r2 = r + 1; r2 < 16; ++r2) v[r2] -= Af[(o + r2) * 65 + o + r] * x;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(o + r) * kTS + o + col] = v[r];
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {
        const int nstrip = (4 - d) * 64;  // blocks (bi, bj) = (m + d, m), 16 rows x 4 strips
        for (int e = tid; e < nstrip; e += 128) {
            const int m = e >> 6, rr = (e >> 2) & 15, c4 = (e & 3) * 4;
            const int bi = m + d, bj = m;
            const float* arow = Af + (16 * bi + rr) * 65;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 16 * bj; k < 16 * bi; ++k) {
                const float a = arow[k];
                const float4 t = *(const float4*)(Tf + k * kTS + 16 * bj + c4);
                acc.x += a * t.x;
                acc.y += a * t.y;
                acc.z += a * t.z;
                acc.w += a * t.w;
            }
            *(float4*)(Mb + m * kMB + rr * kMS + c4) = acc;
        }
        __syncthreads();
        for (int e = tid; e < nstrip; e += 128) {
            const int m = e >> 6, rr = (e >> 2) & 15, c4 = (e & 3) * 4;
            const int bi = m + d, bj = m;
            const float* trow = Tf + (16 * bi + rr) * kTS + 16 * bi;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k <= rr; ++k) {
                const float t = trow[k];
                const float4 mv = *(const float4*)(Mb + m * kMB + k * kMS + c4);
                acc.x += t * mv.x;
                acc.y += t * mv.y;
                acc.z += t * mv.z;
                acc.w += t * mv.w;
            }
            *(float4*)(Tf + (16 * bi + rr) * kTS + 16 * bj + c4) =
                make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
        }
        __syncthreads();
    }
}

// Scales the 128-byte line (64 bf16) of row `row` of a tile by f, in place.
// Lanes of a warp handle different rows; starting each row at a different
// 16-byte chunk keeps the warp's accesses on distinct banks.
__device__ __forceinline__ void scale_line(uint8_t* line, int row, float f) {
#pragma unroll
    for (int qq = 0; qq < 8; ++qq) {
        const int q = (qq + row) & 7;
        uint4 u = *(uint4*)(line + q * 16);
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 x = unpack_bf16(w[p]);
            w[p] = pack_bf16(x.x * f, x.y * f);
        }
        *(uint4*)(line + q * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
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

template <bool kP>
struct IntraSmem {
    static constexpr int QK = 0;                              // kP: [kblk][Q 0-63 | K 64-127][64]
    static constexpr int QKBytes = kP ? 2 * kTile : kTile;    // else [kblk][K 0-63][64]
    static constexpr int Kb = kP ? QK + kHalf : QK;           // K, d_k block 0
    static constexpr int Kblk = kP ? kTile : kHalf;           // distance between K's d_k blocks
    static constexpr int V = QK + QKBytes;                    // [dvblk][64][64]
    static constexpr int Tb = V + kTile;                      // T, bf16 K-major [r][64 i]
    static constexpr int Pst = Tb + kHalf;                    // P staging (kP)
    static constexpr int Af = Pst + (kP ? kHalf : 0);         // fp32 [64][65]
    static constexpr int Tf = Af + 64 * 65 * 4;               // fp32 [64][68]
    static constexpr int Mb = Tf + 64 * 68 * 4;               // fp32 [3][16][20]
    static constexpr int Gs = Mb + 3 * 320 * 4;
    static constexpr int Bs = Gs + 256;
    static constexpr int Bar = Bs + 256;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

template <bool kDelta, bool kP>
__global__ void __launch_bounds__(128)
    intra_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wt,
                    const __grid_constant__ CUtensorMap tm_ut, const __grid_constant__ CUtensorMap tm_p,
                    const __grid_constant__ CUtensorMap tm_t, const Args a) {
    using L = IntraSmem<kP>;
    constexpr bool kKK = kDelta || kP;  // a K K^T (or [Q;K] K^T) product is needed
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Gs = (float*)(sm + L::Gs);
    float* Bs = (float*)(sm + L::Bs);
    float* Af = (float*)(sm + L::Af);
    float* Tf = (float*)(sm + L::Tf);
    float* Mb = (float*)(sm + L::Mb);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk, Lr = min(kChunk, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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
        tmem_alloc(s_tmem, 256);
        // in-chunk inclusive cumsum of g, two tokens per lane
        const int r0 = 2 * lane, r1 = r0 + 1;
        const float g0 = (a.g && r0 < Lr) ? a.g[tok_index(a, b, t0 + r0, h)] : 0.f;
        const float g1 = (a.g && r1 < Lr) ? a.g[tok_index(a, b, t0 + r1, h)] : 0.f;
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
        ed[r0] = __expf(gC - G0);
        ed[r1] = __expf(gC - G1);
        ed[64 + r0] = __expf(G0);
        ed[64 + r1] = __expf(G1);
    } else if (warp == 1) {
        const int r0 = 2 * lane, r1 = r0 + 1;
        if (kDelta) {
            Bs[r0] = (r0 < Lr) ? a.beta[tok_index(a, b, t0 + r0, h)] : 0.f;
            Bs[r1] = (r1 < Lr) ? a.beta[tok_index(a, b, t0 + r1, h)] : 0.f;
        } else {
            Bs[r0] = 1.f;
            Bs[r1] = 1.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tD1 = tmem, tW = tmem + 64, tU = tmem + 128;
    if (tid < kChunk) a.G[(size_t)bh * TP + t0 + tid] = Gs[tid];

    bool ld_pending = false, mma_pending = false;
    uint32_t mph = 0;
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
                    mma_bf16(tD1, sdesc(smem_u32(sm + L::QK) + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024),
                             sdesc(smem_u32(sm + L::Kb) + (ks >> 2) * kTile + (ks & 3) * 32, 16, 1024),
                             id, ks > 0);
            } else {
                constexpr uint32_t id = idesc_bf16(64, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t d = sdesc(smem_u32(sm + L::Kb) + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
                    mma_bf16(tD1, d, d, id, ks > 0);
                }
            }
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
            float v[64];
            tmem_ld32(taddr(tD1, 32 * warp, 0), *(float(*)[32]) & v[0]);
            tmem_ld32(taddr(tD1, 32 * warp, 32), *(float(*)[32]) & v[32]);
            tmem_ld_wait();
            // accumulator row held by this thread
            int row = -1;
            bool is_p = false;
            if (kP) {
                row = tid;
                is_p = row < kChunk;
                if (!is_p) row -= kChunk;
            } else if (lane < 16) {
                row = 16 * warp + lane;
            }
            if (row >= 0) {
                const float Gr = Gs[row];
                if (kP && is_p) {
                    float p[64];
#pragma unroll
                    for (int i = 0; i < 64; ++i) p[i] = (i <= row) ? __expf(Gr - Gs[i]) * v[i] : 0.f;
                    store_row64(sm + L::Pst, row, p);
                } else if (kDelta) {
                    const float br = Bs[row];
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        Af[row * 65 + i] = (i < row) ? br * __expf(Gr - Gs[i]) * v[i] : 0.f;
                }
            }
        }
        __syncthreads();
    }
    if (kDelta) tri_inverse64(Af, Tf, Mb, tid);
    {
        // T as a bf16 K-major tile (identity for linear attention)
        const int r = tid >> 1, q0 = (tid & 1) * 4;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const int q = q0 + qq;
            float t[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                t[e] = kDelta ? Tf[r * kTS + q * 8 + e] : ((q * 8 + e == r) ? 1.f : 0.f);
            uint4 u;
            u.x = pack_bf16(t[0], t[1]);
            u.y = pack_bf16(t[2], t[3]);
            u.z = pack_bf16(t[4], t[5]);
            u.w = pack_bf16(t[6], t[7]);
            *(uint4*)(sm + L::Tb + sw128(r, q)) = u;
        }
        // K_hat = diag(beta gamma) K and V_hat = diag(beta) V, in place
        const int blk = tid & 1;
        if (kDelta) {
            scale_line(sm + L::Kb + blk * L::Kblk + r * 128, r, Bs[r] * __expf(Gs[r]));
            scale_line(sm + L::V + blk * kHalf + r * 128, r, Bs[r]);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        if (kP) {
            tma_store_2d(&tm_p, sm + L::Pst, 0, (bh * NC + c) * kChunk);
            if (kDelta) tma_store_2d(&tm_t, sm + L::Tb, 0, (bh * NC + c) * kChunk);  // for the gradients
            bulk_commit();
        }
        tc_fence_after();
        constexpr uint32_t id = idesc_bf16(128, 64, true, false);
        const uint32_t tb = smem_u32(sm + L::Tb);
        if (kDelta) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tW, sdesc(smem_u32(sm + L::Kb) + ks * 2048, L::Kblk, 1024),
                         sdesc(tb + ks * 32, 16, 1024), id, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tU, sdesc(smem_u32(sm + L::V) + ks * 2048, kHalf, 1024),
                     sdesc(tb + ks * 32, 16, 1024), id, ks > 0);
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
        const int d = tid;  // W^T / U^T row = TMEM lane
        float v[64];
        if (kDelta) {
            tmem_ld32(taddr(tW, 32 * warp, 0), *(float(*)[32]) & v[0]);
            tmem_ld32(taddr(tW, 32 * warp, 32), *(float(*)[32]) & v[32]);
            tmem_ld_wait();
            store_row64(sm + L::QK, d, v);  // W^T staging (Q/K are dead)
        }
        tmem_ld32(taddr(tU, 32 * warp, 0), *(float(*)[32]) & v[0]);
        tmem_ld32(taddr(tU, 32 * warp, 32), *(float(*)[32]) & v[32]);
        tmem_ld_wait();
        store_row64(sm + L::V, d, v);  // U^T staging (V is dead)
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
        bulk_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

struct OutSmem {
    static constexpr int Q = 0;                // [dkblk][64 r][64]
    static constexpr int K = Q + kTile;        // [dkblk][64 r][64]
    static constexpr int St = K + kTile;       // S^T [kblk][128 j][64]
    static constexpr int Dt = St + 2 * kTile;  // Delta^T [128 j][64 r]
    static constexpr int Pb = Dt + kTile;      // P, K-major [r][64 i]
    static constexpr int Gs = Pb + kHalf;
    static constexpr int Bar = Gs + 256;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

__global__ void __launch_bounds__(128)
    output_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_dt,
                     const __grid_constant__ CUtensorMap tm_o, const Args a) {
    using L = OutSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Gs = (float*)(sm + L::Gs);
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
        mbar_expect_tx(bar_ld, 2 * kTile + 2 * kTile + kTile + 256);
        tma_load_4d(sm + L::Q, &tm_q, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K, &tm_k, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K + kHalf, &tm_k, 64, h, t0, b, bar_ld);
        tma_load_2d(sm + L::St, &tm_sc, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::Dt, &tm_dt, 0, (bh * NC + c) * kD, bar_ld);
        bulk_load(Gs, a.G + (size_t)bh * TP + t0, 256, bar_ld);
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
            const float o = __expf(Gs[r]) * x2[r] + x3[r];
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
        bulk_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

template <typename K>
cudaError_t set_smem(K kern, size_t smem) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
        if (e == cudaSuccess) kern<<<grid, 128, smem, s>>>(tm_q, tm_k, tm_v, tm_wt, tm_ut, tm_p, tm_t, a);
    } else {
        const size_t smem = IntraSmem<false>::Size + 1024;
        auto kern = a.beta ? intra_tc_kernel<true, false> : intra_tc_kernel<false, false>;
        e = set_smem(kern, smem);
        if (e == cudaSuccess) kern<<<grid, 128, smem, s>>>(tm_q, tm_k, tm_v, tm_wt, tm_ut, tm_p, tm_t, a);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    timing_end(kind, s);
    return e;
}

cudaError_t launch_output_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
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
