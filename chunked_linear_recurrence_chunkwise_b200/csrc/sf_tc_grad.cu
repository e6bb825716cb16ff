// Tensor-core per-chunk gradient kernel, attention part (sm_100a).
//
// Per chunk-head, with S the state entering the chunk, dS' the gradient of
// the state leaving it, Delta the chunk's corrected values and F = dP .* Gamma:
//   P   = (Q K^T) .* Gamma (lower incl.),   dP = (dO Delta^T) .* lower incl.
//   dQ  = diag(gamma) dO S^T + F K
//   dK  = F^T Q + diag(e^{G_C - G}) Delta dS'^T (+ the delta-rule part dKp)
//   dG  = rowsum(dP.*P) - colsum(dP.*P) + gamma_r <Q_r, (dO S^T)_r>
//         - e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
//         + [last row] (sum_r e^{G_C - G_r} <K_r, (Delta dS'^T)_r> + gamma_C <S, dS'>)
//         (+ the delta-rule part dGp);   dg = reverse in-chunk cumsum of dG.
// All products are M = 64 UMMAs; two accumulators share TMEM columns at lane
// offsets 0 and 16 (rows of dQ-side tiles in lanes 0-15 of each quadrant,
// dK-side tiles in lanes 16-31).  The partial dO S^T and Delta dS'^T are
// rescaled per row in TMEM (tcgen05.st) before the F K and F^T Q UMMAs
// accumulate onto them.

#include <cuda.h>

#include "../../include/sf.h"
#include "sf_internal.h"
#include "tc_common.cuh"

namespace sf {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kTile = 16384;
constexpr int kHalf = 8192;

struct GradSmem {
    static constexpr int Q = 0;                  // [dkblk][64 r][64]
    static constexpr int K = Q + kTile;          // [dkblk][64 r][64]
    static constexpr int dO = K + kTile;         // [dvblk][64 r][64]
    static constexpr int Dt = dO + kTile;        // Delta^T [128 j][64 t]
    static constexpr int St = Dt + kTile;        // S^T   [2 kblk][128 j][64 i]
    static constexpr int dSt = St + 2 * kTile;   // dS'^T [2 kblk][128 j][64 i]
    static constexpr int F = dSt + 2 * kTile;    // F = dP .* Gamma, [64 r][64 t]
    static constexpr int Gs = F + kHalf;         // 64 fp32
    static constexpr int PD = Gs + 256;          // fp32 [64][65]: dP .* P (for column sums)
    static constexpr int dGp = PD + 64 * 65 * 4; // fp32 [2 side][2 half][64] partial dG rows
    static constexpr int red = dGp + 4 * 256;    // fp32 [2][8]: per-warp <S, dS'> and last-row sums
    static constexpr int Bar = red + 64;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

__device__ __forceinline__ size_t tok_index(const Args& a, int b, int t, int h) {
    return ((size_t)b * a.ld_t + t) * a.H + h;
}

// <row r of a 128-byte-swizzled bf16 tile block, x[0..63]>
__device__ __forceinline__ float dot_row64(const uint8_t* blk, int r, const float* x) {
    float acc = 0.f;
#pragma unroll
    for (int qc = 0; qc < 8; ++qc) {
        const uint4 u = *(const uint4*)(blk + sw128(r, qc));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 f = unpack_bf16(w[p]);
            acc += f.x * x[qc * 8 + 2 * p] + f.y * x[qc * 8 + 2 * p + 1];
        }
    }
    return acc;
}

__global__ void __launch_bounds__(256, 1)
    grad_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_dt,
                        const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_dsc,
                        const Args a) {
    using L = GradSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Gs = (float*)(sm + L::Gs);
    float* PD = (float*)(sm + L::PD);
    float* dGp = (float*)(sm + L::dGp);
    float* red = (float*)(sm + L::red);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk, Lr = min(kChunk, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, ch = warp >> 2;  // TMEM lane quadrant, column half
    const bool side_k = lane >= 16;             // lanes 16-31 hold the dK-side tile rows
    const int r = 16 * quad + (lane & 15);      // chunk row of this thread's M = 64 tiles

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *s_abort = 0;
        fence_barrier_init();
        mbar_expect_tx(bar_ld, 4 * kTile + 4 * kTile + 256);
        tma_load_4d(sm + L::Q, &tm_q, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K, &tm_k, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K + kHalf, &tm_k, 64, h, t0, b, bar_ld);
        tma_load_4d(sm + L::dO, &tm_do, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::dO + kHalf, &tm_do, 64, h, t0, b, bar_ld);
        tma_load_2d(sm + L::Dt, &tm_dt, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St, &tm_sc, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::dSt, &tm_dsc, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::dSt + kTile, &tm_dsc, 64, (bh * NC + c) * kD, bar_ld);
        bulk_load(Gs, a.G + (size_t)bh * TP + t0, 256, bar_ld);
    }
    if (warp == 0) tmem_alloc(s_tmem, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane16 = 16u << 16;
    // cols [0, 64): Q K^T (lanes 0-15) | dO Delta^T (lanes 16-31)
    // cols [64, 192): dQ (lanes 0-15)  | dK (lanes 16-31)
    const uint32_t tQK = tmem, tdP = tmem + lane16;
    const uint32_t tdQ = tmem + 64, tdK = tmem + 64 + lane16;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

    bool ld_pending = false, mma_pending = false;
    uint32_t mph = 0;
    if (tid == 0) {
        if (!mbar_wait(bar_ld, 0)) {
            *s_abort = 1;
            ld_pending = true;
            atomicExch(a.err, kErrTimeoutTma);
        } else {
            tc_fence_after();
            const uint32_t q = smem_u32(sm + L::Q), k = smem_u32(sm + L::K), dob = smem_u32(sm + L::dO);
            const uint32_t dt = smem_u32(sm + L::Dt), st = smem_u32(sm + L::St), dst = smem_u32(sm + L::dSt);
            constexpr uint32_t id1 = idesc_bf16(64, 64, false, false);   // Q K^T
            constexpr uint32_t id2 = idesc_bf16(64, 64, false, true);    // dO Delta^T
            constexpr uint32_t id7 = idesc_bf16(64, 128, false, true);   // dO S^T
            constexpr uint32_t id10 = idesc_bf16(64, 128, true, true);   // Delta dS'^T
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(tQK, sdesc(q + o, 16, 1024), sdesc(k + o, 16, 1024), id1, ks > 0);
                mma_bf16(tdP, sdesc(dob + o, 16, 1024), sdesc(dt + ks * 2048, kHalf, 1024), id2, ks > 0);
                mma_bf16(tdQ, sdesc(dob + o, 16, 1024), sdesc(st + ks * 2048, kTile, 1024), id7, ks > 0);
                mma_bf16(tdK, sdesc(dt + ks * 2048, kHalf, 1024), sdesc(dst + ks * 2048, kTile, 1024), id10,
                         ks > 0);
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
        const float Gr = Gs[r];
        // --- P, dP and F on columns [32 ch, 32 ch + 32).  Lane l < 16 holds (Q K^T)[r][.]
        // and lane l + 16 holds (dO Delta^T)[r][.]; after an exchange each lane of the
        // pair finishes 16 of the 32 columns (l < 16 the first, l >= 16 the second).
        float rowpart;
        {
            float v[32];
            tmem_ld32(tQK + lane_base + ch * 32, v);
            tmem_ld_wait();
            float other[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) other[q] = __shfl_xor_sync(0xffffffffu, v[q], 16);
            const int o = side_k ? 16 : 0;
            float rowsum = 0.f;
            float f[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float qk = side_k ? other[o + q] : v[o + q];
                const float dp = side_k ? v[o + q] : other[o + q];
                const int t = ch * 32 + o + q;
                const float gam = (t <= r) ? __expf(Gr - Gs[t]) : 0.f;
                const float pd = gam * qk * dp;
                rowsum += pd;
                PD[r * 65 + t] = pd;
                f[q] = gam * dp;
            }
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                uint4 u;
                u.x = pack_bf16(f[qq * 8 + 0], f[qq * 8 + 1]);
                u.y = pack_bf16(f[qq * 8 + 2], f[qq * 8 + 3]);
                u.z = pack_bf16(f[qq * 8 + 4], f[qq * 8 + 5]);
                u.w = pack_bf16(f[qq * 8 + 6], f[qq * 8 + 7]);
                *(uint4*)(sm + L::F + sw128(r, ch * 4 + (o >> 3) + qq)) = u;
            }
            rowpart = rowsum + __shfl_xor_sync(0xffffffffu, rowsum, 16);  // both halves of the row
        }
        // --- dO S^T (dQ side) / Delta dS'^T (dK side) on columns [64 ch, 64 ch + 64)
        float lastpart = 0.f;
        {
            float x[64];
            tmem_ld32(tdQ + lane_base + ch * 64, *(float(*)[32]) & x[0]);
            tmem_ld32(tdQ + lane_base + ch * 64 + 32, *(float(*)[32]) & x[32]);
            tmem_ld_wait();
            float scale, gpart;
            if (!side_k) {
                scale = __expf(Gr);  // gamma_r
                gpart = rowpart + scale * dot_row64(sm + L::Q + ch * kHalf, r, x);
            } else {
                scale = __expf(Gs[kChunk - 1] - Gr);  // e^{G_C - G_r}
                const float t = scale * dot_row64(sm + L::K + ch * kHalf, r, x);
                gpart = -t;
                lastpart = t;
            }
            dGp[((side_k ? 2 : 0) + ch) * 64 + r] = gpart;
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] *= scale;
            tmem_st32(tdQ + lane_base + ch * 64, *(const float(*)[32]) & x[0]);
            tmem_st32(tdQ + lane_base + ch * 64 + 32, *(const float(*)[32]) & x[32]);
        }
        // --- <S, dS'> over the two identically laid out tiles, and the last-row sum
        {
            float acc = 0.f;
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                const int off = (qq * 256 + tid) * 16;
                const uint4 u = *(const uint4*)(sm + L::St + off);
                const uint4 w = *(const uint4*)(sm + L::dSt + off);
                const uint32_t uu[4] = {u.x, u.y, u.z, u.w}, ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 a2 = unpack_bf16(uu[p]), b2 = unpack_bf16(ww[p]);
                    acc += a2.x * b2.x + a2.y * b2.y;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                acc += __shfl_xor_sync(0xffffffffu, acc, off);
                lastpart += __shfl_xor_sync(0xffffffffu, lastpart, off);
            }
            if (lane == 0) {
                red[warp] = acc;
                red[8 + warp] = lastpart;
            }
        }
    }
    tmem_st_wait();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tc_fence_after();
        const uint32_t f = smem_u32(sm + L::F), k = smem_u32(sm + L::K), q = smem_u32(sm + L::Q);
        constexpr uint32_t id8 = idesc_bf16(64, 128, false, true);  // F K
        constexpr uint32_t id9 = idesc_bf16(64, 128, true, true);   // F^T Q
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            mma_bf16(tdQ, sdesc(f + ks * 32, 16, 1024), sdesc(k + ks * 2048, kHalf, 1024), id8, 1);
            mma_bf16(tdK, sdesc(f + ks * 2048, kHalf, 1024), sdesc(q + ks * 2048, kHalf, 1024), id9, 1);
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
    // --- dG and dg = reverse in-chunk cumsum
    if (warp == 0) {
        float sdot = 0.f, last = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            sdot += red[w];
            last += red[8 + w];
        }
        float v2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int rr = 2 * lane + e;
            float colsum = 0.f;
            for (int i = 0; i < kChunk; ++i) colsum += PD[i * 65 + rr];
            float g = dGp[rr] + dGp[64 + rr] + dGp[128 + rr] + dGp[192 + rr] - colsum;
            if (a.beta) g += a.dGp[(size_t)bh * TP + t0 + rr];
            if (rr == kChunk - 1) g += last + __expf(Gs[kChunk - 1]) * sdot;
            v2[e] = g;
        }
        float incl = v2[0] + v2[1];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, off);
            if (lane + off < 32) incl += y;
        }
        if (a.g) {
            if (2 * lane < Lr) a.dg[tok_index(a, b, t0 + 2 * lane, h)] = incl;
            if (2 * lane + 1 < Lr) a.dg[tok_index(a, b, t0 + 2 * lane + 1, h)] = incl - v2[0];
        }
    }
    // --- dq (lanes 0-15) and dk (lanes 16-31), columns [64 ch, 64 ch + 64)
    {
        float x[64];
        tmem_ld32(tdQ + lane_base + ch * 64, *(float(*)[32]) & x[0]);
        tmem_ld32(tdQ + lane_base + ch * 64 + 32, *(float(*)[32]) & x[32]);
        tmem_ld_wait();
        if (r < Lr) {
            if (side_k && a.beta) {
                const float* kp = a.dKp + ((size_t)bh * TP + t0 + r) * kD + ch * 64;
#pragma unroll
                for (int q = 0; q < 64; q += 4) {
                    const float4 p4 = *(const float4*)(kp + q);
                    x[q] += p4.x;
                    x[q + 1] += p4.y;
                    x[q + 2] += p4.z;
                    x[q + 3] += p4.w;
                }
            }
            __nv_bfloat16* dst = (__nv_bfloat16*)(side_k ? a.dk_ : a.dq) +
                                 tok_index(a, b, t0 + r, h) * kD + ch * 64;
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                uint4 u;
                u.x = pack_bf16(x[qq * 8 + 0], x[qq * 8 + 1]);
                u.y = pack_bf16(x[qq * 8 + 2], x[qq * 8 + 3]);
                u.z = pack_bf16(x[qq * 8 + 4], x[qq * 8 + 5]);
                u.w = pack_bf16(x[qq * 8 + 6], x[qq * 8 + 7]);
                *(uint4*)(dst + qq * 8) = u;
            }
        }
    }

teardown:
    if (tid == 0) {
        if (ld_pending) mbar_wait(bar_ld, 0);
        if (mma_pending) mbar_wait(bar_mma, mph ^ 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}


// ---------------------------------------------------------------------------
// Delta-rule part of the per-chunk gradients (beta given):
//   B = (K K^T) .* Gamma (strictly lower),  T = (I + diag(beta) B)^-1 (stored by the intra kernel)
//   dVhat = T^T dDelta,  dW = -dDelta S^T,  dKhat = T^T dW
//   dA = -(dKhat W^T + dVhat U^T) .* strictly lower,  dB = diag(beta) dA,  E = dB .* Gamma
//   dv = diag(beta) dVhat
//   dbeta_r = <V_r, dVhat_r> + gamma_r <K_r, dKhat_r> + sum_t dA_rt B_rt
//   dKp = diag(beta gamma) dKhat + (E + E^T) K        (added to dk by the attention part)
//   dGp = rowsum(dB .* B) - colsum(dB .* B) + beta_r gamma_r <K_r, dKhat_r>
// M = 64 UMMAs throughout; TMEM columns [0, 64): K K^T (lanes 0-15) | dA (16-31),
// [64, 192): dW then dKhat then dKp (lanes 0-15) | dVhat (lanes 16-31).
struct DeltaSmem {
    static constexpr int K = 0;                    // [dkblk][64 r][64]
    static constexpr int dDt = K + kTile;          // dDelta^T [128 j][64 r]
    static constexpr int St = dDt + kTile;         // S^T [2 kblk][128 j][64 i]
    static constexpr int Wt = St + 2 * kTile;      // W^T [128 i][64 r]
    static constexpr int Ut = Wt + kTile;          // U^T [128 j][64 r]
    static constexpr int Tb = Ut + kTile;          // T, bf16 [r'][64 r] (from the intra kernel)
    static constexpr int dWb = Tb + kHalf;         // dW, then dKhat: bf16 [iblk][64 r][64]
    static constexpr int dVb = dWb + kTile;        // dVhat: bf16 [jblk][64 r][64]
    static constexpr int Bf = dVb + kTile;         // fp32 [64][65] B
    static constexpr int Af = Bf + 64 * 65 * 4;    // fp32 [64][65] E = dB .* Gamma
    static constexpr int Tf = Af + 64 * 65 * 4;    // fp32 [64][65] dB .* B
    static constexpr int Gs = Tf + 64 * 65 * 4;
    static constexpr int Bs = Gs + 256;
    static constexpr int part = Bs + 256;          // fp32 [10][64] partial row sums
    static constexpr int Bar = part + 10 * 256;
    static constexpr int Misc = Bar + 16;
    static constexpr int Size = Misc + 16;
};

__device__ __forceinline__ void store_row_half(uint8_t* tile, int row, int q0, const float* v, int n) {
    // n/8 16-byte chunks starting at chunk q0 of `row` in a 128-byte-swizzled tile
    for (int qq = 0; qq < n / 8; ++qq) {
        uint4 u;
        u.x = pack_bf16(v[qq * 8 + 0], v[qq * 8 + 1]);
        u.y = pack_bf16(v[qq * 8 + 2], v[qq * 8 + 3]);
        u.z = pack_bf16(v[qq * 8 + 4], v[qq * 8 + 5]);
        u.w = pack_bf16(v[qq * 8 + 6], v[qq * 8 + 7]);
        *(uint4*)(tile + sw128(row, q0 + qq)) = u;
    }
}

__global__ void __launch_bounds__(256, 1)
    grad_delta_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_ddt,
                         const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_wt,
                         const __grid_constant__ CUtensorMap tm_ut, const __grid_constant__ CUtensorMap tm_t,
                         const Args a) {
    using L = DeltaSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Gs = (float*)(sm + L::Gs);
    float* Bs = (float*)(sm + L::Bs);
    float* Bf = (float*)(sm + L::Bf);
    float* Af = (float*)(sm + L::Af);
    float* Tf = (float*)(sm + L::Tf);
    float* part = (float*)(sm + L::part);
    float* Ef = Af;  // E = dB .* Gamma, fp32 [64][65]
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);
    uint64_t* bar_mma = bar_ld + 1;
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk, Lr = min(kChunk, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, ch = warp >> 2;
    const bool hi = lane >= 16;               // lanes 16-31: the tile at lane offset 16
    const int r = 16 * quad + (lane & 15);    // chunk row of this thread's M = 64 tiles

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        *s_abort = 0;
        fence_barrier_init();
        mbar_expect_tx(bar_ld, 6 * kTile + kHalf + 256);
        tma_load_2d(sm + L::Tb, &tm_t, 0, (bh * NC + c) * kChunk, bar_ld);  // T from the intra kernel
        tma_load_4d(sm + L::K, &tm_k, 0, h, t0, b, bar_ld);
        tma_load_4d(sm + L::K + kHalf, &tm_k, 64, h, t0, b, bar_ld);
        tma_load_2d(sm + L::dDt, &tm_ddt, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St, &tm_sc, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::Wt, &tm_wt, 0, (bh * NC + c) * kD, bar_ld);
        tma_load_2d(sm + L::Ut, &tm_ut, 0, (bh * NC + c) * kD, bar_ld);
        bulk_load(Gs, a.G + (size_t)bh * TP + t0, 256, bar_ld);
    }
    if (warp == 0) tmem_alloc(s_tmem, 256);
    if (tid < 64) Bs[tid] = (tid < Lr) ? a.beta[tok_index(a, b, t0 + tid, h)] : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane16 = 16u << 16;
    const uint32_t tKK = tmem, tdA = tmem + lane16;      // cols [0, 64)
    const uint32_t tW = tmem + 64, tdV = tmem + 64 + lane16;  // cols [64, 192)
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

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
    // ---- phase A: K K^T and dDelta S^T
    if (tid == 0) {
        if (!mbar_wait(bar_ld, 0)) {
            *s_abort = 1;
            ld_pending = true;
            atomicExch(a.err, kErrTimeoutTma);
        } else {
            tc_fence_after();
            const uint32_t k = smem_u32(sm + L::K), ddt = smem_u32(sm + L::dDt), st = smem_u32(sm + L::St);
            constexpr uint32_t id1 = idesc_bf16(64, 64, false, false);
            constexpr uint32_t id3 = idesc_bf16(64, 128, true, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(tKK, sdesc(k + o, 16, 1024), sdesc(k + o, 16, 1024), id1, ks > 0);
                mma_bf16(tW, sdesc(ddt + ks * 2048, kHalf, 1024), sdesc(st + ks * 2048, kTile, 1024), id3,
                         ks > 0);
            }
            mma_wait();
        }
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        const float Gr = Gs[r];
        float v[32];
        tmem_ld32(tKK + lane_base + ch * 32, v);  // warp-collective; lanes 0-15 hold K K^T
        tmem_ld_wait();
        if (!hi) {
            // B on columns [32 ch, 32 ch + 32) of row r
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int t = ch * 32 + q;
                Bf[r * 65 + t] = (t < r) ? __expf(Gr - Gs[t]) * v[q] : 0.f;
            }
        }
        // dW = -(dDelta S^T), row r, columns [64 ch, 64 ch + 64) -> bf16 MN-major B tile
        float x[64];
        tmem_ld32(tW + lane_base + ch * 64, *(float(*)[32]) & x[0]);
        tmem_ld32(tW + lane_base + ch * 64 + 32, *(float(*)[32]) & x[32]);
        tmem_ld_wait();
        if (!hi) {
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] = -x[q];
            store_row_half(sm + L::dWb + ch * kHalf, r, 0, x, 64);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- phase B: dVhat = T^T dDelta, dKhat = T^T dW
    if (tid == 0) {
        tc_fence_after();
        const uint32_t tb = smem_u32(sm + L::Tb), ddt = smem_u32(sm + L::dDt), dwb = smem_u32(sm + L::dWb);
        constexpr uint32_t idV = idesc_bf16(64, 128, true, false);
        constexpr uint32_t idK = idesc_bf16(64, 128, true, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            mma_bf16(tdV, sdesc(tb + ks * 2048, kHalf, 1024), sdesc(ddt + ks * 32, 16, 1024), idV, ks > 0);
            mma_bf16(tW, sdesc(tb + ks * 2048, kHalf, 1024), sdesc(dwb + ks * 2048, kHalf, 1024), idK, ks > 0);
        }
        mma_wait();
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        const float Gr = Gs[r], gam = __expf(Gr), br = Bs[r];
        float x[64];
        tmem_ld32(tW + lane_base + ch * 64, *(float(*)[32]) & x[0]);  // lanes 0-15 dKhat, 16-31 dVhat
        tmem_ld32(tW + lane_base + ch * 64 + 32, *(float(*)[32]) & x[32]);
        tmem_ld_wait();
        if (!hi) {
            // dKhat: its dot with K, a bf16 copy for dA, then rescale by beta gamma in place
            const float kd = dot_row64(sm + L::K + ch * kHalf, r, x);
            part[(0 + ch) * 64 + r] = gam * kd;           // dbeta term
            part[(2 + ch) * 64 + r] = br * gam * kd;      // dG term
            store_row_half(sm + L::dWb + ch * kHalf, r, 0, x, 64);
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] *= br * gam;
        } else {
            // dVhat: dv = beta dVhat, <V_r, dVhat_r>, bf16 copy for dA
            float vd = 0.f;
            if (r < Lr) {
                const size_t ti = tok_index(a, b, t0 + r, h) * kD + ch * 64;
                const __nv_bfloat16* vrow = (const __nv_bfloat16*)a.v + ti;
                __nv_bfloat16* dvrow = (__nv_bfloat16*)a.dv_ + ti;
#pragma unroll
                for (int qq = 0; qq < 8; ++qq) {
                    const uint4 u = *(const uint4*)(vrow + qq * 8);
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                    uint4 o;
                    uint32_t* ow = &o.x;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 f = unpack_bf16(w[p]);
                        vd += f.x * x[qq * 8 + 2 * p] + f.y * x[qq * 8 + 2 * p + 1];
                        ow[p] = pack_bf16(br * x[qq * 8 + 2 * p], br * x[qq * 8 + 2 * p + 1]);
                    }
                    *(uint4*)(dvrow + qq * 8) = o;
                }
            }
            part[(4 + ch) * 64 + r] = vd;
            store_row_half(sm + L::dVb + ch * kHalf, r, 0, x, 64);
        }
        tmem_st32(tW + lane_base + ch * 64, *(const float(*)[32]) & x[0]);  // dKhat lanes rescaled
        tmem_st32(tW + lane_base + ch * 64 + 32, *(const float(*)[32]) & x[32]);
    }
    tmem_st_wait();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- phase C: dA = dKhat W^T + dVhat U^T (negated and masked by the threads)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t dk = smem_u32(sm + L::dWb), dvb = smem_u32(sm + L::dVb);
        const uint32_t wt = smem_u32(sm + L::Wt), ut = smem_u32(sm + L::Ut);
        constexpr uint32_t id = idesc_bf16(64, 64, false, true);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
            mma_bf16(tdA, sdesc(dk + o, 16, 1024), sdesc(wt + ks * 2048, kHalf, 1024), id, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
            mma_bf16(tdA, sdesc(dvb + o, 16, 1024), sdesc(ut + ks * 2048, kHalf, 1024), id, 1);
        }
        mma_wait();
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        float v[32];
        tmem_ld32(tKK + lane_base + ch * 32, v);  // lanes 16-31: dA row r, columns [32 ch, +32)
        tmem_ld_wait();
        if (hi) {
            const float Gr = Gs[r], br = Bs[r];
            float sab = 0.f, sbb = 0.f;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int t = ch * 32 + q;
                const float da = (t < r) ? -v[q] : 0.f;
                const float bv = Bf[r * 65 + t];
                sab += da * bv;             // sum_t dA B
                sbb += br * da * bv;        // rowsum(dB .* B)
                Ef[r * 65 + t] = (t < r) ? br * da * __expf(Gr - Gs[t]) : 0.f;
                Tf[r * 65 + t] = br * da * bv;  // dB .* B, for the column sums
            }
            part[(6 + ch) * 64 + r] = sab;
            part[(8 + ch) * 64 + r] = sbb;
        }
    }
    __syncthreads();
    {
        // Esym = E + E^T as a bf16 K-major tile [r][64 t] (reuses the T tile)
        const int rr = tid >> 2, q0 = (tid & 3) * 2;
        float e[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = q0 * 8 + i;
            e[i] = Ef[rr * 65 + t] + Ef[t * 65 + rr];
        }
        store_row_half(sm + L::Tb, rr, q0, e, 16);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- phase D: dKp += Esym K (onto diag(beta gamma) dKhat)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t tb = smem_u32(sm + L::Tb), k = smem_u32(sm + L::K);
        constexpr uint32_t id = idesc_bf16(64, 128, false, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tW, sdesc(tb + ks * 32, 16, 1024), sdesc(k + ks * 2048, kHalf, 1024), id, 1);
        mma_wait();
    }
    mph ^= 1;
    __syncthreads();
    if (*s_abort) goto teardown;
    tc_fence_after();
    {
        float x[64];
        tmem_ld32(tW + lane_base + ch * 64, *(float(*)[32]) & x[0]);
        tmem_ld32(tW + lane_base + ch * 64 + 32, *(float(*)[32]) & x[32]);
        tmem_ld_wait();
        if (!hi) {
            float* kp = a.dKp + ((size_t)bh * TP + t0 + r) * kD + ch * 64;
#pragma unroll
            for (int q = 0; q < 64; q += 4) *(float4*)(kp + q) = make_float4(x[q], x[q + 1], x[q + 2], x[q + 3]);
        }
    }
    if (tid < 64) {
        const int rr = tid;
        float colbb = 0.f;
        for (int i = 0; i < kChunk; ++i) colbb += Tf[i * 65 + rr];
        const float db = part[4 * 64 + rr] + part[5 * 64 + rr] + part[0 * 64 + rr] + part[1 * 64 + rr] +
                         part[6 * 64 + rr] + part[7 * 64 + rr];
        const float dg = part[8 * 64 + rr] + part[9 * 64 + rr] - colbb + part[2 * 64 + rr] + part[3 * 64 + rr];
        if (rr < Lr) a.dbeta[tok_index(a, b, t0 + rr, h)] = db;
        a.dGp[(size_t)bh * TP + t0 + rr] = dg;
    }

teardown:
    if (tid == 0) {
        if (ld_pending) mbar_wait(bar_ld, 0);
        if (mma_pending) mbar_wait(bar_mma, mph ^ 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

cudaError_t launch_grad_attn_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
    CUtensorMap tm_q{}, tm_k{}, tm_do{}, tm_dt{}, tm_sc{}, tm_dsc{};
    const bool ok = tmap_tokens(&tm_q, a.q, a, kD) && tmap_tokens(&tm_k, a.k, a, kD) &&
                    tmap_tokens(&tm_do, a.dO, a, kD) && tmap_2d(&tm_dt, a.Dt, 64, rows, 128) &&
                    tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_dsc, a.dSc, kD, rows, 128);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = GradSmem::Size + 1024;
    cudaError_t e = cudaFuncSetAttribute(grad_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_GRAD_ATTN, s);
    grad_attn_tc_kernel<<<dim3(a.NC, BH), 256, smem, s>>>(tm_q, tm_k, tm_do, tm_dt, tm_sc, tm_dsc, a);
    e = cudaGetLastError();
    timing_end(KK_GRAD_ATTN, s);
    return e;
}

cudaError_t launch_grad_delta_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD;
    CUtensorMap tm_k{}, tm_ddt{}, tm_sc{}, tm_wt{}, tm_ut{}, tm_t{};
    const bool ok = tmap_tokens(&tm_k, a.k, a, kD) && tmap_2d(&tm_ddt, a.dDt, 64, rows, 128) &&
                    tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_wt, a.Wt, 64, rows, 128) &&
                    tmap_2d(&tm_ut, a.Ut, 64, rows, 128) &&
                    tmap_2d(&tm_t, a.Tm, 64, (uint64_t)BH * a.NC * kChunk, 64);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = DeltaSmem::Size + 1024;
    cudaError_t e = cudaFuncSetAttribute(grad_delta_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_GRAD_DELTA, s);
    grad_delta_tc_kernel<<<dim3(a.NC, BH), 256, smem, s>>>(tm_k, tm_ddt, tm_sc, tm_wt, tm_ut, tm_t, a);
    e = cudaGetLastError();
    timing_end(KK_GRAD_DELTA, s);
    return e;
}

}  // namespace sf
