// Tensor-core per-chunk gradient kernel, attention part (sm_100a).
//
// Per chunk-head, with S the state entering the chunk, dS' the gradient of
// the state leaving it, Delta the chunk's corrected values and F = dP .* Gamma:
//   P   = (Q K^T) .* Gamma (lower incl.),   dP = (dO Delta^T) .* lower incl.
//   dQ  = diag(gamma) dO S^T + F K
//   dK  = F^T Q + diag(e^{G_C - G}) Delta dS'^T
//   dG  = rowsum(dP.*P) - colsum(dP.*P) + gamma_r <Q_r, (dO S^T)_r>
//         - e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
//         + [last row] (sum_r e^{G_C - G_r} <K_r, (Delta dS'^T)_r> + gamma_C <S, dS'>)
//   dg  = reverse in-chunk cumsum of dG.
// This is the whole per-chunk gradient of (gated) linear attention, where
// Delta = V (no beta); the gated delta rule runs the fused kernel instead.
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
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-aligned, shared window
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

}  // namespace sf
