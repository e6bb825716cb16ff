// Fused per-chunk gradient kernel of the gated delta rule (sm_100a).
//
// One CTA per chunk-head computes dq, dk, dv, dbeta and dg from one load of
// its inputs (the algebra is the chunkwise backward of the delta rule):
//   P = (Q K^T) .* Gamma,  dP = (dO Delta^T) .* lower,  F = dP .* Gamma
//   dQ = diag(gamma) dO S^T + F K
//   dVhat = T^T dDelta,  dW = -dDelta S^T,  dKhat = T^T dW
//   dA = -(dKhat W^T + dVhat U^T) .* strictly lower,  dB = diag(beta) dA,  E = dB .* Gamma
//   dK = F^T Q + diag(e^{G_C - G}) Delta dS'^T + diag(beta gamma) dKhat + (E + E^T) K
//   dV = diag(beta) dVhat
//   dbeta_r = <V_r, dVhat_r> + gamma_r <K_r, dKhat_r> + sum_t dA_rt B_rt
//   dG_r = rowsum(dP.*P) - colsum(dP.*P) + rowsum(dB.*B) - colsum(dB.*B)
//          + gamma_r <(Q S)_r, dO_r> + beta_r gamma_r <K_r, dKhat_r>
//          - e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
//          + [last row] (sum_r e^{G_C - G_r} <K_r, (Delta dS'^T)_r> + gamma_C <S, dS'>)
//   dg = reverse in-chunk cumsum of dG
// with T = (I + diag(beta) B)^-1 taken from the backward intra kernel.
//
// The UMMAs are all M = 64, their accumulators paired at TMEM lane offsets 0
// and 16 (rows 16 w + l of the lane-0 tile sit in lanes 32 w + l, those of the
// lane-16 tile in lanes 32 w + 16 + l):
//   cols [0, 64):    Q K^T          | dA
//   cols [64, 128):  dO Delta^T     | -      (with [128, 256) lanes 0-15: one N = 192 product)
//   cols [128, 256): dQ             | dK
//   cols [256, 384): dW, dKhat, dKp | dVhat
//   cols [384, 448): K K^T          | -
// Shared memory of operands that die early is reused for the later tiles and
// scratch (about 218 KB in all, one CTA per SM).
//
// One thread of a seventeenth warp issues the copies and every UMMA, each as
// soon as its operands are in place: the products of loaded tiles as their five
// copy groups land (committed in three groups), F K and F^T Q once F is
// written, T^T dW and dVhat U^T once dW and dVhat are, dKhat W^T once dKhat
// is, (E + E^T) K once E is.  Sixteen warps share the element-wise work (warp
// w reads TMEM lane quadrant w % 4 and a quarter of the columns, w / 4); they
// hand each stage over through an mbarrier (one arrival per warp) and wait for
// the products they read on the commit barriers, so that the tensor core and
// the element-wise work of the chunk overlap.

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
constexpr int kThreads = 512;          // element-wise warps 0-15
constexpr int kBlock = kThreads + 32;  // + the issuing warp
constexpr int kIss = kThreads;         // the thread that issues copies and UMMAs
constexpr int kLoads = 5;              // operand groups, in the order they are needed

// Per-row partial sums, each kept per column quarter: [term][quarter][64 rows].
enum PartTerm {
    P_ROWQ = 0,  // dG: rowsum(dP .* P) + gamma_r <Q_r, (dO S^T)_r>
    P_KD,        // dG: -e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
    P_BGK,       // dG: beta_r gamma_r <K_r, dKhat_r>
    P_SBB,       // dG: rowsum(dB .* B)
    P_VD,        // dbeta: <V_r, dVhat_r>
    P_GK,        // dbeta: gamma_r <K_r, dKhat_r>
    P_SAB,       // dbeta: sum_t dA_rt B_rt
    P_COUNT
};
constexpr int kDgTerms = P_VD;  // terms [0, kDgTerms) go to dG, the rest to dbeta

struct FusedSmem {
    static constexpr int Q = 0;                   // [dkblk][64 r][64]
    static constexpr int K = Q + kTile;           // [dkblk][64 r][64]
    static constexpr int dO = K + kTile;          // [dvblk][64 r][64]
    static constexpr int Wt = dO + kTile;         // W^T [128 i][64 r]
    static constexpr int Ut = Wt + kTile;         // U^T [128 j][64 r]
    static constexpr int Tb = Ut + kTile;         // T [r'][64 r]
    static constexpr int F = Tb + kHalf;          // F = dP .* Gamma [r][64 t]; later E + E^T
    static constexpr int dDt = F + kHalf;         // dDelta^T [128 j][64 r]; later dVhat (bf16)
    static constexpr int Dt = dDt + kTile;        // Delta^T [128 j][64 t]; later dW (bf16 [iblk][r][64])
    static constexpr int St = Dt + kTile;         // S^T [2][128 j][64 i] (right behind Delta^T: one
                                                  // N = 192 operand [Delta^T | S^T]); later dKhat
    static constexpr int dSt = St + 2 * kTile;    // dS'^T [2][128 j][64 i]; later E (fp32 [64][65])
    static constexpr int PD = dSt + 2 * kTile;    // fp32 [64][65]: dP .* P, then + dB .* B
    static constexpr int Gs = PD + 64 * 65 * 4;   // 64 fp32
    static constexpr int csp = Gs + 256;          // fp32 [8][64]: column sums of PD over 8-row groups
    static constexpr int part = csp + 8 * 256;    // fp32 [P_COUNT][4][64]
    static constexpr int red = part + P_COUNT * 4 * 256;  // fp32 [32]: per-warp <S, dS'>, last-row sums
    static constexpr int Bar = red + 128;         // kLoads + 11 mbarriers
    static constexpr int Misc = Bar + (kLoads + 11) * 8;
    static constexpr int Size = Misc + 16;
};

__device__ __forceinline__ size_t tok_index(const Args& a, int b, int t, int h) {
    return ((size_t)b * a.ld_t + t) * a.H + h;
}

// <row r, 16-byte chunks q0 .. q0 + 3 of a 128-byte-swizzled bf16 tile block, x[0..31]>
__device__ __forceinline__ float dot_row32(const uint8_t* blk, int r, int q0, const float* x) {
    float acc = 0.f;
#pragma unroll
    for (int qc = 0; qc < 4; ++qc) {
        const uint4 u = *(const uint4*)(blk + sw128(r, q0 + qc));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 f = unpack_bf16(w[p]);
            acc += f.x * x[qc * 8 + 2 * p] + f.y * x[qc * 8 + 2 * p + 1];
        }
    }
    return acc;
}

// n fp32 values as bf16 16-byte chunks q0 .. q0 + n/8 - 1 of row `row` of a swizzled tile.
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

__global__ void __launch_bounds__(kBlock, 1)
    grad_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_wt,
                         const __grid_constant__ CUtensorMap tm_ut, const __grid_constant__ CUtensorMap tm_t,
                         const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_ddt,
                         const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_dsc,
                         const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                         const __grid_constant__ CUtensorMap tm_dv, const Args a) {
    using L = FusedSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float* Gs = (float*)(sm + L::Gs);
    float* csp = (float*)(sm + L::csp);
    float* PD = (float*)(sm + L::PD);
    float* Ef = (float*)(sm + L::dSt);
    float* part = (float*)(sm + L::part);
    float* red = (float*)(sm + L::red);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);  // [kLoads] operand groups landed
    uint64_t* bar_a = bar_ld + kLoads;            // [3] products of loaded tiles done
    uint64_t* bar_c = bar_a + 3;                  // [3] later products done
    uint64_t* bar_s = bar_c + 3;                  // [4] element-wise stages handed over (16 warps)
    uint64_t* bar_fin = bar_s + 4;                // teardown after an abort
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk, Lr = min(kChunk, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cq = warp >> 2;  // TMEM lane quadrant, column quarter
    const bool hi = lane >= 16;                 // lanes 16-31: the lane-16 tiles
    const int r = 16 * quad + (lane & 15);      // chunk row of this thread's tiles
    auto P = [&](int term) { return part + (term * 4 + cq) * 64; };

    if (tid == kIss) {
        for (int i = 0; i < kLoads + 11; ++i) mbar_init(bar_ld + i, (i >= kLoads + 6 && i < kLoads + 10) ? 16 : 1);
        *s_abort = 0;
        fence_barrier_init();
        const int rowD = (bh * NC + c) * kD, rowC = (bh * NC + c) * kChunk;
        // 0: Q, K, G (Q K^T, K K^T)
        mbar_expect_tx(&bar_ld[0], 4 * kHalf + 256);
        tma_load_4d(sm + L::Q, &tm_q, 0, h, t0, b, &bar_ld[0]);
        tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, h, t0, b, &bar_ld[0]);
        tma_load_4d(sm + L::K, &tm_k, 0, h, t0, b, &bar_ld[0]);
        tma_load_4d(sm + L::K + kHalf, &tm_k, 64, h, t0, b, &bar_ld[0]);
        bulk_load(Gs, a.G + (size_t)bh * TP + t0, 256, &bar_ld[0]);
        // 1: dO, Delta^T, S^T (dO [Delta^T | S^T])
        mbar_expect_tx(&bar_ld[1], 2 * kHalf + 3 * kTile);
        tma_load_4d(sm + L::dO, &tm_do, 0, h, t0, b, &bar_ld[1]);
        tma_load_4d(sm + L::dO + kHalf, &tm_do, 64, h, t0, b, &bar_ld[1]);
        tma_load_2d(sm + L::Dt, &tm_dt, 0, rowD, &bar_ld[1]);
        tma_load_2d(sm + L::St, &tm_sc, 0, rowD, &bar_ld[1]);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, rowD, &bar_ld[1]);
        // 2: dS'^T (Delta dS'^T)
        mbar_expect_tx(&bar_ld[2], 2 * kTile);
        tma_load_2d(sm + L::dSt, &tm_dsc, 0, rowD, &bar_ld[2]);
        tma_load_2d(sm + L::dSt + kTile, &tm_dsc, 64, rowD, &bar_ld[2]);
        // 3: dDelta^T, T (dDelta S^T, T^T dDelta)
        mbar_expect_tx(&bar_ld[3], kTile + kHalf);
        tma_load_2d(sm + L::dDt, &tm_ddt, 0, rowD, &bar_ld[3]);
        tma_load_2d(sm + L::Tb, &tm_t, 0, rowC, &bar_ld[3]);
        // 4: W^T, U^T (dVhat U^T, dKhat W^T)
        mbar_expect_tx(&bar_ld[4], 2 * kTile);
        tma_load_2d(sm + L::Wt, &tm_wt, 0, rowD, &bar_ld[4]);
        tma_load_2d(sm + L::Ut, &tm_ut, 0, rowD, &bar_ld[4]);
    }
    if (warp == 0) tmem_alloc(s_tmem, 512);
    // beta of this thread's row, held in a register: a load consumed before the
    // block-wide barrier below would hold the issuer's first products back
    const float bpre = (warp < 16 && r < Lr) ? a.beta[tok_index(a, b, t0 + r, h)] : 0.f;
    // this thread's quarter of V's row r (lanes 16-31), read while the tiles load
    uint4 vpre[4] = {};
    if (warp < 16 && hi && r < Lr) {
        const uint4* src = (const uint4*)((const __nv_bfloat16*)a.v + tok_index(a, b, t0 + r, h) * kD + cq * 32);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) vpre[qq] = __ldg(src + qq);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t l16 = 16u << 16;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t c0 = tmem, c64 = tmem + 64, c128 = tmem + 128, c256 = tmem + 256, c384 = tmem + 384;

    // Element-wise warps: a wait that gives up flags the abort (checked before the
    // final stores); every warp passes every barrier whatever happened, so that no
    // wait of another thread runs to its limit.
    auto wait_flag = [&](uint64_t* bar, int err) {
        if (!mbar_wait(bar, 0)) {
            *s_abort = 1;
            atomicExch(a.err, err);
        }
    };
    // Element-wise warps hand their shared- and tensor-memory writes to the issuer.
    auto hand_over = [&](uint64_t* bar) {
        tmem_st_wait();
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
    };
    float lastpart = 0.f;

    // ---------------- the issuer: every UMMA, each as soon as its operands are ready
    if (tid == kIss) {
        const uint32_t q = smem_u32(sm + L::Q), k = smem_u32(sm + L::K), dob = smem_u32(sm + L::dO);
        const uint32_t dt = smem_u32(sm + L::Dt), ddt = smem_u32(sm + L::dDt), tb = smem_u32(sm + L::Tb);
        const uint32_t st = smem_u32(sm + L::St), dst = smem_u32(sm + L::dSt);
        constexpr uint32_t idKK = idesc_bf16(64, 64, false, false);
        constexpr uint32_t idKM = idesc_bf16(64, 64, false, true);
        constexpr uint32_t idKM2 = idesc_bf16(64, 128, false, true);
        constexpr uint32_t idMM2 = idesc_bf16(64, 128, true, true);
        constexpr uint32_t idMK2 = idesc_bf16(64, 128, true, false);
        // a group whose tiles did not land is skipped, its commit still issued so
        // that no element-wise thread waits on it for long
        bool ok = mbar_wait(&bar_ld[0], 0);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c0, sdesc(q + o, 16, 1024), sdesc(k + o, 16, 1024), idKK, ks > 0);  // Q K^T
            }
            ok = mbar_wait(&bar_ld[1], 0);
        }
        if (ok) {
            // dO [Delta^T | S^T]: one N = 192 product, dO Delta^T into columns [64, 128) and
            // dO S^T into [128, 256) of lanes 0-15 (Delta^T and S^T lie 16 KB apart in smem)
            tc_fence_after();
            constexpr uint32_t idKM3 = idesc_bf16(64, 192, false, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c64, sdesc(dob + o, 16, 1024), sdesc(dt + ks * 2048, kTile, 1024), idKM3, ks > 0);
            }
        }
        mma_commit(&bar_a[0]);
        if (ok) ok = mbar_wait(&bar_ld[2], 0);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(c128 + l16, sdesc(dt + ks * 2048, kHalf, 1024), sdesc(dst + ks * 2048, kTile, 1024),
                         idMM2, ks > 0);  // Delta dS'^T
        }
        mma_commit(&bar_a[1]);
        if (ok) ok = mbar_wait(&bar_ld[3], 0);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(c256, sdesc(ddt + ks * 2048, kHalf, 1024), sdesc(st + ks * 2048, kTile, 1024), idMM2,
                         ks > 0);  // dDelta S^T
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c256 + l16, sdesc(tb + ks * 2048, kHalf, 1024), sdesc(ddt + ks * 32, 16, 1024),
                         idMK2, ks > 0);  // T^T dDelta
        }
        mma_commit(&bar_a[2]);
        if (ok) {  // K K^T, first read after dA: behind every product the element-wise stages wait on
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c384, sdesc(k + o, 16, 1024), sdesc(k + o, 16, 1024), idKK, ks > 0);
            }
        }
        // F K and F^T Q accumulate onto the rescaled dO S^T / Delta dS'^T once the
        // element-wise warps have written F and rescaled those ((a), (b))
        bool sok = ok && mbar_wait(&bar_s[0], 0);
        if (sok) {
            tc_fence_after();
            const uint32_t f = smem_u32(sm + L::F);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(c128, sdesc(f + ks * 32, 16, 1024), sdesc(k + ks * 2048, kHalf, 1024), idKM2, 1);
                mma_bf16(c128 + l16, sdesc(f + ks * 2048, kHalf, 1024), sdesc(q + ks * 2048, kHalf, 1024),
                         idMM2, 1);
            }
        }
        // dv is staged, dW and dVhat are written ((c), (d)): dKhat = T^T dW, then dVhat U^T
        sok = sok && mbar_wait(&bar_s[1], 0);
        if (sok) {
            tma_store_4d(&tm_dv, sm + L::dO, 0, h, t0, b);  // rows past the piece's end are clipped
            tma_store_4d(&tm_dv, sm + L::dO + kHalf, 64, h, t0, b);
            bulk_commit();
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c256, sdesc(tb + ks * 2048, kHalf, 1024), sdesc(dt + ks * 2048, kHalf, 1024), idMM2,
                         ks > 0);
        }
        mma_commit(&bar_c[0]);
        const bool sok_pre5 = sok;
        const bool ok5 = sok && mbar_wait(&bar_ld[4], 0);  // W^T, U^T
        if (ok5) {
            tc_fence_after();
            const uint32_t ut = smem_u32(sm + L::Ut);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c0 + l16, sdesc(ddt + o, 16, 1024), sdesc(ut + ks * 2048, kHalf, 1024), idKM,
                         ks > 0);  // dVhat U^T
            }
        }
        // dA += dKhat W^T once dKhat is written (second element-wise stage)
        sok = ok5 && mbar_wait(&bar_s[2], 0);
        if (sok) {
            tc_fence_after();
            const uint32_t wt = smem_u32(sm + L::Wt);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c0 + l16, sdesc(st + o, 16, 1024), sdesc(wt + ks * 2048, kHalf, 1024), idKM, 1);
            }
        }
        mma_commit(&bar_c[1]);
        if (sok) {  // dq, staged in the dW tile (rows past the piece's end are clipped)
            tma_store_4d(&tm_dq, sm + L::Dt, 0, h, t0, b);
            tma_store_4d(&tm_dq, sm + L::Dt + kHalf, 64, h, t0, b);
            bulk_commit();
        }
        // dKp = diag(beta gamma) dKhat + (E + E^T) K once E + E^T is written
        sok = sok && mbar_wait(&bar_s[3], 0);
        if (sok) {
            tc_fence_after();
            const uint32_t f = smem_u32(sm + L::F);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c256, sdesc(f + ks * 32, 16, 1024), sdesc(k + ks * 2048, kHalf, 1024), idKM2, 1);
        }
        mma_commit(&bar_c[2]);
        if (!sok) {  // a copy or an element-wise stage did not arrive in time
            *s_abort = 1;
            atomicExch(a.err, (!ok || (sok_pre5 && !ok5)) ? kErrTimeoutTma : kErrTimeoutMma);
        }
    } else if (warp < 16) {
        // ---------------- the element-wise warps
        // <S, dS'> over the two identically laid out tiles (a dG term of the last row),
        // while the first products run
        wait_flag(&bar_ld[1], kErrTimeoutTma);
        wait_flag(&bar_ld[2], kErrTimeoutTma);
        {
            float acc = 0.f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int off = (qq * kThreads + tid) * 16;
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
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) red[warp] = acc;
        }
        wait_flag(&bar_ld[0], kErrTimeoutTma);  // G, Q, K are read below
        wait_flag(&bar_a[0], kErrTimeoutMma);
        tc_fence_after();
        const float Gr = Gs[r];
        float rowpart;
        // (a) P, dP, F on columns [16 cq, 16 cq + 16): lane l < 16 holds (Q K^T)[r] and
        // (dO Delta^T)[r]; it finishes the first 8 columns and hands the last 8 to
        // lane l + 16.  A warp whose columns all lie past its rows (cq > quad) writes
        // the zeros without reading the products.
        if (cq > quad) {
            const int tb = 16 * cq + (hi ? 8 : 0);
            float f[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                PD[r * 65 + tb + q] = 0.f;
                f[q] = 0.f;
            }
            put_row(sm + L::F, r, tb >> 3, f, 8);
            rowpart = 0.f;
        } else {
            float v[16], u[16];
            tmem_ld16(c0 + lane_base + cq * 16, v);   // lanes 0-15: Q K^T
            tmem_ld16(c64 + lane_base + cq * 16, u);  // lanes 0-15: dO Delta^T
            tmem_ld_wait();
            const int tb = 16 * cq + (hi ? 8 : 0);
            float rowsum = 0.f;
            float f[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float rq = __shfl_xor_sync(0xffffffffu, v[8 + q], 16);
                const float rd = __shfl_xor_sync(0xffffffffu, u[8 + q], 16);
                const float qk = hi ? rq : v[q];
                const float dp = hi ? rd : u[q];
                const int t = tb + q;
                const float gam = (t <= r) ? __expf(Gr - Gs[t]) : 0.f;
                const float pd = gam * qk * dp;
                rowsum += pd;
                PD[r * 65 + t] = pd;
                f[q] = gam * dp;
            }
            put_row(sm + L::F, r, tb >> 3, f, 8);
            rowpart = rowsum + __shfl_xor_sync(0xffffffffu, rowsum, 16);
        }
        // (b) dO S^T (lanes 0-15) / Delta dS'^T (lanes 16-31), columns [32 cq, 32 cq + 32),
        // rescaled in TMEM by gamma_r / e^{G_C - G_r}
        wait_flag(&bar_a[1], kErrTimeoutMma);
        tc_fence_after();
        {
            float x[32];
            tmem_ld32(c128 + lane_base + cq * 32, x);
            tmem_ld_wait();
            const float dot = dot_row32(sm + (hi ? L::K : L::Q) + (cq >> 1) * kHalf, r, (cq & 1) * 4, x);
            float scale;
            if (!hi) {
                scale = __expf(Gr);
                P(P_ROWQ)[r] = rowpart + scale * dot;
            } else {
                scale = __expf(Gs[kChunk - 1] - Gr);
                lastpart = scale * dot;
                P(P_KD)[r] = -lastpart;
            }
#pragma unroll
            for (int q = 0; q < 32; ++q) x[q] *= scale;
            tmem_st32(c128 + lane_base + cq * 32, x);
        }
        hand_over(&bar_s[0]);
        // (c) dW = -(dDelta S^T) (lanes 0-15) and dVhat (lanes 16-31)
        wait_flag(&bar_a[2], kErrTimeoutMma);
        tc_fence_after();
        {
            float x[32];
            tmem_ld32(c256 + lane_base + cq * 32, x);
            tmem_ld_wait();
            if (!hi) {
#pragma unroll
                for (int q = 0; q < 32; ++q) x[q] = -x[q];
                put_row(sm + L::Dt + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);  // MN-major B of T^T dW
            } else {
                const float br = bpre;
                float vd = 0.f;
                uint4 ov[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const uint32_t w[4] = {vpre[qq].x, vpre[qq].y, vpre[qq].z, vpre[qq].w};
                    uint32_t* ow = &ov[qq].x;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 fv = unpack_bf16(w[p]);
                        vd += fv.x * x[qq * 8 + 2 * p] + fv.y * x[qq * 8 + 2 * p + 1];
                        ow[p] = pack_bf16(br * x[qq * 8 + 2 * p], br * x[qq * 8 + 2 * p + 1]);
                    }
                }
                // dv row r into the dO tile (its products are done) for one TMA store
#pragma unroll
                for (int qq = 0; qq < 4; ++qq)
                    *(uint4*)(sm + L::dO + (cq >> 1) * kHalf + sw128(r, (cq & 1) * 4 + qq)) = ov[qq];
                P(P_VD)[r] = vd;
                put_row(sm + L::dDt + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);  // K-major A of dA
            }
        }
        // (d) the last-row sum of e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lastpart += __shfl_xor_sync(0xffffffffu, lastpart, off);
        if (lane == 0) red[16 + warp] = lastpart;
        hand_over(&bar_s[1]);
        // dKhat: dG and dbeta terms, the K-major A operand of dKhat W^T, and
        // diag(beta gamma) dKhat as the start of dKp
        wait_flag(&bar_c[0], kErrTimeoutMma);
        tc_fence_after();
        {
            float x[32];
            tmem_ld32(c256 + lane_base + cq * 32, x);  // lanes 0-15: dKhat
            tmem_ld_wait();
            if (!hi) {
                const float gam = __expf(Gs[r]), br = bpre;
                const float kd = dot_row32(sm + L::K + (cq >> 1) * kHalf, r, (cq & 1) * 4, x);
                P(P_GK)[r] = gam * kd;
                P(P_BGK)[r] = br * gam * kd;
                put_row(sm + L::St + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);  // K-major A of dA
#pragma unroll
                for (int q = 0; q < 32; ++q) x[q] *= br * gam;
            }
            tmem_st32(c256 + lane_base + cq * 32, x);
        }
        {
            // dq (lanes 0-15 of the dQ accumulator) is final: its rows into the dead dW
            // tile for an early store
            float x[32];
            tmem_ld32(c128 + lane_base + cq * 32, x);
            tmem_ld_wait();
            if (!hi) put_row(sm + L::Dt + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);
        }
        hand_over(&bar_s[2]);
        wait_flag(&bar_c[1], kErrTimeoutMma);
        tc_fence_after();
        {
            // B, dA, dB .* B (added onto PD), E on columns [16 cq, 16 cq + 16): lane l < 16
            // holds (K K^T)[r], lane l + 16 dA[r]; each finishes 8 columns as in (a).  A
            // warp whose columns all lie past its rows has B = dA = 0 there: E = 0, PD as is.
            if (cq > quad) {
                const int tb = 16 * cq + (hi ? 8 : 0);
#pragma unroll
                for (int q = 0; q < 8; ++q) Ef[r * 65 + tb + q] = 0.f;
                if (!hi) {
                    P(P_SAB)[r] = 0.f;
                    P(P_SBB)[r] = 0.f;
                }
            } else {
                float va[16], vb[16];
                tmem_ld16(c0 + lane_base + cq * 16, va);   // lanes 16-31: dA (before the sign)
                tmem_ld16(c384 + lane_base + cq * 16, vb);  // lanes 0-15: K K^T
                tmem_ld_wait();
                const int tb = 16 * cq + (hi ? 8 : 0);
                const float Gr = Gs[r], br = bpre;
                float sab = 0.f, sbb = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float recv = __shfl_xor_sync(0xffffffffu, hi ? va[q] : vb[8 + q], 16);
                    const float kk = hi ? recv : vb[q];
                    const float dar = hi ? va[8 + q] : recv;
                    const int t = tb + q;
                    const bool lower = t < r;
                    const float gam = lower ? __expf(Gr - Gs[t]) : 0.f;
                    const float bv = gam * kk;
                    const float da = lower ? -dar : 0.f;
                    sab += da * bv;
                    const float dbb = br * da * bv;
                    sbb += dbb;
                    PD[r * 65 + t] += dbb;  // the same thread wrote dP .* P here in (a)
                    Ef[r * 65 + t] = br * da * gam;
                }
                sab += __shfl_xor_sync(0xffffffffu, sab, 16);
                sbb += __shfl_xor_sync(0xffffffffu, sbb, 16);
                if (!hi) {
                    P(P_SAB)[r] = sab;
                    P(P_SBB)[r] = sbb;
                }
            }
        }
        named_sync(1, kThreads);  // PD and E of every row
        {
            // E + E^T as a bf16 K-major tile [r][64 t] (in the F slot), and the column
            // sums of PD = dP .* P + dB .* B over 8-row groups
            const int rr = tid >> 3, cc = tid & 7;
            float e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = cc * 8 + i;
                e[i] = Ef[rr * 65 + t] + Ef[t * 65 + rr];
            }
            put_row(sm + L::F, rr, cc, e, 8);
            const int col = tid & 63, g = tid >> 6;
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) s += PD[(8 * g + i) * 65 + col];
            csp[g * 64 + col] = s;
        }
        hand_over(&bar_s[3]);
        named_sync(1, kThreads);  // the per-row partial sums and column sums of every warp
        // ---------------- epilogue: dg and dbeta while (E + E^T) K runs, then dk
        if (warp == 0) {  // dG and dg = reverse in-chunk cumsum
            float sdot = 0.f, last = 0.f;
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                sdot += red[w];
                last += red[16 + w];
            }
            float v2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int rr = 2 * lane + e;
                float g = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) g -= csp[i * 64 + rr];
#pragma unroll
                for (int pi = 0; pi < kDgTerms * 4; ++pi) g += part[pi * 64 + rr];
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
        } else if (warp == 1 || warp == 2) {  // dbeta
            const int rr = tid - 32;
            if (rr < Lr) {
                float db = 0.f;
#pragma unroll
                for (int pi = kDgTerms * 4; pi < P_COUNT * 4; ++pi) db += part[pi * 64 + rr];
                a.dbeta[tok_index(a, b, t0 + rr, h)] = db;
            }
        }
        wait_flag(&bar_c[2], kErrTimeoutMma);
        tc_fence_after();
        {
            // dk = dK (lanes 16-31 of the dQ / dK accumulator) + dKp (lanes 0-15), columns
            // [32 cq, 32 cq + 32), into the U^T tile (read by now)
            float x[32], y[32];
            tmem_ld32(c128 + lane_base + cq * 32, x);
            tmem_ld32(c256 + lane_base + cq * 32, y);  // lanes 0-15: dKp
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) x[q] += __shfl_xor_sync(0xffffffffu, y[q], 16);
            if (hi) put_row(sm + L::Ut + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);
        }
        fence_async_smem();
    }
    __syncthreads();
    if (tid == kIss && !*s_abort) {  // rows past the piece's end are clipped by the stores
        tma_store_4d(&tm_dk, sm + L::Ut, 0, h, t0, b);
        tma_store_4d(&tm_dk, sm + L::Ut + kHalf, 64, h, t0, b);
        bulk_commit();
    }
    if (tid == kIss) {
        if (*s_abort) {  // copies still in flight land, and every UMMA issued has
                         // finished, before the CTA exits and frees the TMEM
            for (int i = 0; i < kLoads; ++i) mbar_wait(&bar_ld[i], 0);
            mma_commit(bar_fin);
            mbar_wait(bar_fin, 0);
        }
        bulk_wait_read<0>();  // the output stores have read shared memory
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_grad_fused_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD, rowsC = (uint64_t)BH * a.NC * kChunk;
    CUtensorMap tm_q{}, tm_k{}, tm_do{}, tm_wt{}, tm_ut{}, tm_t{}, tm_dt{}, tm_ddt{}, tm_sc{}, tm_dsc{};
    CUtensorMap tm_dq{}, tm_dk{}, tm_dv{};
    const bool ok = tmap_tokens(&tm_q, a.q, a, kD) && tmap_tokens(&tm_k, a.k, a, kD) &&
                    tmap_tokens(&tm_do, a.dO, a, kD) && tmap_2d(&tm_wt, a.Wt, 64, rows, 128) &&
                    tmap_2d(&tm_ut, a.Ut, 64, rows, 128) && tmap_2d(&tm_t, a.Tm, 64, rowsC, 64) &&
                    tmap_2d(&tm_dt, a.Dt, 64, rows, 128) && tmap_2d(&tm_ddt, a.dDt, 64, rows, 128) &&
                    tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_dsc, a.dSc, kD, rows, 128) &&
                    tmap_tokens(&tm_dq, a.dq, a, kD) && tmap_tokens(&tm_dk, a.dk_, a, kD) &&
                    tmap_tokens(&tm_dv, a.dv_, a, kD);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = FusedSmem::Size + 1024;
    cudaError_t e = cudaFuncSetAttribute(grad_fused_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_GRAD_FUSED, s);
    grad_fused_tc_kernel<<<dim3(a.NC, BH), kBlock, smem, s>>>(tm_q, tm_k, tm_do, tm_wt, tm_ut, tm_t, tm_dt,
                                                                tm_ddt, tm_sc, tm_dsc, tm_dq, tm_dk, tm_dv, a);
    e = cudaGetLastError();
    timing_end(KK_GRAD_FUSED, s);
    return e;
}

}  // namespace sf
