// Fused per-chunk gradient kernel of the gated delta rule (sm_100a).
//
// One CTA per chunk-head computes dq, dk, dv, dbeta and dg from one load of
// its inputs.  The chunkwise backward of the delta rule, with S the state
// entering the chunk, dS' the gradient of the state leaving it, T = (I + A)^-1
// the chunk's UT inverse and Delta = U - W S its corrected values:
//   P = (Q K^T) .* Gamma,  dP = (dO Delta^T) .* lower,  F = dP .* Gamma
//   dQ = diag(gamma) dO S^T + F K
//   dVhat = T^T dDelta,  dv = diag(beta) dVhat
//   dKhat = T^T dW = -dVhat S^T                         (dW = -dDelta S^T)
//   dA = -(dKhat W^T + dVhat U^T) .* strictly lower = -(dVhat Delta^T) .* strictly lower
//   dB = diag(beta) dA,  E = dB .* Gamma,  B = (K K^T) .* Gamma (strictly lower)
//   dK = F^T Q + diag(e^{G_C - G}) Delta dS'^T + diag(beta gamma) dKhat + (E + E^T) K
//   dbeta_r = <V_r, dVhat_r> + gamma_r <K_r, dKhat_r> + sum_t dA_rt B_rt
//   dG_r = rowsum(dP.*P) - colsum(dP.*P) + rowsum(dB.*B) - colsum(dB.*B)
//          + gamma_r <(Q S)_r, dO_r> + beta_r gamma_r <K_r, dKhat_r>
//          - e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
//          + [last row] (sum_r e^{G_C - G_r} <K_r, (Delta dS'^T)_r> + gamma_C <S, dS'>)
//   dg = reverse in-chunk cumsum of dG.
// The two rewritten lines follow from associativity and from U - W S = Delta:
// T^T (dDelta S^T) = dVhat S^T, and dKhat W^T + dVhat U^T = dVhat (U - W S)^T.
// So neither W nor U is read, and dA and dKhat come out of one product,
// dVhat [Delta^T | S^T] (N = 192), two element-wise stages after the loads.
//
// The UMMAs are all M = 64, their accumulators paired at TMEM lane offsets 0
// (lo) and 16 (hi): rows 16 w + l of a lo tile sit in lanes 32 w + l, those of
// a hi tile in lanes 32 w + 16 + l.  Columns:
//   lo [0, 64)     Q K^T                 lo [64, 256)  dO [Delta^T | S^T] -> dP | dQ
//   hi [128, 256)  Delta dS'^T -> dK     lo [256, 384) dVhat = T^T dDelta
//   hi [256, 448)  dVhat [Delta^T | S^T] -> dA | dKhat, then dKp
//   lo [384, 448)  K K^T
//
// One thread of a seventeenth warp issues the copies and every UMMA, each as
// soon as its operands are in place.  Sixteen warps share the element-wise
// work (warp w reads TMEM lane quadrant w % 4 and a quarter of the columns,
// w / 4); they hand each stage over through an mbarrier (one arrival per warp)
// and wait for the products they read on the commit barriers.  Their order is
// the dependent chain first: dVhat (from the first copy group) -> dv, dbeta's
// V term and dVhat in bf16 -> [dA | dKhat] -> E, dKp -> (E + E^T) K -> dk;
// the attention side (P, dP, F, the rescaled dO S^T and Delta dS'^T, then
// F K and F^T Q -> dq) fills the gaps.

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
constexpr int kLoads = 4;              // operand groups, in the order they are needed

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

// Barriers: kLoads copy groups; commits a0 (T^T dDelta), a1 (dO [Delta^T | S^T]),
// a2 (Q K^T, K K^T), a3 (Delta dS'^T), c0 ([dA | dKhat]), c1 (F K, F^T Q),
// c2 ((E + E^T) K); hand-overs s_c, s_ab, s_d, s_q (16 arrivals); fin.
constexpr int kNBar = kLoads + 4 + 3 + 4 + 1;

struct FusedSmem {
    static constexpr int dDt = 0;                 // dDelta^T [128 j][64 r]; later dVhat, bf16 [jblk][64 r][64]
    static constexpr int Tb = dDt + kTile;        // T [r'][64 r]
    static constexpr int dO = Tb + kHalf;         // [dvblk][64 r][64]
    static constexpr int Dt = dO + kTile;         // Delta^T [128 j][64 t]; at the end the dk staging
    static constexpr int St = Dt + kTile;         // S^T [2][128 j][64 i], 16 KB behind Delta^T:
                                                  // [Delta^T | S^T] is one N = 192 operand
    static constexpr int Q = St + 2 * kTile;      // [dkblk][64 r][64]; later the dq staging
    static constexpr int K = Q + kTile;           // [dkblk][64 r][64]
    static constexpr int dSt = K + kTile;         // dS'^T [2][128 j][64 i]; later E, fp32 [64][65]
    static constexpr int F = dSt + 2 * kTile;     // F = dP .* Gamma, bf16 [r][64 t]
    static constexpr int EE = F + kHalf;          // E + E^T, bf16 [r][64 t]
    static constexpr int dVs = EE + kHalf;        // dv staging [dvblk][64 r][64]
    static constexpr int PD = dVs + kTile;        // fp32 [64][65]: dP .* P, then + dB .* B
    static constexpr int Gs = PD + 64 * 65 * 4;   // 64 fp32
    static constexpr int csp = Gs + 256;          // fp32 [8][64]: column sums of PD over 8-row groups
    static constexpr int part = csp + 8 * 256;    // fp32 [P_COUNT][4][64]
    static constexpr int red = part + P_COUNT * 4 * 256;  // fp32 [32]: per-warp <S, dS'>, last-row sums
    static constexpr int Bar = red + 128;
    static constexpr int Misc = Bar + kNBar * 8;
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
                         const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_t,
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
    uint64_t* bar_a = bar_ld + kLoads;            // [4] products of loaded tiles done
    uint64_t* bar_c = bar_a + 4;                  // [3] later products done
    uint64_t* bar_s = bar_c + 3;                  // [4] element-wise hand-overs (16 warps): c, ab, d, q
    uint64_t* bar_fin = bar_s + 4;                // teardown after an abort
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);

    const int c = blockIdx.x, bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
    const int NC = a.NC, TP = NC * kChunk;
    const int t0 = c * kChunk, Lr = min(kChunk, a.T - t0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cq = warp >> 2;  // TMEM lane quadrant, column quarter
    const bool hi = lane >= 16;                 // lanes 16-31: the hi tiles
    const int r = 16 * quad + (lane & 15);      // chunk row of this thread's tiles
    auto P = [&](int term) { return part + (term * 4 + cq) * 64; };

    if (tid == kIss) {
        for (int i = 0; i < kNBar; ++i) {
            const bool hand = i >= kLoads + 7 && i < kLoads + 11;  // the four hand-overs
            mbar_init(bar_ld + i, hand ? 16 : 1);
        }
        *s_abort = 0;
        fence_barrier_init();
        const int rowD = (bh * NC + c) * kD, rowC = (bh * NC + c) * kChunk;
        // 0: dDelta^T, T (T^T dDelta heads the dependent chain)
        mbar_expect_tx(&bar_ld[0], kTile + kHalf);
        tma_load_2d(sm + L::dDt, &tm_ddt, 0, rowD, &bar_ld[0]);
        tma_load_2d(sm + L::Tb, &tm_t, 0, rowC, &bar_ld[0]);
        // 1: dO, Delta^T, S^T (dO [Delta^T | S^T]; [Delta^T | S^T] is also the B of the chain's
        // second product)
        mbar_expect_tx(&bar_ld[1], 2 * kHalf + 3 * kTile);
        tma_load_4d(sm + L::dO, &tm_do, 0, h, t0, b, &bar_ld[1]);
        tma_load_4d(sm + L::dO + kHalf, &tm_do, 64, h, t0, b, &bar_ld[1]);
        tma_load_2d(sm + L::Dt, &tm_dt, 0, rowD, &bar_ld[1]);
        tma_load_2d(sm + L::St, &tm_sc, 0, rowD, &bar_ld[1]);
        tma_load_2d(sm + L::St + kTile, &tm_sc, 64, rowD, &bar_ld[1]);
        // 2: Q, K, G (Q K^T, K K^T)
        mbar_expect_tx(&bar_ld[2], 4 * kHalf + 256);
        tma_load_4d(sm + L::Q, &tm_q, 0, h, t0, b, &bar_ld[2]);
        tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, h, t0, b, &bar_ld[2]);
        tma_load_4d(sm + L::K, &tm_k, 0, h, t0, b, &bar_ld[2]);
        tma_load_4d(sm + L::K + kHalf, &tm_k, 64, h, t0, b, &bar_ld[2]);
        bulk_load(Gs, a.G + (size_t)bh * TP + t0, 256, &bar_ld[2]);
        // 3: dS'^T (Delta dS'^T)
        mbar_expect_tx(&bar_ld[3], 2 * kTile);
        tma_load_2d(sm + L::dSt, &tm_dsc, 0, rowD, &bar_ld[3]);
        tma_load_2d(sm + L::dSt + kTile, &tm_dsc, 64, rowD, &bar_ld[3]);
    }
    if (warp == 0) tmem_alloc(s_tmem, 512);
    // beta of this thread's row, and the 16 columns of V's row r this thread takes in the
    // dVhat stage, read while the tiles load (a load consumed before the block-wide
    // barrier below would hold the issuer's first products back)
    const int cb = cq * 32 + (hi ? 16 : 0);  // first dVhat column of this thread
    const float bpre = (warp < 16 && r < Lr) ? a.beta[tok_index(a, b, t0 + r, h)] : 0.f;
    uint4 vpre[2] = {};
    if (warp < 16 && r < Lr) {
        const uint4* src = (const uint4*)((const __nv_bfloat16*)a.v + tok_index(a, b, t0 + r, h) * kD + cb);
        vpre[0] = __ldg(src);
        vpre[1] = __ldg(src + 1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t l16 = 16u << 16;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t c0 = tmem, c64 = tmem + 64, c128 = tmem + 128, c256 = tmem + 256, c320 = tmem + 320,
                   c384 = tmem + 384;

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

    // ---------------- the issuer: every UMMA, each as soon as its operands are ready
    if (tid == kIss) {
        const uint32_t q = smem_u32(sm + L::Q), k = smem_u32(sm + L::K), dob = smem_u32(sm + L::dO);
        const uint32_t dt = smem_u32(sm + L::Dt), ddt = smem_u32(sm + L::dDt), tb = smem_u32(sm + L::Tb);
        const uint32_t dst = smem_u32(sm + L::dSt);
        constexpr uint32_t idKK = idesc_bf16(64, 64, false, false);
        constexpr uint32_t idKM2 = idesc_bf16(64, 128, false, true);
        constexpr uint32_t idKM3 = idesc_bf16(64, 192, false, true);
        constexpr uint32_t idMM2 = idesc_bf16(64, 128, true, true);
        constexpr uint32_t idMK2 = idesc_bf16(64, 128, true, false);
        // a group whose tiles did not land is skipped, its commit still issued so
        // that no element-wise thread waits on it for long
        bool ok = mbar_wait(&bar_ld[0], 0);
        if (ok) {  // dVhat = T^T dDelta into lo [256, 384)
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c256, sdesc(tb + ks * 2048, kHalf, 1024), sdesc(ddt + ks * 32, 16, 1024), idMK2,
                         ks > 0);
        }
        mma_commit(&bar_a[0]);
        if (ok) ok = mbar_wait(&bar_ld[1], 0);
        if (ok) {
            // dO [Delta^T | S^T]: one N = 192 product, dO Delta^T into lo [64, 128) and
            // dO S^T into lo [128, 256) (Delta^T and S^T lie 16 KB apart in smem)
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c64, sdesc(dob + o, 16, 1024), sdesc(dt + ks * 2048, kTile, 1024), idKM3, ks > 0);
            }
        }
        mma_commit(&bar_a[1]);
        if (ok) ok = mbar_wait(&bar_ld[2], 0);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c0, sdesc(q + o, 16, 1024), sdesc(k + o, 16, 1024), idKK, ks > 0);  // Q K^T
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c384, sdesc(k + o, 16, 1024), sdesc(k + o, 16, 1024), idKK, ks > 0);  // K K^T
            }
        }
        mma_commit(&bar_a[2]);
        if (ok) ok = mbar_wait(&bar_ld[3], 0);
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(c128 + l16, sdesc(dt + ks * 2048, kHalf, 1024), sdesc(dst + ks * 2048, kTile, 1024),
                         idMM2, ks > 0);  // Delta dS'^T
        }
        mma_commit(&bar_a[3]);
        // dVhat is staged in bf16 (and dv for its store): [dA | dKhat] = -dVhat [Delta^T | S^T]
        // (the sign is taken by the element-wise warps), N = 192 into hi [256, 448)
        bool sok = ok && mbar_wait(&bar_s[0], 0);
        if (sok) {
            tma_store_4d(&tm_dv, sm + L::dVs, 0, h, t0, b);  // rows past the piece's end are clipped
            tma_store_4d(&tm_dv, sm + L::dVs + kHalf, 64, h, t0, b);
            bulk_commit();
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                mma_bf16(c256 + l16, sdesc(ddt + o, 16, 1024), sdesc(dt + ks * 2048, kTile, 1024), idKM3,
                         ks > 0);
            }
        }
        mma_commit(&bar_c[0]);
        // F K and F^T Q accumulate onto the rescaled dO S^T / Delta dS'^T once the
        // element-wise warps have written F and rescaled those
        sok = sok && mbar_wait(&bar_s[1], 0);
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
        mma_commit(&bar_c[1]);
        // dKp = diag(beta gamma) dKhat + (E + E^T) K once E + E^T and the scaled dKhat are written
        sok = sok && mbar_wait(&bar_s[2], 0);
        if (sok) {
            tc_fence_after();
            const uint32_t ee = smem_u32(sm + L::EE);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(c320 + l16, sdesc(ee + ks * 32, 16, 1024), sdesc(k + ks * 2048, kHalf, 1024), idKM2,
                         1);
        }
        mma_commit(&bar_c[2]);
        sok = sok && mbar_wait(&bar_s[3], 0);
        if (sok) {  // dq, staged in the Q tile (rows past the piece's end are clipped)
            tma_store_4d(&tm_dq, sm + L::Q, 0, h, t0, b);
            tma_store_4d(&tm_dq, sm + L::Q + kHalf, 64, h, t0, b);
            bulk_commit();
        }
        if (!sok) {  // a copy or an element-wise stage did not arrive in time
            *s_abort = 1;
            atomicExch(a.err, !ok ? kErrTimeoutTma : kErrTimeoutMma);
        }
    } else if (warp < 16) {
        // ---------------- the element-wise warps
        // (c) dVhat (lo [256, 384), columns [32 cq, 32 cq + 32)): lane l < 16 reads row r and
        // hands columns 16-31 of its 32 to lane l + 16, so each thread takes 16 columns from cb:
        // dv = beta_r dVhat for its store, <V_r, dVhat_r>, and dVhat in bf16 as the K-major A
        // of [dA | dKhat]
        wait_flag(&bar_a[0], kErrTimeoutMma);
        tc_fence_after();
        {
            float x[32], y[16];
            tmem_ld32(c256 + lane_base + cq * 32, x);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const float recv = __shfl_xor_sync(0xffffffffu, x[16 + q], 16);
                y[q] = hi ? recv : x[q];
            }
            float vd = 0.f, dv[16];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const uint32_t w[4] = {vpre[qq].x, vpre[qq].y, vpre[qq].z, vpre[qq].w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 fv = unpack_bf16(w[p]);
                    vd += fv.x * y[qq * 8 + 2 * p] + fv.y * y[qq * 8 + 2 * p + 1];
                }
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) dv[q] = bpre * y[q];
            put_row(sm + L::dVs + (cb >> 6) * kHalf, r, (cb & 63) >> 3, dv, 16);
            put_row(sm + L::dDt + (cb >> 6) * kHalf, r, (cb & 63) >> 3, y, 16);
            vd += __shfl_xor_sync(0xffffffffu, vd, 16);
            if (!hi) P(P_VD)[r] = vd;
        }
        hand_over(&bar_s[0]);
        // (a) P, dP, F on columns [16 cq, 16 cq + 16): lane l < 16 holds (Q K^T)[r] and
        // (dO Delta^T)[r]; it finishes the first 8 columns and hands the last 8 to
        // lane l + 16.  A warp whose columns all lie past its rows (cq > quad) writes
        // the zeros without reading the products.
        wait_flag(&bar_ld[2], kErrTimeoutTma);  // G, Q, K are read below
        wait_flag(&bar_a[2], kErrTimeoutMma);
        tc_fence_after();
        const float Gr = Gs[r];
        float rowpart;
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
        // rescaled in TMEM by gamma_r / e^{G_C - G_r}; and <S, dS'> over the two
        // identically laid out tiles (a dG term of the last row)
        wait_flag(&bar_ld[1], kErrTimeoutTma);
        wait_flag(&bar_ld[3], kErrTimeoutTma);
        wait_flag(&bar_a[3], kErrTimeoutMma);
        tc_fence_after();
        {
            float x[32];
            tmem_ld32(c128 + lane_base + cq * 32, x);
            tmem_ld_wait();
            const float dot = dot_row32(sm + (hi ? L::K : L::Q) + (cq >> 1) * kHalf, r, (cq & 1) * 4, x);
            float scale, lastpart = 0.f;
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
            // the last-row sum of e^{G_C - G_r} <K_r, (Delta dS'^T)_r>
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lastpart += __shfl_xor_sync(0xffffffffu, lastpart, off);
            if (lane == 0) red[16 + warp] = lastpart;
        }
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
        hand_over(&bar_s[1]);
        // (d) [dA | dKhat] is done.  Every warp has read dS'^T above before E overwrites it.
        wait_flag(&bar_c[0], kErrTimeoutMma);
        named_sync(1, kThreads);
        tc_fence_after();
        {
            // B, dA, dB .* B (added onto PD), E on columns [16 cq, 16 cq + 16): lane l < 16
            // holds (K K^T)[r], lane l + 16 the unsigned dA[r]; each finishes 8 columns as in
            // (a).  A warp whose columns all lie past its rows has B = dA = 0 there: E = 0, PD as is.
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
                tmem_ld16(c256 + lane_base + cq * 16, va);  // lanes 16-31: dVhat Delta^T
                tmem_ld16(c384 + lane_base + cq * 16, vb);  // lanes 0-15: K K^T
                tmem_ld_wait();
                const int tb = 16 * cq + (hi ? 8 : 0);
                const float br = bpre;
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
        {
            // dKhat = -(dVhat S^T) (lanes 16-31 of hi [320, 448)): the dG and dbeta terms, and
            // diag(beta gamma) dKhat written back in place as the start of dKp (lanes 0-15
            // write back the values they read)
            float x[32];
            tmem_ld32(c320 + lane_base + cq * 32, x);
            tmem_ld_wait();
            if (hi) {
#pragma unroll
                for (int q = 0; q < 32; ++q) x[q] = -x[q];
                const float gam = __expf(Gr), br = bpre;
                const float kd = dot_row32(sm + L::K + (cq >> 1) * kHalf, r, (cq & 1) * 4, x);
                P(P_GK)[r] = gam * kd;
                P(P_BGK)[r] = br * gam * kd;
#pragma unroll
                for (int q = 0; q < 32; ++q) x[q] *= br * gam;
            }
            tmem_st32(c320 + lane_base + cq * 32, x);
        }
        named_sync(1, kThreads);  // PD and E of every row
        {
            // E + E^T as a bf16 K-major tile [r][64 t], and the column sums of
            // PD = dP .* P + dB .* B over 8-row groups
            const int rr = tid >> 3, cc = tid & 7;
            float e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = cc * 8 + i;
                e[i] = Ef[rr * 65 + t] + Ef[t * 65 + rr];
            }
            put_row(sm + L::EE, rr, cc, e, 8);
            const int col = tid & 63, g = tid >> 6;
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) s += PD[(8 * g + i) * 65 + col];
            csp[g * 64 + col] = s;
        }
        hand_over(&bar_s[2]);
        // dq (lanes 0-15 of lo [128, 256)) is final once F K has run: its rows into the Q tile
        // (read by F^T Q, done by then) for the store
        wait_flag(&bar_c[1], kErrTimeoutMma);
        tc_fence_after();
        {
            float x[32];
            tmem_ld32(c128 + lane_base + cq * 32, x);
            tmem_ld_wait();
            if (!hi) put_row(sm + L::Q + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);
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
            // dk = dK (hi [128, 256)) + dKp (hi [320, 448)), columns [32 cq, 32 cq + 32),
            // into the Delta^T tile (every product reading it is done)
            float x[32], y[32];
            tmem_ld32(c128 + lane_base + cq * 32, x);
            tmem_ld32(c320 + lane_base + cq * 32, y);
            tmem_ld_wait();
            if (hi) {
#pragma unroll
                for (int q = 0; q < 32; ++q) x[q] += y[q];
                put_row(sm + L::Dt + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);
            }
        }
        fence_async_smem();
    }
    __syncthreads();
    if (tid == kIss && !*s_abort) {  // rows past the piece's end are clipped by the stores
        tma_store_4d(&tm_dk, sm + L::Dt, 0, h, t0, b);
        tma_store_4d(&tm_dk, sm + L::Dt + kHalf, 64, h, t0, b);
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
    CUtensorMap tm_q{}, tm_k{}, tm_do{}, tm_t{}, tm_dt{}, tm_ddt{}, tm_sc{}, tm_dsc{};
    CUtensorMap tm_dq{}, tm_dk{}, tm_dv{};
    const bool ok = tmap_tokens(&tm_q, a.q, a, kD) && tmap_tokens(&tm_k, a.k, a, kD) &&
                    tmap_tokens(&tm_do, a.dO, a, kD) && tmap_2d(&tm_t, a.Tm, 64, rowsC, 64) &&
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
    grad_fused_tc_kernel<<<dim3(a.NC, BH), kBlock, smem, s>>>(tm_q, tm_k, tm_do, tm_t, tm_dt, tm_ddt, tm_sc,
                                                                tm_dsc, tm_dq, tm_dk, tm_dv, a);
    e = cudaGetLastError();
    timing_end(KK_GRAD_FUSED, s);
    return e;
}

}  // namespace sf
