// Fused per-chunk gradient kernel of the gated delta rule (sm_100a).
//
// For each chunk-head (64 tokens of one batch-head) the kernel computes dq, dk,
// dv, dbeta and dg from one load of its inputs.  The chunkwise backward of the
// delta rule, with S the state
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
// One CTA per SM takes chunk-heads (work items) from a counter until none are
// left, so that CTAs which start late (the SM was busy) take fewer, and
// overlaps them: one thread of a seventeenth warp issues the copies, the stores
// and every UMMA, each as soon as its operands are in place and the tiles or
// TMEM columns it overwrites are dead.  The next item's copies go out as the
// current item's products finish with their tiles: dDelta^T, T, dO, Delta^T,
// S^T, Q, G and V once F K and F^T Q have run (K into the other of two K tiles),
// dS'^T once E, written over it, is consumed; its first product T^T dDelta runs
// behind the current item's last one.  Sixteen warps share the
// element-wise work (warp w reads TMEM lane quadrant w % 4 and a quarter of
// the columns, w / 4); they hand each stage over through an mbarrier (one
// arrival per warp) and wait for the products they read on the commit
// barriers, every barrier completing one phase per item.  Their order is the
// dependent chain first: dVhat -> dv, dbeta's V term and dVhat in bf16 ->
// [dA | dKhat] -> E, dKp -> (E + E^T) K -> dk; the attention side (P, dP, F,
// the rescaled dO S^T and Delta dS'^T, then F K and F^T Q -> dq) fills the
// gaps.  dv, dq and dk leave through TMA stores from staging tiles (dv over V,
// dq in the PD region, dk in its item's K tile).

#include <cuda.h>

#include <algorithm>

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
constexpr int kIss = kThreads;         // the thread that issues copies, stores and UMMAs
constexpr int kLoads = 5;              // operand groups: four in the order the products need
                                       // them, and V (read by the element-wise warps)

// Per-row partial sums, each kept per column quarter: [term][quarter][64 rows].
// Lanes 0-15 and 16-31 of a warp own different terms, and each term is set in
// one stage and added to in a later one by the same thread.
enum PartTerm {
    P_DG_LO = 0,  // dG: rowsum(dP .* P) + gamma_r <Q_r, (dO S^T)_r> + rowsum(dB .* B)
    P_DG_HI,      // dG: -e^{G_C - G_r} <K_r, (Delta dS'^T)_r> + beta_r gamma_r <K_r, dKhat_r>
    P_DB_LO,      // dbeta: <V_r, dVhat_r> + sum_t dA_rt B_rt
    P_DB_HI,      // dbeta: gamma_r <K_r, dKhat_r>
    P_COUNT
};
constexpr int kDgTerms = P_DB_LO;  // terms [0, kDgTerms) go to dG, the rest to dbeta

// Barriers: kLoads copy groups; commits a0 (T^T dDelta), a1 (dO [Delta^T | S^T]),
// a2 (Q K^T), a3 (Delta dS'^T), c0 (K K^T, [dA | dKhat]), c1 (F K, F^T Q),
// c2 ((E + E^T) K); hand-overs s_c, s_ab, s_d, s_q and dk (16 arrivals); pdfree
// (the issuer: the dq store has read the PD region); pub (the issuer: the next
// item is published); fin.
constexpr int kNBar = kLoads + 4 + 3 + 5 + 1 + 1 + 1;

struct FusedSmem {
    static constexpr int dDt = 0;                 // dDelta^T [128 j][64 r]; later dVhat, bf16 [jblk][64 r][64]
    static constexpr int Tb = dDt + kTile;        // T [r'][64 r]
    static constexpr int dO = Tb + kHalf;         // [dvblk][64 r][64]
    static constexpr int Dt = dO + kTile;         // Delta^T [128 j][64 t]
    static constexpr int St = Dt + kTile;         // S^T [2][128 j][64 i], 16 KB behind Delta^T:
                                                  // [Delta^T | S^T] is one N = 192 operand
    static constexpr int Q = St + 2 * kTile;      // [dkblk][64 r][64]
    static constexpr int K = Q + kTile;           // K of even items [dkblk][64 r][64]; then their dk staging
    static constexpr int dSt = K + kTile;         // dS'^T [2][128 j][64 i]; later E, fp32 [64][65]
    static constexpr int F = dSt + 2 * kTile;     // F = dP .* Gamma, bf16 [r][64 t]
    static constexpr int EE = F + kHalf;          // E + E^T, bf16 [r][64 t]
    static constexpr int dVs = EE + kHalf;        // V [dvblk][64 r][64], then the dv staging
    static constexpr int K1 = dVs + kTile;        // K of odd items; then their dk staging
    static constexpr int PD = K1 + kTile;         // fp32 [64][65]: dP .* P, then + dB .* B; then
                                                  // the dq staging [dkblk][64 r][64]
    static constexpr int Gs = PD + 64 * 65 * 4;   // [item parity][64] fp32
    static constexpr int csp = Gs + 512;          // fp32 [8][64]: column sums of PD over 8-row groups
    static constexpr int part = csp + 8 * 256;    // fp32 [P_COUNT][4][64]
    static constexpr int red = part + P_COUNT * 4 * 256;  // fp32 [32]: per-warp <S, dS'>, last-row sums;
                                                          // [32]: the dG sum of rows 32-63
    static constexpr int Bar = red + 256;
    static constexpr int Misc = Bar + kNBar * 8;
    static constexpr int Size = Misc + 16;
};
static_assert(FusedSmem::Size + 1024 <= 232448, "shared memory of one CTA");

__device__ __forceinline__ size_t tok_index(const Args& a, int b, int t, int h) {
    return ((size_t)b * a.ld_t + t) * a.H + h;
}

// A global load that stays where it is written (read-only data; an asm volatile
// load is not moved to its first use), so that its latency overlaps the work that
// follows.
__device__ __forceinline__ float ldg_nc_f32(const float* p) {
    float r;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(r) : "l"(p));
    return r;
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

// Work item n of a launch over NC chunks of every batch-head, the batch-head fastest: the
// chunk-heads in flight at once then cover every head of a few chunks, and their
// token-major loads take whole token rows.
struct Item {
    int c, bh, b, h, t0;
};
__device__ __forceinline__ Item item_of(const Args& a, int n) {
    Item it;
    const int BH = a.B * a.H;
    it.c = n / BH;
    it.bh = n - it.c * BH;
    it.b = it.bh / a.H;
    it.h = it.bh - it.b * a.H;
    it.t0 = it.c * kChunk;
    return it;
}

__global__ void __launch_bounds__(kBlock, 1)
    grad_fused_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_t,
                         const __grid_constant__ CUtensorMap tm_dt, const __grid_constant__ CUtensorMap tm_ddt,
                         const __grid_constant__ CUtensorMap tm_sc, const __grid_constant__ CUtensorMap tm_dsc,
                         const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                         const __grid_constant__ CUtensorMap tm_dv, const __grid_constant__ CUtensorMap tm_v,
                         const Args a) {
    using L = FusedSmem;
    extern __shared__ uint8_t smem_raw[];
    // the 1024-byte aligned base, by pointer arithmetic on the shared array (so that every
    // pointer derived from it is known to address shared memory)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* csp = (float*)(sm + L::csp);
    float* PD = (float*)(sm + L::PD);
    float* Ef = (float*)(sm + L::dSt);
    float* part = (float*)(sm + L::part);
    float* red = (float*)(sm + L::red);
    uint64_t* bar_ld = (uint64_t*)(sm + L::Bar);  // [kLoads] operand groups landed
    uint64_t* bar_a = bar_ld + kLoads;            // [4] products of loaded tiles done
    uint64_t* bar_c = bar_a + 4;                  // [3] later products done
    uint64_t* bar_s = bar_c + 3;                  // [4] element-wise hand-overs (16 warps): c, ab, d, q
    uint64_t* bar_dk = bar_s + 4;                 // dk read from TMEM and staged (16 warps)
    uint64_t* bar_pdfree = bar_dk + 1;            // the dq store has read the PD region (issuer)
    uint64_t* bar_pub = bar_pdfree + 1;           // the next item is published (issuer)
    uint64_t* bar_fin = bar_pub + 1;              // teardown after an abort
    uint32_t* s_tmem = (uint32_t*)(sm + L::Misc);
    volatile int* s_abort = (volatile int*)(sm + L::Misc + 4);
    volatile int* s_item = (volatile int*)(sm + L::Misc + 8);  // [item parity]: chunk-head, or -1

    const int NC = a.NC, TP = NC * kChunk;
    const int total = a.B * a.H * NC;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, cq = warp >> 2;  // TMEM lane quadrant, column quarter
    const bool hi = lane >= 16;                 // lanes 16-31: the hi tiles
    const int r = 16 * quad + (lane & 15);      // chunk row of this thread's tiles
    auto P = [&](int term) { return part + (term * 4 + cq) * 64; };
    // K of item j (by parity: two tiles, so that the next item's K lands while this one's
    // is still read)
    auto k_tile = [&](int j) { return sm + ((j & 1) ? L::K1 : L::K); };
    const int cb = cq * 32 + (hi ? 16 : 0);     // first dVhat column of this thread

    // The issuer's copies of one operand group of the CTA's item j, chunk-head n.  The
    // group's barrier is armed with all of its bytes before its first copy; `pend`
    // marks the groups whose armed phase the issuer has not yet seen complete, and
    // `pend_par` that phase's parity.
    uint32_t pend = 0, pend_par = 0;
    // the next ticket of this CTA (the issuer takes them): chunk-head `ticket` while it is
    // below `total`
    auto take_item = [&]() { return atomicAdd(a.ticket, 1u); };
    auto item_or_none = [&](unsigned t) { return t < (unsigned)total ? (int)t : -1; };
    int cur = -1;  // the issuer's current chunk-head
    auto load_group = [&](int g, int n, int j) {
        const Item it = item_of(a, n);
        const int rowD = (it.bh * NC + it.c) * kD, rowC = (it.bh * NC + it.c) * kChunk;
        if (g == 0) {  // dDelta^T, T (T^T dDelta heads the dependent chain)
            mbar_expect_tx(&bar_ld[0], kTile + kHalf);
            tma_load_2d(sm + L::dDt, &tm_ddt, 0, rowD, &bar_ld[0]);
            tma_load_2d(sm + L::Tb, &tm_t, 0, rowC, &bar_ld[0]);
        } else if (g == 1) {  // dO, Delta^T, S^T (dO [Delta^T | S^T]; [Delta^T | S^T] is
                              // also the B of the chain's second product)
            mbar_expect_tx(&bar_ld[1], 2 * kHalf + 3 * kTile);
            tma_load_4d(sm + L::dO, &tm_do, 0, it.h, it.t0, it.b, &bar_ld[1]);
            tma_load_4d(sm + L::dO + kHalf, &tm_do, 64, it.h, it.t0, it.b, &bar_ld[1]);
            tma_load_2d(sm + L::Dt, &tm_dt, 0, rowD, &bar_ld[1]);
            tma_load_2d(sm + L::St, &tm_sc, 0, rowD, &bar_ld[1]);
            tma_load_2d(sm + L::St + kTile, &tm_sc, 64, rowD, &bar_ld[1]);
        } else if (g == 2) {  // Q, K, G (Q K^T, K K^T); G into the item parity's buffer
            mbar_expect_tx(&bar_ld[2], 4 * kHalf + 256);
            tma_load_4d(sm + L::Q, &tm_q, 0, it.h, it.t0, it.b, &bar_ld[2]);
            tma_load_4d(sm + L::Q + kHalf, &tm_q, 64, it.h, it.t0, it.b, &bar_ld[2]);
            tma_load_4d(k_tile(j), &tm_k, 0, it.h, it.t0, it.b, &bar_ld[2]);
            tma_load_4d(k_tile(j) + kHalf, &tm_k, 64, it.h, it.t0, it.b, &bar_ld[2]);
            bulk_load(sm + L::Gs + (j & 1) * 256, a.G + (size_t)it.bh * TP + it.t0, 256, &bar_ld[2]);
        } else if (g == 3) {  // dS'^T (Delta dS'^T)
            mbar_expect_tx(&bar_ld[3], 2 * kTile);
            tma_load_2d(sm + L::dSt, &tm_dsc, 0, rowD, &bar_ld[3]);
            tma_load_2d(sm + L::dSt + kTile, &tm_dsc, 64, rowD, &bar_ld[3]);
        } else {  // V, into the dv staging tile (rows past the piece's end read as zero)
            mbar_expect_tx(&bar_ld[4], 2 * kHalf);
            tma_load_4d(sm + L::dVs, &tm_v, 0, it.h, it.t0, it.b, &bar_ld[4]);
            tma_load_4d(sm + L::dVs + kHalf, &tm_v, 64, it.h, it.t0, it.b, &bar_ld[4]);
        }
        pend |= 1u << g;
        pend_par = (pend_par & ~(1u << g)) | ((uint32_t)(j & 1) << g);
    };

    if (tid == kIss) {
        for (int i = 0; i < kNBar; ++i) {
            const bool hand = i >= kLoads + 7 && i < kLoads + 12;  // the five hand-overs
            mbar_init(bar_ld + i, hand ? 16 : 1);
        }
        *s_abort = 0;
        cur = item_or_none(take_item());
        s_item[0] = cur;
        fence_barrier_init();
        if (cur >= 0)
            for (int g = 0; g < kLoads; ++g) load_group(g, cur, 0);
    }
    if (warp == 0) tmem_alloc(s_tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t l16 = 16u << 16;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t c0 = tmem, c64 = tmem + 64, c128 = tmem + 128, c256 = tmem + 256, c320 = tmem + 320,
                   c384 = tmem + 384;

    // ---------------- the issuer
    if (tid == kIss) {
        const uint32_t q = smem_u32(sm + L::Q), dob = smem_u32(sm + L::dO);
        const uint32_t dt = smem_u32(sm + L::Dt), ddt = smem_u32(sm + L::dDt), tb = smem_u32(sm + L::Tb);
        const uint32_t dst = smem_u32(sm + L::dSt);
        constexpr uint32_t idKK = idesc_bf16(64, 64, false, false);
        constexpr uint32_t idKM2 = idesc_bf16(64, 128, false, true);
        constexpr uint32_t idKM3 = idesc_bf16(64, 192, false, true);
        constexpr uint32_t idMM2 = idesc_bf16(64, 128, true, true);
        constexpr uint32_t idMK2 = idesc_bf16(64, 128, true, false);
        // A wait that gives up flags the abort; later work is skipped, but every commit and
        // hand-over is still issued so that the element-wise warps pass their waits.
        bool ok = true;
        auto iwait = [&](uint64_t* bar, uint32_t parity) {
            if (ok && !mbar_wait_or_abort(bar, parity, s_abort)) {
                ok = false;
                if (!*s_abort) atomicExch(a.err, kErrTimeoutMma);
                *s_abort = 1;
            }
        };
        auto ld_wait = [&](int g, int j) {
            iwait(&bar_ld[g], (uint32_t)(j & 1));
            if (ok) pend &= ~(1u << g);
        };
        auto store_dk = [&](int n, int j) {  // from item j's K tile; rows past the piece's end are clipped
            const Item it = item_of(a, n);
            if (ok) {
                tma_store_4d(&tm_dk, k_tile(j), 0, it.h, it.t0, it.b);
                tma_store_4d(&tm_dk, k_tile(j) + kHalf, 64, it.h, it.t0, it.b);
            }
            bulk_commit();
        };
        // T^T dDelta of item j into lo [256, 384): item j-1's dVhat there has been read
        auto p_dvhat = [&](int j) {
            ld_wait(0, j);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(c256, sdesc(tb + ks * 2048, kHalf, 1024), sdesc(ddt + ks * 32, 16, 1024), idMK2,
                             ks > 0);
            }
            mma_commit(&bar_a[0]);
        };
        if (cur >= 0) p_dvhat(0);
        int prev = -1, last_j = 0;
        // the ticket after the next one is taken an item ahead, so that the counter's round
        // trip overlaps an item's work (its value is first looked at in the next item)
        unsigned nxt = cur >= 0 ? take_item() : ~0u;
        for (int j = 0; cur >= 0; ++j) {
            const uint32_t ph = (uint32_t)(j & 1);
            // the next item, published for the element-wise warps (its slot was last read for
            // item j - 1 in item j - 2, before the hand-over s_q of j - 2)
            const int next = item_or_none(nxt);
            s_item[(j + 1) & 1] = next;
            mbar_arrive(bar_pub);
            if (j > 0) {  // item j-1's dq store has read the PD region: this item's dP .* P may go there
                bulk_wait_read<0>();
                mbar_arrive(bar_pdfree);
            }
            nxt = next >= 0 ? take_item() : ~0u;
            const bool has_next = next >= 0;
            const Item it = item_of(a, cur);
            const uint32_t k = smem_u32(k_tile(j));
            // dO [Delta^T | S^T]: one N = 192 product, dO Delta^T into lo [64, 128) and dO S^T
            // into lo [128, 256) (Delta^T and S^T lie 16 KB apart in smem); item j-1's dq
            // there was read before its hand-over s_q, waited below for j-1
            ld_wait(1, j);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                    mma_bf16(c64, sdesc(dob + o, 16, 1024), sdesc(dt + ks * 2048, kTile, 1024), idKM3, ks > 0);
                }
            }
            mma_commit(&bar_a[1]);
            ld_wait(2, j);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                    mma_bf16(c0, sdesc(q + o, 16, 1024), sdesc(k + o, 16, 1024), idKK, ks > 0);  // Q K^T
                }
            }
            mma_commit(&bar_a[2]);
            // item j-1's dk has been read from hi [128, 256) and [320, 448) and staged: store
            // it, then Delta dS'^T of item j into hi [128, 256)
            if (j > 0) {
                iwait(bar_dk, ph ^ 1u);
                store_dk(prev, j - 1);
            }
            ld_wait(3, j);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(c128 + l16, sdesc(dt + ks * 2048, kHalf, 1024), sdesc(dst + ks * 2048, kTile, 1024),
                             idMM2, ks > 0);  // Delta dS'^T
            }
            mma_commit(&bar_a[3]);
            // K K^T, read in (d) after the commit of [dA | dKhat]; issued here so that the
            // commits that (a) and (b) wait on come before it
            if (ok) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
                    mma_bf16(c384, sdesc(k + o, 16, 1024), sdesc(k + o, 16, 1024), idKK, ks > 0);
                }
            }
            // dVhat is staged in bf16 (and dv for its store): [dA | dKhat] = -dVhat [Delta^T | S^T]
            // (the sign is taken by the element-wise warps), N = 192 into hi [256, 448)
            iwait(&bar_s[0], ph);
            if (ok) {
                tma_store_4d(&tm_dv, sm + L::dVs, 0, it.h, it.t0, it.b);  // rows past the piece's end are clipped
                tma_store_4d(&tm_dv, sm + L::dVs + kHalf, 64, it.h, it.t0, it.b);
            }
            bulk_commit();
            if (ok) {
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
            iwait(&bar_s[1], ph);
            if (ok) {
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
            // the next item's operands but dS'^T, once every product reading their tiles is done
            // (F K, F^T Q, issued last, complete after the others) and the element-wise reads
            // of S^T and Q came before the hand-over s_ab: dDelta^T (the dVhat written over it
            // is read), T, dO, Delta^T, S^T, Q and G (item j-1's epilogue read its G before item
            // j's hand-over s_ab); V lands in the dv staging tile and K in item j-1's K tile,
            // whose dk was stored, once the stores of item j-1's dk and item j's dv have read
            // their tiles
            if (has_next) {
                iwait(&bar_c[1], ph);
                bulk_wait_read<0>();
                if (ok) {
                    load_group(0, next, j + 1);
                    load_group(4, next, j + 1);
                    load_group(1, next, j + 1);
                    load_group(2, next, j + 1);
                }
            }
            // dKp = diag(beta gamma) dKhat + (E + E^T) K once E + E^T and the scaled dKhat are written
            iwait(&bar_s[2], ph);
            if (ok) {
                tc_fence_after();
                const uint32_t ee = smem_u32(sm + L::EE);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(c320 + l16, sdesc(ee + ks * 32, 16, 1024), sdesc(k + ks * 2048, kHalf, 1024), idKM2,
                             1);
            }
            mma_commit(&bar_c[2]);
            // the next item's dS'^T: E, written over it, has been consumed
            if (has_next && ok) load_group(3, next, j + 1);
            // dq, staged in the PD region (rows past the piece's end are clipped)
            iwait(&bar_s[3], ph);
            if (ok) {
                tma_store_4d(&tm_dq, sm + L::PD, 0, it.h, it.t0, it.b);
                tma_store_4d(&tm_dq, sm + L::PD + kHalf, 64, it.h, it.t0, it.b);
            }
            bulk_commit();
            if (has_next) p_dvhat(j + 1);  // runs behind (E + E^T) K
            prev = cur;
            cur = next;
            last_j = j;
        }
        if (prev >= 0) {
            iwait(bar_dk, (uint32_t)(last_j & 1));
            store_dk(prev, last_j);
        }
        if (!ok) *s_abort = 1;
    } else if (warp < 16) {
        // ---------------- the element-wise warps
        // A wait that gives up flags the abort; every warp still passes every barrier, so
        // that no wait of another thread runs to its limit.
        auto wait_flag = [&](uint64_t* bar, uint32_t parity, int err) {
            if (!mbar_wait_or_abort(bar, parity, s_abort)) {
                if (!*s_abort) atomicExch(a.err, err);
                *s_abort = 1;
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
        // beta of this thread's row in chunk-head n, loaded one item ahead
        auto beta_of = [&](int n) {
            if (n < 0) return 0.f;
            const Item it = item_of(a, n);
            return r < min(kChunk, a.T - it.t0) ? ldg_nc_f32(a.beta + tok_index(a, it.b, it.t0 + r, it.h)) : 0.f;
        };
        int ecur = s_item[0];  // this item's chunk-head
        float bpre = beta_of(ecur);
        // Epilogue of chunk-head n, the CTA's item jj, by warps 0-3: dg and dbeta from the
        // per-row partial sums and column sums.  It runs in the next item while that one
        // waits for its first products (or after the last item).
        auto epilogue = [&](int n, int jj) {
            const Item it = item_of(a, n);
            const int b = it.b, h = it.h, t0 = it.t0, Lr = min(kChunk, a.T - t0);
            const float* Gp = (const float*)(sm + L::Gs) + (jj & 1) * 64;
            if (warp == 0 || warp == 3) {
                // dG of row rr (warp 0: rows 0-31, warp 3: rows 32-63) and dg = its reverse
                // in-chunk cumsum; warp 3 hands the sum of its rows to warp 0 on barrier 3
                const int rr = (warp == 0 ? 0 : 32) + lane;
                float g = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) g -= csp[i * 64 + rr];
#pragma unroll
                for (int pi = 0; pi < kDgTerms * 4; ++pi) g += part[pi * 64 + rr];
                if (warp == 3) {
                    // the last row's terms: sum_w <S, dS'>_w (lanes 0-15) and the last-row
                    // sums (lanes 16-31)
                    float v = red[lane];
#pragma unroll
                    for (int off = 8; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    const float sdot = __shfl_sync(0xffffffffu, v, 0);
                    if (rr == kChunk - 1) g += v + __expf(Gp[kChunk - 1]) * sdot;
                }
                float incl = g;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_down_sync(0xffffffffu, incl, off);
                    if (lane + off < 32) incl += y;
                }
                if (warp == 3) {
                    if (lane == 0) red[32] = incl;
                    named_arrive(3, 64);
                } else {
                    named_sync(3, 64);
                    incl += red[32];
                }
                if (a.g && rr < Lr) a.dg[tok_index(a, b, t0 + rr, h)] = incl;
            } else if (warp == 1 || warp == 2) {  // dbeta
                const int rr = tid - 32;
                if (rr < Lr) {
                    float db = 0.f;
#pragma unroll
                    for (int pi = kDgTerms * 4; pi < P_COUNT * 4; ++pi) db += part[pi * 64 + rr];
                    a.dbeta[tok_index(a, b, t0 + rr, h)] = db;
                }
            }
        };
        int eprev = -1, last_j = 0;  // the last item's chunk-head and index
        bool gave_up = false;        // the same in every element-wise warp
        for (int j = 0; ecur >= 0; ++j) {
            const uint32_t ph = (uint32_t)(j & 1);
            const float* Gs = (const float*)(sm + L::Gs) + (j & 1) * 64;
            const float br = bpre;
            float vdr;  // <V_r, dVhat_r> (lanes 0-15), set down in (a)
            // (c) dVhat (lo [256, 384), columns [32 cq, 32 cq + 32)): lane l < 16 reads row r and
            // hands columns 16-31 of its 32 to lane l + 16, so each thread takes 16 columns from
            // cb: dv = beta_r dVhat for its store, <V_r, dVhat_r>, and dVhat in bf16 as the
            // K-major A of [dA | dKhat].  The dv staging tile was read by the last item's store
            // (its release was waited at the end of that item).
            wait_flag(&bar_a[0], ph, kErrTimeoutMma);
            wait_flag(&bar_ld[4], ph, kErrTimeoutTma);  // V in the dv staging tile
            tc_fence_after();
            {
                uint8_t* vrow = sm + L::dVs + (cb >> 6) * kHalf;
                const uint4 vpre[2] = {*(const uint4*)(vrow + sw128(r, (cb & 63) >> 3)),
                                       *(const uint4*)(vrow + sw128(r, ((cb & 63) >> 3) + 1))};
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
                for (int q = 0; q < 16; ++q) dv[q] = br * y[q];
                put_row(vrow, r, (cb & 63) >> 3, dv, 16);  // over the V values this thread read
                put_row(sm + L::dDt + (cb >> 6) * kHalf, r, (cb & 63) >> 3, y, 16);
                vd += __shfl_xor_sync(0xffffffffu, vd, 16);
                vdr = vd;
            }
            hand_over(&bar_s[0]);
            // the next item (published at the issuer's start of this one) and its beta
            wait_flag(bar_pub, ph, kErrTimeoutMma);
            const int enext = s_item[(j + 1) & 1];
            const float bnext = beta_of(enext);
            // the last item's epilogue (warps 0-3); once all four have read the sums (barrier
            // 4) they arrive on barrier 2, on which the other warps wait before their first
            // write of the sums, in (a)
            if (j > 0 && warp < 4) {
                epilogue(eprev, j - 1);
                named_sync(4, 128);
                named_arrive(2, kThreads);
            }
            // (a) P, dP, F on columns [16 cq, 16 cq + 16): lane l < 16 holds (Q K^T)[r] and
            // (dO Delta^T)[r]; it finishes the first 8 columns and hands the last 8 to
            // lane l + 16.  A warp whose columns all lie past its rows (cq > quad) writes
            // the zeros without reading the products.
            wait_flag(&bar_ld[2], ph, kErrTimeoutTma);  // G, Q, K are read below
            wait_flag(&bar_a[2], ph, kErrTimeoutMma);
            if (j > 0) wait_flag(bar_pdfree, ph ^ 1u, kErrTimeoutTma);  // the last dq store read PD
            if (j > 0 && warp >= 4) named_sync(2, kThreads);  // the last epilogue has read the sums
            if (!hi) P(P_DB_LO)[r] = vdr;
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
            wait_flag(&bar_ld[1], ph, kErrTimeoutTma);
            wait_flag(&bar_ld[3], ph, kErrTimeoutTma);
            wait_flag(&bar_a[3], ph, kErrTimeoutMma);
            tc_fence_after();
            {
                float x[32];
                tmem_ld32(c128 + lane_base + cq * 32, x);
                tmem_ld_wait();
                const float dot = dot_row32((hi ? k_tile(j) : sm + L::Q) + (cq >> 1) * kHalf, r, (cq & 1) * 4, x);
                float scale, lastpart = 0.f;
                if (!hi) {
                    scale = __expf(Gr);
                    P(P_DG_LO)[r] = rowpart + scale * dot;
                } else {
                    scale = __expf(Gs[kChunk - 1] - Gr);
                    lastpart = scale * dot;
                    P(P_DG_HI)[r] = -lastpart;
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
            wait_flag(&bar_c[0], ph, kErrTimeoutMma);
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
                } else {
                    float va[16], vb[16];
                    tmem_ld16(c256 + lane_base + cq * 16, va);  // lanes 16-31: dVhat Delta^T
                    tmem_ld16(c384 + lane_base + cq * 16, vb);  // lanes 0-15: K K^T
                    tmem_ld_wait();
                    const int tb = 16 * cq + (hi ? 8 : 0);
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
                    if (!hi) {  // the same thread set these terms in (c) and (b)
                        P(P_DB_LO)[r] += sab;
                        P(P_DG_LO)[r] += sbb;
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
                    const float gam = __expf(Gr);
                    const float kd = dot_row32(k_tile(j) + (cq >> 1) * kHalf, r, (cq & 1) * 4, x);
                    P(P_DB_HI)[r] = gam * kd;
                    P(P_DG_HI)[r] += br * gam * kd;  // set in (b) by this thread
#pragma unroll
                    for (int q = 0; q < 32; ++q) x[q] *= br * gam;
                }
                tmem_st32(c320 + lane_base + cq * 32, x);
            }
            named_sync(1, kThreads);  // PD and E of every row
            {
                // E + E^T as a bf16 K-major tile [r][64 t] (the last item's (E + E^T) K has read
                // the tile: its commit was waited before that item's dk), and the column sums
                // of PD = dP .* P + dB .* B over 8-row groups
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
            // dq (lanes 0-15 of lo [128, 256)) is final once F K has run: its rows into the PD
            // region for the store, once every warp's column sums have read PD (the barrier
            // also completes every warp's partial sums for the epilogue).  At this barrier the
            // warps also agree on whether a wait of the CTA gave up, and then all leave the
            // loop here: a warp whose wait for the published next item gave up may have read
            // a stale one, and warps that went on to different items would never meet at
            // their named barriers again.
            wait_flag(&bar_c[1], ph, kErrTimeoutMma);
            if (named_sync_or(1, kThreads, *s_abort != 0)) {
                gave_up = true;
                break;
            }
            tc_fence_after();
            {
                float x[32];
                tmem_ld32(c128 + lane_base + cq * 32, x);
                tmem_ld_wait();
                if (!hi) put_row(sm + L::PD + (cq >> 1) * kHalf, r, (cq & 1) * 4, x, 32);
            }
            hand_over(&bar_s[3]);
            // dk = dK (hi [128, 256)) + dKp (hi [320, 448)), columns [32 cq, 32 cq + 32), staged
            // in this item's K tile (read for the last time by (E + E^T) K, and by every warp
            // before the dq stage's barrier); the hand-over lets the issuer store it and reuse
            // those TMEM columns
            wait_flag(&bar_c[2], ph, kErrTimeoutMma);
            tc_fence_after();
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float x[16], y[16];
                tmem_ld16(c128 + lane_base + cq * 32 + hf * 16, x);
                tmem_ld16(c320 + lane_base + cq * 32 + hf * 16, y);
                tmem_ld_wait();
                if (hi) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) x[q] += y[q];
                    put_row(k_tile(j) + (cq >> 1) * kHalf, r, (cq & 1) * 4 + hf * 2, x, 16);
                }
            }
            hand_over(bar_dk);
            eprev = ecur;
            ecur = enext;
            bpre = bnext;
            last_j = j;
        }
        if (!gave_up && eprev >= 0 && warp < 4) epilogue(eprev, last_j);
    }
    __syncthreads();
    if (tid == kIss) {
        if (*s_abort) {  // copies still in flight land, and every UMMA issued has finished,
                         // before the CTA exits and frees the TMEM
            for (int g = 0; g < kLoads; ++g)
                if (pend & (1u << g)) mbar_wait(&bar_ld[g], (pend_par >> g) & 1u);
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
    // the last CTA to finish puts the work counters back to zero for the next launch
    // (every CTA has taken its last item by now)
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(a.ticket + 1, 1u) == gridDim.x - 1) {
            a.ticket[0] = 0;
            a.ticket[1] = 0;
        }
    }
}

// SMs of the current device (cached per device).
int sm_count() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

}  // namespace

cudaError_t launch_grad_fused_tc(const Args& a, cudaStream_t s) {
    const int BH = a.B * a.H;
    if (BH == 0 || a.NC == 0) return cudaSuccess;
    const uint64_t rows = (uint64_t)BH * a.NC * kD, rowsC = (uint64_t)BH * a.NC * kChunk;
    CUtensorMap tm_q{}, tm_k{}, tm_do{}, tm_t{}, tm_dt{}, tm_ddt{}, tm_sc{}, tm_dsc{};
    CUtensorMap tm_dq{}, tm_dk{}, tm_dv{}, tm_v{};
    const bool ok = tmap_tokens(&tm_q, a.q, a, kD) && tmap_tokens(&tm_k, a.k, a, kD) &&
                    tmap_tokens(&tm_do, a.dO, a, kD) && tmap_2d(&tm_t, a.Tm, 64, rowsC, 64) &&
                    tmap_2d(&tm_dt, a.Dt, 64, rows, 128) && tmap_2d(&tm_ddt, a.dDt, 64, rows, 128) &&
                    tmap_2d(&tm_sc, a.Sc, kD, rows, 128) && tmap_2d(&tm_dsc, a.dSc, kD, rows, 128) &&
                    tmap_tokens(&tm_dq, a.dq, a, kD) && tmap_tokens(&tm_dk, a.dk_, a, kD) &&
                    tmap_tokens(&tm_dv, a.dv_, a, kD) && tmap_tokens(&tm_v, a.v, a, kD);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = FusedSmem::Size + 1024;
    cudaError_t e = cudaFuncSetAttribute(grad_fused_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(KK_GRAD_FUSED, s);
    // One CTA per SM it may hold; the CTAs take the chunk-heads from the work counter.
    // a.grad_sms < 0 asks to leave that many SMs to a reverse pass running beside the
    // launch (one CTA per batch-head).  That pays while the pass holds at most a quarter
    // of the SMs: with 32 heads of 148 SMs the pass and the launch take about as long
    // (132 and 139 us per 4096-token piece), while with 64 heads the pass ends long
    // before the launch, which is then faster on every SM.
    const int sms = sm_count();
    const int budget = a.grad_sms > 0                       ? std::min(a.grad_sms, sms)
                       : (a.grad_sms < 0 && -4 * a.grad_sms <= sms) ? sms + a.grad_sms
                                                                     : sms;
    const int ctas = std::min(a.NC * BH, budget);
    grad_fused_tc_kernel<<<ctas, kBlock, smem, s>>>(tm_q, tm_k, tm_do, tm_t, tm_dt, tm_ddt, tm_sc, tm_dsc, tm_dq,
                                                     tm_dk, tm_dv, tm_v, a);
    e = cudaGetLastError();
    timing_end(KK_GRAD_FUSED, s);
    return e;
}

}  // namespace sf
