// SIMT kernels of the chunkwise linear-recurrence layer: fp32 arithmetic on
// CUDA cores, I/O in fp32 or bf16.  They define the chunkwise algebra every
// other kernel of the library must reproduce, and they are the fp32 path.
//
// Per (b, h) and chunk of C = 64 tokens (rows r, i), with G the in-chunk
// inclusive cumsum of g, gamma = exp(G), Gamma_ri = exp(G_r - G_i) and S the
// state entering the chunk (the recurrence is the gated delta rule of Gated
// DeltaNet, evaluated in the StateFlow summary, section 实验设计; the
// chunk / boundary-state structure is the StateFlow summary's section 方法详解):
//
//   B     = (K K^T) .* Gamma, strictly lower          A = diag(beta) B
//   T     = (I + A)^-1 (unit lower triangular)
//   W     = T diag(beta gamma) K,  U = T diag(beta) V  (intra-chunk kernel)
//   Delta = U - W S                                    (state pass)
//   S'    = gamma_C S + Ktil^T Delta,  Ktil = diag(exp(G_C - G)) K
//   O     = diag(gamma) Q S + P Delta,  P = (Q K^T) .* Gamma, lower incl.
//
// Linear attention (no beta) has T = I, W = 0, Delta = V.  The derivation
// unrolls S_r = a_r S_{r-1} + k_r d_r^T with d_r = beta_r (v_r - a_r
// S_{r-1}^T k_r) over the chunk; only exponents <= 0 are ever evaluated.
//
// Backward per chunk with dS' = dL/dS' (from the reverse state pass):
//   dDelta = P^T dO + Ktil dS'
//   dS     = gamma_C dS' + (diag(gamma) Q)^T dO - W^T dDelta
//   dP = (dO Delta^T) .* lower incl.;  dQ = diag(gamma) dO S^T + (dP .* Gamma) K
//   dW = -dDelta S^T;  dKhat = T^T dW;  dVhat = T^T dDelta
//   dA = -(dKhat W^T + dVhat U^T) .* strictly lower;  dB = diag(beta) dA
//   dK = (dP .* Gamma)^T Q + diag(exp(G_C - G)) Delta dS'^T + diag(beta gamma) dKhat
//        + (dB .* Gamma) K + (dB .* Gamma)^T K
//   dV = diag(beta) dVhat
//   dbeta_r = <V_r, dVhat_r> + gamma_r <K_r, dKhat_r> + sum_i dA_ri B_ri
//   dG_r = rowsum(dP.*P) - colsum(dP.*P) + rowsum(dB.*B) - colsum(dB.*B)
//          + gamma_r <(Q S)_r, dO_r> + beta_r gamma_r <K_r, dKhat_r>
//          - <Ktil_r, (Delta dS'^T)_r>
//          (+ sum_i <Ktil_i, (Delta dS'^T)_i> + gamma_C <S, dS'> on the last row)
//   dg = reverse in-chunk cumsum of dG.
// A ragged last chunk is padded with k = v = q = 0, beta = 0, g = 0 rows,
// which leave the state unchanged; nothing is written for padded rows.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "sf_internal.h"
#include "../../include/sf.h"

namespace sf {
namespace {

constexpr int kThreads = 256;
constexpr int kNT = 32;  // d_v columns per CTA in the state passes
constexpr int kNTp = kNT + 1;

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float* p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ size_t tok(const Args& a, int b, int t, int h) {
    return ((size_t)b * a.ld_t + t) * a.H + h;
}
// [BH][NC][d][64] chunk-transposed tile element (x, r)
__device__ __forceinline__ size_t ct(const Args& a, int bh, int c, int d, int x, int r) {
    return (((size_t)bh * a.NC + c) * d + x) * kChunk + r;
}
// [BH][NC][dv][dk] transposed chunk state element (j, i)
__device__ __forceinline__ size_t st(const Args& a, int bh, int c, int j, int i) {
    return (((size_t)bh * a.NC + c) * a.dv + j) * a.dk + i;
}

// Loads the chunk's g into Gs and turns it into the inclusive cumsum (or zeros).
__device__ void load_cumsum(const Args& a, int b, int h, int t0, int L, float* Gs) {
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        Gs[r] = (a.g && r < L) ? a.g[tok(a, b, t0 + r, h)] : 0.f;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float acc = 0.f;
        for (int r = 0; r < kChunk; ++r) {
            acc += Gs[r];
            Gs[r] = acc;
        }
    }
    __syncthreads();
}

// rows [0, 64) of a token-major [.., H, d] tensor into smem [64][ld], zero past L
template <typename TIO>
__device__ void load_rows(const Args& a, const TIO* base, int d, int b, int h, int t0, int L,
                          float* dst, int ld) {
    for (int e = threadIdx.x; e < kChunk * d; e += blockDim.x) {
        const int r = e / d, i = e - r * d;
        dst[r * ld + i] = (r < L) ? ldf(base + tok(a, b, t0 + r, h) * d + i) : 0.f;
    }
}

// chunk-transposed tile [d][64] (global, TW) -> smem [64][ld] (row r, column x)
template <typename TW>
__device__ void load_ct(const TW* src, int d, float* dst, int ld) {
    for (int e = threadIdx.x; e < d * kChunk; e += blockDim.x) {
        const int x = e >> 6, r = e & 63;
        dst[r * ld + x] = ldf(src + e);
    }
}

// ---------------------------------------------------------------- intra fwd
// Grid (NC, H, B).  Writes G and U^T; with beta also W^T.
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) intra_fwd_kernel(Args a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
    const int dk = a.dk, dv = a.dv, nc = dk + dv, ldx = nc + 1;
    extern __shared__ float sm[];
    float* Gs = sm;
    float* bs = Gs + kChunk;
    float* Ks = bs + kChunk;            // [64][dk+1]
    float* X = Ks + kChunk * (dk + 1);  // [64][dk+dv+1]
    float* As = X + kChunk * ldx;       // [64][64]

    load_cumsum(a, b, h, t0, L, Gs);
    if (threadIdx.x < kChunk) a.G[(size_t)bh * TP + t0 + threadIdx.x] = Gs[threadIdx.x];
    if (!a.beta) {  // linear attention: U = V (stored transposed like the delta rule's U)
        for (int e = threadIdx.x; e < dv * kChunk; e += blockDim.x) {
            const int j = e >> 6, r = e & 63;
            const float x = (r < L) ? ldf((const TIO*)a.v + tok(a, b, t0 + r, h) * dv + j) : 0.f;
            stf((TW*)a.Ut + ct(a, bh, c, dv, j, r), x);
        }
        return;
    }
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        bs[r] = (r < L) ? a.beta[tok(a, b, t0 + r, h)] : 0.f;
    }
    load_rows(a, (const TIO*)a.k, dk, b, h, t0, L, Ks, dk + 1);
    for (int e = threadIdx.x; e < kChunk * dv; e += blockDim.x) {
        const int r = e / dv, j = e - r * dv;
        X[r * ldx + dk + j] = (r < L) ? ldf((const TIO*)a.v + tok(a, b, t0 + r, h) * dv + j) : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float val = 0.f;
        if (i < r) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += Ks[r * (dk + 1) + d] * Ks[i * (dk + 1) + d];
            val = bs[r] * __expf(Gs[r] - Gs[i]) * dot;
        }
        As[e] = val;
    }
    for (int e = threadIdx.x; e < kChunk * nc; e += blockDim.x) {
        const int r = e / nc, col = e - r * nc;
        if (col < dk)
            X[r * ldx + col] = bs[r] * __expf(Gs[r]) * Ks[r * (dk + 1) + col];
        else
            X[r * ldx + col] *= bs[r];
    }
    __syncthreads();
    // (I + A) X = RHS by forward substitution; each thread owns whole columns.
    for (int col = threadIdx.x; col < nc; col += blockDim.x) {
        for (int r = 1; r < kChunk; ++r) {
            float acc = X[r * ldx + col];
            for (int i = 0; i < r; ++i) acc -= As[r * kChunk + i] * X[i * ldx + col];
            X[r * ldx + col] = acc;
        }
    }
    __syncthreads();
    TW* Wt = (TW*)a.Wt;
    TW* Ut = (TW*)a.Ut;
    for (int e = threadIdx.x; e < dk * kChunk; e += blockDim.x) {
        const int i = e >> 6, r = e & 63;
        stf(Wt + ct(a, bh, c, dk, i, r), X[r * ldx + i]);
    }
    for (int e = threadIdx.x; e < dv * kChunk; e += blockDim.x) {
        const int j = e >> 6, r = e & 63;
        stf(Ut + ct(a, bh, c, dv, j, r), X[r * ldx + dk + j]);
    }
}

// ---------------------------------------------------------------- state fwd
// Grid (ceil(dv / 32), H, B).  Sequential over chunks; S tile [dk][32] in smem.
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) state_fwd_kernel(Args a) {
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int dk = a.dk, dv = a.dv;
    const int n0 = blockIdx.x * kNT, nt = min(kNT, dv - n0);
    extern __shared__ float sm[];
    float* Ss = sm;                      // [dk][33]
    float* Gs = Ss + kMaxD * kNTp;       // [64]
    float* Us = Gs + kChunk;             // [64][33]  U tile, then Delta
    float* Kt = Us + kChunk * kNTp;      // [64][dk+1]
    float* Ws = Kt + kChunk * (dk + 1);  // [64][dk+1]
    TW* Sc = (TW*)a.Sc;
    TW* Dt = (TW*)a.Dt;

    for (int e = threadIdx.x; e < dk * kNT; e += blockDim.x) {
        const int i = e / kNT, n = e - i * kNT;
        Ss[i * kNTp + n] = (a.S_in && n < nt) ? a.S_in[((size_t)bh * dk + i) * dv + n0 + n] : 0.f;
    }
    for (int c = 0; c < a.NC; ++c) {
        const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * dk; e += blockDim.x) {
            const int n = e / dk, i = e - n * dk;
            stf(Sc + st(a, bh, c, n0 + n, i), Ss[i * kNTp + n]);
        }
        if (threadIdx.x < kChunk) Gs[threadIdx.x] = a.G[(size_t)bh * TP + t0 + threadIdx.x];
        __syncthreads();
        const float gC = Gs[kChunk - 1];
        for (int e = threadIdx.x; e < kChunk * dk; e += blockDim.x) {
            const int r = e / dk, i = e - r * dk;
            Kt[r * (dk + 1) + i] =
                (r < L) ? ldf((const TIO*)a.k + tok(a, b, t0 + r, h) * dk + i) * __expf(gC - Gs[r])
                        : 0.f;
        }
        if (a.beta) load_ct((const TW*)a.Wt + ct(a, bh, c, dk, 0, 0), dk, Ws, dk + 1);
        for (int e = threadIdx.x; e < kNT * kChunk; e += blockDim.x) {
            const int n = e >> 6, r = e & 63;
            float u = 0.f;
            if (n < nt) {
                if (a.beta)
                    u = ldf((const TW*)a.Ut + ct(a, bh, c, dv, n0 + n, r));
                else if (r < L)
                    u = ldf((const TIO*)a.v + tok(a, b, t0 + r, h) * dv + n0 + n);
            }
            Us[r * kNTp + n] = u;
        }
        __syncthreads();
        if (a.beta) {
            for (int e = threadIdx.x; e < kChunk * kNT; e += blockDim.x) {
                const int r = e / kNT, n = e - r * kNT;
                float acc = Us[r * kNTp + n];
                for (int i = 0; i < dk; ++i) acc -= Ws[r * (dk + 1) + i] * Ss[i * kNTp + n];
                Us[r * kNTp + n] = acc;
            }
            __syncthreads();
        }
        for (int e = threadIdx.x; e < nt * kChunk; e += blockDim.x) {
            const int n = e >> 6, r = e & 63;
            stf(Dt + ct(a, bh, c, dv, n0 + n, r), Us[r * kNTp + n]);
        }
        const float gamC = __expf(gC);
        for (int e = threadIdx.x; e < dk * kNT; e += blockDim.x) {
            const int i = e / kNT, n = e - i * kNT;
            float acc = gamC * Ss[i * kNTp + n];
            for (int r = 0; r < kChunk; ++r) acc += Kt[r * (dk + 1) + i] * Us[r * kNTp + n];
            Ss[i * kNTp + n] = acc;
        }
    }
    __syncthreads();
    if (a.S_out) {
        for (int e = threadIdx.x; e < dk * kNT; e += blockDim.x) {
            const int i = e / kNT, n = e - i * kNT;
            if (n < nt) a.S_out[((size_t)bh * dk + i) * dv + n0 + n] = Ss[i * kNTp + n];
        }
    }
}

// ---------------------------------------------------------------- output
// Grid (NC, H, B).  O = diag(gamma) Q S_c + P Delta.
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) output_kernel(Args a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
    const int dk = a.dk, dv = a.dv, ldv = dv + 1;
    extern __shared__ float sm[];
    float* Gs = sm;
    float* Qs = Gs + kChunk;             // [64][dk+1]
    float* Ks = Qs + kChunk * (dk + 1);  // [64][dk+1]
    float* Ps = Ks + kChunk * (dk + 1);  // [64][64]
    float* Ss = Ps + kChunk * kChunk;    // [dk][dv+1]
    float* Ds = Ss + dk * ldv;           // [64][dv+1]

    if (threadIdx.x < kChunk) Gs[threadIdx.x] = a.G[(size_t)bh * TP + t0 + threadIdx.x];
    load_rows(a, (const TIO*)a.q, dk, b, h, t0, L, Qs, dk + 1);
    load_rows(a, (const TIO*)a.k, dk, b, h, t0, L, Ks, dk + 1);
    for (int e = threadIdx.x; e < dv * dk; e += blockDim.x) {
        const int j = e / dk, i = e - j * dk;
        Ss[i * ldv + j] = ldf((const TW*)a.Sc + st(a, bh, c, 0, 0) + e);
    }
    load_ct((const TW*)a.Dt + ct(a, bh, c, dv, 0, 0), dv, Ds, ldv);
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float val = 0.f;
        if (i <= r) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += Qs[r * (dk + 1) + d] * Ks[i * (dk + 1) + d];
            val = __expf(Gs[r] - Gs[i]) * dot;
        }
        Ps[e] = val;
    }
    __syncthreads();
    TIO* o = (TIO*)a.o;
    for (int e = threadIdx.x; e < kChunk * dv; e += blockDim.x) {
        const int r = e / dv, n = e - r * dv;
        if (r >= L) continue;
        float qs = 0.f;
        for (int i = 0; i < dk; ++i) qs += Qs[r * (dk + 1) + i] * Ss[i * ldv + n];
        float pd = 0.f;
        for (int i = 0; i <= r; ++i) pd += Ps[r * kChunk + i] * Ds[i * ldv + n];
        stf(o + tok(a, b, t0 + r, h) * dv + n, __expf(Gs[r]) * qs + pd);
    }
}

// ---------------------------------------------------------------- dDelta pre
// Grid (NC, H, B).  dDelta^T = (P^T dO)^T, the part of dDelta that does not need dS.
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) dd_pre_kernel(Args a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
    const int dk = a.dk, dv = a.dv;
    extern __shared__ float sm[];
    float* Gs = sm;
    float* Qs = Gs + kChunk;
    float* Ks = Qs + kChunk * (dk + 1);
    float* Ps = Ks + kChunk * (dk + 1);
    float* dOs = Ps + kChunk * kChunk;  // [64][dv]

    if (threadIdx.x < kChunk) Gs[threadIdx.x] = a.G[(size_t)bh * TP + t0 + threadIdx.x];
    load_rows(a, (const TIO*)a.q, dk, b, h, t0, L, Qs, dk + 1);
    load_rows(a, (const TIO*)a.k, dk, b, h, t0, L, Ks, dk + 1);
    load_rows(a, (const TIO*)a.dO, dv, b, h, t0, L, dOs, dv);
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float val = 0.f;
        if (i <= r) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += Qs[r * (dk + 1) + d] * Ks[i * (dk + 1) + d];
            val = __expf(Gs[r] - Gs[i]) * dot;
        }
        Ps[e] = val;
    }
    __syncthreads();
    TW* dDt = (TW*)a.dDt;
    for (int e = threadIdx.x; e < dv * kChunk; e += blockDim.x) {
        const int n = e >> 6, i = e & 63;
        float acc = 0.f;
        for (int r = i; r < kChunk; ++r) acc += Ps[r * kChunk + i] * dOs[r * dv + n];
        stf(dDt + ct(a, bh, c, dv, n, i), acc);
    }
}

// ---------------------------------------------------------------- state bwd
// Grid (ceil(dv / 32), H, B).  Reverse pass over chunks carrying dS [dk][32].
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) state_bwd_kernel(Args a) {
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int dk = a.dk, dv = a.dv;
    const int n0 = blockIdx.x * kNT, nt = min(kNT, dv - n0);
    extern __shared__ float sm[];
    float* dSs = sm;                     // [dk][33]
    float* Gs = dSs + kMaxD * kNTp;      // [64]
    float* dOs = Gs + kChunk;            // [64][33]
    float* dDs = dOs + kChunk * kNTp;    // [64][33]
    float* Kt = dDs + kChunk * kNTp;     // [64][dk+1]
    float* Qg = Kt + kChunk * (dk + 1);  // [64][dk+1]
    float* Ws = Qg + kChunk * (dk + 1);  // [64][dk+1]
    TW* dSc = (TW*)a.dSc;
    TW* dDt = (TW*)a.dDt;

    for (int e = threadIdx.x; e < dk * kNT; e += blockDim.x) {
        const int i = e / kNT, n = e - i * kNT;
        dSs[i * kNTp + n] =
            (a.dS_out && n < nt) ? a.dS_out[((size_t)bh * dk + i) * dv + n0 + n] : 0.f;
    }
    for (int c = a.NC - 1; c >= 0; --c) {
        const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < nt * dk; e += blockDim.x) {
            const int n = e / dk, i = e - n * dk;
            stf(dSc + st(a, bh, c, n0 + n, i), dSs[i * kNTp + n]);
        }
        if (threadIdx.x < kChunk) Gs[threadIdx.x] = a.G[(size_t)bh * TP + t0 + threadIdx.x];
        __syncthreads();
        const float gC = Gs[kChunk - 1];
        for (int e = threadIdx.x; e < kChunk * dk; e += blockDim.x) {
            const int r = e / dk, i = e - r * dk;
            const size_t ti = tok(a, b, t0 + r, h) * dk + i;
            Kt[r * (dk + 1) + i] = (r < L) ? ldf((const TIO*)a.k + ti) * __expf(gC - Gs[r]) : 0.f;
            Qg[r * (dk + 1) + i] = (r < L) ? ldf((const TIO*)a.q + ti) * __expf(Gs[r]) : 0.f;
        }
        if (a.beta) load_ct((const TW*)a.Wt + ct(a, bh, c, dk, 0, 0), dk, Ws, dk + 1);
        for (int e = threadIdx.x; e < kNT * kChunk; e += blockDim.x) {
            const int n = e >> 6, r = e & 63;
            float x = 0.f, y = 0.f;
            if (n < nt) {
                if (r < L) x = ldf((const TIO*)a.dO + tok(a, b, t0 + r, h) * dv + n0 + n);
                y = ldf(dDt + ct(a, bh, c, dv, n0 + n, r));
            }
            dOs[r * kNTp + n] = x;
            dDs[r * kNTp + n] = y;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < kChunk * kNT; e += blockDim.x) {
            const int r = e / kNT, n = e - r * kNT;
            float acc = dDs[r * kNTp + n];
            for (int i = 0; i < dk; ++i) acc += Kt[r * (dk + 1) + i] * dSs[i * kNTp + n];
            dDs[r * kNTp + n] = acc;
            if (!a.beta && n < nt && r < L)
                stf((TIO*)a.dv_ + tok(a, b, t0 + r, h) * dv + n0 + n, acc);
        }
        __syncthreads();
        for (int e = threadIdx.x; e < nt * kChunk; e += blockDim.x) {
            const int n = e >> 6, r = e & 63;
            stf(dDt + ct(a, bh, c, dv, n0 + n, r), dDs[r * kNTp + n]);
        }
        const float gamC = __expf(gC);
        for (int e = threadIdx.x; e < dk * kNT; e += blockDim.x) {
            const int i = e / kNT, n = e - i * kNT;
            float acc = gamC * dSs[i * kNTp + n];
            for (int r = 0; r < kChunk; ++r) acc += Qg[r * (dk + 1) + i] * dOs[r * kNTp + n];
            if (a.beta)
                for (int r = 0; r < kChunk; ++r) acc -= Ws[r * (dk + 1) + i] * dDs[r * kNTp + n];
            dSs[i * kNTp + n] = acc;
        }
    }
    __syncthreads();
    if (a.dS_in) {
        for (int e = threadIdx.x; e < dk * kNT; e += blockDim.x) {
            const int i = e / kNT, n = e - i * kNT;
            if (n < nt) a.dS_in[((size_t)bh * dk + i) * dv + n0 + n] = dSs[i * kNTp + n];
        }
    }
}

// ---------------------------------------------------------------- grad delta
// Grid (NC, H, B), delta rule only.  Writes dv, dbeta and the delta-rule parts
// of dk (dKp) and dG (dGp).
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) grad_delta_kernel(Args a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
    const int dk = a.dk, dv = a.dv;
    const int ldk = dk + 1, ldv = dv + 1;
    extern __shared__ float sm[];
    float* Gs = sm;                      // 64
    float* bs = Gs + kChunk;             // 64
    float* db1 = bs + kChunk;            // 64
    float* red = db1 + kChunk;           // 64
    float* Ks = red + kChunk;            // [64][dk+1]
    float* Bs = Ks + kChunk * ldk;       // [64][64]
    float* Ts = Bs + kChunk * kChunk;    // [64][64]   T, later E = dB .* Gamma
    float* dAs = Ts + kChunk * kChunk;   // [64][64]
    float* dDs = dAs + kChunk * kChunk;  // [64][dv+1]
    float* R = dDs + kChunk * ldv;       // region: dVhat+U | S | W
    const int Rsize = max(2 * kChunk * ldv, max(dk * ldv, kChunk * ldk));
    float* dWs = R + Rsize;              // [64][dk+1]  dW, then dKhat

    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        Gs[r] = a.G[(size_t)bh * TP + t0 + r];
        bs[r] = (r < L) ? a.beta[tok(a, b, t0 + r, h)] : 0.f;
        db1[r] = 0.f;
        red[r] = 0.f;
    }
    load_rows(a, (const TIO*)a.k, dk, b, h, t0, L, Ks, ldk);
    load_ct((const TW*)a.dDt + ct(a, bh, c, dv, 0, 0), dv, dDs, ldv);
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float val = 0.f;
        if (i < r) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += Ks[r * ldk + d] * Ks[i * ldk + d];
            val = __expf(Gs[r] - Gs[i]) * dot;
        }
        Bs[e] = val;
    }
    __syncthreads();
    // T = (I + diag(beta) B)^-1, column by column (thread c owns column c).
    if (threadIdx.x < kChunk) {
        const int cc = threadIdx.x;
        for (int r = 0; r < kChunk; ++r) {
            float val;
            if (r < cc) {
                val = 0.f;
            } else if (r == cc) {
                val = 1.f;
            } else {
                float acc = 0.f;
                for (int i = cc; i < r; ++i) acc += Bs[r * kChunk + i] * Ts[i * kChunk + cc];
                val = -bs[r] * acc;
            }
            Ts[r * kChunk + cc] = val;
        }
    }
    __syncthreads();
    float* dVh = R;                  // [64][dv+1]
    float* Us = R + kChunk * ldv;    // [64][dv+1]
    load_ct((const TW*)a.Ut + ct(a, bh, c, dv, 0, 0), dv, Us, ldv);
    for (int e = threadIdx.x; e < kChunk * dv; e += blockDim.x) {
        const int r = e / dv, n = e - r * dv;
        float acc = 0.f;
        for (int i = r; i < kChunk; ++i) acc += Ts[i * kChunk + r] * dDs[i * ldv + n];
        dVh[r * ldv + n] = acc;
        if (r < L) stf((TIO*)a.dv_ + tok(a, b, t0 + r, h) * dv + n, bs[r] * acc);
    }
    __syncthreads();
    // <V_r, dVhat_r>, summed in a fixed order (one thread per row) so that results
    // do not depend on the scheduling of the threads
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        float acc = 0.f;
        if (r < L) {
            const TIO* vr = (const TIO*)a.v + tok(a, b, t0 + r, h) * dv;
            for (int n = 0; n < dv; ++n) acc += ldf(vr + n) * dVh[r * ldv + n];
        }
        db1[r] = acc;
    }
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float acc = 0.f;
        if (i < r)
            for (int n = 0; n < dv; ++n) acc += dVh[r * ldv + n] * Us[i * ldv + n];
        dAs[e] = acc;
    }
    __syncthreads();
    float* Ss = R;  // [dk][dv+1], S[i][n]
    for (int e = threadIdx.x; e < dv * dk; e += blockDim.x) {
        const int n = e / dk, i = e - n * dk;
        Ss[i * ldv + n] = ldf((const TW*)a.Sc + st(a, bh, c, 0, 0) + e);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * dk; e += blockDim.x) {
        const int r = e / dk, i = e - r * dk;
        float acc = 0.f;
        for (int n = 0; n < dv; ++n) acc += dDs[r * ldv + n] * Ss[i * ldv + n];
        dWs[r * ldk + i] = -acc;
    }
    __syncthreads();
    // dKhat = T^T dW in place: row r needs rows >= r, so go top to bottom per column.
    for (int col = threadIdx.x; col < dk; col += blockDim.x) {
        for (int r = 0; r < kChunk; ++r) {
            float acc = 0.f;
            for (int i = r; i < kChunk; ++i) acc += Ts[i * kChunk + r] * dWs[i * ldk + col];
            dWs[r * ldk + col] = acc;
        }
    }
    __syncthreads();
    float* Wsm = R;  // [64][dk+1]
    load_ct((const TW*)a.Wt + ct(a, bh, c, dk, 0, 0), dk, Wsm, ldk);
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float acc = dAs[e];
        if (i < r)
            for (int d = 0; d < dk; ++d) acc += dWs[r * ldk + d] * Wsm[i * ldk + d];
        dAs[e] = (i < r) ? -acc : 0.f;
    }
    if (threadIdx.x < kChunk) {  // <K_r, dKhat_r>, one thread per row
        const int r = threadIdx.x;
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc += Ks[r * ldk + i] * dWs[r * ldk + i];
        red[r] = acc;
    }
    __syncthreads();
    // dbeta and dG (delta part); E = dB .* Gamma into Ts.
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        const float gam = __expf(Gs[r]);
        float sAB = 0.f, rowBB = 0.f, colBB = 0.f;
        for (int i = 0; i < kChunk; ++i) {
            sAB += dAs[r * kChunk + i] * Bs[r * kChunk + i];
            rowBB += bs[r] * dAs[r * kChunk + i] * Bs[r * kChunk + i];
            colBB += bs[i] * dAs[i * kChunk + r] * Bs[i * kChunk + r];
        }
        if (r < L) a.dbeta[tok(a, b, t0 + r, h)] = db1[r] + gam * red[r] + sAB;
        a.dGp[(size_t)bh * TP + t0 + r] = rowBB - colBB + bs[r] * gam * red[r];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        Ts[e] = (i < r) ? bs[r] * dAs[e] * __expf(Gs[r] - Gs[i]) : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * dk; e += blockDim.x) {
        const int r = e / dk, d = e - r * dk;
        float acc = bs[r] * __expf(Gs[r]) * dWs[r * ldk + d];
        for (int i = 0; i < kChunk; ++i)
            acc += (Ts[r * kChunk + i] + Ts[i * kChunk + r]) * Ks[i * ldk + d];
        a.dKp[((size_t)bh * TP + t0 + r) * dk + d] = acc;
    }
}

// ---------------------------------------------------------------- grad attn
// Grid (NC, H, B).  Writes dq, dk and dg.
template <typename TIO, typename TW>
__global__ void __launch_bounds__(kThreads) grad_attn_kernel(Args a) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * a.H + h, TP = a.NC * kChunk;
    const int t0 = c * kChunk, L = min(kChunk, a.T - t0);
    const int dk = a.dk, dv = a.dv;
    const int ldk = dk + 1, ldv = dv + 1;
    constexpr int kMaxE = kChunk * kMaxD / kThreads;  // 32 outputs per thread at most
    extern __shared__ float sm[];
    float* Gs = sm;                      // 64
    float* dGs = Gs + kChunk;            // 64
    float* scal = dGs + kChunk;          // 128: <S, dS'>, -, per-warp partials, then per-row terms
    float* Qs = scal + 2 * kChunk;       // [64][dk+1]
    float* Ks = Qs + kChunk * ldk;       // [64][dk+1]
    float* dOs = Ks + kChunk * ldk;      // [64][dv+1]
    float* Ds = dOs + kChunk * ldv;      // [64][dv+1]
    float* R = Ds + kChunk * ldv;        // P, dP | S | dS'
    float* Ps = R;
    float* dPs = R + kChunk * kChunk;
    const TW* Scg = (const TW*)a.Sc + st(a, bh, c, 0, 0);
    const TW* dScg = (const TW*)a.dSc + st(a, bh, c, 0, 0);

    if (threadIdx.x < kChunk) {
        Gs[threadIdx.x] = a.G[(size_t)bh * TP + t0 + threadIdx.x];
        dGs[threadIdx.x] = 0.f;
        scal[threadIdx.x] = 0.f;
        scal[kChunk + threadIdx.x] = 0.f;
    }
    load_rows(a, (const TIO*)a.q, dk, b, h, t0, L, Qs, ldk);
    load_rows(a, (const TIO*)a.k, dk, b, h, t0, L, Ks, ldk);
    load_rows(a, (const TIO*)a.dO, dv, b, h, t0, L, dOs, ldv);
    load_ct((const TW*)a.Dt + ct(a, bh, c, dv, 0, 0), dv, Ds, ldv);
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        float p = 0.f, dp = 0.f;
        if (i <= r) {
            float dot = 0.f;
            for (int d = 0; d < dk; ++d) dot += Qs[r * ldk + d] * Ks[i * ldk + d];
            p = __expf(Gs[r] - Gs[i]) * dot;
            for (int n = 0; n < dv; ++n) dp += dOs[r * ldv + n] * Ds[i * ldv + n];
        }
        Ps[e] = p;
        dPs[e] = dp;
    }
    __syncthreads();
    if (threadIdx.x < kChunk) {
        const int r = threadIdx.x;
        float acc = 0.f;
        for (int i = 0; i < kChunk; ++i)
            acc += dPs[r * kChunk + i] * Ps[r * kChunk + i] - dPs[i * kChunk + r] * Ps[i * kChunk + r];
        dGs[r] = acc;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kChunk; e += blockDim.x) {
        const int r = e >> 6, i = e & 63;
        dPs[e] *= (i <= r) ? __expf(Gs[r] - Gs[i]) : 0.f;  // F = dP .* Gamma
    }
    __syncthreads();
    float dq[kMaxE], dkk[kMaxE];
#pragma unroll
    for (int j = 0; j < kMaxE; ++j) {
        const int e = threadIdx.x + j * kThreads;
        dq[j] = 0.f;
        dkk[j] = 0.f;
        if (e < kChunk * dk) {
            const int r = e / dk, d = e - r * dk;
            float x = 0.f, y = 0.f;
            for (int i = 0; i < kChunk; ++i) {
                x += dPs[r * kChunk + i] * Ks[i * ldk + d];
                y += dPs[i * kChunk + r] * Qs[i * ldk + d];
            }
            dq[j] = x;
            dkk[j] = y;
        }
    }
    __syncthreads();
    float* Ss = R;  // [dk][dv+1], S[i][n]
    for (int e = threadIdx.x; e < dv * dk; e += blockDim.x) {
        const int n = e / dk, i = e - n * dk;
        Ss[i * ldv + n] = ldf(Scg + e);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kMaxE; ++j) {
        const int e = threadIdx.x + j * kThreads;
        if (e < kChunk * dk) {
            const int r = e / dk, d = e - r * dk;
            float x = 0.f;
            for (int n = 0; n < dv; ++n) x += dOs[r * ldv + n] * Ss[d * ldv + n];
            dq[j] += __expf(Gs[r]) * x;
        }
    }
    // gamma_r <Q_r, (dO S^T)_r> per row, one warp per row in a fixed order of summation
    // (lanes over d, then a shuffle tree), so that results do not depend on scheduling
    for (int r = threadIdx.x >> 5; r < kChunk; r += kThreads / 32) {
        const int lane = threadIdx.x & 31;
        float acc = 0.f;
        for (int d = lane; d < dk; d += 32) {
            float x = 0.f;
            for (int n = 0; n < dv; ++n) x += dOs[r * ldv + n] * Ss[d * ldv + n];
            acc += Qs[r * ldk + d] * x;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) dGs[r] += __expf(Gs[r]) * acc;
    }
    __syncthreads();
    float* dSp = R;  // [dk][dv+1], dS'[i][n]
    float sdot = 0.f;
    for (int e = threadIdx.x; e < dv * dk; e += blockDim.x) {
        const int n = e / dk, i = e - n * dk;
        const float x = ldf(dScg + e);
        dSp[i * ldv + n] = x;
        sdot += x * ldf(Scg + e);
    }
    // <S, dS'>: per-warp shuffle trees, then warp 0's lanes in order
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, off);
    if ((threadIdx.x & 31) == 0) scal[2 + (threadIdx.x >> 5)] = sdot;
    __syncthreads();
    if (threadIdx.x == 0) {
        float acc = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) acc += scal[2 + w];
        scal[0] = acc;
    }
    const float gC = Gs[kChunk - 1];
#pragma unroll
    for (int j = 0; j < kMaxE; ++j) {
        const int e = threadIdx.x + j * kThreads;
        if (e < kChunk * dk) {
            const int r = e / dk, d = e - r * dk;
            float x = 0.f;
            for (int n = 0; n < dv; ++n) x += Ds[r * ldv + n] * dSp[d * ldv + n];
            dkk[j] += __expf(gC - Gs[r]) * x;
        }
    }
    // e^{G_C - G_r} <K_r, (Delta dS'^T)_r> per row (one warp per row, fixed order), kept in
    // red[r] for its last-row sum
    float* red = scal + 2 + kThreads / 32;
    for (int r = threadIdx.x >> 5; r < kChunk; r += kThreads / 32) {
        const int lane = threadIdx.x & 31;
        float acc = 0.f;
        for (int d = lane; d < dk; d += 32) {
            float x = 0.f;
            for (int n = 0; n < dv; ++n) x += Ds[r * ldv + n] * dSp[d * ldv + n];
            acc += Ks[r * ldk + d] * x;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            const float t = __expf(gC - Gs[r]) * acc;
            dGs[r] -= t;
            red[r] = t;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float lastsum = 0.f;
        for (int r = 0; r < kChunk; ++r) lastsum += red[r];
        dGs[kChunk - 1] += lastsum + __expf(gC) * scal[0];
        float acc = 0.f;
        for (int r = kChunk - 1; r >= 0; --r) {
            acc += dGs[r] + (a.beta ? a.dGp[(size_t)bh * TP + t0 + r] : 0.f);
            dGs[r] = acc;
        }
    }
    __syncthreads();
    if (a.g && threadIdx.x < L) a.dg[tok(a, b, t0 + threadIdx.x, h)] = dGs[threadIdx.x];
#pragma unroll
    for (int j = 0; j < kMaxE; ++j) {
        const int e = threadIdx.x + j * kThreads;
        if (e < kChunk * dk) {
            const int r = e / dk, d = e - r * dk;
            if (r < L) {
                const size_t ti = tok(a, b, t0 + r, h) * dk + d;
                float kval = dkk[j];
                if (a.beta) kval += a.dKp[((size_t)bh * TP + t0 + r) * dk + d];
                stf((TIO*)a.dq + ti, dq[j]);
                stf((TIO*)a.dk_ + ti, kval);
            }
        }
    }
}

// ---------------------------------------------------------------- launchers
size_t smem_intra(const Args& a) {
    return sizeof(float) *
           (2 * kChunk + kChunk * (a.dk + 1) + kChunk * (a.dk + a.dv + 1) + kChunk * kChunk);
}
size_t smem_state_fwd(const Args& a) {
    return sizeof(float) * (kMaxD * kNTp + kChunk + kChunk * kNTp + 2 * kChunk * (a.dk + 1));
}
size_t smem_output(const Args& a) {
    return sizeof(float) * (kChunk + 2 * kChunk * (a.dk + 1) + kChunk * kChunk +
                            a.dk * (a.dv + 1) + kChunk * (a.dv + 1));
}
size_t smem_dd_pre(const Args& a) {
    return sizeof(float) * (kChunk + 2 * kChunk * (a.dk + 1) + kChunk * kChunk + kChunk * a.dv);
}
size_t smem_state_bwd(const Args& a) {
    return sizeof(float) * (kMaxD * kNTp + kChunk + 2 * kChunk * kNTp + 3 * kChunk * (a.dk + 1));
}
size_t smem_grad_delta(const Args& a) {
    const int ldk = a.dk + 1, ldv = a.dv + 1;
    const int Rsize = std::max(2 * kChunk * ldv, std::max(a.dk * ldv, kChunk * ldk));
    return sizeof(float) *
           (4 * kChunk + kChunk * ldk + 3 * kChunk * kChunk + kChunk * ldv + Rsize + kChunk * ldk);
}
size_t smem_grad_attn(const Args& a) {
    const int ldk = a.dk + 1, ldv = a.dv + 1;
    const int Rsize = std::max(2 * kChunk * kChunk, a.dk * ldv);
    return sizeof(float) * (4 * kChunk + 2 * kChunk * ldk + 2 * kChunk * ldv + Rsize);
}

template <typename K>
cudaError_t launch(K kernel, int kind, dim3 grid, size_t smem, const Args& a, cudaStream_t s) {
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    timing_begin(kind, s);
    kernel<<<grid, kThreads, smem, s>>>(a);
    e = cudaGetLastError();
    timing_end(kind, s);
    return e;
}

dim3 chunk_grid(const Args& a) { return dim3(a.NC, a.H, a.B); }
dim3 tile_grid(const Args& a) { return dim3((a.dv + kNT - 1) / kNT, a.H, a.B); }

}  // namespace

// bf16 I/O keeps bf16 intermediates; fp32 I/O keeps fp32 intermediates.
#define SF_DISPATCH(KERNEL, KIND, GRID, SMEM)                                                   \
    (a.dtype == SF_BF16 ? launch(KERNEL<__nv_bfloat16, __nv_bfloat16>, KIND, GRID, SMEM, a, s)   \
                        : launch(KERNEL<float, float>, KIND, GRID, SMEM, a, s))

cudaError_t launch_intra_fwd(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(intra_fwd_kernel, KK_INTRA_FWD, chunk_grid(a), smem_intra(a));
}
cudaError_t launch_state_fwd(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(state_fwd_kernel, KK_STATE_FWD, tile_grid(a), smem_state_fwd(a));
}
cudaError_t launch_output(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(output_kernel, KK_OUTPUT, chunk_grid(a), smem_output(a));
}
cudaError_t launch_dd_pre(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(dd_pre_kernel, KK_DD_PRE, chunk_grid(a), smem_dd_pre(a));
}
cudaError_t launch_state_bwd(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(state_bwd_kernel, KK_STATE_BWD, tile_grid(a), smem_state_bwd(a));
}
cudaError_t launch_grad_delta(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(grad_delta_kernel, KK_GRAD_DELTA, chunk_grid(a), smem_grad_delta(a));
}
cudaError_t launch_grad_attn(const Args& a, cudaStream_t s) {
    return SF_DISPATCH(grad_attn_kernel, KK_GRAD_ATTN, chunk_grid(a), smem_grad_attn(a));
}

}  // namespace sf
