// One-tile GEMM through the library's UMMA helpers, used by the GPU tests to
// check the shared-memory descriptor encodings (K-major / MN-major, 128-byte
// swizzle), the TMEM accumulator lane layout for M = 64 and M = 128, and the
// layout of an A operand held in tensor memory (a_tmem).
// C[M][N] = A[M][K] * B[K][N]; A, B bf16 row-major in global memory, C fp32.
#include "../../chunked_linear_recurrence_chunkwise_b200/csrc/tc_common.cuh"

using namespace sf::tc;

__global__ void __launch_bounds__(128, 1)
    umma_probe_kernel(const __nv_bfloat16* A, const __nv_bfloat16* B, float* C, int M, int N,
                      int K, int a_mn, int b_mn, int neg_a, int lane16, int restore, int a_tmem,
                      int* err) {
    extern __shared__ uint8_t raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
    uint8_t* As = sm;                 // up to 128 x 128 bf16 = 32 KB
    uint8_t* Bs = sm + 32768;         // up to 128 x 128 bf16 = 32 KB
    uint64_t* bar = (uint64_t*)(sm + 65536);
    uint32_t* s_tmem = (uint32_t*)(sm + 65536 + 8);
    const int tid = threadIdx.x, warp = tid >> 5;
    // A element (m, k)
    for (int e = tid; e < M * K; e += blockDim.x) {
        const int m = e / K, k = e % K;
        uint32_t off;
        if (!a_mn) off = (k / 64) * (M * 128) + sw128(m, (k % 64) / 8) + (k % 8) * 2;
        else       off = (m / 64) * (K * 128) + sw128(k, (m % 64) / 8) + (m % 8) * 2;
        *(__nv_bfloat16*)(As + off) = A[e];
    }
    // B element (k, n)
    for (int e = tid; e < K * N; e += blockDim.x) {
        const int k = e / N, n = e % N;
        uint32_t off;
        if (!b_mn) off = (k / 64) * (N * 128) + sw128(n, (k % 64) / 8) + (k % 8) * 2;
        else       off = (n / 64) * (K * 128) + sw128(k, (n % 64) / 8) + (n % 8) * 2;
        *(__nv_bfloat16*)(Bs + off) = B[e];
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(s_tmem, 256);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // a_tmem (M = 128): row m = 32 warp + lane of A into lane m, columns [128, 128 + K / 2),
    // two bf16 per column, the lower K index in the low half
    if (a_tmem) {
        const int m = warp * 32 + (tid & 31);
        for (int k0 = 0; k0 < K; k0 += 16) {
            uint32_t w[8];
            for (int q = 0; q < 8; ++q) {
                const __nv_bfloat16 lo = A[m * K + k0 + 2 * q], hi = A[m * K + k0 + 2 * q + 1];
                w[q] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
            }
            tmem_st8u(taddr(tmem, warp * 32, 128 + k0 / 2), w);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    // lane16: an M = 64 accumulator placed at TMEM lane offset 16 (lanes 16-31 of each quadrant)
    const uint32_t tD = tmem + ((lane16 ? 16u : 0u) << 16);
    const uint32_t id = idesc_bf16(M, N, a_mn, b_mn, neg_a != 0);
    const uint32_t a0 = smem_u32(As), b0 = smem_u32(Bs);
    auto issue = [&](uint32_t acc0) {
        for (int ks = 0; ks < K / 16; ++ks) {
            const uint64_t ad = a_mn ? sdesc(a0 + ks * 2048, K * 128, 1024)
                                     : sdesc(a0 + (ks / 4) * (M * 128) + (ks % 4) * 32, 16, 1024);
            const uint64_t bd = b_mn ? sdesc(b0 + ks * 2048, K * 128, 1024)
                                     : sdesc(b0 + (ks / 4) * (N * 128) + (ks % 4) * 32, 16, 1024);
            if (a_tmem) mma_bf16_ts(tD, tmem + 128 + 8 * ks, bd, id, (ks > 0) || acc0);
            else mma_bf16(tD, ad, bd, id, (ks > 0) || acc0);
        }
    };
    if (tid == 0) {
        issue(0);
        mma_commit(bar);
        if (!mbar_wait(bar, 0)) atomicExch(err, 1);
    }
    __syncthreads();
    tc_fence_after();
    const int lane = tid & 31;
    // restore: read the accumulator, double it, store it back, accumulate A*B once more (3 A*B)
    if (restore) {
        for (int n0 = 0; n0 < N; n0 += 32) {
            float v[32];
            tmem_ld32(taddr(tmem, warp * 32, n0), v);
            tmem_ld_wait();
            for (int q = 0; q < 32; ++q) v[q] *= 2.f;
            tmem_st32(taddr(tmem, warp * 32, n0), v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            issue(1);
            mma_commit(bar);
            if (!mbar_wait(bar, 1)) atomicExch(err, 1);
        }
        __syncthreads();
        tc_fence_after();
    }
    for (int n0 = 0; n0 < N; n0 += 32) {
        float v[32];
        tmem_ld32(taddr(tmem, warp * 32, n0), v);
        tmem_ld_wait();
        int row = -1;
        if (M == 128) row = warp * 32 + lane;
        else if (!lane16 && lane < 16) row = warp * 16 + lane;
        else if (lane16 && lane >= 16) row = warp * 16 + lane - 16;
        if (row >= 0)
            for (int q = 0; q < 32; ++q) C[row * N + n0 + q] = v[q];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

extern "C" int umma_probe(const void* A, const void* B, void* C, int M, int N, int K, int a_mn,
                          int b_mn, int neg_a, int lane16, int restore, int a_tmem, void* err,
                          void* stream) {
    if (!(M == 64 || M == 128) || N % 32 || N > 256 || K % 64 || K > 128 || (lane16 && M != 64) ||
        (a_tmem && M != 128) || K * N * 2 > 32768)
        return 1;
    const int smem = 65536 + 64 + 1024;
    cudaFuncSetAttribute(umma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    umma_probe_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, (float*)C, M, N, K, a_mn, b_mn,
        neg_a, lane16, restore, a_tmem, (int*)err);
    return (int)cudaGetLastError();
}
