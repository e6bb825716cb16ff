// Failure detection without a fault: one thread waits, through the library's
// bounded mbarrier wait, on a barrier that nothing arrives on.  The wait must
// give up after its cycle limit and the kernel must return normally, writing
// the error code the library's kernels write, so that the host reads a status
// and the context stays usable.
#include "../../chunked_linear_recurrence_chunkwise_b200/csrc/tc_common.cuh"

using namespace sf::tc;

__global__ void wait_probe_kernel(int* err, long long* cycles, int abort_early) {
    __shared__ uint64_t bar;
    __shared__ int s_abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const long long t0 = clock64();
        bool ok;
        if (abort_early) {
            s_abort = 1;  // another thread of the CTA has already given up
            ok = mbar_wait_or_abort(&bar, 0, &s_abort);
        } else {
            ok = mbar_wait(&bar, 0);  // nothing ever arrives
        }
        *cycles = clock64() - t0;
        if (!ok) atomicExch(err, kErrTimeoutMma);
    }
}

__global__ void add_one_kernel(int* x) { atomicAdd(x, 1); }

extern "C" int wait_probe(void* err, void* cycles, int abort_early, void* stream) {
    wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((int*)err, (long long*)cycles, abort_early);
    return (int)cudaGetLastError();
}

extern "C" int add_one(void* x, void* stream) {
    add_one_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((int*)x);
    return (int)cudaGetLastError();
}

extern "C" long long wait_limit_cycles() { return kWaitCycles; }
