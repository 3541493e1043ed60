// wait_timeout.cu -- the kernels' bounded wait, made to run out on purpose
// without faulting: one thread waits on a shared-memory barrier that nothing
// ever arrives on, through the same mbar_wait the kernels use (common.cuh).
// After its time limit the wait gives up, sets SPATTN_DEV_WAIT_TIMEOUT in the
// device status word and returns false; the kernel then ends normally.  The
// host checks the launch succeeded, the status bit, the wait's result, and
// that the context still runs a kernel afterwards.  Prints one line and
// exits 0 when all hold, 1 otherwise.
#include <cstdio>

#include "common.cuh"

using namespace spattn;

__global__ void wait_for_nobody(int *result, unsigned long long *elapsed_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = global_ns();
        const bool ok = mbar_wait(&bar, 0);   // the phase never completes
        *elapsed_ns = global_ns() - t0;
        *result = ok ? 1 : 0;
    }
}

__global__ void add_one(int *x) { x[threadIdx.x] += 1; }

int main() {
    int *d = nullptr;
    unsigned long long *t = nullptr;
    if (cudaMalloc(&d, 64 * sizeof(int)) != cudaSuccess || cudaMalloc(&t, sizeof(*t)) != cudaSuccess) {
        std::printf("FAIL allocation\n");
        return 1;
    }
    cudaMemset(d, 0, 64 * sizeof(int));
    cudaMemset(d, 0xff, sizeof(int));   // result slot: -1 until the kernel writes it
    const int32_t zero = 0;
    cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    wait_for_nobody<<<1, 32>>>(d, t);
    const cudaError_t e1 = cudaDeviceSynchronize();
    int32_t status = 0;
    int result = -1;
    unsigned long long ns = 0;
    cudaMemcpyFromSymbol(&status, g_status, sizeof(status));
    cudaMemcpy(&result, d, sizeof(int), cudaMemcpyDeviceToHost);
    cudaMemcpy(&ns, t, sizeof(ns), cudaMemcpyDeviceToHost);
    // the context is still usable: a plain kernel runs and its result comes back
    add_one<<<1, 64>>>(d);
    const cudaError_t e2 = cudaDeviceSynchronize();
    int after = 0;
    cudaMemcpy(&after, d + 1, sizeof(int), cudaMemcpyDeviceToHost);
    const bool pass = e1 == cudaSuccess && e2 == cudaSuccess && (status & SPATTN_DEV_WAIT_TIMEOUT) && result == 0 &&
                      ns >= kWaitLimitNs && after == 1;
    std::printf("%s launch=%s status=%#x wait_result=%d waited_ms=%.1f after=%d\n", pass ? "ok" : "FAIL",
                cudaGetErrorString(e1), (unsigned)status, result, ns / 1e6, after);
    cudaFree(d);
    cudaFree(t);
    return pass ? 0 : 1;
}
