// nf4lora_check_bounded_wait: a self-check of the give-up path that every
// kernel of the library shares.
//
// Each wait of a kernel on a shared-memory barrier is bounded; a wait that
// runs out sets the CTA's abort flag and the device status word, every role
// leaves its loop, the copies still in flight are drained, tensor memory is
// freed, and the kernel returns.  In a healthy run no wait ever runs out, so
// this kernel makes one run out on purpose, in a form that cannot fault or
// hang: it holds tensor memory and has a bulk copy in flight, exactly as a
// layer kernel does, and then waits, with a short caller-given limit, on a
// barrier that nothing ever arrives on.  Every thread of the CTA waits; the
// one whose limit runs out first raises the abort flag and the others leave
// on it.  The host then reads NF4_ERR_TIMEOUT from nf4lora_device_status().
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "nf4lora.h"
#include "trace.h"

namespace nf4lora {

namespace {

constexpr uint32_t kCheckCopyBytes = 1024;
constexpr uint32_t kCheckTmemCols = 32;

// The source of the bulk copy kept in flight (never read back).
__device__ __align__(128) uint8_t g_check_src[kCheckCopyBytes];

__global__ void __launch_bounds__(128) k_bounded_wait_check(uint64_t limit_ns) {
    __shared__ __align__(128) uint8_t buf[kCheckCopyBytes];
    __shared__ uint64_t bar_copy, bar_never;
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        mbar_init(&bar_copy, 1);
        mbar_init(&bar_never, 1);  // nothing arrives on it
        s_abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (warp == 1) {
        tmem_alloc(&tmem_base, kCheckTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_copy, kCheckCopyBytes);
        bulk_load(buf, g_check_src, kCheckCopyBytes, &bar_copy);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    volatile int* abort_flag = &s_abort;
    mbar_wait_for(&bar_never, 0, abort_flag, limit_ns);
    __syncthreads();
    if (tid == 0) mbar_drain(&bar_copy, 0);  // the copy lands before the CTA exits
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kCheckTmemCols);
    }
}

}  // namespace

}  // namespace nf4lora

extern "C" int nf4lora_check_bounded_wait(int64_t limit_ns, void* stream) {
    using namespace nf4lora;
    if (limit_ns < 100000 || limit_ns > 1000000000) return NF4_ERR_INVALID_ARG;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return NF4_ERR_CUDA;
    if (major != 10) return NF4_ERR_DEVICE;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    TraceScope trace("bounded_wait_check", st);
    k_bounded_wait_check<<<1, 128, 0, st>>>(static_cast<uint64_t>(limit_ns));
    return cudaGetLastError() == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}
