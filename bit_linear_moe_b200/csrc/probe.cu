// A kernel whose producer never delivers, for checking the bounded waits
// without faulting or hanging the GPU (Ignis README, "Credits": a per-request
// error boundary).  One CTA initialises an mbarrier that nothing arrives on and
// waits for it with the same bounded wait every TMA/tensor-core kernel of the
// library uses; nothing is in flight while it waits.  The wait runs out after
// `limit_cycles`, records NVFP4_ERR_DEVICE_TIMEOUT in the library status word
// (read by nvfp4_read_device_status) and the kernel returns normally, so the
// context stays usable.
#include "internal.h"
#include "tma.cuh"

namespace nvfp4 {

__global__ void __launch_bounds__(32) wait_timeout_probe_kernel(int* status, long long limit_cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, status, limit_cycles);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_debug_wait_timeout(int64_t limit_cycles, void* stream) {
    if (limit_cycles < 1 || limit_cycles > kWaitCycles) return NVFP4_ERR_SHAPE;
    int major = 0, minor = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
        minor != 0)
        return NVFP4_ERR_ARCH;
    int* status = device_status_ptr();
    if (!status) return NVFP4_ERR_LAUNCH;
    wait_timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, (long long)limit_cycles);
    return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_LAUNCH;
}
