// Device-side error word.  Kernels that contain a bounded wait get its
// address as a kernel argument and set it (atomicOr of a reason code) when a
// wait gives up, then return; the host reads and clears it with
// gdn_device_status().
#include <cuda_runtime.h>

#include <atomic>

#include "../../include/gdn.h"
#include "gdn_internal.h"

namespace gdn {

__device__ int g_device_error = 0;

static std::atomic<long long> g_launches{0};

void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

cudaError_t device_error_word(int **ptr)
{
    // A device symbol's address is per device: look it up with the
    // caller's device current, every time (cheap), never cache across devices.
    return cudaGetSymbolAddress(reinterpret_cast<void **>(ptr), g_device_error);
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, int *err)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    int *p = nullptr;
    e = device_error_word(&p);
    if (e != cudaSuccess) return e;
    e = cudaMemcpy(err, p, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return e;
    if (*err) {
        const int zero = 0;
        e = cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    }
    return e;
}

}  // namespace gdn

extern "C" long long gdn_kernel_launches(void)
{
    return gdn::g_launches.load(std::memory_order_relaxed);
}
