// Device status word: kernels record the first error they detect here (an
// out-of-range index they skipped, a bounded wait that gave up) instead of
// trapping, so the CUDA context stays usable and the host can read the code.
#include "internal.h"

#include <mutex>

namespace mfsdp {
namespace {
__device__ int32_t g_status_word = 0;

constexpr int kMaxDevices = 64;
int32_t* g_status_addr[kMaxDevices] = {nullptr};
std::mutex g_status_mu;
}  // namespace

int32_t* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_status_addr[dev] = static_cast<int32_t*>(p);
    }
    return g_status_addr[dev];
}

}  // namespace mfsdp
