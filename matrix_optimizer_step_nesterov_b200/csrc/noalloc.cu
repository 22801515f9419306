// mfsdp_muon_step_noalloc: the grouped Muon step for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain a workspace at step time: plugins and
// inference or training hosts that own every byte of device memory through
// their own pre-planned pools and forbid driver allocations, and
// latency-critical loops that must not enter an allocator, which may
// synchronise the device.  This entry point takes the step's scratch from a
// fixed array compiled into the library instead of from the caller.
//
// The scratch is kNoAllocScratchBytes (64 MiB) of device memory per GPU that
// loads the library, held until the process exits.  It fits small owner
// lists: the bf16 step needs about 8 B per element of each matrix plus 8 B
// per element of its r x r Gram matrix (r = the shorter side), e.g. one
// 2048 x 1024 or several 512 x 512 matrices.  Larger lists are rejected with
// MFSDP_ERR_WORKSPACE_TOO_SMALL before any GPU work.
//
// Every call shares the one array, so every call re-uploads its own
// descriptor and tile tables into it (enqueued on the caller's stream before
// the step's kernels) rather than trusting what an earlier call left there.
#include "../../include/mfsdp.h"
#include "internal.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

// The step's scratch: one array per device, shared by every call of this
// entry point.  In host code this name is only a host-side stand-in; the
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of this device's scratch, resolved once per device with the
// device current.  Returns MFSDP_OK or MFSDP_ERR_CUDA.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MFSDP_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return MFSDP_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return MFSDP_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MFSDP_OK;
}

}  // namespace

extern "C" int mfsdp_muon_step_noalloc(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                                       void* stream) {
    // host-only validation and sizing first: nothing reaches the GPU on error
    size_t need = 0;
    int st = mfsdp_muon_workspace_size(mats, n, hp, &need);
    if (st != MFSDP_OK) return st;
    if (need > kNoAllocScratchBytes) return MFSDP_ERR_WORKSPACE_TOO_SMALL;
    if (need == 0) return MFSDP_OK;   // empty list or only zero-size matrices: no-op
    void* scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != MFSDP_OK) return st;
    // The step writes every scratch byte it later reads (tables, partial sums,
    // X, A and B buffers), so the previous call's contents need no clearing;
    // the tables are uploaded on every call, whatever the previous call left.
    return mfsdp::muon_step_impl(mats, nullptr, n, hp, scratch, kNoAllocScratchBytes, stream,
                                 /*always_upload=*/true);
}
