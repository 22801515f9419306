// Per-kernel-class CUDA-event timing of the library's own launches, and an
// NVTX range named after the kernel class around every launch (free unless a
// profiler is attached).
#include "../../include/mfsdp.h"
#include "internal.h"

#include <nvtx3/nvToolsExt.h>

#include <mutex>
#include <vector>

namespace mfsdp {
namespace {

struct Slot {
    int cls;
    cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_active = false;
int g_capacity = 0;
std::vector<Slot> g_slots;   // created lazily, reused across sessions
int g_used = 0;

}  // namespace

const char* const kRangeNames[MFSDP_KCLASS_COUNT] = {
    "mfsdp:momentum", "mfsdp:norm", "mfsdp:gram", "mfsdp:poly",
    "mfsdp:apply", "mfsdp:write", "mfsdp:adamw", "mfsdp:final",
};

int prof_before(int cls, cudaStream_t s) {
    nvtxRangePushA((cls >= 0 && cls < MFSDP_KCLASS_COUNT) ? kRangeNames[cls] : "mfsdp");
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_active || g_used >= g_capacity) return -1;
    Slot& sl = g_slots[g_used];
    if (cudaEventRecord(sl.start, s) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    sl.cls = cls;
    return g_used++;
}

void prof_after(int slot, cudaStream_t s) {
    nvtxRangePop();
    if (slot < 0) return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (slot < static_cast<int>(g_slots.size()) && cudaEventRecord(g_slots[slot].stop, s) != cudaSuccess) {
        cudaGetLastError();
        g_slots[slot].cls = -1;
    }
}

}  // namespace mfsdp

using namespace mfsdp;

extern "C" int mfsdp_profile_begin(int32_t max_launches) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_active || max_launches < 1) return MFSDP_ERR_INVALID_ARG;
    while (static_cast<int>(g_slots.size()) < max_launches) {
        Slot sl{-1, nullptr, nullptr};
        if (cudaEventCreate(&sl.start) != cudaSuccess || cudaEventCreate(&sl.stop) != cudaSuccess) {
            cudaGetLastError();
            return MFSDP_ERR_CUDA;
        }
        g_slots.push_back(sl);
    }
    g_capacity = max_launches;
    g_used = 0;
    g_active = true;
    return MFSDP_OK;
}

extern "C" int mfsdp_profile_end(mfsdp_profile* out) {
    if (!out) return MFSDP_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_active) return MFSDP_ERR_INVALID_ARG;
    g_active = false;
    for (int k = 0; k < MFSDP_KCLASS_COUNT; ++k) {
        out->launches[k] = 0;
        out->ms[k] = 0.0;
    }
    int status = MFSDP_OK;
    for (int i = 0; i < g_used; ++i) {
        Slot& sl = g_slots[i];
        if (sl.cls < 0 || sl.cls >= MFSDP_KCLASS_COUNT) continue;
        float ms = 0.f;
        if (cudaEventSynchronize(sl.stop) != cudaSuccess || cudaEventElapsedTime(&ms, sl.start, sl.stop) != cudaSuccess) {
            cudaGetLastError();
            status = MFSDP_ERR_CUDA;
            continue;
        }
        out->launches[sl.cls] += 1;
        out->ms[sl.cls] += ms;
    }
    g_used = 0;
    return status;
}
