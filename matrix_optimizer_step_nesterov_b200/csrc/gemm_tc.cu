// tcgen05 engine: not yet enabled in this build; the bf16 phases run on the SIMT engine.
#include "gemm_tc.h"

namespace mfsdp {

bool tc_available() { return false; }

void tc_build_tiles(const std::vector<MatDev>&, std::vector<TileDev>&, std::vector<TileDev>&) {}

cudaError_t launch_gemm_tc(Phase, const MatDev*, int32_t, const TileDev*, int32_t, int32_t,
                           const StepScalars&, const float*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace mfsdp
