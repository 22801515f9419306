// Tensor-core (tcgen05 / TMEM / TMA) engine of the Newton-Schulz GEMM phases.
#pragma once

#include <vector>

#include "internal.h"

namespace mfsdp {

// true when the bf16 phases run on the tcgen05 engine of this build
bool tc_available();

// grouped tile tables of the engine (symmetric phases, general phases)
void tc_build_tiles(const std::vector<MatDev>& mats, std::vector<TileDev>& sym, std::vector<TileDev>& gen);

cudaError_t launch_gemm_tc(Phase ph, const MatDev* d_mats, int32_t nmats, const TileDev* d_tiles,
                           int32_t ntiles, int32_t iter, const StepScalars& sc, const float* s,
                           cudaStream_t st);

}  // namespace mfsdp
