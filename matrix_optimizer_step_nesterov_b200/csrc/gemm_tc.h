// Tensor-core (tcgen05 / TMEM / TMA) engine of the Newton-Schulz GEMM phases.
#pragma once

#include <cstddef>
#include <vector>

#include "internal.h"

namespace mfsdp {

// true when the bf16 phases run on the tcgen05 engine (compiled for sm_100a)
bool tc_available();

// bytes of the per-matrix TMA descriptor table (64-byte aligned entries)
size_t tc_maps_bytes(size_t nmats);

// encode every matrix's TMA descriptors (needs the workspace pointers filled in)
bool tc_encode_maps(const std::vector<MatDev>& mats, void* host_out);

// grouped tile tables of the engine: GRAM and POLY (upper-triangle tiles, each
// ordered longest-K first) and APPLY (all tiles)
void tc_build_tiles(const std::vector<MatDev>& mats, std::vector<TileDev>& gram, std::vector<TileDev>& poly,
                    std::vector<TileDev>& gen);

// output tile edges of the engine's tiles (rows of a tile, columns of a tile)
int tc_tile_rows();
int tc_tile_cols();

// one CTA whose single wait runs out after limit_ns (failure-detection test)
cudaError_t launch_bounded_wait_selftest(unsigned long long limit_ns, cudaStream_t st);

cudaError_t launch_gemm_tc(Phase ph, const MatDev* d_mats, const void* d_maps, int32_t nmats,
                           const TileDev* d_tiles, int32_t ntiles, int32_t iter, const StepScalars& sc,
                           const float* s, cudaStream_t st);

}  // namespace mfsdp
