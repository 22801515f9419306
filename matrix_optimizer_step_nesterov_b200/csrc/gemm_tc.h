// Tensor-core (tcgen05 / TMEM / TMA) engine of the Newton-Schulz GEMM phases.
#pragma once

#include <cstddef>
#include <vector>

#include "internal.h"

namespace mfsdp {

// bytes of the per-matrix TMA descriptor table (64-byte aligned entries)
size_t tc_maps_bytes(size_t nmats);

// encode every matrix's TMA descriptors (needs the workspace pointers filled in)
bool tc_encode_maps(const std::vector<MatDev>& mats, void* host_out);

// CTA-pair clusters of the engine's persistent grid that fit on the current
// device at once (computed once per device; 0 on a CUDA error)
int tc_max_clusters();

// clusters a phase over ntiles tiles launches
int tc_launch_clusters(int ntiles, int max_clusters);

// grouped tile tables of the engine: GRAM and POLY (upper-triangle tiles) and
// APPLY (all tiles), each sorted longest-K first, then partitioned over the
// tc_launch_clusters(size, max_clusters) clusters of its launch by a
// longest-processing-time assignment; *_seg get the clusters + 1 offsets of
// the clusters' segments
void tc_build_tiles(const std::vector<MatDev>& mats, int max_clusters, std::vector<TileDev>& gram,
                    std::vector<TileDev>& poly, std::vector<TileDev>& gen, std::vector<int32_t>& gram_seg,
                    std::vector<int32_t>& poly_seg, std::vector<int32_t>& gen_seg);

// output tile edges of the engine's tiles (rows of a tile, columns of a tile)
int tc_tile_rows();
int tc_tile_cols();

// one CTA whose single wait runs out after limit_ns (failure-detection test)
cudaError_t launch_bounded_wait_selftest(unsigned long long limit_ns, cudaStream_t st);

// one phase over the tiles of d_tiles, partitioned by d_seg over `clusters` clusters
// ring: the stages of the operand ring the launch cycles through (tc_ring_depth)
cudaError_t launch_gemm_tc(Phase ph, const MatDev* d_mats, const void* d_maps, int32_t nmats,
                           const TileDev* d_tiles, const int32_t* d_seg, int32_t clusters, int32_t iter, int32_t ring,
                           const StepScalars& sc, const float* s, cudaStream_t st);

// the ring depth for a phase launch of `tiles` tiles over `clusters` clusters on
// these matrices: 4 for a long launch whose operands fit in the device's L2, else
// all the stages the kernel allocates
int tc_ring_depth(Phase ph, const std::vector<MatDev>& mats, int64_t tiles, int32_t clusters);

}  // namespace mfsdp
