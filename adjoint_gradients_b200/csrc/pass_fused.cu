// pass_fused.cu -- instances of the pass kernel with fused SU(2) rotations:
// CNOT entanglers (the one-layer schedules of the gather path, and the fused
// schedule whose passes apply each layer's map as a permutation of the tile).
#include "pass_kernel.cuh"

#define QML_FUSED_INSTANCES(X)                                                                   \
  X(false, 0, 0, 0) X(true, 0, 0, 0) X(false, 1, 0, 0) X(true, 1, 0, 0) X(false, 1, 1, 0)          \
  X(true, 1, 1, 0) X(false, 2, 0, 0) X(true, 2, 0, 0) X(false, 2, 1, 0) X(true, 2, 1, 0)

QML_DEFINE_PASS_UNIT(pass_fused, QML_FUSED_INSTANCES)

namespace qml {

// Resident blocks per SM of a pass kernel (every form shares the register
// and shared-memory budget of its mode; the fused-form instances stand in).
cudaError_t pass_occupancy(bool backward, int mode, size_t smem, int* blocks_per_sm) {
  if (backward)
    return mode == 0   ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<true, 0, 0, 0>, kThreads, smem)
           : mode == 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<true, 1, 1, 0>, kThreads, smem)
                       : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<true, 2, 1, 0>, kThreads, smem);
  return mode == 0   ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<false, 0, 0, 0>, kThreads, smem)
         : mode == 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<false, 1, 1, 0>, kThreads, smem)
                     : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<false, 2, 1, 0>, kThreads, smem);
}

}  // namespace qml
