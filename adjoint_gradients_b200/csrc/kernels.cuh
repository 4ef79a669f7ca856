// kernels.cuh -- launch wrappers of the sm_100a kernels (host-callable).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "device_plan.h"

namespace qml {

// Arguments of one pass launch (forward or backward).
struct PassArgs {
  const DevPass* passes;
  int pass_idx;
  int n, B, U;           // qubits, samples, batch units (forward: ceil(B/2); backward: B)
  long long N;           // 2^n
  int n_tiles;           // tiles in this pass
  float2* buf0;          // forward: psi; backward: psi (plane 0)
  float2* buf1;          // backward: lambda (plane 1)
  float2* dummy;         // forward: partner plane of the last unit when B is odd
  const float4* coef;    // [L*n][4] broadcast gate coefficients (forward U, or U^dagger)
  const float2* enc;     // forward: [U][n][2] (cos, sin)(x/2) pairs
  const float* g;        // backward: dL/dE [B]
  void* ckpt;            // checkpoint slots
  int storage;           // 0 fp32, 1 bf16
  int bmax;              // samples per checkpoint slot (slot stride)
  float* partials;       // backward gradient partials
  unsigned* status;
};

size_t pass_smem_bytes(int max_slots);

// `slow`: some register bit indexes a batch unit (only when n < 5); the
// generic per-position code then replaces the single-unit fast path.
cudaError_t launch_pass(bool backward, bool slow, const PassArgs& a, int grid, size_t smem, cudaStream_t s);
cudaError_t set_pass_smem_attr(size_t smem);
cudaError_t pass_occupancy(bool backward, bool slow, size_t smem, int* blocks_per_sm);

cudaError_t launch_prep_coef(const float* theta, int L, int n, float4* coef_fwd, float4* coef_inv,
                             cudaStream_t s);
cudaError_t launch_prep_enc(const float* x, int B, int n, float2* enc, cudaStream_t s);
cudaError_t launch_expect(const float2* psi, int B, int n, double* partial, float* E,
                          unsigned* status, cudaStream_t s);
size_t expect_partial_count(int B, int n);
cudaError_t launch_grad_reduce(const DevPass* passes, const int* slot_pass, const int* slot_index,
                               const float* partials, int grid, const float* theta, int L, int n,
                               float* grad, unsigned* status, cudaStream_t s);
cudaError_t launch_loss_seed(const float* E, const float* y, int B, float* g, float* loss,
                             cudaStream_t s);
cudaError_t launch_bwd_init(float2* psi, float2* lam, const float* g, int B, int n, cudaStream_t s);
cudaError_t launch_encode(const float* x, int B, int n, float2* psi, cudaStream_t s);
cudaError_t launch_ckpt_copy(bool save, const float2* psi_in, float2* psi_out, void* slot,
                             int storage, long long count, cudaStream_t s);

}  // namespace qml
