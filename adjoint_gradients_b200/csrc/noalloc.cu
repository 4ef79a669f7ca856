// noalloc.cu -- an allocation-free variant of the Z0 expectation reduction.
//
// Some callers cannot hand this library a workspace, because they may not
// call cudaMalloc at all: a plugin living inside a host application whose
// framework owns every byte of device memory through its own pooling
// allocator (an allocation behind the framework's back defeats its
// accounting and can fragment its pool), or a latency-critical loop in which
// a cudaMalloc / cudaFree, which may synchronise the device, is not allowed.
// For them, qml_expect_z0_static keeps its scratch -- the per-chunk partial
// sums of the two-stage reduction -- in a fixed-size array compiled into the
// library.  The array lives on every GPU that loads the library until the
// process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.cuh"
#include "qml.h"

namespace {

// Scratch of qml_expect_z0_static: one double per (sample, 2^16-amplitude chunk).
constexpr size_t kStaticPartials = 32768;  // 256 KiB
static __device__ __align__(256) double g_static_partials[kStaticPartials];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
double* g_partials_ptr[kMaxDevices] = {};
unsigned long long g_ctx_id[kMaxDevices] = {};  // context the cached address belongs to (0: none)

// Driver's unique id of the current context (ids are never reused, unlike
// context handles), through the runtime's driver entry points; 0 if unknown.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static bool probed = false;
  if (!probed) {
    probed = true;
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(fn);
    cudaGetLastError();
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.  The cache belongs to the
// device's context: after cudaDeviceReset the next call runs in a new context,
// whose id differs, and looks the address up again.
cudaError_t scratch_on_current_device(double** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = current_context_id();
  if (!g_partials_ptr[dev] || id == 0 || id != g_ctx_id[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_partials);  // also makes the device's context current
    if (e != cudaSuccess) return e;
    g_partials_ptr[dev] = static_cast<double*>(p);
    g_ctx_id[dev] = current_context_id();
  }
  *out = g_partials_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" qml_status qml_expect_z0_static(const float* psi_dev, int n_qubits, int B, float* expect_dev,
                                           void* stream) {
  if (!psi_dev || !expect_dev || B < 1 || n_qubits < 1 || n_qubits > 30) return QML_ERR_INVALID_ARG;
  if (((uintptr_t)psi_dev) % 8 != 0) return QML_ERR_INVALID_ARG;
  if (qml::expect_partial_count(B, n_qubits) > kStaticPartials) return QML_ERR_WORKSPACE;
  double* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return QML_ERR_CUDA;
  // Every partial slot that stage 2 reads is written by stage 1 of this call,
  // so nothing left over from an earlier call is ever read.
  cudaError_t e = qml::launch_expect(reinterpret_cast<const float2*>(psi_dev), B, n_qubits, scratch, expect_dev,
                                     nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QML_OK : QML_ERR_CUDA;
}
