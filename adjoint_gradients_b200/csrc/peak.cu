// peak.cu -- measured FMA throughput of the GPU (the ALU roofline denominators).
//
// Every thread runs kChains independent FMA chains (x <- x * m + a), so the
// pipe sees kChains independent instructions per warp between dependences; the
// grid fills every SM with several blocks.  fp32 uses the packed f32x2 FMA the
// pass kernels use, fp64 the DFMA of the fp64 mode.  The result is stored (to
// a small array compiled into the library) only when it equals a value it
// never takes in practice, which keeps the loop alive.
#include <cuda_runtime.h>

#include "qml.h"

namespace {

constexpr int kChains = 8;
constexpr int kThreads = 256;
constexpr int kSink = 4096;
__device__ double g_sink[kSink];

__global__ void __launch_bounds__(kThreads) fma_f32x2_kernel(int iters, float2 m, float2 a) {
  float2 x[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) x[c] = make_float2(1.f + 0.01f * c, 0.5f + 0.01f * threadIdx.x);
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = __ffma2_rn(x[c], m, a);
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += x[c].x + x[c].y;
  if (s == 1234.5f) g_sink[blockIdx.x % kSink] = s;
}

__global__ void __launch_bounds__(kThreads) fma_f64_kernel(int iters, double m, double a) {
  double x[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) x[c] = 1.0 + 0.01 * c + 1e-3 * threadIdx.x;
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = fma(x[c], m, a);
  }
  double s = 0.0;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += x[c];
  if (s == 1234.5) g_sink[blockIdx.x % kSink] = s;
}

}  // namespace

extern "C" qml_status qml_measure_fma_peak(int fp64, int iters, void* stream, double* tflops, float* ms_out) {
  if (!tflops || iters < 1) return QML_ERR_INVALID_ARG;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return QML_ERR_CUDA;
  cudaError_t e = fp64 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fma_f64_kernel, kThreads, 0)
                       : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fma_f32x2_kernel, kThreads, 0);
  if (e != cudaSuccess || per_sm < 1) return QML_ERR_CUDA;
  const int grid = sms * per_sm;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t a = nullptr, b = nullptr;
  if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return QML_ERR_CUDA;
  e = cudaEventRecord(a, s);
  if (e == cudaSuccess) {
    if (fp64) fma_f64_kernel<<<grid, kThreads, 0, s>>>(iters, 0.9999999, 1e-7);
    else fma_f32x2_kernel<<<grid, kThreads, 0, s>>>(iters, make_float2(0.9999f, 0.9999f), make_float2(1e-4f, 1e-4f));
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaEventRecord(b, s);
  if (e == cudaSuccess) e = cudaEventSynchronize(b);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (e != cudaSuccess || ms <= 0.f) return QML_ERR_CUDA;
  const double lanes = fp64 ? 1.0 : 2.0;  // FMAs per instruction and thread
  const double fma = (double)grid * kThreads * (double)iters * kChains * lanes;
  *tflops = 2.0 * fma / (ms * 1e-3) / 1e12;
  if (ms_out) *ms_out = ms;
  return QML_OK;
}
