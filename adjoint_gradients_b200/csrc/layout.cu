// layout.cu -- conversion between the standard amplitude order and the
// working-state order of a plan (a permutation of the lowest index bits, the
// same for every aligned chunk of the state).
#include <algorithm>
#include <cstdint>

#include "kernels.cuh"

namespace qml {

namespace {

constexpr int kChunkBits = kTileBits;         // 4096 elements (32 KB) per chunk
constexpr int kChunk = 1 << kChunkBits;
constexpr int kPermThreads = 256;
constexpr int kPerThread = kChunk / kPermThreads;  // 16 elements, 8 float4

// The permutation and the shared-memory swizzle, both linear maps over the
// bits of a chunk index, given by the images of single bits:
//   wcol[k]: shared position of element 2^k (the swizzle; XORs into bits 1-3
//            only, so element pairs (2m, 2m+1) stay adjacent);
//   rcol[k]: shared position of the element that lands at 2^k.
struct BitPerm {
  int wcol[kChunkBits];
  int rcol[kChunkBits];
};

__device__ __forceinline__ int lin(const int (&col)[kChunkBits], int lo, int v, int nbits) {
  int r = 0;
#pragma unroll
  for (int k = 0; k < nbits; ++k)
    if ((v >> k) & 1) r ^= col[lo + k];
  return r;
}

// One chunk per block iteration: the chunk is read whole into registers
// (16-byte loads), written to shared memory in the swizzled order, and written
// back permuted (each warp stores 256 contiguous bytes).  The next chunk's
// loads are issued before the current one is written back.  A chunk maps onto
// itself, so the in-place update is race-free.
__global__ void __launch_bounds__(kPermThreads) permute_bits_kernel(float2* buf, long long chunks, const BitPerm pm) {
  __shared__ __align__(16) float2 sh[kChunk];
  float4* sh4 = reinterpret_cast<float4*>(sh);
  const int t = threadIdx.x;
  // unit m = t + 256 i holds elements 2m, 2m + 1: element bits 1-8 from t, 9-11 from i
  const int wt = lin(pm.wcol, 1, t, 8);
  // destination j = t + 256 i: bits 0-7 from t, 8-11 from i
  const int rt = lin(pm.rcol, 0, t, 8);
  long long c = blockIdx.x;
  float4 v[kPerThread / 2];
  if (c < chunks) {
    const float4* src = reinterpret_cast<const float4*>(buf + (size_t)c * kChunk);
#pragma unroll
    for (int i = 0; i < kPerThread / 2; ++i) v[i] = src[t + kPermThreads * i];
  }
  for (; c < chunks; c += gridDim.x) {
#pragma unroll
    for (int i = 0; i < kPerThread / 2; ++i) sh4[(wt ^ lin(pm.wcol, 9, i, 3)) >> 1] = v[i];
    __syncthreads();
    const long long cn = c + gridDim.x;
    if (cn < chunks) {
      const float4* src = reinterpret_cast<const float4*>(buf + (size_t)cn * kChunk);
#pragma unroll
      for (int i = 0; i < kPerThread / 2; ++i) v[i] = src[t + kPermThreads * i];
    }
    float2* dst = buf + (size_t)c * kChunk;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) dst[t + kPermThreads * i] = sh[rt ^ lin(pm.rcol, 8, i, 4)];
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_permute_bits(float2* buf, long long count, int cb, const int* to, int sms, cudaStream_t s) {
  if (cb < 0 || cb > kChunkBits || (count & (kChunk - 1)) != 0 || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0)
    return cudaErrorInvalidValue;
  int to12[kChunkBits], from[kChunkBits];
  for (int b = 0; b < kChunkBits; ++b) to12[b] = b < cb ? to[b] : b;
  for (int b = 0; b < kChunkBits; ++b) from[b] = -1;
  for (int b = 0; b < kChunkBits; ++b) {
    if (to12[b] < 0 || to12[b] >= kChunkBits || from[to12[b]] >= 0) return cudaErrorInvalidValue;
    from[to12[b]] = b;
  }
  // Swizzle columns a[c] (3 bits, applied to shared bits 1-3) for element bits
  // 4 + c.  A warp reads the sources of 32 consecutive destinations; their
  // source bits from[0..4] should reach all 16 low shared positions (bank
  // pairs), so the source bits >= 4 among them fill the bits 1-3 that the
  // ones below 4 leave out.
  int a[kChunkBits - 4] = {};
  int missing = 0xE;  // bits 1, 2, 3
  for (int k = 0; k < 5; ++k)
    if (from[k] >= 1 && from[k] <= 3) missing &= ~(1 << from[k]);
  for (int k = 0; k < 5 && missing; ++k)
    if (from[k] >= 4) {
      const int bit = __builtin_ctz(missing);
      missing &= missing - 1;
      a[from[k] - 4] = 1 << (bit - 1);
    }
  BitPerm pm{};
  auto phys = [&](int b) { return b < 4 ? (1 << b) : ((1 << b) ^ (a[b - 4] << 1)); };  // position of element 2^b
  for (int k = 0; k < kChunkBits; ++k) {
    pm.wcol[k] = phys(k);
    pm.rcol[k] = phys(from[k]);
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, permute_bits_kernel, kPermThreads, 0);
  if (e != cudaSuccess) return e;
  const long long chunks = count >> kChunkBits;
  const long long grid = std::min<long long>(chunks, (long long)sms * std::max(per_sm, 1));
  if (grid == 0) return cudaSuccess;
  permute_bits_kernel<<<(unsigned)grid, kPermThreads, 0, s>>>(buf, chunks, pm);
  return cudaGetLastError();
}

}  // namespace qml
