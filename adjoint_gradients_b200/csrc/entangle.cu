// entangle.cu -- CNOT entanglers.
//
// A layer's CNOT list (CNOT(c, t): bit t of the index flips where bit c is
// set; the pages name CNOT gates as the other entangler their kernels fuse by
// recomputing indices with shifts and masks, [Deep-dive] sec. 3.2) is, as a
// whole, a linear map M of the index bits over GF(2): the layer sends the
// amplitude at index b to index M b.  Applying it is therefore a gather,
// psi'(j) = psi(M^-1 j), and un-applying it the gather psi(b) = psi'(M b).
// The map is given by the images of single bits (col[k] = image of 2^k).
// A CNOT moves amplitudes across any tile boundary, so the gather is its own
// pass between the fused rotation passes, out of place into a second buffer.
#include <cuda_bf16.h>

#include <algorithm>

#include "kernels.cuh"

namespace qml {

namespace {

// Gather dst[b][j] = src[b][m(j)] (SCATTER false), or the same permutation
// written as a scatter dst[b][m(j)] = src[b][j] (SCATTER true, m being the
// inverse map), for every sample b; m(j) = XOR of col[k] over the set bits k
// of j.  The side indexed by e is coalesced; the host picks the form whose
// other side keeps a warp's 32 consecutive indices close together (for the
// CNOT ladder M^-1 j = j ^ (j << 1) stays within 64 elements, M j = prefix
// XOR of j spreads over the whole state).
// m(j) = t0[j & 1023] ^ t1[(j >> 10) & 1023] ^ t2[j >> 20] from three
// 1024-entry shared tables (n <= 30).
template <bool SCATTER, class T>
__global__ void permute_state_kernel(const T* __restrict__ src, T* __restrict__ dst, int n, long long total,
                                     const LinMap m) {
  __shared__ uint32_t t0[1024], t1[1024], t2[1024];
  for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
    uint32_t a = 0, b = 0, c = 0;
#pragma unroll
    for (int k = 0; k < 10; ++k)
      if ((i >> k) & 1) {
        a ^= k < n ? m.col[k] : 0u;
        b ^= k + 10 < n ? m.col[k + 10] : 0u;
        c ^= k + 20 < n ? m.col[k + 20] : 0u;
      }
    t0[i] = a;
    t1[i] = b;
    t2[i] = c;
  }
  __syncthreads();
  const long long stride = (long long)gridDim.x * blockDim.x;
  const uint32_t mask = (uint32_t)((1ull << n) - 1);
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const uint32_t j = (uint32_t)e & mask;
    const uint32_t s = t0[j & 1023u] ^ t1[(j >> 10) & 1023u] ^ t2[(j >> 20) & 1023u];
    const long long o = (e & ~(long long)mask) | s;
    if (SCATTER) dst[o] = __ldg(&src[e]);
    else dst[e] = __ldg(&src[o]);
  }
}

// Highest index bit that a warp's five lowest index bits reach under m.
int spread(const LinMap& m, int n) {
  int hi = 0;
  for (int k = 0; k < 5 && k < n; ++k)
    if (m.col[k]) hi = std::max(hi, 31 - __builtin_clz(m.col[k]));
  return hi;
}

// The psi lanes of the backward planes from a checkpoint slot (standard
// layout): plane0[i].x = Re slot[i], plane1[i].x = Im slot[i].
__global__ void restore_planes_kernel(float2* plane0, float2* plane1, const void* slot, int storage,
                                      long long count) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    float re, im;
    if (storage == 1) {
      const __nv_bfloat162 v = reinterpret_cast<const __nv_bfloat162*>(slot)[i];
      re = __bfloat162float(v.x);
      im = __bfloat162float(v.y);
    } else {
      const float2 v = reinterpret_cast<const float2*>(slot)[i];
      re = v.x;
      im = v.y;
    }
    plane0[i].x = re;
    plane1[i].x = im;
  }
}

// A checkpoint slot (standard layout, sample-major) from the forward pass's
// working layout: unit u = samples 2u, 2u+1 keeps (Re psi_2u, Re psi_2u+1) at
// sample 2u's positions and (Im psi_2u, Im psi_2u+1) at sample 2u+1's (or in
// `partner` for an odd batch's last unit).
__global__ void slot_from_planes_kernel(const float2* buf, const float2* partner, void* slot, int storage, int B,
                                        int n) {
  const long long N = 1ll << n, count = (long long)B << n;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += stride) {
    const int b = (int)(e >> n);
    const long long i = e & (N - 1);
    const int u = b >> 1;
    const float2 p0 = buf[(size_t)(2 * u) * N + i];
    const float2 p1 = (2 * u + 1 < B) ? buf[(size_t)(2 * u + 1) * N + i] : partner[i];
    const float re = (b & 1) ? p0.y : p0.x, im = (b & 1) ? p1.y : p1.x;
    if (storage == 1) reinterpret_cast<__nv_bfloat162*>(slot)[e] = __floats2bfloat162_rn(re, im);
    else reinterpret_cast<float2*>(slot)[e] = make_float2(re, im);
  }
}

// fp64 mode (standard layout): slot <- psi (save) or psi <- slot, the slot in
// fp64 (storage 2), fp32 (0) or bf16 (1, round to nearest even).
__global__ void slot_copy64_kernel(bool save, double2* psi, void* slot, int storage, long long count) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    if (save) {
      const double2 v = psi[i];
      if (storage == 2) reinterpret_cast<double2*>(slot)[i] = v;
      else if (storage == 1)
        reinterpret_cast<__nv_bfloat162*>(slot)[i] = __floats2bfloat162_rn((float)v.x, (float)v.y);
      else reinterpret_cast<float2*>(slot)[i] = make_float2((float)v.x, (float)v.y);
    } else {
      double2 v;
      if (storage == 2) {
        v = reinterpret_cast<const double2*>(slot)[i];
      } else if (storage == 1) {
        const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(slot)[i]);
        v = make_double2(f.x, f.y);
      } else {
        const float2 f = reinterpret_cast<const float2*>(slot)[i];
        v = make_double2(f.x, f.y);
      }
      psi[i] = v;
    }
  }
}

unsigned grid_for(long long count, int sms) {
  const long long blocks = (count + 255) / 256;
  return (unsigned)std::min<long long>(blocks, (long long)sms * 16);
}

}  // namespace

template <class T>
cudaError_t permute_state(const T* src, T* dst, int n, int B, const LinMap& m, const LinMap& m_inv, int sms,
                          cudaStream_t s) {
  const long long total = (long long)B << n;
  if (n > kMaxQubits) return cudaErrorInvalidValue;  // three 10-bit tables
  if (total == 0) return cudaSuccess;
  if (spread(m, n) <= spread(m_inv, n))
    permute_state_kernel<false, T><<<grid_for(total, sms), 256, 0, s>>>(src, dst, n, total, m);
  else
    permute_state_kernel<true, T><<<grid_for(total, sms), 256, 0, s>>>(src, dst, n, total, m_inv);
  return cudaGetLastError();
}

cudaError_t launch_gather_bits(const float2* src, float2* dst, int n, int B, const LinMap& m, const LinMap& m_inv,
                               int sms, cudaStream_t s) {
  return permute_state(src, dst, n, B, m, m_inv, sms, s);
}

cudaError_t launch_gather_bits64(const double2* src, double2* dst, int n, int B, const LinMap& m,
                                 const LinMap& m_inv, int sms, cudaStream_t s) {
  return permute_state(src, dst, n, B, m, m_inv, sms, s);
}

cudaError_t launch_slot_copy64(bool save, double2* psi, void* slot, int storage, long long count, int sms,
                               cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  slot_copy64_kernel<<<grid_for(count, sms), 256, 0, s>>>(save, psi, slot, storage, count);
  return cudaGetLastError();
}

cudaError_t launch_slot_from_planes(const float2* buf, const float2* partner, void* slot, int storage, int B, int n,
                                   int sms, cudaStream_t s) {
  const long long count = (long long)B << n;
  if (count == 0) return cudaSuccess;
  slot_from_planes_kernel<<<grid_for(count, sms), 256, 0, s>>>(buf, partner, slot, storage, B, n);
  return cudaGetLastError();
}

cudaError_t launch_restore_planes(float2* plane0, float2* plane1, const void* slot, int storage, long long count,
                                  int sms, cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  restore_planes_kernel<<<grid_for(count, sms), 256, 0, s>>>(plane0, plane1, slot, storage, count);
  return cudaGetLastError();
}

}  // namespace qml
