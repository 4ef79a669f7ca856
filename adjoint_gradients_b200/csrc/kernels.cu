// kernels.cu -- the helper kernels of the fused HEA forward / adjoint path
// (encoding angles, Z0 and Pauli-sum expectations, loss seed, lambda seed,
// gradient reduction, stand-alone encoding and checkpoint copies) and the
// host side of the pass launches.  The pass kernel itself is in
// pass_kernel.cuh, instantiated by pass_split.cu, pass_fused.cu and
// pass_reup.cu.
#include "pass_kernel.cuh"

namespace qml {
namespace {

// ----------------------------------------------------------------- helpers

// (cos, sin)(x/2) for the two samples of each forward unit.
__global__ void prep_enc_kernel(const float* x, int B, int n, float2* enc) {
  const int U = (B + 1) / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= U * n) return;
  const int u = idx / n, q = idx % n;
  double s0, c0, s1 = 0.0, c1 = 1.0;
  sincos(0.5 * (double)x[(2 * u) * n + q], &s0, &c0);
  if (2 * u + 1 < B) sincos(0.5 * (double)x[(2 * u + 1) * n + q], &s1, &c1);
  enc[idx * 2 + 0] = make_float2((float)c0, (float)c1);
  enc[idx * 2 + 1] = make_float2((float)s0, (float)s1);
}

constexpr int kExpThreads = 256;
constexpr int kExpChunkLog = 16;  // amplitudes per block

__global__ void expect_partial_kernel(const float2* psi, int n, double* partial) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExpChunkLog) - 1) >> kExpChunkLog);
  const int b = blockIdx.y, c = blockIdx.x;
  const long long lo = (long long)c << kExpChunkLog;
  const long long hi = min(N, lo + (1ll << kExpChunkLog));
  const float2* p = psi + (size_t)b * N;
  float s = 0.f;
  for (long long i = lo + threadIdx.x; i < hi; i += kExpThreads) {
    const float2 v = p[i];
    const float pr = fmaf(v.x, v.x, v.y * v.y);
    s += (i & 1) ? -pr : pr;
  }
  __shared__ double red[kExpThreads];
  red[threadIdx.x] = (double)s;
  __syncthreads();
  for (int w = kExpThreads / 2; w; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[(size_t)b * chunks + c] = red[0];
}

__global__ void expect_final_kernel(const double* partial, int chunks, int B, float* E,
                                    unsigned* status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  double s = 0.0;
  for (int c = 0; c < chunks; ++c) s += partial[(size_t)b * chunks + c];
  E[b] = (float)s;
  if (!isfinite(s) && status) atomicOr(status, kErrNumeric);
}

// grad[l][q] from the per-block partial sums (fixed order, fp64), rotating
// (s_x, s_y, s_z) = Im<lambda|(X, Y, Z)|psi> into the three angle gradients:
//   d/dg = s_z,  d/db = cos g s_y - sin g s_x,
//   d/da = cos b (cos g s_x + sin g s_y) - sin b s_z.
// Split form (gfix non-null): the sums were taken after Ry of the rotation,
// in the backward state's frame; gfix[.][0] takes them to the split circuit's
// states and Rz(phi1) (gfix[.][1]) to the state after the whole rotation:
// Rz(f)^dagger X Rz(f) = cos f X - sin f Y, Rz(f)^dagger Y Rz(f) = sin f X + cos f Y.
// One warp per (layer, qubit): lane i sums rows i, i + 32, ... in fp64, then
// a fixed butterfly combines the lanes, so the order (and the result) does
// not depend on timing.
__global__ void grad_reduce_kernel(const DevPass* passes, const int* slot_pass,
                                   const int* slot_index, const float* partials, int grid,
                                   const float* theta, const double* gfix, int L, int n, float* grad,
                                   unsigned* status) {
  const int idx = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (idx >= L * n) return;  // whole warps leave together
  const int p = slot_pass[idx], s = slot_index[idx];
  const DevPass& ps = passes[p];
  const int stride = ps.nslots * 3;
  const float* base = partials + ps.partial_off + s * 3;
  double sx = 0.0, sy = 0.0, sz = 0.0;
  for (int c = lane; c < grid; c += 32) {
    sx += base[(size_t)c * stride + 0];
    sy += base[(size_t)c * stride + 1];
    sz += base[(size_t)c * stride + 2];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sx += __shfl_xor_sync(0xffffffffu, sx, o);
    sy += __shfl_xor_sync(0xffffffffu, sy, o);
    sz += __shfl_xor_sync(0xffffffffu, sz, o);
  }
  if (lane != 0) return;
  if (gfix) {
    const double sc = gfix[(size_t)idx * 2 + 0], f = gfix[(size_t)idx * 2 + 1];
    double sf, cf;
    sincos(f, &sf, &cf);
    sx *= sc;
    sy *= sc;
    sz *= fabs(sc);
    const double tx = cf * sx - sf * sy;
    sy = sf * sx + cf * sy;
    sx = tx;
  }
  const double be = theta[idx * 3 + 1], ga = theta[idx * 3 + 2];
  double sb, cb, sg, cg;
  sincos(be, &sb, &cb);
  sincos(ga, &sg, &cg);
  const double gz = sz;
  const double gy = cg * sy - sg * sx;
  const double gx = cb * (cg * sx + sg * sy) - sb * sz;
  grad[idx * 3 + 0] = (float)gx;
  grad[idx * 3 + 1] = (float)gy;
  grad[idx * 3 + 2] = (float)gz;
  if (!(isfinite(gx) && isfinite(gy) && isfinite(gz)) && status) atomicOr(status, kErrNumeric);
}

// g[b] = 2 (E[b] - y[b]) / B, loss = mean (E - y)^2 (fixed-order fp64 sum).
__global__ void loss_seed_kernel(const float* E, const float* y, int B, float* g, float* loss) {
  __shared__ double red[256];
  double s = 0.0;
  for (int b = threadIdx.x; b < B; b += 256) {
    const double d = (double)E[b] - (double)y[b];
    if (g) g[b] = (float)(2.0 * d / B);
    s += d * d;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0 && loss) *loss = (float)(red[0] / B);
}

// Start of the adjoint walk: lambda = dL/dE[b] Z0 psi, written together with
// psi into the plane layout the backward passes use: plane 0 (the psi buffer,
// in place) holds (Re psi, Re lambda), plane 1 (the lambda buffer) holds
// (Im psi, Im lambda).
// ---------------------------------------------- observables: sums of Pauli strings
//
// O = sum_k c_k P_k with P_k = i^ny X^x Z^z (x: qubits carrying X or Y, z:
// qubits carrying Z or Y, ny: the number of Y), so that
//   (P psi)(j) = i^ny (-1)^popcount((j ^ x) & z) psi(j ^ x),
//   <psi|P|psi> = sum_j conj(psi(j)) (P psi)(j).
// Terms are grouped by x, so each group reads psi(j ^ x) once.  The general
// observable of E(theta) = <psi|O|psi> ([Deep-dive] sec. 1.2), evaluated
// matrix-free by bit flips ([Deep-dive] sec. 3.2, the expectation listing).

// sum over the group's terms of c_k i^ny (-1)^popcount(m & z_k), m = j ^ x
__device__ __forceinline__ double2 obs_weight(const ObsTerm* t, int count, uint32_t m) {
  double wr = 0.0, wi = 0.0;
  for (int k = 0; k < count; ++k) {
    const double c = (__popc(m & t[k].z) & 1) ? -t[k].c : t[k].c;
    switch (t[k].ny & 3) {
      case 0: wr += c; break;
      case 1: wi += c; break;
      case 2: wr -= c; break;
      default: wi -= c; break;
    }
  }
  return make_double2(wr, wi);
}

__global__ void obs_expect_partial_kernel(const float2* psi, int n, const ObsGroup* groups, int ngroups,
                                          const ObsTerm* terms, double* partial) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExpChunkLog) - 1) >> kExpChunkLog);
  const int b = blockIdx.y, c = blockIdx.x;
  const long long lo = (long long)c << kExpChunkLog;
  const long long hi = min(N, lo + (1ll << kExpChunkLog));
  const float2* p = psi + (size_t)b * N;
  double s = 0.0;
  for (int gi = 0; gi < ngroups; ++gi) {
    const ObsGroup G = groups[gi];
    for (long long j = lo + threadIdx.x; j < hi; j += kExpThreads) {
      const uint32_t m = (uint32_t)j ^ G.x;
      const float2 a = p[j], q = p[m];
      // conj(a) * q
      const double wr = (double)a.x * q.x + (double)a.y * q.y;
      const double wi = (double)a.x * q.y - (double)a.y * q.x;
      const double2 d = obs_weight(terms + G.first, G.count, m);
      s += wr * d.x - wi * d.y;
    }
  }
  __shared__ double red[kExpThreads];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = kExpThreads / 2; w; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[(size_t)b * chunks + c] = red[0];
}

// lambda = g_b O psi in the standard layout (psi and lambda are different buffers)
__global__ void obs_lambda_kernel(const float2* psi, float2* lam, const float* g, int B, int n,
                                  const ObsGroup* groups, int ngroups, const ObsTerm* terms) {
  const long long N = 1ll << n;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)B * N) return;
  const int b = (int)(idx >> n);
  const uint32_t j = (uint32_t)(idx & (N - 1));
  const float2* p = psi + (size_t)b * N;
  double ar = 0.0, ai = 0.0;
  for (int gi = 0; gi < ngroups; ++gi) {
    const ObsGroup G = groups[gi];
    const uint32_t m = j ^ G.x;
    const float2 q = p[m];
    const double2 d = obs_weight(terms + G.first, G.count, m);
    ar += d.x * q.x - d.y * q.y;
    ai += d.x * q.y + d.y * q.x;
  }
  const double gs = (double)__ldg(&g[b]);
  lam[idx] = make_float2((float)(gs * ar), (float)(gs * ai));
}

// psi, lambda (standard layout) -> the backward planes, in place, position by position
__global__ void planes_kernel(float2* psi, float2* lam, long long count) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= count) return;
  const float2 v = psi[idx], l = lam[idx];
  psi[idx] = make_float2(v.x, l.x);
  lam[idx] = make_float2(v.y, l.y);
}

__global__ void bwd_init_kernel(float2* psi, float2* lam, const float* g, int B, int n) {
  const long long N = 1ll << n;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)B * N) return;
  const int b = (int)(idx >> n);
  const float gs = (idx & 1) ? -__ldg(&g[b]) : __ldg(&g[b]);
  const float2 v = psi[idx];
  psi[idx] = make_float2(v.x, gs * v.x);
  lam[idx] = make_float2(v.y, gs * v.y);
}

// Encoded product state, standard layout, one thread per amplitude.
__global__ void encode_kernel(const float* x, int B, int n, float2* psi) {
  const long long N = 1ll << n;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)B * N) return;
  const int b = (int)(idx >> n);
  const long long i = idx & (N - 1);
  float v = 1.f;
  for (int q = 0; q < n; ++q) {
    float s, c;
    sincosf(0.5f * x[b * n + q], &s, &c);
    v *= ((i >> q) & 1) ? s : c;
  }
  psi[idx] = make_float2(v, 0.f);
}

__global__ void ckpt_copy_kernel(bool save, const float2* in, float2* out, void* slot,
                                 int storage, long long count) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= count) return;
  if (save) {
    if (storage == 0) reinterpret_cast<float2*>(slot)[idx] = in[idx];
    else reinterpret_cast<__nv_bfloat162*>(slot)[idx] = __floats2bfloat162_rn(in[idx].x, in[idx].y);
  } else {
    if (storage == 0) out[idx] = reinterpret_cast<const float2*>(slot)[idx];
    else out[idx] = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(slot)[idx]);
  }
}

}  // namespace

size_t pass_smem_bytes(int max_slots, bool tma) {
  return pass_buf_bytes(tma) + sizeof(BlockCtx) + (size_t)(kThreads / 32) * max_slots * 3 * sizeof(float);
}

size_t pass_multi_smem_bytes() { return multi_stage_offset() + sizeof(MultiStage); }

cudaError_t set_pass_smem_attr(size_t smem_thr, size_t smem_tma) {
  cudaError_t e = pass_split_attr(smem_thr, smem_tma);
  if (e == cudaSuccess) e = pass_fused_attr(smem_thr, smem_tma);
  if (e == cudaSuccess) e = pass_reup_attr(smem_thr, smem_tma);
  if (e == cudaSuccess) e = pass_csplit_attr(smem_thr, smem_tma);
  if (e == cudaSuccess) e = pass_single_attr(smem_thr, smem_tma);
  return e;
}

int debug_layouts(int* out, int cap) {
  int v[2 * 3 * 12 + 2 * (kTileBits + 1)];
  int k = 0;
  for (int P = 0; P < kPhases; ++P)
    for (int V = 0; V < 2; ++V) {
      for (int m = 0; m < kThrBits; ++m)
        v[k++] = P == 0 ? thr_tbit<0, 0>(m) : P == 1 ? (V ? thr_tbit<1, 1>(m) : thr_tbit<1, 0>(m)) : thr_tbit<2, 0>(m);
      for (int r = 0; r < kRegBits; ++r) v[k++] = P == 0 ? reg_tbit<0>(r) : P == 1 ? reg_tbit<1>(r) : reg_tbit<2>(r);
    }
  for (int b = 0; b < kTileBits; ++b) v[k++] = (int)wbit(b);
  v[k++] = kSmemSlots;
  for (int b = 0; b < kTileBits; ++b) v[k++] = (int)wbit8(b);
  v[k++] = kExch8Slots;
  for (int i = 0; i < k && i < cap; ++i) out[i] = v[i];
  return k;
}

cudaError_t launch_pass(bool backward, const PassArgs& a, const DevPass& p, const PassMaps& maps, int grid,
                        size_t smem, cudaStream_t s, const CoefRegion* coef) {
  const int mode = p.slow ? 0 : p.tma ? 2 : 1;
  // re-uploading: form 2 where the tile holds a batch-unit bit, else 1;
  // split-form passes: 3; the fused SU(2) form: 0
  int form = 0;
  for (int o = 0; o < p.nops; ++o)
    if (p.ops[o].kind == OP_RY || p.ops[o].kind == OP_DIAG) form = 3;
  if (a.reupload) {
    form = 1;
    for (int b = 0; b < kTileBits; ++b)
      if (p.tile_q[b] < 0) form = 2;
  }
  if (form == 3 && p.cnot) form = 4;
  if (form == 3 && !backward && a.npass > 0 && a.zf) form = 5;
  if (form == 5) return pass_single_launch(backward, mode, p.variant, form, a, p, maps, grid, smem, coef, s);
  if (form == 4) return pass_csplit_launch(backward, mode, p.variant, form, a, p, maps, grid, smem, coef, s);
  if (form == 3) return pass_split_launch(backward, mode, p.variant, form, a, p, maps, grid, smem, coef, s);
  if (form == 0) return pass_fused_launch(backward, mode, p.variant, form, a, p, maps, grid, smem, coef, s);
  return pass_reup_launch(backward, mode, p.variant, form, a, p, maps, grid, smem, coef, s);
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;
bool g_encode_probed = false;
}  // namespace

cudaError_t encode_pass_maps(const DevPass& p, int n, int B, bool backward, const void* buf0, const void* buf1,
                             PassMaps* maps) {
  // forward: buf1 is the one-sample partner buffer of an odd batch's last unit
  const int samples[2] = {B, backward ? B : 1};
  std::memset(maps, 0, sizeof(*maps));
  if (!p.tma) return cudaSuccess;
  if (!g_encode_probed) {
    g_encode_probed = true;
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cudaGetLastError();
  }
  if (!g_encode_tiled) return cudaErrorNotSupported;
  void* bases[2] = {const_cast<void*>(buf0), const_cast<void*>(buf1)};
  void* outs[2] = {maps->m0, maps->m1};
  if (p.tma_kind[0] != TD_IN || p.tma_qlo[0] != 0) return cudaErrorInvalidValue;
  for (int i = 0; i < 2; ++i) {
    if (!bases[i] || (reinterpret_cast<uintptr_t>(bases[i]) & 15u)) return cudaErrorInvalidValue;
    cuuint64_t dims[kTmaRank], strides[kTmaRank];
    cuuint32_t box[kTmaRank], estr[kTmaRank];
    const cuuint64_t esz = sizeof(float2);
    for (int d = 0; d < kTmaRank; ++d) {
      const int k = p.tma_kind[d];
      estr[d] = 1;
      if (k == TD_IN || k == TD_OUT) {
        dims[d] = 1ull << p.tma_bits[d];
        strides[d] = esz << p.tma_qlo[d];
        box[d] = k == TD_IN ? (cuuint32_t)(1u << p.tma_bits[d]) : 1u;
      } else if (k == TD_SAMPLE) {
        dims[d] = (cuuint64_t)samples[i];
        strides[d] = esz << n;
        box[d] = 1;
      } else if (k == TD_OUT_SAMPLE) {
        dims[d] = (cuuint64_t)samples[i] << p.tma_bits[d];
        strides[d] = esz << p.tma_qlo[d];
        box[d] = 1;
      } else {  // padding
        dims[d] = 1;
        strides[d] = d > 0 ? strides[d - 1] * dims[d - 1] : esz;
        box[d] = 1;
      }
    }
    CUresult r = g_encode_tiled(reinterpret_cast<CUtensorMap*>(outs[i]), CU_TENSOR_MAP_DATA_TYPE_FLOAT64, kTmaRank,
                                bases[i], dims, strides + 1, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_prep_enc(const float* x, int B, int n, float2* enc, cudaStream_t s) {
  const int tot = ((B + 1) / 2) * n;
  prep_enc_kernel<<<(tot + 127) / 128, 128, 0, s>>>(x, B, n, enc);
  return cudaGetLastError();
}

size_t expect_partial_count(int B, int n) {
  const long long N = 1ll << n;
  const long long chunks = (N + (1ll << kExpChunkLog) - 1) >> kExpChunkLog;
  return (size_t)B * (size_t)chunks;
}

cudaError_t launch_expect(const float2* psi, int B, int n, double* partial, float* E,
                          unsigned* status, cudaStream_t s) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExpChunkLog) - 1) >> kExpChunkLog);
  dim3 grid(chunks, B);
  expect_partial_kernel<<<grid, kExpThreads, 0, s>>>(psi, n, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expect_final_kernel<<<(B + 127) / 128, 128, 0, s>>>(partial, chunks, B, E, status);
  return cudaGetLastError();
}

cudaError_t launch_expect_final(const double* partial, int chunks, int B, float* E, unsigned* status,
                               cudaStream_t s) {
  expect_final_kernel<<<(B + 127) / 128, 128, 0, s>>>(partial, chunks, B, E, status);
  return cudaGetLastError();
}

cudaError_t launch_grad_reduce(const DevPass* passes, const int* slot_pass, const int* slot_index,
                               const float* partials, int grid, const float* theta, const double* gfix, int L,
                               int n, float* grad, unsigned* status, cudaStream_t s) {
  const long long threads = (long long)L * n * 32;  // one warp per (layer, qubit)
  grad_reduce_kernel<<<(unsigned)((threads + 127) / 128), 128, 0, s>>>(passes, slot_pass, slot_index, partials,
                                                                       grid, theta, gfix, L, n, grad, status);
  return cudaGetLastError();
}

cudaError_t launch_loss_seed(const float* E, const float* y, int B, float* g, float* loss,
                             cudaStream_t s) {
  loss_seed_kernel<<<1, 256, 0, s>>>(E, y, B, g, loss);
  return cudaGetLastError();
}

cudaError_t launch_encode(const float* x, int B, int n, float2* psi, cudaStream_t s) {
  const long long tot = (long long)B << n;
  const long long blocks = (tot + 255) / 256;
  encode_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, B, n, psi);
  return cudaGetLastError();
}

cudaError_t launch_obs_expect(const float2* psi, int B, int n, const ObsGroup* groups, int ngroups,
                              const ObsTerm* terms, double* partial, float* E, unsigned* status, cudaStream_t s) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExpChunkLog) - 1) >> kExpChunkLog);
  dim3 grid(chunks, B);
  obs_expect_partial_kernel<<<grid, kExpThreads, 0, s>>>(psi, n, groups, ngroups, terms, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expect_final_kernel<<<(B + 127) / 128, 128, 0, s>>>(partial, chunks, B, E, status);
  return cudaGetLastError();
}

cudaError_t launch_obs_bwd_init(float2* psi, float2* lam, const float* g, int B, int n, const ObsGroup* groups,
                                int ngroups, const ObsTerm* terms, cudaStream_t s) {
  const long long tot = (long long)B << n;
  const unsigned blocks = (unsigned)((tot + 255) / 256);
  obs_lambda_kernel<<<blocks, 256, 0, s>>>(psi, lam, g, B, n, groups, ngroups, terms);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  planes_kernel<<<blocks, 256, 0, s>>>(psi, lam, tot);
  return cudaGetLastError();
}

cudaError_t launch_bwd_init(float2* psi, float2* lam, const float* g, int B, int n, cudaStream_t s) {
  const long long tot = (long long)B << n;
  bwd_init_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(psi, lam, g, B, n);
  return cudaGetLastError();
}

cudaError_t launch_ckpt_copy(bool save, const float2* psi_in, float2* psi_out, void* slot,
                             int storage, long long count, cudaStream_t s) {
  const long long blocks = (count + 255) / 256;
  ckpt_copy_kernel<<<(unsigned)blocks, 256, 0, s>>>(save, psi_in, psi_out, slot, storage, count);
  return cudaGetLastError();
}

}  // namespace qml
