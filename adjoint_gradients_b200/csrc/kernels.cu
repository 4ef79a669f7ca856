// kernels.cu -- sm_100a kernels of the fused HEA forward / adjoint path.
//
// Method (Kawase, "Fast and memory-efficient classical simulation of quantum
// machine learning via forward and backward gate fusion"; cited below by the
// page that states it):
//   * forward gate fusion: many gates per read/write of the state vector
//     [Deep-dive blog sec. 1.4 item 1; gist.science Technical Summary sec. 2];
//   * backward gate fusion: inside a fused block, rebuild the input state of
//     each gate with U^dagger next to the adjoint state, and form the gradient
//     [Deep-dive sec. 1.2 (adjoint equations), sec. 1.4 item 2];
//   * CZ ladders as a sign from index bits [Deep-dive sec. 3.2, "Listing 1"];
//   * matrix-free Z expectation [Deep-dive sec. 3.2, "Listing 3"];
//   * bf16 storage with fp32 compute [gist.science Technical Summary sec. 2].
//
// Data layout on chip.  A tile is 4096 positions of one batch unit; each of
// the 128 threads keeps 32 positions in registers as two float2 values:
//   forward : re = (Re psi_b, Re psi_{b+1}), im = (Im psi_b, Im psi_{b+1})
//             -- two samples of a pair share every gate, so one packed
//             f32x2 FMA updates both;
//   backward: re = (Re psi, Re lambda),     im = (Im psi, Im lambda)
//             -- psi and lambda share every U^dagger.
// In HBM the working state keeps the same pairing ("planes"): plane 0 holds
// the re pairs and plane 1 the im pairs, each as [2^n] float2 at the same
// byte positions the standard (re, im) layout uses, so converting between
// layouts is always in place.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace qml {
namespace {

constexpr unsigned kErrNumeric = 1u << 6;  // bit (QML_ERR_NUMERIC)

// ---------------------------------------------------------------- gate math

struct Coef {
  float2 ar, ai, nai, br, bi, nbi, nbr;  // broadcast (v, v) pairs
};

__device__ __forceinline__ Coef load_coef(const float4* p) {
  const float4 f0 = __ldg(p), f1 = __ldg(p + 1), f2 = __ldg(p + 2), f3 = __ldg(p + 3);
  Coef c;
  c.ar = make_float2(f0.x, f0.y);
  c.ai = make_float2(f0.z, f0.w);
  c.nai = make_float2(f1.x, f1.y);
  c.br = make_float2(f1.z, f1.w);
  c.bi = make_float2(f2.x, f2.y);
  c.nbi = make_float2(f2.z, f2.w);
  c.nbr = make_float2(f3.x, f3.y);
  return c;
}

// (x, y) <- [[a, b], [-conj b, conj a]] (x, y) on two lanes at once.
__device__ __forceinline__ void su2(float2& xr, float2& xi, float2& yr, float2& yi, const Coef& c) {
  float2 o0r = __fmul2_rn(c.ar, xr);
  o0r = __ffma2_rn(c.nai, xi, o0r);
  o0r = __ffma2_rn(c.br, yr, o0r);
  o0r = __ffma2_rn(c.nbi, yi, o0r);
  float2 o0i = __fmul2_rn(c.ar, xi);
  o0i = __ffma2_rn(c.ai, xr, o0i);
  o0i = __ffma2_rn(c.br, yi, o0i);
  o0i = __ffma2_rn(c.bi, yr, o0i);
  float2 o1r = __fmul2_rn(c.nbr, xr);
  o1r = __ffma2_rn(c.nbi, xi, o1r);
  o1r = __ffma2_rn(c.ar, yr, o1r);
  o1r = __ffma2_rn(c.ai, yi, o1r);
  float2 o1i = __fmul2_rn(c.nbr, xi);
  o1i = __ffma2_rn(c.bi, xr, o1i);
  o1i = __ffma2_rn(c.ar, yi, o1i);
  o1i = __ffma2_rn(c.nai, yr, o1i);
  xr = o0r;
  xi = o0i;
  yr = o1r;
  yi = o1i;
}

template <int K>
__device__ __forceinline__ void rot_fwd(float2 (&re)[kPos], float2 (&im)[kPos], const Coef& c) {
#pragma unroll
  for (int j = 0; j < kPos; ++j)
    if (!(j & (1 << K))) su2(re[j], im[j], re[j | (1 << K)], im[j | (1 << K)], c);
}

// Gradient terms of one qubit at the state just after its fused rotation, then
// U^dagger on psi and lambda.  With psi in lane x and lambda in lane y:
//   s_z = Im<lambda|Z|psi>, s_x = Im<lambda|X|psi>, s_y = Im<lambda|Y|psi>.
// 2 Re<lambda|(-i/2) P|psi> = Im<lambda|P|psi>, so these are the gradients of
// the three rotation angles up to a known rotation (applied in grad_reduce).
template <int K>
__device__ __forceinline__ float3 rot_bwd(float2 (&re)[kPos], float2 (&im)[kPos], const Coef& c) {
  float sx = 0.f, sy = 0.f, sz = 0.f;
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    if (j & (1 << K)) continue;
    const int jj = j | (1 << K);
    const float p0r = re[j].x, l0r = re[j].y, p0i = im[j].x, l0i = im[j].y;
    const float p1r = re[jj].x, l1r = re[jj].y, p1i = im[jj].x, l1i = im[jj].y;
    sz = fmaf(l0r, p0i, sz);
    sz = fmaf(-l0i, p0r, sz);
    sz = fmaf(-l1r, p1i, sz);
    sz = fmaf(l1i, p1r, sz);
    sx = fmaf(l0r, p1i, sx);
    sx = fmaf(-l0i, p1r, sx);
    sx = fmaf(l1r, p0i, sx);
    sx = fmaf(-l1i, p0r, sx);
    sy = fmaf(-l0r, p1r, sy);
    sy = fmaf(-l0i, p1i, sy);
    sy = fmaf(l1r, p0r, sy);
    sy = fmaf(l1i, p0i, sy);
    su2(re[j], im[j], re[jj], im[jj], c);
  }
  return make_float3(sx, sy, sz);
}

__device__ __forceinline__ void rot_fwd_k(int k, float2 (&re)[kPos], float2 (&im)[kPos],
                                          const Coef& c) {
  static_assert(kRegBits == 4, "dispatch below covers four register bits");
  switch (k) {
    case 0: rot_fwd<0>(re, im, c); break;
    case 1: rot_fwd<1>(re, im, c); break;
    case 2: rot_fwd<2>(re, im, c); break;
    default: rot_fwd<3>(re, im, c); break;
  }
}

__device__ __forceinline__ float3 rot_bwd_k(int k, float2 (&re)[kPos], float2 (&im)[kPos],
                                            const Coef& c) {
  switch (k) {
    case 0: return rot_bwd<0>(re, im, c);
    case 1: return rot_bwd<1>(re, im, c);
    case 2: return rot_bwd<2>(re, im, c);
    default: return rot_bwd<3>(re, im, c);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void flip(float2& v, uint32_t signbit) {
  v.x = __uint_as_float(__float_as_uint(v.x) ^ signbit);
  v.y = __uint_as_float(__float_as_uint(v.y) ^ signbit);
}

// ------------------------------------------------------------ tile geometry

struct ThreadCtx {
  uint32_t aq;    // qubit-space index of this thread's register position 0
  uint32_t ut;    // batch unit of register position 0
  uint32_t slot;  // swizzled shared-memory slot of register position 0
};

__device__ __forceinline__ ThreadCtx thread_ctx(const DevPhase& ph, int tid, uint32_t base_q,
                                                uint32_t unit_base) {
  ThreadCtx t;
  t.aq = base_q;
  t.ut = unit_base;
  t.slot = 0;
#pragma unroll
  for (int k = 0; k < kThrBits; ++k)
    if ((tid >> k) & 1) {
      if (ph.thr_q[k] >= 0) t.aq |= 1u << ph.thr_q[k];
      else t.ut += 1u << ph.thr_u[k];
      t.slot ^= ph.thr_phys[k];
    }
  return t;
}

struct RegMaps {
  uint32_t q[kRegBits];     // qubit bit of register bit k (0 if a unit bit)
  uint32_t u[kRegBits];     // unit increment of register bit k (0 if a qubit)
  uint32_t phys[kRegBits];  // shared-memory slot bit(s) of register bit k
};

__device__ __forceinline__ RegMaps reg_maps(const DevPhase& ph) {
  RegMaps m;
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) {
    m.q[k] = ph.reg_q[k] >= 0 ? (1u << ph.reg_q[k]) : 0u;
    m.u[k] = ph.reg_u[k] >= 0 ? (1u << ph.reg_u[k]) : 0u;
    m.phys[k] = ph.reg_phys[k];
  }
  return m;
}

#define REG_COMBINE(arr, j, op)                                   \
  ([&]() {                                                        \
    uint32_t r_ = 0;                                              \
    _Pragma("unroll") for (int k_ = 0; k_ < kRegBits; ++k_) if ((j) & (1 << k_)) r_ op arr[k_]; \
    return r_;                                                    \
  }())

__device__ void exchange(float2 (&re)[kPos], float2 (&im)[kPos], float4* tile,
                         const DevPhase& from, const DevPhase& to, int tid) {
  const ThreadCtx tf = thread_ctx(from, tid, 0, 0);
  const ThreadCtx tt = thread_ctx(to, tid, 0, 0);
  const RegMaps mf = reg_maps(from);
  const RegMaps mt = reg_maps(to);
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t s = tf.slot ^ REG_COMBINE(mf.phys, j, ^=);
    tile[s] = make_float4(re[j].x, re[j].y, im[j].x, im[j].y);
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t s = tt.slot ^ REG_COMBINE(mt.phys, j, ^=);
    const float4 v = tile[s];
    re[j] = make_float2(v.x, v.y);
    im[j] = make_float2(v.z, v.w);
  }
}

// CZ(q, q+1) for every q: sign (-1)^{sum_q i_q i_{q+1}} of the global index i.
// With i = a | b (a: thread and out-of-tile bits, b: register bits, disjoint),
// the exponent is Q(a) + Q(b) + parity(b & ((a << 1) ^ (a >> 1))).
__device__ __forceinline__ void apply_cz(float2 (&re)[kPos], float2 (&im)[kPos],
                                         const DevPhase& ph, uint32_t aq) {
  const uint32_t qa = __popc(aq & (aq >> 1)) & 1u;
  const uint32_t m = (aq << 1) ^ (aq >> 1);
  uint32_t w = ph.cz_reg ^ (qa ? 0xffffffffu : 0u);
  const uint32_t pat[5] = {0xAAAAAAAAu, 0xCCCCCCCCu, 0xF0F0F0F0u, 0xFF00FF00u, 0xFFFF0000u};
#pragma unroll
  for (int k = 0; k < kRegBits; ++k)
    if (ph.reg_q[k] >= 0 && ((m >> ph.reg_q[k]) & 1u)) w ^= pat[k];
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t sb = (w << (31 - j)) & 0x80000000u;
    flip(re[j], sb);
    flip(im[j], sb);
  }
}

// Value of register position j for a runtime j (slow paths for n < 5 only).
__device__ __forceinline__ float2 sel(const float2 (&v)[kPos], int j) {
  float2 r = v[0];
#pragma unroll
  for (int k = 1; k < kPos; ++k)
    if (k == j) r = v[k];
  return r;
}

__device__ __forceinline__ void put(float2 (&v)[kPos], int j, float2 x) {
#pragma unroll
  for (int k = 0; k < kPos; ++k)
    if (k == j) v[k] = x;
}

// Register position j's batch unit and qubit index, for a runtime j.
__device__ __forceinline__ void pos_of(const RegMaps& m, const ThreadCtx& tc, int j, uint32_t* u,
                                       uint32_t* i) {
  uint32_t uu = tc.ut, ii = tc.aq;
#pragma unroll
  for (int k = 0; k < kRegBits; ++k)
    if (j & (1 << k)) { uu += m.u[k]; ii |= m.q[k]; }
  *u = uu;
  *i = ii;
}

// ------------------------------------------------------------------ planes

template <bool BWD>
struct Planes {
  __device__ static float2* p0(const PassArgs& a, uint32_t u) {
    return BWD ? a.buf0 + (size_t)u * a.N : a.buf0 + (size_t)(2 * u) * a.N;
  }
  __device__ static float2* p1(const PassArgs& a, uint32_t u) {
    if (BWD) return a.buf1 + (size_t)u * a.N;
    return (2 * u + 1 < (uint32_t)a.B) ? a.buf0 + (size_t)(2 * u + 1) * a.N : a.dummy;
  }
};

template <bool BWD, bool SLOW>
__device__ void load_planes(const PassArgs& a, const DevPhase& ph, const ThreadCtx& tc,
                            float2 (&re)[kPos], float2 (&im)[kPos]) {
  const RegMaps m = reg_maps(ph);
  if constexpr (!SLOW) {
    if (tc.ut < (uint32_t)a.U) {
      const float2* p0 = Planes<BWD>::p0(a, tc.ut) + tc.aq;
      const float2* p1 = Planes<BWD>::p1(a, tc.ut) + tc.aq;
#pragma unroll
      for (int j = 0; j < kPos; ++j) {
        const uint32_t b = REG_COMBINE(m.q, j, |=);
        re[j] = p0[b];
        im[j] = p1[b];
      }
    } else {
#pragma unroll
      for (int j = 0; j < kPos; ++j) re[j] = im[j] = make_float2(0.f, 0.f);
    }
  } else {
#pragma unroll 1
    for (int j = 0; j < kPos; ++j) {
      uint32_t u, i;
      pos_of(m, tc, j, &u, &i);
      float2 r = make_float2(0.f, 0.f), v = r;
      if (u < (uint32_t)a.U) {
        r = Planes<BWD>::p0(a, u)[i];
        v = Planes<BWD>::p1(a, u)[i];
      }
      put(re, j, r);
      put(im, j, v);
    }
  }
}

template <bool BWD, bool SLOW>
__device__ void store_planes(const PassArgs& a, const DevPhase& ph, const ThreadCtx& tc,
                             const float2 (&re)[kPos], const float2 (&im)[kPos]) {
  const RegMaps m = reg_maps(ph);
  if constexpr (!SLOW) {
    if (tc.ut < (uint32_t)a.U) {
      float2* p0 = Planes<BWD>::p0(a, tc.ut) + tc.aq;
      float2* p1 = Planes<BWD>::p1(a, tc.ut) + tc.aq;
#pragma unroll
      for (int j = 0; j < kPos; ++j) {
        const uint32_t b = REG_COMBINE(m.q, j, |=);
        p0[b] = re[j];
        p1[b] = im[j];
      }
    }
  } else {
#pragma unroll 1
    for (int j = 0; j < kPos; ++j) {
      uint32_t u, i;
      pos_of(m, tc, j, &u, &i);
      if (u < (uint32_t)a.U) {
        Planes<BWD>::p0(a, u)[i] = sel(re, j);
        Planes<BWD>::p1(a, u)[i] = sel(im, j);
      }
    }
  }
}

// Forward, last pass: write the standard (re, im) layout of both samples.
template <bool SLOW>
__device__ void store_standard_fwd(const PassArgs& a, const DevPhase& ph, const ThreadCtx& tc,
                                   const float2 (&re)[kPos], const float2 (&im)[kPos]) {
  const RegMaps m = reg_maps(ph);
  if constexpr (!SLOW) {
    const uint32_t u = tc.ut;
    if (u >= (uint32_t)a.U) return;
    float2* s0 = a.buf0 + (size_t)(2 * u) * a.N + tc.aq;
    float2* s1 = s0 + a.N;
    const bool has1 = 2 * u + 1 < (uint32_t)a.B;
#pragma unroll
    for (int j = 0; j < kPos; ++j) {
      const uint32_t b = REG_COMBINE(m.q, j, |=);
      s0[b] = make_float2(re[j].x, im[j].x);
      if (has1) s1[b] = make_float2(re[j].y, im[j].y);
    }
  } else {
#pragma unroll 1
  for (int j = 0; j < kPos; ++j) {
    uint32_t u = tc.ut, i = tc.aq;
    for (int k = 0; k < kRegBits; ++k)
      if (j & (1 << k)) { u += m.u[k]; i |= m.q[k]; }
    if (u < (uint32_t)a.U) {
      const float2 r = sel(re, j), v = sel(im, j);
      a.buf0[(size_t)(2 * u) * a.N + i] = make_float2(r.x, v.x);
      if (2 * u + 1 < (uint32_t)a.B) a.buf0[(size_t)(2 * u + 1) * a.N + i] = make_float2(r.y, v.y);
    }
  }
  }
}

// Forward: checkpoint slot (standard layout, fp32 or bf16 round-to-nearest-even).
template <bool SLOW>
__device__ void store_ckpt_fwd(const PassArgs& a, int slot, const DevPhase& ph,
                               const ThreadCtx& tc, const float2 (&re)[kPos],
                               const float2 (&im)[kPos], int bmax) {
  const RegMaps m = reg_maps(ph);
  if constexpr (!SLOW) {
    const uint32_t u = tc.ut;
    if (u >= (uint32_t)a.U) return;
    const size_t e0 = ((size_t)slot * bmax + 2 * u) * a.N + tc.aq;
    const bool has1 = 2 * u + 1 < (uint32_t)a.B;
    if (a.storage == 0) {
      float2* s0 = reinterpret_cast<float2*>(a.ckpt) + e0;
      float2* s1 = s0 + a.N;
#pragma unroll
      for (int j = 0; j < kPos; ++j) {
        const uint32_t b = REG_COMBINE(m.q, j, |=);
        s0[b] = make_float2(re[j].x, im[j].x);
        if (has1) s1[b] = make_float2(re[j].y, im[j].y);
      }
    } else {
      __nv_bfloat162* s0 = reinterpret_cast<__nv_bfloat162*>(a.ckpt) + e0;
      __nv_bfloat162* s1 = s0 + a.N;
#pragma unroll
      for (int j = 0; j < kPos; ++j) {
        const uint32_t b = REG_COMBINE(m.q, j, |=);
        s0[b] = __floats2bfloat162_rn(re[j].x, im[j].x);
        if (has1) s1[b] = __floats2bfloat162_rn(re[j].y, im[j].y);
      }
    }
  } else {
#pragma unroll 1
  for (int j = 0; j < kPos; ++j) {
    uint32_t u = tc.ut, i = tc.aq;
    for (int k = 0; k < kRegBits; ++k)
      if (j & (1 << k)) { u += m.u[k]; i |= m.q[k]; }
    if (u >= (uint32_t)a.U) continue;
    const float2 r = sel(re, j), v = sel(im, j);
    const size_t e0 = ((size_t)slot * bmax + 2 * u) * a.N + i;
    const bool has1 = 2 * u + 1 < (uint32_t)a.B;
    if (a.storage == 0) {
      float2* s = reinterpret_cast<float2*>(a.ckpt);
      s[e0] = make_float2(r.x, v.x);
      if (has1) s[e0 + a.N] = make_float2(r.y, v.y);
    } else {
      __nv_bfloat162* s = reinterpret_cast<__nv_bfloat162*>(a.ckpt);
      s[e0] = __floats2bfloat162_rn(r.x, v.x);
      if (has1) s[e0 + a.N] = __floats2bfloat162_rn(r.y, v.y);
    }
  }
  }
}

// Backward: replace the psi lanes by the checkpointed state of slot `slot`.
template <bool SLOW>
__device__ void restore_ckpt_bwd(const PassArgs& a, int slot, const DevPhase& ph,
                                 const ThreadCtx& tc, float2 (&re)[kPos], float2 (&im)[kPos],
                                 int bmax) {
  const RegMaps m = reg_maps(ph);
  if constexpr (!SLOW) {
    const uint32_t u = tc.ut;
    if (u >= (uint32_t)a.U) return;
    const size_t e = ((size_t)slot * bmax + u) * a.N + tc.aq;
#pragma unroll
    for (int j = 0; j < kPos; ++j) {
      const uint32_t b = REG_COMBINE(m.q, j, |=);
      float2 v;
      if (a.storage == 0) v = reinterpret_cast<const float2*>(a.ckpt)[e + b];
      else v = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.ckpt)[e + b]);
      re[j].x = v.x;
      im[j].x = v.y;
    }
  } else {
#pragma unroll 1
  for (int j = 0; j < kPos; ++j) {
    uint32_t u, i;
    pos_of(m, tc, j, &u, &i);
    if (u >= (uint32_t)a.U) continue;
    const size_t e = ((size_t)slot * bmax + u) * a.N + i;
    float2 v;
    if (a.storage == 0) v = reinterpret_cast<const float2*>(a.ckpt)[e];
    else v = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.ckpt)[e]);
    float2 r = sel(re, j), w = sel(im, j);
    r.x = v.x;
    w.x = v.y;
    put(re, j, r);
    put(im, j, w);
  }
  }
}

// Forward: the angle-encoded product state prod_q (cos, sin)(x_q/2)[bit q].
template <bool SLOW>
__device__ void gen_state(const PassArgs& a, const DevPhase& ph, const ThreadCtx& tc,
                          float2 (&re)[kPos], float2 (&im)[kPos]) {
  const RegMaps m = reg_maps(ph);
  const int n = a.n;
  if constexpr (!SLOW) {
    if (tc.ut >= (uint32_t)a.U) {
#pragma unroll
      for (int j = 0; j < kPos; ++j) re[j] = im[j] = make_float2(0.f, 0.f);
      return;
    }
    const float2* e = a.enc + (size_t)tc.ut * n * 2;
    uint32_t regq = 0;
#pragma unroll
    for (int k = 0; k < kRegBits; ++k) regq |= m.q[k];
    float2 c = make_float2(1.f, 1.f);
    for (int q = 0; q < n; ++q)
      if (!((regq >> q) & 1u)) c = __fmul2_rn(c, __ldg(&e[2 * q + ((tc.aq >> q) & 1u)]));
    float2 e0[kRegBits], e1[kRegBits];
#pragma unroll
    for (int k = 0; k < kRegBits; ++k) {
      const int q = ph.reg_q[k];
      e0[k] = __ldg(&e[2 * q]);
      e1[k] = __ldg(&e[2 * q + 1]);
    }
#pragma unroll
    for (int j = 0; j < kPos; ++j) {
      float2 v = c;
#pragma unroll
      for (int k = 0; k < kRegBits; ++k) v = __fmul2_rn(v, (j & (1 << k)) ? e1[k] : e0[k]);
      re[j] = v;
      im[j] = make_float2(0.f, 0.f);
    }
  } else {
#pragma unroll 1
    for (int j = 0; j < kPos; ++j) {
      uint32_t u, i;
      pos_of(m, tc, j, &u, &i);
      float2 v = make_float2(0.f, 0.f);
      if (u < (uint32_t)a.U) {
        const float2* e = a.enc + (size_t)u * n * 2;
        v = make_float2(1.f, 1.f);
        for (int q = 0; q < n; ++q) v = __fmul2_rn(v, __ldg(&e[2 * q + ((i >> q) & 1u)]));
      }
      put(re, j, v);
      put(im, j, make_float2(0.f, 0.f));
    }
  }
}

// ----------------------------------------------------------- the pass kernel

template <bool BWD, bool SLOW>
__global__ void __launch_bounds__(kThreads, 2) pass_kernel(const PassArgs a) {
  const int bmax = a.bmax;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float4* tile = reinterpret_cast<float4*>(smem_raw);
  unsigned char* prog = smem_raw + (size_t)kTilePos * sizeof(float4);
  DevPass* P = reinterpret_cast<DevPass*>(prog);
  const DevPass& gp = a.passes[a.pass_idx];
  DevPhase* PH = reinterpret_cast<DevPhase*>(prog + ((sizeof(DevPass) + 15) & ~size_t(15)));
  const int tid = threadIdx.x;

  // copy the pass program into shared memory
  {
    const int* src = reinterpret_cast<const int*>(&gp);
    int* dst = reinterpret_cast<int*>(P);
    for (int i = tid; i < (int)(sizeof(DevPass) / 4); i += kThreads) dst[i] = src[i];
  }
  __syncthreads();
  DevOp* OPS = reinterpret_cast<DevOp*>(reinterpret_cast<unsigned char*>(PH) +
                                       sizeof(DevPhase) * P->nphases);
  {
    const int* src = reinterpret_cast<const int*>(a.phases + P->phase0);
    int* dst = reinterpret_cast<int*>(PH);
    for (int i = tid; i < (int)(P->nphases * sizeof(DevPhase) / 4); i += kThreads) dst[i] = src[i];
    const int* so = reinterpret_cast<const int*>(a.ops + P->op0);
    int* dso = reinterpret_cast<int*>(OPS);
    for (int i = tid; i < P->nops * 4; i += kThreads) dso[i] = so[i];
  }
  constexpr int kWarps = kThreads / 32;
  float* acc = reinterpret_cast<float*>(prog + a.smem_prog);  // [warps][nslots*3]
  const int nacc = P->nslots * 3;
  if (BWD)
    for (int i = tid; i < kWarps * nacc; i += kThreads) acc[i] = 0.f;
  __syncthreads();

  const int n_out = P->n_out;
  const int warp = tid >> 5, lane = tid & 31;

  for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
    const uint32_t o = (uint32_t)t & ((1u << n_out) - 1u);
    const uint32_t ug = (uint32_t)t >> n_out;
    uint32_t base_q = 0;
    for (int k = 0; k < n_out; ++k)
      if ((o >> k) & 1u) base_q |= 1u << P->out_q[k];
    const uint32_t unit_base = ug << P->unit_bits;

    float2 re[kPos], im[kPos];
    int cur = BWD ? P->store_phase : P->load_phase;
    {
      const ThreadCtx tc = thread_ctx(PH[cur], tid, base_q, unit_base);
      if (!BWD) {
        if (P->gen) gen_state<SLOW>(a, PH[cur], tc, re, im);
        else load_planes<false, SLOW>(a, PH[cur], tc, re, im);
      } else {
        load_planes<true, SLOW>(a, PH[cur], tc, re, im);
        if (P->ckpt >= 0) restore_ckpt_bwd<SLOW>(a, P->ckpt, PH[cur], tc, re, im, bmax);
      }
    }

    if (!BWD) {
      for (int oi = 0; oi < P->nops; ++oi) {
        const DevOp op = OPS[oi];
        if (op.kind == OP_EXCH) {
          exchange(re, im, tile, PH[op.a], PH[op.b], tid);
          cur = op.b;
        } else if (op.kind == OP_ROT) {
          for (int k = 0; k < kRegBits; ++k)
            if ((op.b >> k) & 1) {
              const int q = PH[cur].reg_q[k];
              const Coef c = load_coef(a.coef + ((size_t)op.a * a.n + q) * 4);
              rot_fwd_k(k, re, im, c);
            }
        } else if (op.kind == OP_CZ) {
          const ThreadCtx tc = thread_ctx(PH[cur], tid, base_q, unit_base);
          apply_cz(re, im, PH[cur], tc.aq);
        }
      }
      const ThreadCtx tc = thread_ctx(PH[cur], tid, base_q, unit_base);
      if (P->ckpt >= 0) store_ckpt_fwd<SLOW>(a, P->ckpt, PH[cur], tc, re, im, bmax);
      if (P->last) store_standard_fwd<SLOW>(a, PH[cur], tc, re, im);
      else store_planes<false, SLOW>(a, PH[cur], tc, re, im);
    } else {
      for (int oi = P->nops - 1; oi >= 0; --oi) {
        const DevOp op = OPS[oi];
        if (op.kind == OP_EXCH) {
          exchange(re, im, tile, PH[op.b], PH[op.a], tid);
          cur = op.a;
        } else if (op.kind == OP_ROT) {
          for (int k = kRegBits - 1; k >= 0; --k)
            if ((op.b >> k) & 1) {
              const int q = PH[cur].reg_q[k];
              const Coef c = load_coef(a.coef + ((size_t)op.a * a.n + q) * 4);
              float3 s = rot_bwd_k(k, re, im, c);
              s.x = warp_sum(s.x);
              s.y = warp_sum(s.y);
              s.z = warp_sum(s.z);
              if (lane == 0) {
                const int slot = op.c + __popc((unsigned)op.b & ((1u << k) - 1u));
                float* w = acc + warp * nacc + slot * 3;
                w[0] += s.x;
                w[1] += s.y;
                w[2] += s.z;
              }
            }
        } else if (op.kind == OP_CZ) {
          const ThreadCtx tc = thread_ctx(PH[cur], tid, base_q, unit_base);
          apply_cz(re, im, PH[cur], tc.aq);
        }
      }
      if (!P->gen) {
        const ThreadCtx tc = thread_ctx(PH[cur], tid, base_q, unit_base);
        store_planes<true, SLOW>(a, PH[cur], tc, re, im);
      }
    }
  }

  if (BWD) {
    __syncthreads();
    float* out = a.partials + P->partial_off + (size_t)blockIdx.x * nacc;
    for (int i = tid; i < nacc; i += kThreads) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += acc[w * nacc + i];
      out[i] = v;
    }
  }
}

// ----------------------------------------------------------------- helpers

// Gate coefficients of U = Rz(g) Ry(b) Rx(a) = [[A, B], [-conj B, conj A]] in
// fp64, rounded to fp32 broadcast pairs, and of U^dagger = [[conj A, -B], ...].
__global__ void prep_coef_kernel(const float* theta, int L, int n, float4* cf, float4* ci) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= L * n) return;
  const double al = theta[idx * 3 + 0], be = theta[idx * 3 + 1], ga = theta[idx * 3 + 2];
  double sa, ca, sb, cb, sg, cg;
  sincos(0.5 * al, &sa, &ca);
  sincos(0.5 * be, &sb, &cb);
  sincos(0.5 * ga, &sg, &cg);
  // e^{-i g/2} = cg - i sg
  const double p_re = cb * ca, p_im = sb * sa;     // (Ry Rx)[0][0]
  const double q_re = -sb * ca, q_im = -cb * sa;   // (Ry Rx)[0][1]
  const double ar = cg * p_re + sg * p_im, ai = cg * p_im - sg * p_re;
  const double br = cg * q_re + sg * q_im, bi = cg * q_im - sg * q_re;
  const float far = (float)ar, fai = (float)ai, fbr = (float)br, fbi = (float)bi;
  cf[idx * 4 + 0] = make_float4(far, far, fai, fai);
  cf[idx * 4 + 1] = make_float4(-fai, -fai, fbr, fbr);
  cf[idx * 4 + 2] = make_float4(fbi, fbi, -fbi, -fbi);
  cf[idx * 4 + 3] = make_float4(-fbr, -fbr, 0.f, 0.f);
  // U^dagger: A' = conj A, B' = -B
  ci[idx * 4 + 0] = make_float4(far, far, -fai, -fai);
  ci[idx * 4 + 1] = make_float4(fai, fai, -fbr, -fbr);
  ci[idx * 4 + 2] = make_float4(-fbi, -fbi, fbi, fbi);
  ci[idx * 4 + 3] = make_float4(fbr, fbr, 0.f, 0.f);
}

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
__global__ void grad_reduce_kernel(const DevPass* passes, const int* slot_pass,
                                   const int* slot_index, const float* partials, int grid,
                                   const float* theta, int L, int n, float* grad,
                                   unsigned* status) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= L * n) return;
  const int p = slot_pass[idx], s = slot_index[idx];
  const DevPass& ps = passes[p];
  const int stride = ps.nslots * 3;
  const float* base = partials + ps.partial_off + s * 3;
  double sx = 0.0, sy = 0.0, sz = 0.0;
  for (int c = 0; c < grid; ++c) {
    sx += base[(size_t)c * stride + 0];
    sy += base[(size_t)c * stride + 1];
    sz += base[(size_t)c * stride + 2];
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

size_t pass_smem_bytes(int prog_bytes, int max_slots) {
  return (size_t)kTilePos * sizeof(float4) + (size_t)prog_bytes + (size_t)(kThreads / 32) * max_slots * 3 * sizeof(float);
}

cudaError_t set_pass_smem_attr(size_t smem) {
  const int v = (int)smem;
  cudaError_t e = cudaFuncSetAttribute(pass_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, v);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(pass_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, v);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(pass_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, v);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(pass_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, v);
  return e;
}

cudaError_t pass_occupancy(bool backward, bool slow, size_t smem, int* blocks_per_sm) {
  if (backward)
    return slow ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<true, true>, kThreads, smem)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<true, false>, kThreads, smem);
  return slow ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<false, true>, kThreads, smem)
              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, pass_kernel<false, false>, kThreads, smem);
}

cudaError_t launch_pass(bool backward, bool slow, const PassArgs& a, int grid, size_t smem, cudaStream_t s) {
  if (backward) {
    if (slow) pass_kernel<true, true><<<grid, kThreads, smem, s>>>(a);
    else pass_kernel<true, false><<<grid, kThreads, smem, s>>>(a);
  } else {
    if (slow) pass_kernel<false, true><<<grid, kThreads, smem, s>>>(a);
    else pass_kernel<false, false><<<grid, kThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_prep_coef(const float* theta, int L, int n, float4* cf, float4* ci,
                             cudaStream_t s) {
  const int tot = L * n;
  prep_coef_kernel<<<(tot + 127) / 128, 128, 0, s>>>(theta, L, n, cf, ci);
  return cudaGetLastError();
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

cudaError_t launch_grad_reduce(const DevPass* passes, const int* slot_pass, const int* slot_index,
                               const float* partials, int grid, const float* theta, int L, int n,
                               float* grad, unsigned* status, cudaStream_t s) {
  const int tot = L * n;
  grad_reduce_kernel<<<(tot + 127) / 128, 128, 0, s>>>(passes, slot_pass, slot_index, partials,
                                                       grid, theta, L, n, grad, status);
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
