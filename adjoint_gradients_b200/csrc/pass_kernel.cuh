// pass_kernel.cuh -- the fused pass kernel of the HEA forward / adjoint path
// and its device helpers, included by the translation units that instantiate
// it (pass_split.cu, pass_fused.cu, pass_reup.cu: compiled in parallel) and by
// kernels.cu (which uses the layout helpers only).
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
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "kernels.cuh"

namespace qml {

namespace {

// Gate coefficients of the current pass, per context region (CoefRegion in
// kernels.cuh).  Read through the constant cache with warp-uniform indices,
// they feed the packed FMAs from uniform registers instead of the vector
// register file.  Each translation unit that includes this file has its own
// copy, filled by its own launch function (QML_DEFINE_PASS_UNIT below).
__constant__ CoefRegion c_reg[kCoefRegions];

constexpr unsigned kErrNumeric = 1u << 6;  // bit (QML_ERR_NUMERIC)
constexpr unsigned kErrBounds = 1u << 7;   // bit (QML_ERR_BOUNDS)
constexpr unsigned kErrTimeout = 1u << 8;  // bit (QML_ERR_TIMEOUT)
// Polls of an mbarrier before a wait is declared failed (each poll may
// suspend the thread briefly, so this bounds the wait to well under a second).
constexpr uint32_t kWaitLimit = 1u << 22;

// ---------------------------------------------------------------- gate math

struct Coef {
  float2 ar, ai, nai, br, bi, nbi, nbr;  // broadcast (v, v) pairs
};

__device__ __forceinline__ Coef const_coef(int region, int slot) {
  const float4 f0 = c_reg[region].rot[slot][0], f1 = c_reg[region].rot[slot][1];
  const float4 f2 = c_reg[region].rot[slot][2], f3 = c_reg[region].rot[slot][3];
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
// Term order: every x term comes first, so x is dead before the last term of
// each output, and the final terms read only the y value that is overwritten
// by, or already consumed before, the instruction that writes them.  The
// results can then land in the registers of (x, y) without extra moves.
__device__ __forceinline__ void su2(float2& xr, float2& xi, float2& yr, float2& yi, const Coef& c) {
  float2 o0r = __fmul2_rn(c.ar, xr);
  float2 o0i = __fmul2_rn(c.ar, xi);
  float2 o1r = __fmul2_rn(c.nbr, xr);
  float2 o1i = __fmul2_rn(c.nbr, xi);
  o0r = __ffma2_rn(c.nai, xi, o0r);
  o0i = __ffma2_rn(c.ai, xr, o0i);
  o1r = __ffma2_rn(c.nbi, xi, o1r);
  o1i = __ffma2_rn(c.bi, xr, o1i);
  o0r = __ffma2_rn(c.br, yr, o0r);
  o0i = __ffma2_rn(c.br, yi, o0i);
  o1r = __ffma2_rn(c.ai, yi, o1r);
  o1i = __ffma2_rn(c.nai, yr, o1i);
  xr = __ffma2_rn(c.nbi, yi, o0r);
  xi = __ffma2_rn(c.bi, yr, o0i);
  yr = __ffma2_rn(c.ar, yr, o1r);
  yi = __ffma2_rn(c.ar, yi, o1i);
}

// cf(j) gives the coefficients for register pair (j, j | 1 << K).
template <int K, class CF>
__device__ __forceinline__ void rot_fwd(float2 (&re)[kPos], float2 (&im)[kPos], const CF& cf) {
#pragma unroll
  for (int j = 0; j < kPos; ++j)
    if (!(j & (1 << K))) su2(re[j], im[j], re[j | (1 << K)], im[j | (1 << K)], cf(j));
}

// The same coefficients for every register pair.
struct SameCoef {
  Coef c;
  __device__ __forceinline__ Coef operator()(int) const { return c; }
};

__device__ __forceinline__ float2 swap2(float2 v) { return make_float2(v.y, v.x); }

template <class CF>
__device__ __forceinline__ void rot_fwd_k(int k, float2 (&re)[kPos], float2 (&im)[kPos], const CF& cf) {
  static_assert(kRegBits == 5, "dispatch below covers five register bits");
  switch (k) {
    case 0: rot_fwd<0>(re, im, cf); break;
    case 1: rot_fwd<1>(re, im, cf); break;
    case 2: rot_fwd<2>(re, im, cf); break;
    case 3: rot_fwd<3>(re, im, cf); break;
    default: rot_fwd<4>(re, im, cf); break;
  }
}

// Split form: the real rotation Ry on register pairs (x, y) = (j, j | 1 << K)
// with one packed FMA per output, p = (t, t) and np = (-t, -t):
//   tangent form   x <- x + np y,  y <- y + p x   ([[1, -t], [t, 1]] for p = t)
//   cotangent form x <- y + np x,  y <- x + p y   ([[-u, 1], [1, u]] for p = u)
// The backward pass un-applies a tangent-form rotation with p = -t (the
// inverse up to the scale 1 + t^2) and a cotangent-form one with the same p
// (that matrix squares to (1 + u^2) I).
// INPLACE (tangent form only): no copy of the old x: x <- x - t y, then
// y <- t x' + (1 + t^2) y (= y + t x; q = (1 + t^2, 1 + t^2)); one more
// packed product per output pair, and no register moves.  Measured faster in
// the tensor-copy passes whose rotations are all in tangent form (the
// flip-tracked ones), slower where the two forms mix.
template <bool COT, bool INPLACE = false>
__device__ __forceinline__ void ry_pair(float2& xr, float2& xi, float2& yr, float2& yi, float2 p, float2 np,
                                        float2 q) {
  const float2 x0r = xr, x0i = xi;
  if (!COT && INPLACE) {
    xr = __ffma2_rn(np, yr, xr);
    xi = __ffma2_rn(np, yi, xi);
    yr = __ffma2_rn(p, xr, __fmul2_rn(q, yr));
    yi = __ffma2_rn(p, xi, __fmul2_rn(q, yi));
  } else if (!COT) {
    xr = __ffma2_rn(np, yr, x0r);
    xi = __ffma2_rn(np, yi, x0i);
    yr = __ffma2_rn(p, x0r, yr);
    yi = __ffma2_rn(p, x0i, yi);
  } else {
    xr = __ffma2_rn(np, x0r, yr);
    xi = __ffma2_rn(np, x0i, yi);
    yr = __ffma2_rn(p, yr, x0r);
    yi = __ffma2_rn(p, yi, x0i);
  }
}

template <int K, bool COT, bool INPLACE>
__device__ __forceinline__ void ry_fwd(float2 (&re)[kPos], float2 (&im)[kPos], float2 p, float2 np, float2 q) {
#pragma unroll
  for (int j = 0; j < kPos; ++j)
    if (!(j & (1 << K))) ry_pair<COT, INPLACE>(re[j], im[j], re[j | (1 << K)], im[j | (1 << K)], p, np, q);
}

template <bool COT, bool INPLACE = false>
__device__ __forceinline__ void ry_fwd_k(int k, float2 (&re)[kPos], float2 (&im)[kPos], float2 p, float2 np) {
  const float2 q = INPLACE ? __ffma2_rn(p, p, make_float2(1.f, 1.f)) : make_float2(0.f, 0.f);
  switch (k) {
    case 0: ry_fwd<0, COT, INPLACE>(re, im, p, np, q); break;
    case 1: ry_fwd<1, COT, INPLACE>(re, im, p, np, q); break;
    case 2: ry_fwd<2, COT, INPLACE>(re, im, p, np, q); break;
    case 3: ry_fwd<3, COT, INPLACE>(re, im, p, np, q); break;
    default: ry_fwd<4, COT, INPLACE>(re, im, p, np, q); break;
  }
}

// Complex-lane form (the one-sample forward of single-tile circuits, RE 5):
// a register pair is one amplitude (re, im).  Ry is real, so the same
// packed FMAs as ry_pair apply to the pair, one per output amplitude.
template <int K, bool COT>
__device__ __forceinline__ void ry1_fwd(float2 (&z)[kPos], float2 p, float2 np) {
#pragma unroll
  for (int j = 0; j < kPos; ++j)
    if (!(j & (1 << K))) {
      const float2 x = z[j], y = z[j | (1 << K)];
      if (!COT) {
        z[j] = __ffma2_rn(np, y, x);
        z[j | (1 << K)] = __ffma2_rn(p, x, y);
      } else {
        z[j] = __ffma2_rn(np, x, y);
        z[j | (1 << K)] = __ffma2_rn(p, y, x);
      }
    }
}

template <bool COT>
__device__ __forceinline__ void ry1_fwd_k(int k, float2 (&z)[kPos], float2 p, float2 np) {
  switch (k) {
    case 0: ry1_fwd<0, COT>(z, p, np); break;
    case 1: ry1_fwd<1, COT>(z, p, np); break;
    case 2: ry1_fwd<2, COT>(z, p, np); break;
    case 3: ry1_fwd<3, COT>(z, p, np); break;
    default: ry1_fwd<4, COT>(z, p, np); break;
  }
}

// Applier of a register pair's 2x2 gate for rot_bwd_red: the fused SU(2)
// with per-pair coefficients.
template <class CF>
struct Su2Ap {
  CF cf;
  __device__ __forceinline__ void operator()(int j, float2& xr, float2& xi, float2& yr, float2& yi) const {
    su2(xr, xi, yr, yi, cf(j));
  }
};

// Gradient terms of one qubit at the state just after its fused rotation, then
// U^dagger on psi and lambda.  With psi in lane x and lambda in lane y:
//   s_z = Im<lambda|Z|psi>, s_x = Im<lambda|X|psi>, s_y = Im<lambda|Y|psi>.
// 2 Re<lambda|(-i/2) P|psi> = Im<lambda|P|psi>, so these are the gradients of
// the three rotation angles up to a known rotation (applied in grad_reduce).
// The products lambda * psi are formed as packed products of a pair with a
// lane-swapped pair, e.g. (p0r, l0r) * (l0i, p0i) = (p0r l0i, l0r p0i), whose
// lane difference is Im(conj(l0) p0); the differences are taken at the end.
// The same call also finishes the warp sum of the previous qubit's terms
// (pv): the shuffle steps of warp_reduce3 are spread over the pair loop so
// that their latency hides behind this qubit's FMAs.  *r_prev receives the
// sum as warp_reduce3 returns it.  ap(j, ...) un-applies the gate on register
// pair (j, j | 1 << K).
template <int K, class AP>
__device__ __forceinline__ float3 rot_bwd_red(float2 (&re)[kPos], float2 (&im)[kPos], const AP& ap, float3 pv,
                                              int lane, float* r_prev) {
  const bool h16 = (lane & 16) != 0, h8 = (lane & 8) != 0;
  float k0 = h16 ? pv.z : pv.x, k1 = h16 ? 0.f : pv.y;
  const float s0 = h16 ? pv.x : pv.z, s1 = h16 ? pv.y : 0.f;
  float v = 0.f;
  float2 ax = make_float2(0.f, 0.f), ay = ax, az0 = ax, az1 = ax;
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    if (j & (1 << K)) continue;
    const int pi = (j & ((1 << K) - 1)) | ((j >> (K + 1)) << K);  // pair index 0..15
    if (pi == 0) {
      k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
      k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    } else if (pi == 3) {
      v = h8 ? k1 : k0;
      v += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
    } else if (pi == 6) {
      v += __shfl_xor_sync(0xffffffffu, v, 4);
    } else if (pi == 9) {
      v += __shfl_xor_sync(0xffffffffu, v, 2);
    } else if (pi == 12) {
      v += __shfl_xor_sync(0xffffffffu, v, 1);
    }
    const int jj = j | (1 << K);
    const float2 si0 = swap2(im[j]), si1 = swap2(im[jj]), sr1 = swap2(re[jj]);
    az0 = __ffma2_rn(re[j], si0, az0);   // y - x: Im(conj l0 p0)
    az1 = __ffma2_rn(re[jj], si1, az1);  // y - x: Im(conj l1 p1)
    ax = __ffma2_rn(re[j], si1, ax);     // y - x: l0r p1i - p0r l1i
    ax = __ffma2_rn(re[jj], si0, ax);    // y - x: l1r p0i - p1r l0i
    ay = __ffma2_rn(re[j], sr1, ay);     // x - y: p0r l1r - l0r p1r
    ay = __ffma2_rn(im[j], si1, ay);     // x - y: p0i l1i - l0i p1i
    ap(j, re[j], im[j], re[jj], im[jj]);
  }
  *r_prev = v;
  return make_float3(ax.y - ax.x, ay.x - ay.y, (az0.y - az0.x) - (az1.y - az1.x));
}

// Split form: only the gradient sums of qubit K (with the warp sum of the
// previous qubit finished inside, as in rot_bwd_red); the caller then
// un-applies Ry with ry_fwd.
template <int K>
__device__ __forceinline__ float3 rot_bwd_sums(const float2 (&re)[kPos], const float2 (&im)[kPos], float3 pv,
                                               int lane, float* r_prev) {
  const bool h16 = (lane & 16) != 0, h8 = (lane & 8) != 0;
  float k0 = h16 ? pv.z : pv.x, k1 = h16 ? 0.f : pv.y;
  const float s0 = h16 ? pv.x : pv.z, s1 = h16 ? pv.y : 0.f;
  float v = 0.f;
  float2 ax = make_float2(0.f, 0.f), ay = ax, az0 = ax, az1 = ax;
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    if (j & (1 << K)) continue;
    const int pi = (j & ((1 << K) - 1)) | ((j >> (K + 1)) << K);
    if (pi == 0) {
      k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
      k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
    } else if (pi == 3) {
      v = h8 ? k1 : k0;
      v += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
    } else if (pi == 6) {
      v += __shfl_xor_sync(0xffffffffu, v, 4);
    } else if (pi == 9) {
      v += __shfl_xor_sync(0xffffffffu, v, 2);
    } else if (pi == 12) {
      v += __shfl_xor_sync(0xffffffffu, v, 1);
    }
    const int jj = j | (1 << K);
    const float2 si0 = swap2(im[j]), si1 = swap2(im[jj]), sr1 = swap2(re[jj]);
    az0 = __ffma2_rn(re[j], si0, az0);
    az1 = __ffma2_rn(re[jj], si1, az1);
    ax = __ffma2_rn(re[j], si1, ax);
    ax = __ffma2_rn(re[jj], si0, ax);
    ay = __ffma2_rn(re[j], sr1, ay);
    ay = __ffma2_rn(im[j], si1, ay);
  }
  *r_prev = v;
  return make_float3(ax.y - ax.x, ay.x - ay.y, (az0.y - az0.x) - (az1.y - az1.x));
}

__device__ __forceinline__ float3 rot_bwd_sums_k(int k, const float2 (&re)[kPos], const float2 (&im)[kPos],
                                                 float3 pv, int lane, float* r_prev) {
  switch (k) {
    case 0: return rot_bwd_sums<0>(re, im, pv, lane, r_prev);
    case 1: return rot_bwd_sums<1>(re, im, pv, lane, r_prev);
    case 2: return rot_bwd_sums<2>(re, im, pv, lane, r_prev);
    case 3: return rot_bwd_sums<3>(re, im, pv, lane, r_prev);
    default: return rot_bwd_sums<4>(re, im, pv, lane, r_prev);
  }
}

template <class AP>
__device__ __forceinline__ float3 rot_bwd_red_ap(int k, float2 (&re)[kPos], float2 (&im)[kPos], const AP& ap,
                                                 float3 pv, int lane, float* r_prev) {
  switch (k) {
    case 0: return rot_bwd_red<0>(re, im, ap, pv, lane, r_prev);
    case 1: return rot_bwd_red<1>(re, im, ap, pv, lane, r_prev);
    case 2: return rot_bwd_red<2>(re, im, ap, pv, lane, r_prev);
    case 3: return rot_bwd_red<3>(re, im, ap, pv, lane, r_prev);
    default: return rot_bwd_red<4>(re, im, ap, pv, lane, r_prev);
  }
}

template <class CF>
__device__ __forceinline__ float3 rot_bwd_red_k(int k, float2 (&re)[kPos], float2 (&im)[kPos], const CF& cf,
                                                float3 pv, int lane, float* r_prev) {
  return rot_bwd_red_ap(k, re, im, Su2Ap<CF>{cf}, pv, lane, r_prev);
}

// Data re-uploading: Ry(x_q) (forward) or Ry(-x_q) (backward) on qubit K's
// register pairs, with per-sample angles.  Forward lanes are two samples, so
// the (cos, sin)(x/2) pairs are per lane; backward lanes are psi and lambda of
// one sample, so both lanes take that sample's values.
template <bool BWD>
__device__ __forceinline__ void enc_coef(const PassArgs& a, uint32_t unit, int q, float2* c, float2* s) {
  if (!BWD) {
    const float2* e = a.enc + ((size_t)unit * a.n + q) * 2;
    *c = __ldg(&e[0]);
    *s = __ldg(&e[1]);
  } else {
    const float2* e = a.enc + ((size_t)(unit >> 1) * a.n + q) * 2;
    const float2 c2 = __ldg(&e[0]), s2 = __ldg(&e[1]);
    const float cv = (unit & 1u) ? c2.y : c2.x, sv = (unit & 1u) ? s2.y : s2.x;
    *c = make_float2(cv, cv);
    *s = make_float2(sv, sv);
  }
}

// Data re-uploading folded into the layer's rotation: the SU(2) coefficients
// of U Ry(x) (forward, c holding U) or of Ry(-x) U^dagger (backward, c holding
// U^dagger), with (cs, sn) = (cos, sin)(x/2) per lane.  With U = [[a, b],
// [-conj b, conj a]]: U Ry(x) has a' = a cs + b sn, b' = b cs - a sn, and
// Ry(-x) U^dagger has a' = a cs - conj(b) sn, b' = b cs + conj(a) sn.
template <bool BWD>
__device__ __forceinline__ Coef reup_coef(const Coef& c, float2 cs, float2 sn) {
  const float2 nsn = make_float2(-sn.x, -sn.y);
  Coef m;
  if (!BWD) {
    m.ar = __ffma2_rn(c.br, sn, __fmul2_rn(c.ar, cs));
    m.ai = __ffma2_rn(c.bi, sn, __fmul2_rn(c.ai, cs));
    m.nai = __ffma2_rn(c.nbi, sn, __fmul2_rn(c.nai, cs));
    m.br = __ffma2_rn(c.ar, nsn, __fmul2_rn(c.br, cs));
    m.bi = __ffma2_rn(c.nai, sn, __fmul2_rn(c.bi, cs));
    m.nbi = __ffma2_rn(c.ai, sn, __fmul2_rn(c.nbi, cs));
    m.nbr = __ffma2_rn(c.ar, sn, __fmul2_rn(c.nbr, cs));
  } else {
    m.ar = __ffma2_rn(c.nbr, sn, __fmul2_rn(c.ar, cs));
    m.ai = __ffma2_rn(c.bi, sn, __fmul2_rn(c.ai, cs));
    m.nai = __ffma2_rn(c.nbi, sn, __fmul2_rn(c.nai, cs));
    m.br = __ffma2_rn(c.ar, sn, __fmul2_rn(c.br, cs));
    m.bi = __ffma2_rn(c.nai, sn, __fmul2_rn(c.bi, cs));
    m.nbi = __ffma2_rn(c.ai, sn, __fmul2_rn(c.nbi, cs));
    m.nbr = __ffma2_rn(c.ar, nsn, __fmul2_rn(c.nbr, cs));
  }
  return m;
}

// U Ry(x) (forward) or Ry(-x) U^dagger (backward) per register pair, for
// register bits that also span batch units: pair j takes the coefficients of
// its own unit (unit plus the mu[k] of its set bits; mu[k] is 0 unless
// register bit k is a batch-unit bit, which happens only for n < 10).
template <bool BWD>
struct ReupPairCoef {
  Coef c;
  const PassArgs& a;
  int q;
  uint32_t unit;
  const uint32_t (&mu)[kRegBits];
  __device__ __forceinline__ Coef operator()(int j) const {
    uint32_t du = 0;
#pragma unroll
    for (int k = 0; k < kRegBits; ++k)
      if ((j >> k) & 1) du += mu[k];
    // padding units past the batch hold zero amplitudes; their angles are
    // not written, so take unit 0's (any finite coefficients keep them zero)
    const uint32_t u = unit + du < (uint32_t)a.U ? unit + du : 0u;
    float2 cs, sn;
    enc_coef<BWD>(a, u, q, &cs, &sn);
    return reup_coef<BWD>(c, cs, sn);
  }
};

// Sum (a, b, c) over the warp with six shuffles; afterwards lanes 0, 8 and 16
// hold the totals of a, b and c.
__device__ __forceinline__ float warp_reduce3(float a, float b, float c, int lane) {
  // 4 values (a, b, c, 0) over 32 lanes: halve the value count at offsets 16 and 8
  const bool h16 = (lane & 16) != 0;
  float k0 = h16 ? c : a, k1 = h16 ? 0.f : b;
  const float s0 = h16 ? a : c, s1 = h16 ? b : 0.f;
  k0 += __shfl_xor_sync(0xffffffffu, s0, 16);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 16);
  const bool h8 = (lane & 8) != 0;
  float v = h8 ? k1 : k0;
  v += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;  // value index (lane >> 3): 0 = a, 1 = b, 2 = c, 3 = pad
}

__device__ __forceinline__ void flip(float2& v, uint32_t signbit) {
  v.x = __uint_as_float(__float_as_uint(v.x) ^ signbit);
  v.y = __uint_as_float(__float_as_uint(v.y) ^ signbit);
}

// ------------------------------------------------------------ tile geometry

// Shared-memory slot (16 bytes) of tile position t: slot(t) = sum over the set
// bits b of t of wbit(b), i.e. t plus one pad slot every 32 positions plus a
// small offset for tile bits 10 and 11.  The map is injective and additive
// over disjoint bits, so register offsets are compile-time constants, and in
// every layout below the eight lanes of a quarter warp (one 128-byte
// wavefront of 16-byte accesses) hit eight different bank groups.
__host__ __device__ constexpr uint32_t wbit(int b) {
  return b < 5 ? (1u << b) : (1u << b) + (1u << (b - 5)) + (b == 10 ? 2u : b == 11 ? 4u : 0u);
}

// Tile bit addressed by register-index bit k in phase P.
template <int P>
__host__ __device__ constexpr int reg_tbit(int k) {
  return P == 0 ? k : P == 1 ? 5 + k : (k < 2 ? 10 + k : k - 2);
}

// Tile bit addressed by thread-index bit m in phase P (V: layout variant).
template <int P, int V>
__host__ __device__ constexpr int thr_tbit(int m) {
  if (P == 0) return 5 + m;  // 5..11
  if (P == 1) {
    if (V == 0) return m < 5 ? m : 5 + m;  // 0,1,2,3,4,10,11; V1: 10,11,0,1,2,3,4
    constexpr int o[7] = {10, 11, 0, 1, 2, 3, 4};
    return o[m];
  }
  constexpr int o2[7] = {5, 6, 7, 3, 4, 8, 9};
  return o2[m];
}

template <int P>
__host__ __device__ constexpr uint32_t reg_slot(int j) {
  uint32_t s = 0;
  for (int k = 0; k < kRegBits; ++k)
    if ((j >> k) & 1) s += wbit(reg_tbit<P>(k));
  return s;
}

template <int P, int V>
__device__ __forceinline__ uint32_t thr_slot(uint32_t tid) {
  uint32_t s = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) s += wbit(thr_tbit<P, V>(m));
  return s;
}

// Per-block tile-bit maps of the pass.
struct BlockCtx {
  uint32_t qbit[kTileBits];  // tile bit -> 1 << qubit (0 for a unit bit)
  uint32_t ubit[kTileBits];  // tile bit -> unit increment (0 for a qubit)
  uint32_t abit[kTileBits];  // tile bit -> its address bit in the working state (0 for a unit bit)
  unsigned long long mbar;   // completion barrier of the tile's tensor copies
  int tma_c[2][kTmaRank];    // tensor coordinates of the next tile's copies
  int tma_sel;               // plane 1 of the next tile comes through tm1
  uint32_t cz_w[kPhases][kThreads];  // per layout and thread: entangler terms of the thread bits
  uint32_t cz_n[kPhases][kThreads];  // per layout and thread: xor of the thread bits' neighbours
  double ez[kThreads / 32][2];       // Z0 epilogue: per warp, the two samples' partial sums
};

// Qubit-space index and batch unit of (thread, register 0) in phase P.
template <int P, int V>
__device__ __forceinline__ void thread_pos(const BlockCtx& bc, uint32_t tid, uint32_t* aq, uint32_t* ut) {
  uint32_t q = 0, u = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) {
      q |= bc.qbit[thr_tbit<P, V>(m)];
      u += bc.ubit[thr_tbit<P, V>(m)];
    }
  *aq = q;
  *ut = u;
}

struct RegMaps {
  uint32_t q[kRegBits];  // qubit bit of register bit k (0 if a unit bit)
  uint32_t u[kRegBits];  // unit increment of register bit k (0 if a qubit)
  uint32_t a[kRegBits];  // working-state address bit of register bit k (0 if a unit bit)
};

// Working-state address bits of this thread's fixed tile bits in layout P.
template <int P, int V>
__device__ __forceinline__ uint32_t thread_addr(const BlockCtx& bc, uint32_t tid) {
  uint32_t x = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) x |= bc.abit[thr_tbit<P, V>(m)];
  return x;
}

template <int P>
__device__ __forceinline__ RegMaps reg_maps(const BlockCtx& bc) {
  RegMaps m;
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) {
    m.q[k] = bc.qbit[reg_tbit<P>(k)];
    m.u[k] = bc.ubit[reg_tbit<P>(k)];
    m.a[k] = bc.abit[reg_tbit<P>(k)];
  }
  return m;
}

#define REG_COMBINE(arr, j, op)                                   \
  ([&]() {                                                        \
    uint32_t r_ = 0;                                              \
    _Pragma("unroll") for (int k_ = 0; k_ < kRegBits; ++k_) if ((j) & (1 << k_)) r_ op arr[k_]; \
    return r_;                                                    \
  }())

template <int X, int Y, int V>
__device__ __forceinline__ void exchange_t(float2 (&re)[kPos], float2 (&im)[kPos], float4* tile, uint32_t tid) {
  const uint32_t sx = thr_slot<X, V>(tid);
  const uint32_t sy = thr_slot<Y, V>(tid);
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) tile[sx + reg_slot<X>(j)] = make_float4(re[j].x, re[j].y, im[j].x, im[j].y);
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const float4 v = tile[sy + reg_slot<Y>(j)];
    re[j] = make_float2(v.x, v.y);
    im[j] = make_float2(v.z, v.w);
  }
}

template <int V>
__device__ __forceinline__ void exchange(int x, int y, float2 (&re)[kPos], float2 (&im)[kPos], float4* tile,
                                         uint32_t tid) {
  switch (x * 3 + y) {
    case 1: exchange_t<0, 1, V>(re, im, tile, tid); break;
    case 2: exchange_t<0, 2, V>(re, im, tile, tid); break;
    case 3: exchange_t<1, 0, V>(re, im, tile, tid); break;
    case 5: exchange_t<1, 2, V>(re, im, tile, tid); break;
    case 6: exchange_t<2, 0, V>(re, im, tile, tid); break;
    default: exchange_t<2, 1, V>(re, im, tile, tid); break;
  }
}

// Tensor-copy passes keep the copied tile in a landing buffer of its own, so
// their layout exchanges go through a second, smaller buffer: the re pairs
// first, then the im pairs, 8 bytes per position.  Slot of position t:
// sum over the set bits b of t of wbit8(b) (additive and injective; every
// half warp of every layout's 8-byte accesses hits 16 different bank pairs).
__host__ __device__ constexpr uint32_t wbit8(int b) {
  return b < 5 ? (1u << b) : b == 5 ? 33u : b == 6 ? 66u : b == 7 ? 132u : b == 8 ? 264u : b == 9 ? 528u : b == 10 ? 1060u
                                                                                                                 : 2120u;
}
constexpr int kExch8Slots = 4235;  // largest slot (sum of all wbit8) + 1

template <int P>
__host__ __device__ constexpr uint32_t reg_slot8(int j) {
  uint32_t s = 0;
  for (int k = 0; k < kRegBits; ++k)
    if ((j >> k) & 1) s += wbit8(reg_tbit<P>(k));
  return s;
}

template <int P, int V>
__device__ __forceinline__ uint32_t thr_slot8(uint32_t tid) {
  uint32_t s = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) s += wbit8(thr_tbit<P, V>(m));
  return s;
}

// An exchange between layouts X and Y is local to each warp when both take
// the warp index from tile bits 10 and 11: the warp's 1024 positions then
// stay in the warp, in a slot range of its own (the largest slot of tile bits
// 0-9 is 1054 < wbit8(10) = 1060), so a warp barrier orders it.
template <int X, int Y, int V>
__host__ __device__ constexpr bool exchange8_warp_local() {
  return thr_tbit<X, V>(5) == 10 && thr_tbit<X, V>(6) == 11 && thr_tbit<Y, V>(5) == 10 && thr_tbit<Y, V>(6) == 11;
}

// Thread-index bit of layout (Y, V) that holds tile bit t (-1: none).
template <int Y, int V>
__host__ __device__ constexpr int thr_index_of(int t) {
  for (int m = 0; m < kThrBits; ++m)
    if (thr_tbit<Y, V>(m) == t) return m;
  return -1;
}

// Pending bit flips of layout X's register bits (fl, bit k: register bit k;
// see the split-form rotations in pass_kernel) as thread-index bits of
// layout Y: a register bit of phase 0 or 1 is a thread bit of the other.
template <int X, int Y, int V>
__device__ __forceinline__ uint32_t flip_thr(uint32_t fl) {
  uint32_t m = 0;
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) {
    const int mm = thr_index_of<Y, V>(reg_tbit<X>(k));
    if (mm >= 0 && ((fl >> k) & 1u)) m |= 1u << mm;
  }
  return m;
}

// ONE: the complex-lane form, whose state is the re array alone.  fl: bit
// flips pending on X's register bits (register j holds the amplitude of
// position j ^ fl); the writes go to the registers' own slots, and the reads
// take the flipped positions, whose flipped bits are thread bits in Y (phases
// 0 and 1), so only the reading thread's slot base changes.
template <int X, int Y, int V, bool ONE>
__device__ __forceinline__ void exchange8_t(float2 (&re)[kPos], float2 (&im)[kPos], float2* ex, uint32_t tid,
                                            uint32_t fl) {
  // (ONE keeps block barriers: its layouts' reads may cross warps)
  constexpr bool WL = !ONE && exchange8_warp_local<X, Y, V>();
  const uint32_t sx = thr_slot8<X, V>(tid);
  const uint32_t sy = thr_slot8<Y, V>(tid ^ flip_thr<X, Y, V>(fl));
  auto sync = []() {
    if constexpr (WL) __syncwarp();
    else __syncthreads();
  };
  sync();
#pragma unroll
  for (int j = 0; j < kPos; ++j) ex[sx + reg_slot8<X>(j)] = re[j];
  sync();
#pragma unroll
  for (int j = 0; j < kPos; ++j) re[j] = ex[sy + reg_slot8<Y>(j)];
  if constexpr (ONE) return;  // the next exchange starts with a barrier
  sync();
#pragma unroll
  for (int j = 0; j < kPos; ++j) ex[sx + reg_slot8<X>(j)] = im[j];
  sync();
#pragma unroll
  for (int j = 0; j < kPos; ++j) im[j] = ex[sy + reg_slot8<Y>(j)];
}

template <int V, bool ONE = false>
__device__ __forceinline__ void exchange8(int x, int y, float2 (&re)[kPos], float2 (&im)[kPos], float2* ex,
                                          uint32_t tid, uint32_t fl = 0) {
  switch (x * 3 + y) {
    case 1: exchange8_t<0, 1, V, ONE>(re, im, ex, tid, fl); break;
    case 2: exchange8_t<0, 2, V, ONE>(re, im, ex, tid, fl); break;
    case 3: exchange8_t<1, 0, V, ONE>(re, im, ex, tid, fl); break;
    case 5: exchange8_t<1, 2, V, ONE>(re, im, ex, tid, fl); break;
    case 6: exchange8_t<2, 0, V, ONE>(re, im, ex, tid, fl); break;
    default: exchange8_t<2, 1, V, ONE>(re, im, ex, tid, fl); break;
  }
}

// Fused CNOT layers: a layout exchange whose reads are permuted.  Each
// thread writes its positions (layout X) at perm_slot of their tile position,
// then reads for its position y (layout Y) the slot G y + G_o o of the
// direction's gather map, given as columns already in slot space: cy is the
// part of the thread bits and the out-of-tile bits, dc[k] the column of
// register bit k (perm_slot is linear, so the slot of a gathered position is
// the xor of these).
template <int P>
__host__ __device__ constexpr uint32_t reg_pattern(int j) {
  uint32_t t = 0;
  for (int k = 0; k < kRegBits; ++k)
    if ((j >> k) & 1) t |= 1u << reg_tbit<P>(k);
  return t;
}

template <int P, int V>
__device__ __forceinline__ uint32_t thr_pattern(uint32_t tid) {
  uint32_t t = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m) t |= ((tid >> m) & 1u) << thr_tbit<P, V>(m);
  return t;
}

template <int X, int Y, int V>
__device__ __forceinline__ void exchange8p_t(float2 (&re)[kPos], float2 (&im)[kPos], float2* ex, uint32_t tid,
                                             const DevPass& Pp, int dir, uint32_t co, uint32_t fl) {
  // pending flips fl of X's register bits: register j holds position j ^ fl,
  // written at that position's slot (perm_slot is linear: one xor)
  uint32_t ft = 0;
#pragma unroll
  for (int k = 0; k < kRegBits; ++k)
    if ((fl >> k) & 1u) ft |= 1u << reg_tbit<X>(k);
  const uint32_t sx = perm_slot(thr_pattern<X, V>(tid)) ^ perm_slot(ft);
  uint32_t cy = co;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) cy ^= Pp.pcol[dir][thr_tbit<Y, V>(m)];
  uint32_t dc[kRegBits];
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) dc[k] = Pp.pcol[dir][reg_tbit<Y>(k)];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) ex[sx ^ perm_slot(reg_pattern<X>(j))] = re[j];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) re[j] = ex[cy ^ REG_COMBINE(dc, j, ^=)];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) ex[sx ^ perm_slot(reg_pattern<X>(j))] = im[j];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPos; ++j) im[j] = ex[cy ^ REG_COMBINE(dc, j, ^=)];
  // the reads above cross warps and slot ranges: a following warp-local
  // exchange (warp barrier only) must not write before every warp has read
  __syncthreads();
}

template <int V>
__device__ __forceinline__ void exchange8p(int x, int y, float2 (&re)[kPos], float2 (&im)[kPos], float2* ex,
                                           uint32_t tid, const DevPass& Pp, int dir, uint32_t co, uint32_t fl = 0) {
  switch (x * 3 + y) {
    case 0: exchange8p_t<0, 0, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 1: exchange8p_t<0, 1, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 2: exchange8p_t<0, 2, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 3: exchange8p_t<1, 0, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 4: exchange8p_t<1, 1, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 5: exchange8p_t<1, 2, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 6: exchange8p_t<2, 0, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    case 7: exchange8p_t<2, 1, V>(re, im, ex, tid, Pp, dir, co, fl); break;
    default: exchange8p_t<2, 2, V>(re, im, ex, tid, Pp, dir, co, fl); break;
  }
}

// CZ on every bond (a, b) of the entangler: sign (-1)^{S(i)}, S(i) = sum over
// bonds of i_a i_b, of the global index i.  Split i = T | O | R (thread bits,
// out-of-tile bits, register bits; disjoint).  S is a quadratic form, so
//   S(i) = S(T) + S(O) + S(R) + parity(O & N(T)) + sum_k R_k [parity(T & nb(q_k))
//          + parity(O & nb(q_k))],
// N(T) = xor of the neighbour masks of T's qubits, nb(q) = q's neighbours.
// Per thread and layout the terms in T alone are one 32-bit word over the
// register index (with the per-pass table S(R)), kept in shared memory; S(O)
// is computed once per tile.
// Bit j of the returned word: the entangler parity of this thread's position j.
__device__ __forceinline__ uint32_t cz_word(uint32_t w_t, uint32_t n_t, const uint32_t (&nb)[kRegBits],
                                           uint32_t base_q, uint32_t s_o) {
  const uint32_t qo = (s_o ^ (uint32_t)__popc(base_q & n_t)) & 1u;
  uint32_t w = w_t ^ (qo ? 0xffffffffu : 0u);
  const uint32_t pat[5] = {0xAAAAAAAAu, 0xCCCCCCCCu, 0xF0F0F0F0u, 0xFF00FF00u, 0xFFFF0000u};
#pragma unroll
  for (int k = 0; k < kRegBits; ++k)
    if (__popc(base_q & nb[k]) & 1) w ^= pat[k];
  return w;
}

__device__ __forceinline__ void apply_cz(float2 (&re)[kPos], float2 (&im)[kPos], uint32_t w_t, uint32_t n_t,
                                         const uint32_t (&nb)[kRegBits], uint32_t base_q, uint32_t s_o) {
  const uint32_t w = cz_word(w_t, n_t, nb, base_q, s_o);
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t sb = (w << (31 - j)) & 0x80000000u;
    flip(re[j], sb);
    flip(im[j], sb);
  }
}

// S(A) = sum over bonds within the qubit mask A (nbhi: neighbours above).
__device__ __forceinline__ uint32_t bond_parity(uint32_t aq, const PassArgs& a) {
  uint32_t s = 0, rem = aq;
  while (rem) {
    const int q = __ffs(rem) - 1;
    rem &= rem - 1u;
    s ^= (uint32_t)__popc(aq & a.cz_nbhi[q]);
  }
  return s & 1u;
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

// What a pass does to HBM at its start or end, in the memory layout P.
enum MemOp { M_LOAD, M_STORE, M_STORE_STD, M_GEN, M_CKPT_STORE, M_CKPT_RESTORE };

// The state in the buffers is stored at working-state addresses
// (DevPass::tile_abit / out_abit; the identity unless the plan has three or
// more qubit sets, in which case separate kernels convert it from and to the
// standard order at the ends of the pass chain).  The encoding and the
// checkpoint slots use the standard index, i.e. the qubit bits.  ZF: the
// complex-lane forward (one sample per batch unit, re[j] its amplitude;
// encoding, checkpoint and standard-order stores only).
template <bool BWD, bool SLOW, int P, int V, int OP, bool ZF = false>
__device__ __forceinline__ void mem_t(const PassArgs& a, const BlockCtx& bc, uint32_t tid, uint32_t base_q,
                                      uint32_t base_a, uint32_t unit_base, float2 (&re)[kPos], float2 (&im)[kPos],
                                      int slot, float rs, uint32_t fl) {
  uint32_t aq, ut;
  thread_pos<P, V>(bc, tid, &aq, &ut);
  constexpr bool std_index = !(OP == M_LOAD || OP == M_STORE || OP == M_STORE_STD);
  float ez0 = 0.f, ez1 = 0.f;  // M_STORE_STD with a.epart: sum of |psi|^2 (1 - 2 b0) of the two lanes
  if (std_index) aq |= base_q;
  else aq = thread_addr<P, V>(bc, tid) | base_a;
  ut += unit_base;
  const RegMaps m = reg_maps<P>(bc);
  const int n = a.n;
  // stores with pending flips fl: register j holds position j ^ fl
  const uint32_t fx = fl ? (std_index ? REG_COMBINE(m.q, fl, |=) : REG_COMBINE(m.a, fl, |=)) : 0u;
  if constexpr (OP == M_GEN && !SLOW) {
    // The product state of one batch unit (no unit bit among the register
    // bits): the factors of the qubits outside the register bits once, then
    // those of the register bits as a product tree over the positions.
    const bool ok = ut < (uint32_t)a.U;
    const float2* e = a.enc + (size_t)(ZF ? ut >> 1 : ut) * n * 2;
    const bool hi = ZF && (ut & 1u);  // ZF: the sample's lane of the pair table
    auto fac = [&](int q, uint32_t bit) {
      const float2 f = __ldg(&e[2 * q + bit]);
      return ZF ? (hi ? make_float2(f.y, f.y) : make_float2(f.x, f.x)) : f;
    };
    uint32_t rq = 0;
#pragma unroll
    for (int k = 0; k < kRegBits; ++k) rq |= m.q[k];
    float2 v[kPos];
    v[0] = ok ? make_float2(1.f, 1.f) : make_float2(0.f, 0.f);
    if (ok)
      for (int q = 0; q < n; ++q)
        if (!((rq >> q) & 1u)) v[0] = __fmul2_rn(v[0], fac(q, (aq >> q) & 1u));
#pragma unroll
    for (int k = 0; k < kRegBits; ++k) {
      float2 f0 = make_float2(1.f, 1.f), f1 = f0;
      if (ok && m.q[k]) {
        const int q = __ffs(m.q[k]) - 1;
        f0 = fac(q, 0u);
        f1 = fac(q, 1u);
      }
#pragma unroll
      for (int j = 0; j < (1 << k); ++j) {
        v[j | (1 << k)] = __fmul2_rn(v[j], f1);
        v[j] = __fmul2_rn(v[j], f0);
      }
    }
#pragma unroll
    for (int j = 0; j < kPos; ++j) {
      if (ZF) {
        re[j] = make_float2(v[j].x, 0.f);
      } else {
        re[j] = v[j];
        im[j] = make_float2(0.f, 0.f);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < kPos; ++j) {
      const uint32_t i = (aq | (std_index ? REG_COMBINE(m.q, j, |=) : REG_COMBINE(m.a, j, |=))) ^ fx;
      const uint32_t u = SLOW ? ut + REG_COMBINE(m.u, j, +=) : ut;
      const bool ok = u < (uint32_t)a.U;
      if constexpr (OP == M_LOAD) {
        if (ok) {
          re[j] = Planes<BWD>::p0(a, u)[i];
          im[j] = Planes<BWD>::p1(a, u)[i];
        } else {
          re[j] = im[j] = make_float2(0.f, 0.f);
        }
      } else if constexpr (OP == M_STORE) {
        if (ok) {
          Planes<BWD>::p0(a, u)[i] = re[j];
          Planes<BWD>::p1(a, u)[i] = im[j];
        }
      } else if constexpr (OP == M_STORE_STD && ZF) {
        if (ok) a.buf0[(size_t)u * a.N + i] = re[j];
        const float pr = fmaf(re[j].x, re[j].x, re[j].y * re[j].y);
        if (i & 1u) ez0 -= pr;
        else ez0 += pr;
      } else if constexpr (OP == M_STORE_STD) {  // forward only
        if (ok) {
          a.buf0[(size_t)(2 * u) * a.N + i] = make_float2(re[j].x, im[j].x);
          if (2 * u + 1 < (uint32_t)a.B) a.buf0[(size_t)(2 * u + 1) * a.N + i] = make_float2(re[j].y, im[j].y);
        }
        const float2 pr = __ffma2_rn(re[j], re[j], __fmul2_rn(im[j], im[j]));  // |psi|^2 of both lanes
        if (i & 1u) ez0 -= pr.x, ez1 -= pr.y;
        else ez0 += pr.x, ez1 += pr.y;
      } else if constexpr (OP == M_GEN) {  // forward only, generic addressing: angle-encoded product state
        float2 v = make_float2(0.f, 0.f);
        if (ok) {
          const float2* e = a.enc + (size_t)u * n * 2;
          v = make_float2(1.f, 1.f);
          for (int q = 0; q < n; ++q) v = __fmul2_rn(v, __ldg(&e[2 * q + ((i >> q) & 1u)]));
        }
        re[j] = v;
        im[j] = make_float2(0.f, 0.f);
      } else if constexpr (OP == M_CKPT_STORE && ZF) {
        if (ok) {
          const size_t e0 = ((size_t)slot * a.bmax + u) * a.N + i;
          if (a.storage == 0) reinterpret_cast<float2*>(a.ckpt)[e0] = re[j];
          else reinterpret_cast<__nv_bfloat162*>(a.ckpt)[e0] = __floats2bfloat162_rn(re[j].x, re[j].y);
        }
      } else if constexpr (OP == M_CKPT_STORE) {  // forward only
        if (ok) {
          const size_t e0 = ((size_t)slot * a.bmax + 2 * u) * a.N + i;
          const bool has1 = 2 * u + 1 < (uint32_t)a.B;
          if (a.storage == 0) {
            float2* s = reinterpret_cast<float2*>(a.ckpt);
            s[e0] = make_float2(re[j].x, im[j].x);
            if (has1) s[e0 + a.N] = make_float2(re[j].y, im[j].y);
          } else {
            __nv_bfloat162* s = reinterpret_cast<__nv_bfloat162*>(a.ckpt);
            s[e0] = __floats2bfloat162_rn(re[j].x, im[j].x);
            if (has1) s[e0 + a.N] = __floats2bfloat162_rn(re[j].y, im[j].y);
          }
        }
      } else {  // M_CKPT_RESTORE, backward only: psi lanes from the slot
        if (ok) {
          const size_t e = ((size_t)slot * a.bmax + u) * a.N + i;
          float2 v;
          if (a.storage == 0) v = reinterpret_cast<const float2*>(a.ckpt)[e];
          else v = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.ckpt)[e]);
          re[j].x = v.x * rs;
          im[j].x = v.y * rs;
        }
      }
    }
  }
  if constexpr (OP == M_STORE_STD) {
    // Z0 epilogue: the tile's two partial sums (lanes x, y = samples 2u,
    // 2u + 1) in a fixed order: warp butterfly, then the warps in order.
    // slot: the tile's out-of-tile index (tiles of one unit, no unit bits).
    if (a.epart) {
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        ez0 += __shfl_xor_sync(0xffffffffu, ez0, o);
        ez1 += __shfl_xor_sync(0xffffffffu, ez1, o);
      }
      BlockCtx& w = const_cast<BlockCtx&>(bc);
      if ((tid & 31) == 0) w.ez[tid >> 5][0] = ez0, w.ez[tid >> 5][1] = ez1;
      __syncthreads();
      if (tid == 0 && ut < (uint32_t)a.U) {
        double s0 = 0.0, s1 = 0.0;
        for (int k = 0; k < kThreads / 32; ++k) s0 += w.ez[k][0], s1 += w.ez[k][1];
        const size_t tps = (size_t)1 << (n > kTileBits ? n - kTileBits : 0);  // tiles per sample
        if (ZF) {
          a.epart[(size_t)ut * tps + (size_t)slot] = s0;
        } else {
          a.epart[(size_t)(2 * ut) * tps + (size_t)slot] = s0;
          if (2 * ut + 1 < (uint32_t)a.B) a.epart[(size_t)(2 * ut + 1) * tps + (size_t)slot] = s1;
        }
      }
      __syncthreads();
    }
  }
}

template <bool BWD, bool SLOW, int V, int OP, bool ZF = false>
__device__ __forceinline__ void mem_op(int phase, const PassArgs& a, const BlockCtx& bc, uint32_t tid,
                                       uint32_t base_q, uint32_t base_a, uint32_t unit_base, float2 (&re)[kPos],
                                       float2 (&im)[kPos], int slot = 0, float rs = 1.f, uint32_t fl = 0) {
  // memory ops run in phase 0 or 1 (the planner never picks phase 2)
  if (phase == 0) mem_t<BWD, SLOW, 0, V, OP, ZF>(a, bc, tid, base_q, base_a, unit_base, re, im, slot, rs, fl);
  else mem_t<BWD, SLOW, 1, V, OP, ZF>(a, bc, tid, base_q, base_a, unit_base, re, im, slot, rs, fl);
}

// Prefetch of the block's next tile: each thread copies its own positions of
// the load layout P into the shared-memory slots it will read them from, with
// cp.async (zero fill for batch units past the end).
template <bool BWD, int P, int V>
__device__ __forceinline__ void prefetch_t(const PassArgs& a, const BlockCtx& bc, uint32_t tid, uint32_t base_q,
                                           uint32_t base_a, uint32_t unit_base, float4* tile) {
  uint32_t aq, ut;
  thread_pos<P, V>(bc, tid, &aq, &ut);
  aq = thread_addr<P, V>(bc, tid) | base_a;
  ut += unit_base;
  RegMaps m = reg_maps<P>(bc);
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) m.q[k] = m.a[k];
  const bool ok = ut < (uint32_t)a.U;
  const float2* p0 = Planes<BWD>::p0(a, ok ? ut : 0u) + (ok ? aq : 0u);
  const float2* p1 = Planes<BWD>::p1(a, ok ? ut : 0u) + (ok ? aq : 0u);
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(tile) + thr_slot<P, V>(tid) * 16u;
  const int nbytes = ok ? 8 : 0;
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t b = ok ? REG_COMBINE(m.q, j, |=) : 0u;
    const uint32_t dst = sbase + reg_slot<P>(j) * 16u;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(p0 + b), "r"(nbytes) : "memory");
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst + 8u), "l"(p1 + b), "r"(nbytes) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <bool BWD, int V>
__device__ __forceinline__ void prefetch_op(int phase, const PassArgs& a, const BlockCtx& bc, uint32_t tid,
                                            uint32_t base_q, uint32_t base_a, uint32_t unit_base, float4* tile) {
  if (phase == 0) prefetch_t<BWD, 0, V>(a, bc, tid, base_q, base_a, unit_base, tile);
  else prefetch_t<BWD, 1, V>(a, bc, tid, base_q, base_a, unit_base, tile);
}

// Registers of layout P from the thread's own prefetched slots.
template <int P, int V>
__device__ __forceinline__ void load_prefetched_t(float2 (&re)[kPos], float2 (&im)[kPos], const float4* tile,
                                                  uint32_t tid) {
  asm volatile("cp.async.wait_all;" ::: "memory");
  const uint32_t s0 = thr_slot<P, V>(tid);
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const float4 v = tile[s0 + reg_slot<P>(j)];
    re[j] = make_float2(v.x, v.y);
    im[j] = make_float2(v.z, v.w);
  }
}

template <int V>
__device__ __forceinline__ void load_prefetched(int phase, float2 (&re)[kPos], float2 (&im)[kPos], const float4* tile,
                                                uint32_t tid) {
  if (phase == 0) load_prefetched_t<0, V>(re, im, tile, tid);
  else load_prefetched_t<1, V>(re, im, tile, tid);
}


// ------------------------------------------------ tensor-copy (TMA) tile loads
//
// With a tensor map per plane buffer, one thread loads a whole tile (both
// planes, 64 KB) into the shared tile buffer with two bulk tensor copies that
// signal an mbarrier; no other thread issues a memory instruction for it.  The
// copied layout is the tensor's dimension order (see kTmaRank); sstride gives
// each tile bit's element offset in it, plane 1 sits 4096 elements after
// plane 0.

// Tensor coordinates of both planes of tile `tile` (computed by the issuing
// thread ahead of time, so that the issue point needs few registers).  In the
// forward pass plane 1 of unit u is sample 2u+1; when that sample does not
// exist (odd B, last unit) the plane lives in the one-sample partner buffer,
// whose map is tm1, at sample 0.
__device__ __forceinline__ void tma_coords(const DevPass& P, bool bwd, int B, int tile, int (&c)[2][kTmaRank],
                                           int* sel) {
  const uint32_t o = (uint32_t)tile & ((1u << P.n_out) - 1u);
  const uint32_t u = (uint32_t)tile >> P.n_out;
  const bool partner = !bwd && 2u * u + 1u >= (uint32_t)B;
  *sel = bwd || partner;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const uint32_t smp = bwd ? u : (p == 1 && partner) ? 0u : 2u * u + (uint32_t)p;
#pragma unroll
    for (int d = 0; d < kTmaRank; ++d) {
      const int k = P.tma_kind[d];
      const uint32_t ob = (o >> P.tma_shift[d]) & ((1u << P.tma_bits[d]) - 1u);
      c[p][d] = k == TD_OUT ? (int)ob : k == TD_SAMPLE ? (int)smp : k == TD_OUT_SAMPLE ? (int)(ob | (smp << P.tma_bits[d])) : 0;
    }
  }
}

__device__ __forceinline__ void tma_load_tile(const CUtensorMap* m0, const CUtensorMap* m1, int sel,
                                              const int (&c)[2][kTmaRank], uint32_t dst, uint32_t mbar) {
  // the shared buffer was last written through the generic proxy (exchanges)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(kTilePos * 16) : "memory");
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const CUtensorMap* m = (p == 1 && sel) ? m1 : m0;
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
        "%6}], [%7];" ::"r"(dst + (uint32_t)p * (kTilePos * 8)),
        "l"(m), "r"(c[p][0]), "r"(c[p][1]), "r"(c[p][2]), "r"(c[p][3]), "r"(c[p][4]), "r"(mbar)
        : "memory");
  }
}

// Bounded wait for the phase with the given parity; false if it never came.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Registers of layout P from the copied tile.
template <int P, int V>
__device__ __forceinline__ void load_tma_t(float2 (&re)[kPos], float2 (&im)[kPos], const float2* buf,
                                           const DevPass& Pp, uint32_t tid) {
  uint32_t s0 = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) s0 += (uint32_t)Pp.sstride[thr_tbit<P, V>(m)];
  uint32_t r[kRegBits];
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) r[k] = (uint32_t)Pp.sstride[reg_tbit<P>(k)];
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t off = s0 + REG_COMBINE(r, j, +=);
    re[j] = buf[off];
    im[j] = buf[off + kTilePos];
  }
}

// Backward checkpoint restore on the copied tile: replace the psi lanes of
// this thread's positions (layout P) with the slot's values, before the tile
// is read into registers (so no state registers are live here).  The 32
// positions go in four groups of eight (register bits 3 and 4 per group), the
// eight loads of a group in flight together.
template <int P, int V>
__device__ __forceinline__ void restore_tma_t(const PassArgs& a, const BlockCtx& bc, const DevPass& Pp, uint32_t tid,
                                              uint32_t base_q, uint32_t unit_base, float2* buf, int slot, float rs) {
  uint32_t aq, ut;
  thread_pos<P, V>(bc, tid, &aq, &ut);
  aq |= base_q;
  ut += unit_base;
  if (ut >= (uint32_t)a.U) return;
  uint32_t s0 = 0;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) s0 += (uint32_t)Pp.sstride[thr_tbit<P, V>(m)];
  uint32_t r[kRegBits];
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) r[k] = (uint32_t)Pp.sstride[reg_tbit<P>(k)];
  const RegMaps m = reg_maps<P>(bc);
  const size_t e0 = ((size_t)slot * a.bmax + ut) * a.N + aq;
  const bool f32 = a.storage == 0;
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    const uint32_t gq = ((g & 1) ? m.q[3] : 0u) | ((g & 2) ? m.q[4] : 0u);
    const uint32_t go = s0 + ((g & 1) ? r[3] : 0u) + ((g & 2) ? r[4] : 0u);
    float2 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const size_t e = e0 + (gq | REG_COMBINE(m.q, i, |=));
      if (f32) v[i] = reinterpret_cast<const float2*>(a.ckpt)[e];
      else v[i] = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(a.ckpt)[e]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t off = go + REG_COMBINE(r, i, +=);
      buf[off].x = v[i].x * rs;
      buf[off + kTilePos].x = v[i].y * rs;
    }
  }
}

template <int V>
__device__ __forceinline__ void load_tma(int phase, float2 (&re)[kPos], float2 (&im)[kPos], const float2* buf,
                                         const DevPass& Pp, uint32_t tid) {
  if (phase == 0) load_tma_t<0, V>(re, im, buf, Pp, tid);
  else load_tma_t<1, V>(re, im, buf, Pp, tid);
}

// Fused CNOT layers: registers of layout P gathered from the copied tile
// through the direction's map (columns as landing-buffer offsets: the offset
// of a tile position is a bit permutation of it, so the offset of a gathered
// position is the xor of the columns of its set bits, co for the out-of-tile
// bits).
template <int P, int V>
__device__ __forceinline__ void load_tma_perm_t(float2 (&re)[kPos], float2 (&im)[kPos], const float2* buf,
                                                const DevPass& Pp, int dir, uint32_t co, uint32_t tid) {
  uint32_t s0 = co;
#pragma unroll
  for (int m = 0; m < kThrBits; ++m)
    if ((tid >> m) & 1u) s0 ^= Pp.pcol[dir][thr_tbit<P, V>(m)];
  uint32_t r[kRegBits];
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) r[k] = Pp.pcol[dir][reg_tbit<P>(k)];
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const uint32_t off = s0 ^ REG_COMBINE(r, j, ^=);
    re[j] = buf[off];
    im[j] = buf[off + kTilePos];
  }
}

template <int V>
__device__ __forceinline__ void load_tma_perm(int phase, float2 (&re)[kPos], float2 (&im)[kPos], const float2* buf,
                                              const DevPass& Pp, int dir, uint32_t co, uint32_t tid) {
  if (phase == 0) load_tma_perm_t<0, V>(re, im, buf, Pp, dir, co, tid);
  else load_tma_perm_t<1, V>(re, im, buf, Pp, dir, co, tid);
}

// Out-of-tile qubit bits and first batch unit of tile t.
// (out-of-tile bits as qubit bits and as working-state address bits)
__device__ __forceinline__ void tile_base(const DevPass& P, int t, uint32_t* base_q, uint32_t* base_a,
                                          uint32_t* unit_base) {
  const int n_out = P.n_out;
  const uint32_t o = (uint32_t)t & ((1u << n_out) - 1u);
  uint32_t bq = 0, ba = 0;
  for (int k = 0; k < n_out; ++k)
    if ((o >> k) & 1u) bq |= 1u << P.out_q[k], ba |= P.out_abit[k];
  *base_q = bq;
  *base_a = ba;
  *unit_base = ((uint32_t)t >> n_out) << P.unit_bits;
}

template <int P, int V>
__device__ __forceinline__ void cz_t(float2 (&re)[kPos], float2 (&im)[kPos], const BlockCtx& bc, const DevPass& Pp,
                                     uint32_t tid, uint32_t base_q, uint32_t s_o) {
  uint32_t nb[kRegBits];
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) nb[k] = Pp.cz_nb[P][k];
  apply_cz(re, im, bc.cz_w[P][tid], bc.cz_n[P][tid], nb, base_q, s_o);
}

template <int V>
__device__ __forceinline__ void cz_op(int phase, float2 (&re)[kPos], float2 (&im)[kPos], const BlockCtx& bc,
                                      const DevPass& Pp, uint32_t tid, uint32_t base_q, uint32_t s_o) {
  switch (phase) {
    case 0: cz_t<0, V>(re, im, bc, Pp, tid, base_q, s_o); break;
    case 1: cz_t<1, V>(re, im, bc, Pp, tid, base_q, s_o); break;
    default: cz_t<2, V>(re, im, bc, Pp, tid, base_q, s_o); break;
  }
}

// Split form: the diagonal op d (layer l).  A position i = T | O | R (thread,
// out-of-tile and register bits) is multiplied by
//   (-1)^{S(i)} * f(T) f(O) * R_d[j],
// with S the entangler parity (l >= 0 only), f the product of the per-qubit
// factors dq[l + 1][q][bit] over the bits named, and R_d[j] the pass's
// constant table for the register part j (the global scale folded in).  The
// factor applies to both lanes of a pair (two samples, or psi and lambda).
// Only the thread part depends on the layout P; the loop over positions is
// shared by all layouts (one copy of its code).
template <int P, int V>
__device__ __forceinline__ void diag_thread_t(const BlockCtx& bc, const DevPass& Pp, const float2* dq, int l,
                                              uint32_t tid, uint32_t base_q, uint32_t s_o, float* fr_out,
                                              float* fi_out, uint32_t* w_out) {
  float fr = 1.f, fi = 0.f;
  auto mul = [&](float2 v) {
    const float r = fr * v.x - fi * v.y;
    fi = fmaf(fr, v.y, fi * v.x);
    fr = r;
  };
#pragma unroll
  for (int m = 0; m < kThrBits; ++m) {
    const int q = Pp.tile_q[thr_tbit<P, V>(m)];
    if (q >= 0) mul(__ldg(&dq[2 * q + ((tid >> m) & 1u)]));
  }
  for (int k = 0; k < Pp.n_out; ++k) {
    const int q = Pp.out_q[k];
    mul(__ldg(&dq[2 * q + ((base_q >> q) & 1u)]));
  }
  uint32_t w = 0;
  if (l >= 0) {
    uint32_t nb[kRegBits];
#pragma unroll
    for (int k = 0; k < kRegBits; ++k) nb[k] = Pp.cz_nb[P][k];
    w = cz_word(bc.cz_w[P][tid], bc.cz_n[P][tid], nb, base_q, s_o);
  }
  *fr_out = fr;
  *fi_out = fi;
  *w_out = w;
}

template <int V, bool ZF = false>
__device__ __forceinline__ void diag_op(int phase, float2 (&re)[kPos], float2 (&im)[kPos], const BlockCtx& bc,
                                        const DevPass& Pp, const PassArgs& a, const CoefRegion* C, int d, int l,
                                        uint32_t tid, uint32_t base_q, uint32_t s_o, uint32_t fl = 0) {
  const float2* dq = a.dq + (size_t)(l + 1) * a.n * 2;
  float fr, fi;
  uint32_t w;
  switch (phase) {
    case 0: diag_thread_t<0, V>(bc, Pp, dq, l, tid, base_q, s_o, &fr, &fi, &w); break;
    case 1: diag_thread_t<1, V>(bc, Pp, dq, l, tid, base_q, s_o, &fr, &fi, &w); break;
    default: diag_thread_t<2, V>(bc, Pp, dq, l, tid, base_q, s_o, &fr, &fi, &w); break;
  }
  // pending flips fl: register j holds position j ^ fl, whose factor is
  // table entry j ^ fl and whose sign is bit j ^ fl of the sign word
  if (fl) {
    const uint32_t pat[5] = {0xAAAAAAAAu, 0xCCCCCCCCu, 0xF0F0F0F0u, 0xFF00FF00u, 0xFFFF0000u};
#pragma unroll
    for (int k = 0; k < kRegBits; ++k)
      if ((fl >> k) & 1u) w = ((w & pat[k]) >> (1 << k)) | ((w & ~pat[k]) << (1 << k));
  }
  // per position: the factor (scalar complex, table entries from the constant
  // bank), its sign, then the product with both lanes
#pragma unroll
  for (int j = 0; j < kPos; ++j) {
    const float2 r = C->diag[d][j ^ fl];
    const uint32_t sb = (w << (31 - j)) & 0x80000000u;
    const float gr = __uint_as_float(__float_as_uint(fmaf(-fi, r.y, fr * r.x)) ^ sb);
    const float gi = __uint_as_float(__float_as_uint(fmaf(fr, r.y, fi * r.x)) ^ sb);
    if constexpr (ZF) {  // complex-lane form: the pair is one amplitude
      const float2 z = re[j];
      re[j] = make_float2(fmaf(gr, z.x, -gi * z.y), fmaf(gi, z.x, gr * z.y));
    } else {
      const float2 xr = re[j], xi = im[j];
      re[j] = make_float2(fmaf(gr, xr.x, -gi * xi.x), fmaf(gr, xr.y, -gi * xi.y));
      im[j] = make_float2(fmaf(gi, xr.x, gr * xi.x), fmaf(gi, xr.y, gr * xi.y));
    }
  }
}

// The thread's batch unit, the register bits' unit increments and qubits in
// layout P (for data re-uploading).
template <int P, int V>
__device__ __forceinline__ void unit_maps_t(const BlockCtx& bc, uint32_t tid, uint32_t unit_base, uint32_t* unit,
                                            uint32_t (&mu)[kRegBits], int (&rq)[kRegBits]) {
  uint32_t aq, ut;
  thread_pos<P, V>(bc, tid, &aq, &ut);
  *unit = unit_base + ut;
#pragma unroll
  for (int k = 0; k < kRegBits; ++k) {
    mu[k] = bc.ubit[reg_tbit<P>(k)];
    const uint32_t qb = bc.qbit[reg_tbit<P>(k)];
    rq[k] = qb ? __ffs(qb) - 1 : -1;
  }
}

template <int V>
__device__ __forceinline__ void unit_maps(int phase, const BlockCtx& bc, uint32_t tid, uint32_t unit_base,
                                          uint32_t* unit, uint32_t (&mu)[kRegBits], int (&rq)[kRegBits]) {
  switch (phase) {
    case 0: unit_maps_t<0, V>(bc, tid, unit_base, unit, mu, rq); break;
    case 1: unit_maps_t<1, V>(bc, tid, unit_base, unit, mu, rq); break;
    default: unit_maps_t<2, V>(bc, tid, unit_base, unit, mu, rq); break;
  }
}

// Entangler terms of this thread's fixed bits in layout P (see apply_cz).
template <int P, int V>
__device__ __forceinline__ void cz_thread_terms(BlockCtx& bc, const DevPass& Pp, const PassArgs& a, uint32_t tid) {
  uint32_t tq, ut;
  thread_pos<P, V>(bc, tid, &tq, &ut);
  uint32_t n_t = 0;
  for (uint32_t rem = tq; rem; rem &= rem - 1u) n_t ^= a.cz_nb[__ffs(rem) - 1];
  uint32_t w = Pp.cz_reg[P] ^ (bond_parity(tq, a) ? 0xffffffffu : 0u);
  const uint32_t pat[5] = {0xAAAAAAAAu, 0xCCCCCCCCu, 0xF0F0F0F0u, 0xFF00FF00u, 0xFFFF0000u};
#pragma unroll
  for (int k = 0; k < kRegBits; ++k)
    if (__popc(tq & Pp.cz_nb[P][k]) & 1) w ^= pat[k];
  bc.cz_w[P][tid] = w;
  bc.cz_n[P][tid] = n_t;
}

// ----------------------------------------------------------- the pass kernel
//
// One launch runs one pass over every tile of the batch (persistent blocks,
// tiles assigned round-robin).  The pass record arrives as a kernel parameter
// so that its ops and slot numbers are uniform across the warp.
//
// MODE 0: a memory layout has a batch-unit register bit (n < 5), generic
// addressing.  MODE 1: tiles are loaded by the threads (the next tile with
// cp.async).  MODE 2: tiles are loaded by tensor copies through tm0 / tm1.
// RE: data re-uploading (every layer starts with the encoding again), folded
// into the layer's rotations.  RE 1: the tile holds no batch-unit bit, so each
// thread's amplitudes belong to one batch unit and each rotation takes one set
// of coefficients.  RE 2: tiles with batch-unit bits (n < 12), coefficients
// per register pair.  RE 3: the split form (OP_RY and OP_DIAG ops; no
// re-uploading).  RE 4: the split form of the fused CNOT schedule (also
// OP_PERM; tensor copies only).  RE 0: the fused SU(2) form (OP_ROT and
// OP_CZ, and OP_PERM with tensor copies).

// Shared memory of a pass block.  Tensor-copy passes (MODE 2): the landing
// buffer of the copied tile (both planes, 64 KB), then the 8-byte exchange
// buffer; the next tile's copy is issued as soon as the current tile is in
// registers, so it is in flight during the whole tile (two blocks per SM).
// Other passes: one buffer for the exchanges and the cp.async prefetch (three
// blocks per SM).  Then the block's context and gradient accumulators.
constexpr size_t kLandBytes = (size_t)kTilePos * 16;
constexpr size_t kExch8Bytes = ((size_t)kExch8Slots * 8 + 127) & ~(size_t)127;
__host__ __device__ constexpr size_t pass_buf_bytes(bool tma) {
  return tma ? kLandBytes + kExch8Bytes : (size_t)kSmemSlots * sizeof(float4);
}

// Split passes of single-tile circuits (all passes in one launch): the ops
// and coefficients of the running pass, staged after the block's context and
// accumulators (the launch asks for pass_stage_bytes() more shared memory).
// The backward's gradient rows of every pass of the launch are kept here
// too (block-private, summed over the block's tiles) when they fit, and
// written out once at the end.
constexpr int kMultiRows = 2048;
struct MultiStage {
  CoefRegion coef;
  DevOp ops[kMaxOps];
  int nops;
  float rows[kMultiRows];
};
__host__ __device__ constexpr size_t multi_stage_offset() {
  return (pass_buf_bytes(false) + sizeof(BlockCtx) + (size_t)(kThreads / 32) * kMaxSlots * 3 * sizeof(float) + 15) &
         ~(size_t)15;
}
__device__ __forceinline__ MultiStage* multi_stage(unsigned char* smem) {
  return reinterpret_cast<MultiStage*>(smem + multi_stage_offset());
}

// Register budget: the split-form passes (tensor copies, and the one-launch
// passes of single-tile circuits) and the fused-SU(2) tensor-copy passes
// (CNOT entanglers, with their permuted exchanges) may use up to 255
// registers (two blocks per SM); the re-uploading forms are held to 168
// (three blocks' worth), where their code does not spill, although the
// shared memory of a tensor-copy block still allows only two per SM.
template <bool BWD, int MODE, int V, int RE>
__global__ void __launch_bounds__(kThreads, (RE >= 3 || (RE == 0 && MODE == 2)) ? kBlocksPerSmTma : kBlocksPerSm)
    pass_kernel(const PassArgs a, const __grid_constant__ DevPass P, const __grid_constant__ CUtensorMap tm0,
                const __grid_constant__ CUtensorMap tm1) {
  constexpr bool SLOW = MODE == 0;
  constexpr bool TMA = MODE == 2;
  constexpr bool REUP = RE == 1 || RE == 2;  // data re-uploading folded into the fused rotations
  constexpr bool SPLIT = RE >= 3;            // split form: OP_RY / OP_DIAG instead of OP_ROT / OP_CZ
  // split passes of circuits that fit one tile (n <= 12): every pass in one
  // launch, coefficients from the workspace (see MULTI below)
  constexpr bool MULTI = SPLIT && !TMA;
  // fused CNOT layers (OP_PERM): passes loaded by tensor copies, in the
  // fused SU(2) form (RE 0) or the split form (RE 4)
  constexpr bool CNOTF = TMA && (RE == 0 || RE == 4);
  // RE 5: the complex-lane forward of single-tile circuits (one sample per
  // batch unit, its amplitude (re, im) in the re array; im unused)
  constexpr bool ZF = !BWD && RE == 5;
  // split-form tensor-copy passes: a cotangent-form rotation [[-u, 1], [1, u]]
  // is applied as its tangent-form factor T(-u) = [[1, u], [-u, 1]] followed
  // by a flip X of the qubit's register bit that is not carried out: register
  // j then holds the amplitude of position j ^ fl.  A later rotation of a
  // flipped bit takes the negated coefficient (X T(t) X = T(-t)), its backward
  // sums the negated y and z parts (X Y X = -Y, X Z X = -Z), a diagonal op
  // the flipped table index and sign bit, and the next exchange (plain or
  // permuted, for the CNOT maps) or store the flipped positions, which ends
  // the flips.  One rotation code per register bit, no branch on the form,
  // and the tangent form updated in place.
  constexpr bool FLIP = SPLIT && TMA && (RE == 3 || RE == 4);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  float4* tile = reinterpret_cast<float4*>(smem_raw);  // MODE 2: the landing buffer
  float2* ex8 = reinterpret_cast<float2*>(smem_raw + kLandBytes);  // MODE 2: the exchange buffer
  BlockCtx* bc = reinterpret_cast<BlockCtx*>(smem_raw + pass_buf_bytes(TMA));
  float* acc = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(bc) + sizeof(BlockCtx));  // [warps][nslots*3]
  const uint32_t tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kThreads / 32;
  const int region = a.region;
  const int nacc = P.nslots * 3;
  const bool loads = BWD || !P.gen;  // the forward's encoding pass reads nothing
  const float rs = (BWD && a.rscale) ? __ldg(a.rscale) : 1.f;  // scale of a restored checkpoint (split form)
  const uint32_t tile_s = (uint32_t)__cvta_generic_to_shared(tile);
  const uint32_t mbar = (uint32_t)__cvta_generic_to_shared(&bc->mbar);

  if (tid < kTileBits) {
    const int q = P.tile_q[tid];
    bc->qbit[tid] = q >= 0 ? (1u << q) : 0u;
    bc->ubit[tid] = q >= 0 ? 0u : (1u << (-1 - q));
    bc->abit[tid] = P.tile_abit[tid];
  }
  if (BWD)
    for (int i = tid; i < kWarps * nacc; i += kThreads) acc[i] = 0.f;
  if (TMA) {
    if ((tile_s & 127u) != 0) {  // tensor copies need a 128-byte aligned destination
      if (tid == 0) atomicOr(a.status, kErrBounds);
      return;
    }
    if (tid == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar) : "memory");
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
  }
  __syncthreads();
  cz_thread_terms<0, V>(*bc, P, a, tid);
  cz_thread_terms<1, V>(*bc, P, a, tid);
  cz_thread_terms<2, V>(*bc, P, a, tid);
  if (TMA && loads && tid == 0 && (int)blockIdx.x < a.n_tiles) {
    tma_coords(P, BWD, a.B, blockIdx.x, bc->tma_c, &bc->tma_sel);
    tma_load_tile(&tm0, &tm1, bc->tma_sel, bc->tma_c, tile_s, mbar);
  }
  uint32_t parity = 0;

  // Without tensor copies the next tile is fetched into the shared tile
  // buffer once the buffer is free (after the pass's last exchange), so its
  // latency hides behind the last register phase; n < 5 loads directly.  The
  // tensor copy of the next tile is issued right after the current tile is in
  // registers.
  const bool can_pf = !SLOW && loads && !MULTI;
  const int mem_ph = BWD ? P.store_phase : P.load_phase;
  const int pf_at = BWD ? P.pf_bwd : P.pf_fwd;  // op index after which to prefetch (-1: after the load)
  bool have_pf = false;
  uint32_t pco = 0;  // fused CNOT layers: the out-of-tile part of the tile's gather

  // The ops of one pass on the registers, forward order (PP: the pass, C: its
  // coefficients; the layout is P's, the same for every pass of a launch).
  auto run_fwd_ops = [&](const DevPass& PP, const auto& OPS, int nops, const CoefRegion* C, uint32_t base_q,
                         uint32_t s_o, uint32_t unit_base,
                         float2 (&re)[kPos], float2 (&im)[kPos], bool pf_next, auto&& prefetch_next, uint32_t& fl) {
    for (int oi = 0; oi < nops; ++oi) {
      const DevOp op = OPS[oi];
      if (op.kind == OP_EXCH) {
        if constexpr (ZF) exchange8<V, true>(op.a, op.b, re, im, reinterpret_cast<float2*>(tile), tid);
        else if constexpr (FLIP) exchange8<V>(op.a, op.b, re, im, ex8, tid, fl);
        else if constexpr (TMA) exchange8<V>(op.a, op.b, re, im, ex8, tid);
        else exchange<V>(op.a, op.b, re, im, tile, tid);
        fl = 0;
      } else if constexpr (SPLIT) {
        if (op.kind == OP_RY) {
          int slot = op.d;
#pragma unroll
          for (int k = 0; k < kRegBits; ++k)
            if ((op.b >> k) & 1) {
              const float4 f0 = C->rot[slot][0];
              const bool cot = C->rot[slot][1].x != 0.f;
              ++slot;
              const float2 p = make_float2(f0.x, f0.y), np = make_float2(f0.z, f0.w);
              if constexpr (ZF) {
                if (cot) ry1_fwd_k<true>(k, re, p, np);
                else ry1_fwd_k<false>(k, re, p, np);
              } else if constexpr (FLIP) {
                // tangent form with t (tangent), -u (cotangent), negated on a flipped bit
                const bool neg = cot != (((fl >> k) & 1u) != 0u);
                ry_fwd_k<false, true>(k, re, im, neg ? np : p, neg ? p : np);
                if (cot) fl ^= 1u << k;
              } else {
                if (cot) ry_fwd_k<true>(k, re, im, p, np);
                else ry_fwd_k<false>(k, re, im, p, np);
              }
            }
        } else if (op.kind == OP_DIAG) {
          diag_op<V, ZF>(op.a, re, im, *bc, P, a, C, op.d, op.c, tid, base_q, s_o, fl);
        } else if (op.kind == OP_PERM) {
          if constexpr (CNOTF)
            if (PP.perm_at[0] == 2) {
              exchange8p<V>(op.a, op.b, re, im, ex8, tid, PP, 0, pco, fl);
              fl = 0;
            }
        }
      } else if (op.kind == OP_ROT) {
        int slot = op.d;
        if (REUP) {  // the encoding again, folded into the layer's rotations
          uint32_t unit, mu[kRegBits];
          int rq[kRegBits];
          unit_maps<V>(op.a, *bc, tid, unit_base, &unit, mu, rq);
#pragma unroll
          for (int k = 0; k < kRegBits; ++k)
            if ((op.b >> k) & 1) {
              const Coef c = const_coef(region, slot++);
              if (RE == 1) {
                float2 cs, sn;
                enc_coef<false>(a, unit, rq[k], &cs, &sn);
                rot_fwd_k(k, re, im, SameCoef{reup_coef<false>(c, cs, sn)});
              } else {
                rot_fwd_k(k, re, im, ReupPairCoef<false>{c, a, rq[k], unit, mu});
              }
            }
        } else {
#pragma unroll
          for (int k = 0; k < kRegBits; ++k)
            if ((op.b >> k) & 1) rot_fwd_k(k, re, im, SameCoef{const_coef(region, slot++)});
        }
      } else if (op.kind == OP_CZ) {
        cz_op<V>(op.a, re, im, *bc, P, tid, base_q, s_o);
      } else if (op.kind == OP_PERM) {
        if constexpr (CNOTF)
          if (PP.perm_at[0] == 2) exchange8p<V>(op.a, op.b, re, im, ex8, tid, PP, 0, pco);
      }
      if (pf_next && oi == pf_at) prefetch_next();
    }
  };

  // The ops of one pass in reverse (un-applied), with the gradient sums into acc.
  auto run_bwd_ops = [&](const DevPass& PP, const auto& OPS, int nops, const CoefRegion* C, uint32_t base_q,
                         uint32_t s_o, uint32_t unit_base,
                         float2 (&re)[kPos], float2 (&im)[kPos], bool pf_next, auto&& prefetch_next, uint32_t& fl) {
    const int pacc = PP.nslots * 3;  // row stride of the pass's sums
    for (int oi = nops - 1; oi >= 0; --oi) {
      const DevOp op = OPS[oi];
      if (op.kind == OP_EXCH) {
        if constexpr (FLIP) exchange8<V>(op.b, op.a, re, im, ex8, tid, fl);
        else if constexpr (TMA) exchange8<V>(op.b, op.a, re, im, ex8, tid);
        else exchange<V>(op.b, op.a, re, im, tile, tid);
        fl = 0;
      } else if constexpr (SPLIT) {
        if (op.kind == OP_RY) {
          // the same sums, then Ry un-applied (tangent or cotangent form)
          int slot = op.d, pslot = -1;
          float3 pend = make_float3(0.f, 0.f, 0.f);
#pragma unroll
          for (int k = 0; k < kRegBits; ++k)
            if ((op.b >> k) & 1) {
              float r;
              float3 v;
              const float4 f0 = C->rot[slot][0];
              const bool cot = C->rot[slot][1].x != 0.f;
              const float2 p = make_float2(f0.x, f0.y), np = make_float2(f0.z, f0.w);
              v = rot_bwd_sums_k(k, re, im, pend, lane, &r);
              if constexpr (FLIP) {
                const bool fk = ((fl >> k) & 1u) != 0u;
                if (fk) v.y = -v.y, v.z = -v.z;  // sums of the flipped bit's qubit
                const bool neg = cot != fk;
                ry_fwd_k<false, true>(k, re, im, neg ? np : p, neg ? p : np);
                if (cot) fl ^= 1u << k;
              } else {
                if (cot) ry_fwd_k<true>(k, re, im, p, np);
                else ry_fwd_k<false>(k, re, im, p, np);
              }
              if (pslot >= 0 && (lane & 7) == 0 && lane < 24) acc[warp * pacc + pslot * 3 + (lane >> 3)] += r;
              pend = v;
              pslot = slot++;
            }
          if (pslot >= 0) {
            const float r = warp_reduce3(pend.x, pend.y, pend.z, lane);
            if ((lane & 7) == 0 && lane < 24) acc[warp * pacc + pslot * 3 + (lane >> 3)] += r;
          }
        } else if (op.kind == OP_DIAG) {
          // the diagonal before layer 0 needs no un-applying: nothing reads the state after it
          if (op.c >= 0) diag_op<V>(op.a, re, im, *bc, P, a, C, op.d, op.c, tid, base_q, s_o, fl);
        } else if (op.kind == OP_PERM) {
          if constexpr (CNOTF)
            if (PP.perm_at[1] == 2) {
              exchange8p<V>(op.b, op.a, re, im, ex8, tid, PP, 1, pco, fl);
              fl = 0;
            }
        }
      } else if (op.kind == OP_ROT) {
        // each rotation finishes the warp sum of the previous one
        int slot = op.d, pslot = -1;
        float3 pend = make_float3(0.f, 0.f, 0.f);
        // re-uploading: Ry(-x) of the layer's encoding joins U^dagger
        uint32_t unit = 0, mu[kRegBits] = {0u, 0u, 0u, 0u, 0u};
        int rq[kRegBits] = {0, 0, 0, 0, 0};
        if (REUP) unit_maps<V>(op.a, *bc, tid, unit_base, &unit, mu, rq);
#pragma unroll
        for (int k = 0; k < kRegBits; ++k)
          if ((op.b >> k) & 1) {
            float r;
            float3 v;
            const Coef c = const_coef(region, slot);
            if (RE == 0) {
              v = rot_bwd_red_k(k, re, im, SameCoef{c}, pend, lane, &r);
            } else if (RE == 1) {
              float2 cs, sn;
              enc_coef<true>(a, unit, rq[k], &cs, &sn);
              v = rot_bwd_red_k(k, re, im, SameCoef{reup_coef<true>(c, cs, sn)}, pend, lane, &r);
            } else {
              v = rot_bwd_red_k(k, re, im, ReupPairCoef<true>{c, a, rq[k], unit, mu}, pend, lane, &r);
            }
            if (pslot >= 0 && (lane & 7) == 0 && lane < 24) acc[warp * pacc + pslot * 3 + (lane >> 3)] += r;
            pend = v;
            pslot = slot++;
          }
        if (pslot >= 0) {
          const float r = warp_reduce3(pend.x, pend.y, pend.z, lane);
          if ((lane & 7) == 0 && lane < 24) acc[warp * pacc + pslot * 3 + (lane >> 3)] += r;
        }
      } else if (op.kind == OP_CZ) {
        cz_op<V>(op.a, re, im, *bc, P, tid, base_q, s_o);
      } else if (op.kind == OP_PERM) {
        if constexpr (CNOTF)
          if (PP.perm_at[1] == 2) exchange8p<V>(op.b, op.a, re, im, ex8, tid, PP, 1, pco);
      }
      if (pf_next && oi == pf_at) prefetch_next();
    }
  };

  if constexpr (MULTI) {
    // Every pass of the launch (a.npass of them, all with P's tile layout) on
    // each tile, the state kept in registers in between.  The backward's sums
    // go to the block's row of each pass after that pass, so start the rows
    // at zero.
    // (a pass's rows start at partial_off = gridDim.x x the rows of the
    // passes before it, so partial_off / gridDim.x is its offset in the
    // block's own rows)
    MultiStage* stg = multi_stage(smem_raw);
    const DevPass& PLast = a.passes[a.npass - 1];
    const int nrows = (int)(PLast.partial_off / gridDim.x) + PLast.nslots * 3;
    const bool srows = BWD && nrows <= kMultiRows;
    if (srows) {
      for (int i = tid; i < nrows; i += kThreads) stg->rows[i] = 0.f;
    } else if (BWD) {
      for (int pi = 0; pi < a.npass; ++pi) {
        const int pn = a.passes[pi].nslots * 3;
        float* row = a.partials + a.passes[pi].partial_off + (size_t)blockIdx.x * pn;
        for (int i = tid; i < pn; i += kThreads) row[i] = 0.f;
      }
    }
    auto none = []() {};
    uint32_t nofl = 0;  // (no flips outside the tensor-copy split passes)
    // each pass's ops and coefficients are staged in shared memory before
    // the pass runs (read from global memory they would stall every op)
    auto stage = [&](int pi) {
      __syncthreads();  // the previous pass is done with the stage
      const DevPass& PP = a.passes[pi];
      const int* so = reinterpret_cast<const int*>(PP.ops);
      int* dop = reinterpret_cast<int*>(stg->ops);
      for (int i = tid; i < kMaxOps * 5; i += kThreads) dop[i] = so[i];
      const float4* sc = reinterpret_cast<const float4*>(a.coef + pi);
      float4* dc = reinterpret_cast<float4*>(&stg->coef);
      for (int i = tid; i < (int)(sizeof(CoefRegion) / 16); i += kThreads) dc[i] = sc[i];
      if (tid == 0) stg->nops = PP.nops;
      __syncthreads();
    };
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
      uint32_t base_q, base_a, unit_base;
      tile_base(P, t, &base_q, &base_a, &unit_base);
      const uint32_t s_o = bond_parity(base_q, a);
      float2 re[kPos], im[kPos];
      if (ZF) {
        // the complex-lane form starts from the encoding and ends with the
        // standard-order state (the host launches it for no other chain)
        if (!a.passes[0].gen || !a.passes[a.npass - 1].last) {
          if (tid == 0) atomicOr(a.status, kErrBounds);
          return;
        }
        const DevPass& P0 = a.passes[0];
        mem_op<false, SLOW, V, M_GEN, ZF>(P0.load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
        for (int pi = 0; pi < a.npass; ++pi) {
          const DevPass& PP = a.passes[pi];
          stage(pi);
          run_fwd_ops(PP, stg->ops, stg->nops, &stg->coef, base_q, s_o, unit_base, re, im, false, none, nofl);
          if (PP.ckpt >= 0)
            mem_op<false, SLOW, V, M_CKPT_STORE, ZF>(PP.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im,
                                                     PP.ckpt);
        }
        const DevPass& PL = a.passes[a.npass - 1];
        mem_op<false, SLOW, V, M_STORE_STD, ZF>(PL.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im,
                                                t & ((1 << PL.n_out) - 1));
      } else if (!BWD) {
        const DevPass& P0 = a.passes[0];
        if (P0.gen) mem_op<false, SLOW, V, M_GEN>(P0.load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
        else mem_op<false, SLOW, V, M_LOAD>(P0.load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
        for (int pi = 0; pi < a.npass; ++pi) {
          const DevPass& PP = a.passes[pi];
          stage(pi);
          run_fwd_ops(PP, stg->ops, stg->nops, &stg->coef, base_q, s_o, unit_base, re, im, false, none, nofl);
          if (PP.ckpt >= 0)
            mem_op<false, SLOW, V, M_CKPT_STORE>(PP.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im, PP.ckpt);
        }
        const DevPass& PL = a.passes[a.npass - 1];
        if (PL.last)
          mem_op<false, SLOW, V, M_STORE_STD>(PL.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im,
                                              t & ((1 << PL.n_out) - 1));
        else mem_op<false, SLOW, V, M_STORE>(PL.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
      } else {
        const DevPass& PL = a.passes[a.npass - 1];
        mem_op<true, SLOW, V, M_LOAD>(PL.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
        for (int pi = a.npass - 1; pi >= 0; --pi) {
          const DevPass& PP = a.passes[pi];
          if (PP.ckpt >= 0)
            mem_op<true, SLOW, V, M_CKPT_RESTORE>(PP.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im,
                                                  PP.ckpt, a.rscale ? __ldg(a.rscale + pi) : 1.f);
          for (int i = tid; i < kWarps * kMaxSlots * 3; i += kThreads) acc[i] = 0.f;
          stage(pi);
          run_bwd_ops(PP, stg->ops, stg->nops, &stg->coef, base_q, s_o, unit_base, re, im, false, none, nofl);
          __syncthreads();
          const int pn = PP.nslots * 3;
          float* row = srows ? stg->rows + PP.partial_off / gridDim.x : a.partials + PP.partial_off + (size_t)blockIdx.x * pn;
          for (int i = tid; i < pn; i += kThreads) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += acc[w * pn + i];
            row[i] += v;
          }
          __syncthreads();
        }
        // the first pass is the encoding pass: nothing reads the state after it
        if (!a.passes[0].gen) mem_op<true, SLOW, V, M_STORE>(a.passes[0].load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
      }
    }
    if (srows) {  // the block's rows, summed over its tiles, written once
      __syncthreads();
      for (int pi = 0; pi < a.npass; ++pi) {
        const DevPass& PP = a.passes[pi];
        const int pn = PP.nslots * 3;
        const float* src = stg->rows + PP.partial_off / gridDim.x;
        float* row = a.partials + PP.partial_off + (size_t)blockIdx.x * pn;
        for (int i = tid; i < pn; i += kThreads) row[i] = src[i];
      }
    }
    return;
  }

  const CoefRegion* creg = &c_reg[region];
  for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
    uint32_t base_q, base_a, unit_base;
    tile_base(P, t, &base_q, &base_a, &unit_base);
    const uint32_t s_o = bond_parity(base_q, a);  // entangler terms of the out-of-tile bits
    if constexpr (CNOTF) {
      if (P.perm_at[BWD]) {
        const uint32_t o = (uint32_t)t & ((1u << P.n_out) - 1u);
        pco = 0;
        for (int k = 0; k < P.n_out; ++k)
          if ((o >> k) & 1u) pco ^= P.pcol_o[BWD][k];
      }
    }
    const int tn = t + (int)gridDim.x;
    const bool pf_next = can_pf && tn < a.n_tiles;
    auto prefetch_next = [&]() {
      if constexpr (!TMA) {
        __syncthreads();  // every thread is done with the tile buffer
        uint32_t bq, ba, ub;
        tile_base(P, tn, &bq, &ba, &ub);
        prefetch_op<BWD, V>(mem_ph, a, *bc, tid, bq, ba, ub, tile);
      }
    };

    if (TMA && pf_next && tid == 0) tma_coords(P, BWD, a.B, tn, bc->tma_c, &bc->tma_sel);
    float2 re[kPos], im[kPos];
    if (TMA && loads) {
      const uint32_t ph = parity;
      parity ^= 1u;
      const bool ok = mbar_wait(mbar, ph);
      if (__syncthreads_or(!ok)) {
        // the copy never completed: report, give it one more bounded wait, stop
        if (tid == 0) {
          atomicOr(a.status, kErrTimeout);
          mbar_wait(mbar, ph);
        }
        return;
      }
      float2* tb = reinterpret_cast<float2*>(tile);
      if (BWD && P.ckpt >= 0) {
        if (mem_ph == 0) restore_tma_t<0, V>(a, *bc, P, tid, base_q, unit_base, tb, P.ckpt, rs);
        else restore_tma_t<1, V>(a, *bc, P, tid, base_q, unit_base, tb, P.ckpt, rs);
      }
      if (CNOTF && P.perm_at[BWD] == 1) {
        load_tma_perm<V>(mem_ph, re, im, tb, P, BWD ? 1 : 0, pco, tid);
      } else {
        load_tma<V>(mem_ph, re, im, tb, P, tid);
      }
      __syncthreads();  // every thread has its positions: the landing buffer is free
      if (pf_next && tid == 0) tma_load_tile(&tm0, &tm1, bc->tma_sel, bc->tma_c, tile_s, mbar);
    }
    if (!BWD) {
      if (P.gen) mem_op<false, SLOW, V, M_GEN>(P.load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
      else if (TMA) {
      } else if (have_pf) load_prefetched<V>(P.load_phase, re, im, tile, tid);
      else mem_op<false, SLOW, V, M_LOAD>(P.load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
      if (pf_next && pf_at < 0) prefetch_next();
      uint32_t fl = 0;  // pending flips (FLIP passes)
      run_fwd_ops(P, P.ops, P.nops, creg, base_q, s_o, unit_base, re, im, pf_next, prefetch_next, fl);
      if (P.ckpt >= 0)
        mem_op<false, SLOW, V, M_CKPT_STORE>(P.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im, P.ckpt, 1.f,
                                             fl);
      if (P.last)
        mem_op<false, SLOW, V, M_STORE_STD>(P.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im,
                                            t & ((1 << P.n_out) - 1), 1.f, fl);
      else mem_op<false, SLOW, V, M_STORE>(P.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im, 0, 1.f, fl);
    } else {
      if (TMA) {
      } else if (have_pf) load_prefetched<V>(P.store_phase, re, im, tile, tid);
      else mem_op<true, SLOW, V, M_LOAD>(P.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im);
      if (!TMA && P.ckpt >= 0)
        mem_op<true, SLOW, V, M_CKPT_RESTORE>(P.store_phase, a, *bc, tid, base_q, base_a, unit_base, re, im, P.ckpt, rs);
      if (pf_next && pf_at < 0) prefetch_next();
      uint32_t fl = 0;  // pending flips (FLIP passes)
      run_bwd_ops(P, P.ops, P.nops, creg, base_q, s_o, unit_base, re, im, pf_next, prefetch_next, fl);
      if (!P.gen) mem_op<true, SLOW, V, M_STORE>(P.load_phase, a, *bc, tid, base_q, base_a, unit_base, re, im, 0, 1.f, fl);
    }
    have_pf = pf_next;
  }

  if (BWD) {
    __syncthreads();
    float* out = a.partials + P.partial_off + (size_t)blockIdx.x * nacc;
    for (int i = tid; i < nacc; i += kThreads) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += acc[w * nacc + i];
      out[i] = v;
    }
  }
}

// Copy one pass's gate coefficients (device memory) into this unit's
// constant-memory region, in stream order: the first nslots rotation slots,
// and with diagonal ops the whole region (its tables follow the slots).
inline cudaError_t copy_coef_here(int region, const CoefRegion* src, int nslots, int ndiag, cudaStream_t s) {
  const size_t off = (size_t)region * sizeof(CoefRegion);
  const size_t bytes = ndiag > 0 ? sizeof(CoefRegion) : (size_t)nslots * sizeof(src->rot[0]);
  if (bytes == 0) return cudaSuccess;
  return cudaMemcpyToSymbolAsync(c_reg, src, bytes, off, cudaMemcpyDeviceToDevice, s);
}

}  // namespace
}  // namespace qml

// Launch and attribute functions of one translation unit's instances: LIST(X)
// names them as X(backward, mode, variant, form).
#define QML_PASS_LAUNCH_CASE(B, M, V, R)                                                            \
  if (backward == B && mode == M && variant == V && form == R) {                                     \
    if (coef) {                                                                                      \
      const cudaError_t ce = copy_coef_here(a.region, coef, p.nslots, p.ndiag, s);                  \
      if (ce != cudaSuccess) return ce;                                                              \
    }                                                                                                \
    pass_kernel<B, M, V, R><<<grid, kThreads, smem, s>>>(a, p, m0, m1);                              \
    return cudaGetLastError();                                                                       \
  }
#define QML_PASS_ATTR_CASE(B, M, V, R)                                                                \
  if (e == cudaSuccess)                                                                              \
    e = cudaFuncSetAttribute(pass_kernel<B, M, V, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                             (int)(M == 2 ? smem_tma : smem_thr));                                   \
  if (e == cudaSuccess)                                                                              \
    e = cudaFuncSetAttribute(pass_kernel<B, M, V, R>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
#define QML_DEFINE_PASS_UNIT(NAME, LIST)                                                             \
  namespace qml {                                                                                     \
  cudaError_t NAME##_launch(bool backward, int mode, int variant, int form, const PassArgs& a,        \
                            const DevPass& p, const PassMaps& maps, int grid, size_t smem,            \
                            const CoefRegion* coef, cudaStream_t s) {                                 \
    const CUtensorMap& m0 = *reinterpret_cast<const CUtensorMap*>(maps.m0);                          \
    const CUtensorMap& m1 = *reinterpret_cast<const CUtensorMap*>(maps.m1);                          \
    LIST(QML_PASS_LAUNCH_CASE)                                                                        \
    return cudaErrorInvalidValue;                                                                     \
  }                                                                                                   \
  cudaError_t NAME##_attr(size_t smem_thr, size_t smem_tma) {                                         \
    cudaError_t e = cudaSuccess;                                                                      \
    LIST(QML_PASS_ATTR_CASE)                                                                          \
    return e;                                                                                         \
  }                                                                                                   \
  }
