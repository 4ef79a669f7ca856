// f64.cu -- fp64 compute mode: the same fused forward and adjoint backward
// passes with complex128 state vectors (re, im doubles) and fp64 arithmetic.
//
// The method is the one of kernels.cu (forward gate fusion, backward gate
// fusion that rebuilds psi next to lambda, CZ entanglers as index-parity
// signs; Kawase, "Fast and memory-efficient classical simulation of quantum
// machine learning via forward and backward gate fusion", [Deep-dive] sec. 1.2
// and 1.4, sec. 3.2).  The pages state that the simulator runs in double as
// well as single precision ([Gist-EN] Technical Summary sec. 2 and 4).
//
// Layout and schedule.  The passes of the fp32 schedule are reused: the ops
// are the same rotations and CZ layers, and a pass's tile holds the qubits
// the schedule gives it, less one qubit that the pass does not rotate when the
// schedule's tile has 12 (so a tile is at most 2^11 positions and two blocks
// fit on an SM).  The state stays in the standard index order throughout.  A
// block keeps one sample's tile in shared memory (psi, and lambda in the
// backward: 36 KB per plane with one pad element per eight), and a rotation
// op is applied in chunks of up to three qubits: each thread takes the eight
// positions of one chunk group into registers, applies the chunk's 2x2
// unitaries (and, backward, accumulates the three Im<lambda|P|psi> terms of
// each qubit first), and writes them back.
#include <cuda_bf16.h>

#include <algorithm>

#include "kernels.cuh"

namespace qml {

namespace {

constexpr unsigned kErrNumeric = 1u << 6;  // QML_ERR_NUMERIC
constexpr unsigned kErrBounds = 1u << 7;   // QML_ERR_BOUNDS

constexpr int kW = kF64Warps;
constexpr int kT = kF64Threads;

__device__ __forceinline__ int padp(int p) { return p + (p >> 3); }
// shared positions of one plane for tiles of up to 2^tmax positions
constexpr int plane_slots(int tmax) { return (1 << tmax) + ((1 << tmax) >> 3); }

// Per-block schedule data, built at kernel start.
struct Ctx64 {
  int T, n_out;
  int tq[kTileBits];      // position bit -> qubit (ascending)
  int oq[kMaxQubits];     // out-of-tile qubits (ascending)
  int pos_of_q[kMaxQubits];
  uint32_t off_lo[64], off_hi[64];  // index offset of position bits 0-5 / 6-11
  uint32_t s_off[kTilePos / 32];    // entangler parity of the in-tile part of each position
  double4 coef[kMaxSlots];          // (ar, ai, br, bi): U forward, U^dagger backward; split form: (p, cot, 0, 0)
  double cs[kMaxQubits], sn[kMaxQubits];  // (cos, sin)(x/2) of the tile's sample
  double2 dlo[64], dhi[64];         // split form, diagonal op: factors of position bits 0-5 / 6-11
  uint32_t pcol[kMaxQubits];        // fused CNOT layers: tile position of the gather map's image of each qubit
};

size_t f64_smem_bytes(bool bwd, int tmax) {
  size_t b = sizeof(double2) * (size_t)plane_slots(tmax) * (bwd ? 2 : 1) + sizeof(Ctx64);
  if (bwd) b += sizeof(double) * (size_t)kW * kMaxSlots * 3;
  return b;
}

// (x, y) <- (a x + b y, -conj(b) x + conj(a) y), u = (ar, ai, br, bi)
__device__ __forceinline__ void su2_64(double2& x, double2& y, const double4& u) {
  const double xr = x.x, xi = x.y, yr = y.x, yi = y.y;
  x.x = fma(u.x, xr, fma(-u.y, xi, fma(u.z, yr, -u.w * yi)));
  x.y = fma(u.x, xi, fma(u.y, xr, fma(u.z, yi, u.w * yr)));
  y.x = fma(-u.z, xr, fma(-u.w, xi, fma(u.x, yr, u.y * yi)));
  y.y = fma(-u.z, xi, fma(u.w, xr, fma(u.x, yi, -u.y * yr)));
}

// Re-uploading folded into the rotation (one sample per tile): U Ry(x)
// forward, Ry(-x) U^dagger backward (u holding U^dagger); (c, s) = (cos,
// sin)(x/2).  U Ry(x): a' = a c + b s, b' = b c - a s.  Ry(-x) U^dagger:
// a' = a c - conj(b) s, b' = b c + conj(a) s.
template <bool BWD>
__device__ __forceinline__ double4 reup64(double4 u, double c, double s) {
  if (!BWD) return make_double4(u.x * c + u.z * s, u.y * c + u.w * s, u.z * c - u.x * s, u.w * c - u.y * s);
  return make_double4(u.x * c - u.z * s, u.y * c + u.w * s, u.z * c + u.x * s, u.w * c - u.y * s);
}

// Split form: Ry on the pair (x, y), p = u.x, cotangent form when u.y != 0
// (the same forms and the same parameter convention as the fp32 passes:
// tangent x <- x - p y, y <- y + p x; cotangent x <- y - p x, y <- x + p y;
// the backward pass un-applies with -p (tangent) or p (cotangent)).
__device__ __forceinline__ void ry64(double2& x, double2& y, const double4& u) {
  const double p = u.x;
  const double2 x0 = x;
  if (u.y == 0.0) {
    x = make_double2(fma(-p, y.x, x0.x), fma(-p, y.y, x0.y));
    y = make_double2(fma(p, x0.x, y.x), fma(p, x0.y, y.y));
  } else {
    x = make_double2(fma(-p, x0.x, y.x), fma(-p, x0.y, y.y));
    y = make_double2(fma(p, y.x, x0.x), fma(p, y.y, x0.y));
  }
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double2 slot_load(const Pass64Args& a, int slot, size_t g) {
  const size_t i = (size_t)slot * a.slot_elems + g;
  if (a.storage == 2) return reinterpret_cast<const double2*>(a.ckpt)[i];
  if (a.storage == 1) {
    const __nv_bfloat162 v = reinterpret_cast<const __nv_bfloat162*>(a.ckpt)[i];
    return make_double2((double)__bfloat162float(v.x), (double)__bfloat162float(v.y));
  }
  const float2 v = reinterpret_cast<const float2*>(a.ckpt)[i];
  return make_double2((double)v.x, (double)v.y);
}

__device__ __forceinline__ void slot_store(const Pass64Args& a, int slot, size_t g, double2 v) {
  const size_t i = (size_t)slot * a.slot_elems + g;
  if (a.storage == 2) {
    reinterpret_cast<double2*>(a.ckpt)[i] = v;
  } else if (a.storage == 1) {
    __nv_bfloat162 h;
    h.x = __float2bfloat16_rn((float)v.x);  // fp64 -> fp32 -> bf16, both round to nearest even
    h.y = __float2bfloat16_rn((float)v.y);
    reinterpret_cast<__nv_bfloat162*>(a.ckpt)[i] = h;
  } else {
    reinterpret_cast<float2*>(a.ckpt)[i] = make_float2((float)v.x, (float)v.y);
  }
}

// One rotation chunk of K qubits (slots s0 .. s0+K-1) over the tile.
template <bool BWD, int K, bool SPLIT>
__device__ void rot_chunk(const Pass64Args& a, const DevPass& P, const Ctx64& cx, double2* tp, double2* tl,
                          double* acc, int s0, int warp, int lane) {
  int pb[K], srt[K];
  double4 u[K];
#pragma unroll
  for (int i = 0; i < K; ++i) {
    const int q = P.slot_lq[s0 + i] % a.n;
    pb[i] = cx.pos_of_q[q];
    u[i] = cx.coef[s0 + i];
    if (a.reupload) u[i] = reup64<BWD>(u[i], cx.cs[q], cx.sn[q]);
    srt[i] = pb[i];
  }
#pragma unroll
  for (int i = 1; i < K; ++i)  // ascending, for inserting the chunk bits
#pragma unroll
    for (int j = K - 1; j >= i; --j)
      if (srt[j - 1] > srt[j]) {
        const int t = srt[j];
        srt[j] = srt[j - 1];
        srt[j - 1] = t;
      }
  double sx[K], sy[K], sz[K];
#pragma unroll
  for (int i = 0; i < K; ++i) sx[i] = sy[i] = sz[i] = 0.0;
  const int G = (1 << cx.T) >> K;
  for (int g = threadIdx.x; g < G; g += kT) {
    int p0 = g;
#pragma unroll
    for (int i = 0; i < K; ++i) p0 = ((p0 >> srt[i]) << (srt[i] + 1)) | (p0 & ((1 << srt[i]) - 1));
    // position of register j: p0 plus the chunk bits set in j
    auto pos = [&](int j) {
      int p = p0;
#pragma unroll
      for (int i = 0; i < K; ++i)
        if ((j >> i) & 1) p |= 1 << pb[i];
      return padp(p);
    };
    double2 v[1 << K], w[1 << K];
#pragma unroll
    for (int j = 0; j < (1 << K); ++j) {
      v[j] = tp[pos(j)];
      if (BWD) w[j] = tl[pos(j)];
    }
#pragma unroll
    for (int i = 0; i < K; ++i) {
#pragma unroll
      for (int j = 0; j < (1 << K); ++j) {
        if ((j >> i) & 1) continue;
        const int jj = j | (1 << i);
        if (BWD) {
          // terms at the state just after this qubit's rotation (psi = v, lambda = w)
          const double2 p0v = v[j], p1v = v[jj], l0 = w[j], l1 = w[jj];
          sx[i] += l0.x * p1v.y - l0.y * p1v.x + l1.x * p0v.y - l1.y * p0v.x;  // Im(conj l0 p1 + conj l1 p0)
          sy[i] += l1.x * p0v.x + l1.y * p0v.y - l0.x * p1v.x - l0.y * p1v.y;  // Re(conj l1 p0 - conj l0 p1)
          sz[i] += l0.x * p0v.y - l0.y * p0v.x - l1.x * p1v.y + l1.y * p1v.x;  // Im(conj l0 p0 - conj l1 p1)
          if (SPLIT) ry64(w[j], w[jj], u[i]);
          else su2_64(w[j], w[jj], u[i]);
        }
        if (SPLIT) ry64(v[j], v[jj], u[i]);
        else su2_64(v[j], v[jj], u[i]);
      }
    }
#pragma unroll
    for (int j = 0; j < (1 << K); ++j) {
      tp[pos(j)] = v[j];
      if (BWD) tl[pos(j)] = w[j];
    }
  }
  if (BWD) {
    // warp sums of the chunk's 3K terms as one reduce-scatter: the terms sit
    // in 16 slots (the unused ones zero); each xor step sends half of a
    // lane's remaining slots to its partner and adds the other half, so after
    // four steps lane l holds slot ((l >> 1) & 15) summed over 16 lanes, and
    // a last step completes it (16 shuffles for up to 9 terms, instead of 5
    // per term)
    double r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = 0.0;
#pragma unroll
    for (int i = 0; i < K; ++i) {
      r[3 * i + 0] = sx[i];
      r[3 * i + 1] = sy[i];
      r[3 * i + 2] = sz[i];
    }
#pragma unroll
    for (int st = 0; st < 4; ++st) {
      const int half = 8 >> st, off = 16 >> st;
      const bool up = (lane & off) != 0;  // keep the upper half of the remaining slots
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const double send = up ? r[i] : r[i + half];
        const double got = __shfl_xor_sync(0xffffffffu, send, off);
        r[i] = (up ? r[i + half] : r[i]) + got;
      }
    }
    const double v = r[0] + __shfl_xor_sync(0xffffffffu, r[0], 1);
    // lane l now holds the full sum of slot (l>>4)*8 + ((l>>3)&1)*4 + ((l>>2)&1)*2 + ((l>>1)&1)
    const int slot = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
    if ((lane & 1) == 0 && slot < 3 * K) acc[((size_t)warp * kMaxSlots + s0 + slot / 3) * 3 + slot % 3] += v;
  }
}

// SPLIT: the split form (OP_RY / OP_DIAG passes, a.srot set); otherwise the
// fused SU(2) (OP_ROT / OP_CZ).
template <bool BWD, bool SPLIT>
__global__ void __launch_bounds__(kT, BWD ? 2 : 3) pass64_kernel(const Pass64Args a, const __grid_constant__ DevPass P) {
  extern __shared__ __align__(16) unsigned char smem64[];
  double2* tp = reinterpret_cast<double2*>(smem64);
  const int plane = plane_slots(a.tmax);
  double2* tl = tp + plane;
  Ctx64& cx = *reinterpret_cast<Ctx64*>(smem64 + sizeof(double2) * plane * (BWD ? 2 : 1));
  double* acc = reinterpret_cast<double*>(reinterpret_cast<unsigned char*>(&cx) + sizeof(Ctx64));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = a.n;

  if (tid == 0) {
    const uint32_t inmask = a.tile_mask;  // this pass's tile qubits
    int T = 0, no = 0;
    for (int q = 0; q < n; ++q) {
      cx.pos_of_q[q] = -1;
      if ((inmask >> q) & 1u) {
        cx.pos_of_q[q] = T;
        cx.tq[T++] = q;
      } else {
        cx.oq[no++] = q;
      }
    }
    cx.T = T;
    cx.n_out = no;
  }
  // gate coefficients of the pass's slots: U = Rz Ry Rx, in fp64; split
  // form: the tangent-form parameter of Ry (backward: its inverse's)
  constexpr bool split = SPLIT;
  for (int s = tid; s < P.nslots && split; s += kT) {
    const SplitRot r = a.srot[P.slot_lq[s]];
    const double pr = (BWD && !r.cot) ? -r.tau : r.tau;
    cx.coef[s] = make_double4(pr, (double)r.cot, 0.0, 0.0);
  }
  for (int s = tid; s < P.nslots && !split; s += kT) {
    const int lq = P.slot_lq[s];
    double sa, ca, sb, cb, sg, cg;
    sincos(0.5 * a.theta[lq * 3 + 0], &sa, &ca);
    sincos(0.5 * a.theta[lq * 3 + 1], &sb, &cb);
    sincos(0.5 * a.theta[lq * 3 + 2], &sg, &cg);
    // (Ry Rx)[0][0] = cb ca + i sb sa, (Ry Rx)[0][1] = -sb ca - i cb sa; Rz row 0 is e^{-i g/2}
    const double p_re = cb * ca, p_im = sb * sa, q_re = -sb * ca, q_im = -cb * sa;
    const double ar = cg * p_re + sg * p_im, ai = cg * p_im - sg * p_re;
    const double br = cg * q_re + sg * q_im, bi = cg * q_im - sg * q_re;
    cx.coef[s] = BWD ? make_double4(ar, -ai, -br, -bi) : make_double4(ar, ai, br, bi);  // U^dagger: (conj a, -b)
  }
  if (BWD)
    for (int i = tid; i < kW * kMaxSlots * 3; i += kT) acc[i] = 0.0;
  __syncthreads();
  const int T = cx.T, P2 = 1 << T, no = cx.n_out;
  if (T != a.T || T > a.tmax) {  // the host's tile does not fit: touch nothing
    if (tid == 0) atomicOr(a.status, kErrBounds);
    return;
  }
  for (int i = tid; i < 64; i += kT) {
    uint32_t lo = 0, hi = 0;
    for (int k = 0; k < 6; ++k)
      if ((i >> k) & 1) {
        if (k < T) lo |= 1u << cx.tq[k];
        if (k + 6 < T) hi |= 1u << cx.tq[k + 6];
      }
    cx.off_lo[i] = lo;
    cx.off_hi[i] = hi;
  }
  __syncthreads();
  // entangler parity of the in-tile part of every position
  for (int v0 = warp * 32; v0 < kTilePos; v0 += kT) {
    const int v = v0 + lane;
    const uint32_t i = cx.off_lo[v & 63] | cx.off_hi[(v >> 6) & 63];
    uint32_t par = 0;
    for (uint32_t r = i; r; r &= r - 1u) par ^= (uint32_t)__popc(i & a.nbhi[__ffs(r) - 1]);
    const uint32_t bits = __ballot_sync(0xffffffffu, v < P2 && (par & 1u));
    if (lane == 0) cx.s_off[v0 >> 5] = bits;
  }
  __syncthreads();

  const bool enc = (!BWD && P.gen) || a.reupload;
  for (long long t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
    const int b = (int)(t >> no);
    const uint32_t o = (uint32_t)(t & ((1ll << no) - 1));
    uint32_t base = 0;
    for (int k = 0; k < no; ++k)
      if ((o >> k) & 1u) base |= 1u << cx.oq[k];
    const size_t gbase = ((size_t)b << n) + base;
    if (enc) {
      for (int q = tid; q < n; q += kT) sincos(0.5 * a.x[(size_t)b * n + q], &cx.sn[q], &cx.cs[q]);
      __syncthreads();
    }
    // entangler parity of the out-of-tile part and of its bonds into the tile
    uint32_t s_base = 0, cm = 0;
    for (uint32_t r = base; r; r &= r - 1u) s_base ^= (uint32_t)__popc(base & a.nbhi[__ffs(r) - 1]);
    for (int k = 0; k < T; ++k) cm |= ((uint32_t)__popc(base & a.nb[cx.tq[k]]) & 1u) << k;
    s_base &= 1u;

    for (int v = tid; v < P2; v += kT) {
      const uint32_t idx = cx.off_lo[v & 63] | cx.off_hi[(v >> 6) & 63];
      const size_t g = gbase + idx;
      double2 pv;
      if (!BWD && P.gen) {
        const uint32_t i = base | idx;
        double r = 1.0;
        for (int q = 0; q < n; ++q) r *= ((i >> q) & 1u) ? cx.sn[q] : cx.cs[q];
        pv = make_double2(r, 0.0);
      } else if (BWD && P.ckpt >= 0) {
        pv = slot_load(a, P.ckpt, g);  // the checkpoint replaces the uncomputed state
        if (a.rscale) {  // split form: in the backward state's scale
          const double r = *a.rscale;
          pv = make_double2(pv.x * r, pv.y * r);
        }
      } else {
        pv = a.psi[g];
      }
      tp[padp(v)] = pv;
      if (BWD) tl[padp(v)] = a.lam[g];
    }
    // the block's next tile into L2 while this one is computed (its loads then
    // hit L2): each thread its own positions of both planes
    const long long tn = t + gridDim.x;
    if (tn < a.n_tiles && (BWD || !P.gen)) {
      const int bn = (int)(tn >> no);
      const uint32_t on = (uint32_t)(tn & ((1ll << no) - 1));
      uint32_t bsn = 0;
      for (int k = 0; k < no; ++k)
        if ((on >> k) & 1u) bsn |= 1u << cx.oq[k];
      const size_t gn = ((size_t)bn << n) + bsn;
      for (int v = tid; v < P2; v += kT) {
        const size_t g = gn + (cx.off_lo[v & 63] | cx.off_hi[(v >> 6) & 63]);
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a.psi + g));
        if (BWD) asm volatile("prefetch.global.L2 [%0];" ::"l"(a.lam + g));
      }
    }
    __syncthreads();

    for (int k = 0; k < P.nops; ++k) {
      const DevOp op = P.ops[BWD ? P.nops - 1 - k : k];
      if (op.kind == OP_ROT || op.kind == OP_RY) {
        const int m = __popc((unsigned)op.b);
        for (int c0 = 0; c0 < m; c0 += 3) {
          const int kk = min(3, m - c0);
          if (split) {
            if (kk == 3) rot_chunk<BWD, 3, true>(a, P, cx, tp, tl, acc, op.d + c0, warp, lane);
            else if (kk == 2) rot_chunk<BWD, 2, true>(a, P, cx, tp, tl, acc, op.d + c0, warp, lane);
            else rot_chunk<BWD, 1, true>(a, P, cx, tp, tl, acc, op.d + c0, warp, lane);
          } else {
            if (kk == 3) rot_chunk<BWD, 3, false>(a, P, cx, tp, tl, acc, op.d + c0, warp, lane);
            else if (kk == 2) rot_chunk<BWD, 2, false>(a, P, cx, tp, tl, acc, op.d + c0, warp, lane);
            else rot_chunk<BWD, 1, false>(a, P, cx, tp, tl, acc, op.d + c0, warp, lane);
          }
          __syncthreads();
        }
      } else if (SPLIT && op.kind == OP_DIAG) {
        // split form: position v (global index base | idx(v)) times
        // dlo[v & 63] dhi[v >> 6] f_out scale, and the entangler sign (l >= 0)
        const int l = op.c;
        if (BWD && l < 0) continue;  // nothing reads the state before layer 0's rotations
        const double2* dq = a.dq + (size_t)(l + 1) * n * 2;
        if (tid < 128) {
          const int i = tid & 63, hi = tid >> 6;
          double2 f = make_double2(1.0, 0.0);
          for (int k = 0; k < 6; ++k) {
            const int pb = k + 6 * hi;
            if (pb >= T) break;
            const double2 d = dq[2 * cx.tq[pb] + ((i >> k) & 1)];
            f = make_double2(f.x * d.x - f.y * d.y, f.x * d.y + f.y * d.x);
          }
          if (hi) cx.dhi[i] = f;
          else cx.dlo[i] = f;
        }
        double sc = 1.0;
        if (l >= 0) sc = BWD ? a.slay[l].gam / (l + 1 < a.L ? a.slay[l + 1].rho : 1.0) : 1.0 / a.slay[l].gam;
        double2 fo = make_double2(sc, 0.0);
        for (int k = 0; k < no; ++k) {
          const int q = cx.oq[k];
          const double2 d = dq[2 * q + ((base >> q) & 1u)];
          fo = make_double2(fo.x * d.x - fo.y * d.y, fo.x * d.y + fo.y * d.x);
        }
        __syncthreads();
        for (int v = tid; v < P2; v += kT) {
          const double2 fl = cx.dlo[v & 63], fh = cx.dhi[(v >> 6) & 63];
          const double2 f1 = make_double2(fl.x * fh.x - fl.y * fh.y, fl.x * fh.y + fl.y * fh.x);
          double2 f = make_double2(f1.x * fo.x - f1.y * fo.y, f1.x * fo.y + f1.y * fo.x);
          if (l >= 0) {
            const uint32_t par = s_base ^ ((cx.s_off[v >> 5] >> (v & 31)) & 1u) ^ ((uint32_t)__popc(v & cm) & 1u);
            if (par) f = make_double2(-f.x, -f.y);
          }
          const int pp = padp(v);
          const double2 x = tp[pp];
          tp[pp] = make_double2(f.x * x.x - f.y * x.y, f.x * x.y + f.y * x.x);
          if (BWD) {
            const double2 y = tl[pp];
            tl[pp] = make_double2(f.x * y.x - f.y * y.y, f.x * y.y + f.y * y.x);
          }
        }
        __syncthreads();
      } else if (!SPLIT && op.kind == OP_PERM) {
        // fused CNOT layers (fused-SU(2) passes only): the tile's positions
        // gathered through the factor's map G (forward M_g^-1, backward
        // M_g): position v takes the position of G (idx(v) | base).  G
        // changes only bits of this pass's qubit set, all in the tile, and
        // the tile position of a qubit pattern is linear in it, so the
        // source position is the xor of per-qubit columns (pcol: the tile
        // position of G's image of each qubit's bit), those of v's bits and
        // of the tile's out-of-tile bits.  psi, then lambda.
        constexpr int kPer = (1 << 11) / kT;  // positions per thread (tiles of up to 2^11)
        if (P2 > kPer * kT) {  // (fused CNOT plans have two qubit sets: 11-qubit tiles at most)
          if (tid == 0) atomicOr(a.status, kErrBounds);
          continue;
        }
        if (tid < n) {
          // (constant indices into the parameter block: no pointer into it)
          uint32_t img = 0;
#pragma unroll
          for (int q = 0; q < kMaxQubits; ++q)
            if (q == tid)
              img = op.c == 0 ? (BWD ? a.perm_bwd[0][q] : a.perm_fwd[0][q]) : (BWD ? a.perm_bwd[1][q] : a.perm_fwd[1][q]);
          uint32_t u = 0;
          for (int k = 0; k < T; ++k) u |= ((img >> cx.tq[k]) & 1u) << k;
          cx.pcol[tid] = u;
        }
        __syncthreads();
        uint32_t ub = 0;  // the out-of-tile bits' part, then this thread's fixed position bits
        for (uint32_t r = base; r; r &= r - 1u) ub ^= cx.pcol[__ffs(r) - 1];
        for (int k = 0; k < T && (1 << k) < kT; ++k)
          if ((tid >> k) & 1) ub ^= cx.pcol[cx.tq[k]];
        for (int plane = 0; plane < (BWD ? 2 : 1); ++plane) {
          double2* tb = plane ? tl : tp;
          double2 tv[kPer];
#pragma unroll
          for (int i = 0; i < kPer; ++i) {
            const int v = tid + i * kT;
            if (v >= P2) break;
            uint32_t u = ub;
#pragma unroll
            for (int k = 0; k < 3; ++k)  // position bits 8-10 come from i (kT = 256)
              if ((i >> k) & 1) u ^= cx.pcol[cx.tq[8 + k]];
            tv[i] = tb[padp((int)u)];
          }
          __syncthreads();
#pragma unroll
          for (int i = 0; i < kPer; ++i) {
            const int v = tid + i * kT;
            if (v >= P2) break;
            tb[padp(v)] = tv[i];
          }
          __syncthreads();
        }
      } else if (!SPLIT && op.kind == OP_CZ) {
        for (int v = tid; v < P2; v += kT) {
          const uint32_t par = s_base ^ ((cx.s_off[v >> 5] >> (v & 31)) & 1u) ^ ((uint32_t)__popc(v & cm) & 1u);
          if (par) {
            const int p = padp(v);
            tp[p] = make_double2(-tp[p].x, -tp[p].y);
            if (BWD) tl[p] = make_double2(-tl[p].x, -tl[p].y);
          }
        }
        __syncthreads();
      }
    }

    if (!BWD || !P.gen) {
      for (int v = tid; v < P2; v += kT) {
        const size_t g = gbase + (cx.off_lo[v & 63] | cx.off_hi[(v >> 6) & 63]);
        const double2 pv = tp[padp(v)];
        if (!BWD && P.ckpt >= 0) slot_store(a, P.ckpt, g, pv);
        a.psi[g] = pv;
        if (BWD) a.lam[g] = tl[padp(v)];
      }
    }
    __syncthreads();  // the tile buffers are reused by the next tile
  }
  if (BWD) {
    const int nacc = P.nslots * 3;
    for (int i = tid; i < nacc; i += kT) {
      double s = 0.0;
      for (int w = 0; w < kW; ++w) s += acc[((size_t)w * kMaxSlots) * 3 + i];  // fixed warp order
      a.partials[P.partial_off + (long long)blockIdx.x * nacc + i] = s;
    }
  }
}

// lambda = g[b] Z0 psi (separate buffer; psi unchanged).
__global__ void bwd_init64_kernel(const double2* psi, double2* lam, const double* g, int n, long long tot) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= tot) return;
  const double gs = (idx & 1) ? -g[idx >> n] : g[idx >> n];
  const double2 v = psi[idx];
  lam[idx] = make_double2(gs * v.x, gs * v.y);
}

constexpr int kExp64Threads = 256;
constexpr int kExp64ChunkLog = 16;

__global__ void expect64_partial_kernel(const double2* psi, int n, double* partial) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExp64ChunkLog) - 1) >> kExp64ChunkLog);
  const int b = blockIdx.y, c = blockIdx.x;
  const long long lo = (long long)c << kExp64ChunkLog;
  const long long hi = min(N, lo + (1ll << kExp64ChunkLog));
  const double2* p = psi + (size_t)b * N;
  double s = 0.0;
  for (long long i = lo + threadIdx.x; i < hi; i += kExp64Threads) {
    const double2 v = p[i];
    const double m = v.x * v.x + v.y * v.y;
    s += (i & 1) ? -m : m;
  }
  __shared__ double red[kExp64Threads];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = kExp64Threads / 2; w; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[(size_t)b * chunks + c] = red[0];
}

__global__ void expect64_final_kernel(const double* partial, int chunks, int B, double* E, unsigned* status) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  double s = 0.0;
  for (int c = 0; c < chunks; ++c) s += partial[(size_t)b * chunks + c];
  E[b] = s;
  if (!isfinite(s) && status) atomicOr(status, kErrNumeric);
}

// Observable O = sum_k c_k i^ny X^x Z^z with terms grouped by x (the same
// grouping as the fp32 path): the group's weight at m = j ^ x is
// sum_k c_k i^ny (-1)^popcount(m & z_k).
__device__ __forceinline__ double2 obs_weight64(const ObsTerm* t, int count, uint32_t m) {
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

// Partial sums of <psi|O|psi> = sum_j sum_groups conj(psi(j)) w(j ^ x) psi(j ^ x)
// over chunks of 2^16 amplitudes (fp64).
__global__ void obs64_expect_partial_kernel(const double2* psi, int n, const ObsGroup* groups, int ngroups,
                                            const ObsTerm* terms, double* partial) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExp64ChunkLog) - 1) >> kExp64ChunkLog);
  const int b = blockIdx.y, c = blockIdx.x;
  const long long lo = (long long)c << kExp64ChunkLog;
  const long long hi = min(N, lo + (1ll << kExp64ChunkLog));
  const double2* p = psi + (size_t)b * N;
  double s = 0.0;
  for (int gi = 0; gi < ngroups; ++gi) {
    const ObsGroup G = groups[gi];
    for (long long j = lo + threadIdx.x; j < hi; j += kExp64Threads) {
      const uint32_t m = (uint32_t)j ^ G.x;
      const double2 a = p[j], q = p[m];
      const double wr = a.x * q.x + a.y * q.y;  // conj(a) q
      const double wi = a.x * q.y - a.y * q.x;
      const double2 d = obs_weight64(terms + G.first, G.count, m);
      s += wr * d.x - wi * d.y;
    }
  }
  __shared__ double red[kExp64Threads];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = kExp64Threads / 2; w; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[(size_t)b * chunks + c] = red[0];
}

// lambda = g_b O psi (separate buffer; psi unchanged).
__global__ void obs64_lambda_kernel(const double2* psi, double2* lam, const double* g, int n, long long tot,
                                    const ObsGroup* groups, int ngroups, const ObsTerm* terms) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= tot) return;
  const long long N = 1ll << n;
  const int b = (int)(idx >> n);
  const uint32_t j = (uint32_t)(idx & (N - 1));
  const double2* p = psi + (size_t)b * N;
  double ar = 0.0, ai = 0.0;
  for (int gi = 0; gi < ngroups; ++gi) {
    const ObsGroup G = groups[gi];
    const uint32_t m = j ^ G.x;
    const double2 q = p[m];
    const double2 d = obs_weight64(terms + G.first, G.count, m);
    ar += d.x * q.x - d.y * q.y;
    ai += d.x * q.y + d.y * q.x;
  }
  lam[idx] = make_double2(g[b] * ar, g[b] * ai);
}

// gfix (split form, else null): as in the fp32 reduction, the sums scaled to
// the split circuit's states and rotated by phi1 first.
__global__ void grad_reduce64_kernel(const DevPass* passes, const int* slot_pass, const int* slot_index,
                                     const double* partials, int grid, const double* theta, const double* gfix,
                                     int L, int n, double* grad, unsigned* status) {
  // one warp per (layer, qubit): strided lane sums, then a fixed butterfly
  const int idx = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (idx >= L * n) return;  // whole warps leave together
  const int p = slot_pass[idx], s = slot_index[idx];
  const DevPass& ps = passes[p];
  const int stride = ps.nslots * 3;
  const double* base = partials + ps.partial_off + s * 3;
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
  // (s_x, s_y, s_z) are Im<lambda|P|psi> at the rotation's output; the angle
  // gradients take X and Y back through the Rz and Ry that follow them
  double sb, cb, sg, cg;
  sincos(theta[idx * 3 + 1], &sb, &cb);
  sincos(theta[idx * 3 + 2], &sg, &cg);
  const double gz = sz;
  const double gy = cg * sy - sg * sx;
  const double gx = cb * (cg * sx + sg * sy) - sb * sz;
  grad[idx * 3 + 0] = gx;
  grad[idx * 3 + 1] = gy;
  grad[idx * 3 + 2] = gz;
  if (!(isfinite(gx) && isfinite(gy) && isfinite(gz)) && status) atomicOr(status, kErrNumeric);
}

// g[b] = 2 (E[b] - y[b]) / B, loss = mean (E - y)^2 (fixed-order sum).
__global__ void loss_seed64_kernel(const double* E, const double* y, int B, double* g, double* loss) {
  __shared__ double red[256];
  double s = 0.0;
  for (int b = threadIdx.x; b < B; b += 256) {
    const double d = E[b] - y[b];
    if (g) g[b] = 2.0 * d / B;
    s += d * d;
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0 && loss) loss[0] = red[0] / B;
}

}  // namespace

size_t pass64_smem_bytes(bool backward, int tmax) { return f64_smem_bytes(backward, tmax); }

cudaError_t pass64_setup(int tmax, int* blocks_fwd, int* blocks_bwd) {
  cudaError_t e = cudaSuccess;
  for (int sp = 0; sp < 2 && e == cudaSuccess; ++sp) {
    e = cudaFuncSetAttribute(sp ? pass64_kernel<false, true> : pass64_kernel<false, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)f64_smem_bytes(false, kTileBits));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(sp ? pass64_kernel<true, true> : pass64_kernel<true, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)f64_smem_bytes(true, kTileBits));
  }
  // the grid is the same for both forms: take the smaller occupancy
  int f0 = 0, f1 = 0, b0 = 0, b1 = 0;
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&f0, pass64_kernel<false, false>, kT, f64_smem_bytes(false, tmax));
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&f1, pass64_kernel<false, true>, kT, f64_smem_bytes(false, tmax));
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b0, pass64_kernel<true, false>, kT, f64_smem_bytes(true, tmax));
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b1, pass64_kernel<true, true>, kT, f64_smem_bytes(true, tmax));
  *blocks_fwd = std::min(f0, f1);
  *blocks_bwd = std::min(b0, b1);
  return e;
}

cudaError_t launch_pass64(bool backward, const Pass64Args& a, const DevPass& p, int grid, cudaStream_t s) {
  if (a.tmax < a.T || a.tmax > kTileBits) return cudaErrorInvalidValue;
  const bool split = a.srot != nullptr;
  const size_t smem = f64_smem_bytes(backward, a.tmax);
  if (backward) {
    if (split) pass64_kernel<true, true><<<grid, kT, smem, s>>>(a, p);
    else pass64_kernel<true, false><<<grid, kT, smem, s>>>(a, p);
  } else {
    if (split) pass64_kernel<false, true><<<grid, kT, smem, s>>>(a, p);
    else pass64_kernel<false, false><<<grid, kT, smem, s>>>(a, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_init64(const double2* psi, double2* lam, const double* g, int B, int n, cudaStream_t s) {
  const long long tot = (long long)B << n;
  bwd_init64_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(psi, lam, g, n, tot);
  return cudaGetLastError();
}

size_t expect64_partial_count(int B, int n) {
  const long long N = 1ll << n;
  return (size_t)B * (size_t)((N + (1ll << kExp64ChunkLog) - 1) >> kExp64ChunkLog);
}

cudaError_t launch_expect64(const double2* psi, int B, int n, double* partial, double* E, unsigned* status,
                            cudaStream_t s) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExp64ChunkLog) - 1) >> kExp64ChunkLog);
  expect64_partial_kernel<<<dim3(chunks, B), kExp64Threads, 0, s>>>(psi, n, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expect64_final_kernel<<<(B + 127) / 128, 128, 0, s>>>(partial, chunks, B, E, status);
  return cudaGetLastError();
}

cudaError_t launch_obs_expect64(const double2* psi, int B, int n, const ObsGroup* groups, int ngroups,
                                const ObsTerm* terms, double* partial, double* E, unsigned* status, cudaStream_t s) {
  const long long N = 1ll << n;
  const int chunks = (int)((N + (1ll << kExp64ChunkLog) - 1) >> kExp64ChunkLog);
  obs64_expect_partial_kernel<<<dim3(chunks, B), kExp64Threads, 0, s>>>(psi, n, groups, ngroups, terms, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  expect64_final_kernel<<<(B + 127) / 128, 128, 0, s>>>(partial, chunks, B, E, status);
  return cudaGetLastError();
}

cudaError_t launch_obs_bwd_init64(const double2* psi, double2* lam, const double* g, int B, int n,
                                  const ObsGroup* groups, int ngroups, const ObsTerm* terms, cudaStream_t s) {
  const long long tot = (long long)B << n;
  obs64_lambda_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(psi, lam, g, n, tot, groups, ngroups, terms);
  return cudaGetLastError();
}

cudaError_t launch_grad_reduce64(const DevPass* passes, const int* slot_pass, const int* slot_index,
                                 const double* partials, int grid, const double* theta, const double* gfix, int L,
                                 int n, double* grad, unsigned* status, cudaStream_t s) {
  const long long threads = (long long)L * n * 32;  // one warp per (layer, qubit)
  grad_reduce64_kernel<<<(unsigned)((threads + 127) / 128), 128, 0, s>>>(passes, slot_pass, slot_index, partials,
                                                                         grid, theta, gfix, L, n, grad, status);
  return cudaGetLastError();
}

cudaError_t launch_loss_seed64(const double* E, const double* y, int B, double* g, double* loss, cudaStream_t s) {
  loss_seed64_kernel<<<1, 256, 0, s>>>(E, y, B, g, loss);
  return cudaGetLastError();
}

}  // namespace qml
