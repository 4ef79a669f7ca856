// coef.cu -- gate coefficients of the passes, computed on the device from
// theta in fp64: the fused SU(2) of every rotation slot (and its inverse),
// and the tables of the split form (see kernels.cuh, SplitRot).
//
// The rotation of a (layer, qubit) is U = Rz(g) Ry(b) Rx(a) (the ansatz of
// the Deep-dive blog sec. 2.1); the split form rewrites it exactly as
// Rz(phi1) Ry(vt) Rz(phi2).
#include "kernels.cuh"

namespace qml {

namespace {

constexpr int kPos = 1 << kRegBits;

// U = Rz(g) Ry(b) Rx(a) = [[A, B], [-conj B, conj A]] in fp64 (half angles).
template <class T>
__device__ __forceinline__ void su2_of(const T* th, double* ar, double* ai, double* br, double* bi) {
  const double al = th[0], be = th[1], ga = th[2];
  double sa, ca, sb, cb, sg, cg;
  sincos(0.5 * al, &sa, &ca);
  sincos(0.5 * be, &sb, &cb);
  sincos(0.5 * ga, &sg, &cg);
  // (Ry Rx)[0][0] = cb ca + i sb sa, (Ry Rx)[0][1] = -sb ca - i cb sa; row 0 of Rz is e^{-i g/2}
  const double p_re = cb * ca, p_im = sb * sa;
  const double q_re = -sb * ca, q_im = -cb * sa;
  *ar = cg * p_re + sg * p_im;
  *ai = cg * p_im - sg * p_re;
  *br = cg * q_re + sg * q_im;
  *bi = cg * q_im - sg * q_re;
}

// Gate coefficients of every pass slot: U computed in fp64 and rounded to
// fp32 broadcast pairs, and U^dagger = [[conj A, -B], ...] for the backward
// passes.  Output: one CoefRegion per pass and direction.
__global__ void prep_pass_coef_kernel(const DevPass* passes, int n_passes, const float* theta, CoefRegion* cf,
                                      CoefRegion* ci) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_passes * kMaxSlots) return;
  const int p = idx / kMaxSlots, s = idx % kMaxSlots;
  if (s >= passes[p].nslots) return;
  const int lq = passes[p].slot_lq[s];
  double ar, ai, br, bi;
  su2_of(theta + lq * 3, &ar, &ai, &br, &bi);
  const float far = (float)ar, fai = (float)ai, fbr = (float)br, fbi = (float)bi;
  float4* f = cf[p].rot[s];
  f[0] = make_float4(far, far, fai, fai);
  f[1] = make_float4(-fai, -fai, fbr, fbr);
  f[2] = make_float4(fbi, fbi, -fbi, -fbi);
  f[3] = make_float4(-fbr, -fbr, 0.f, 0.f);
  // U^dagger: A' = conj A, B' = -B
  float4* g = ci[p].rot[s];
  g[0] = make_float4(far, far, -fai, -fai);
  g[1] = make_float4(fai, fai, -fbr, -fbr);
  g[2] = make_float4(-fbi, -fbi, fbi, fbi);
  g[3] = make_float4(fbr, fbr, 0.f, 0.f);
}

// ----------------------------------------------------- split-form tables
//
// U = Rz(g) Ry(b) Rx(a) = Rz(phi1) Ry(vt) Rz(phi2) with A = e^{-i sig} c,
// B = -e^{-i del} s, c = |A|, s = |B|, sig = (phi1 + phi2) / 2,
// del = (phi1 - phi2) / 2.  Every state the split passes hold is the split
// circuit's state times a "frame": a real scale and a sign (-1 on the 0 half)
// for each qubit rotated in cotangent form since the last diagonal op.  Each
// diagonal op removes the frame of its layer's rotations (forward) or restores
// it (backward), so that the last pass leaves the exact final state.

template <class T>
__device__ void split_rot_item(const T* theta, int idx, SplitRot* out) {
  double ar, ai, br, bi;
  su2_of(theta + (size_t)idx * 3, &ar, &ai, &br, &bi);
  const double c = sqrt(ar * ar + ai * ai), s = sqrt(br * br + bi * bi);
  const double sig = -atan2(ai, ar), del = -atan2(-bi, -br);
  SplitRot r;
  r.phi1 = sig + del;
  r.phi2 = sig - del;
  r.cot = s > c ? 1 : 0;
  r.tau = r.cot ? c / s : s / c;
  r.g = r.cot ? -1.0 / s : 1.0 / c;
  r.k2 = r.g * r.g;
  r.pad = 0;
  out[idx] = r;
}

template <class T>
__global__ void split_rot_kernel(const T* theta, int total, SplitRot* out) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < total) split_rot_item(theta, idx, out);
}

// Per layer: the frame of all its rotations, and per rotation the scale of
// the backward sums.  At the sum of rotation j the backward state is
// rho * gam * Z^m times the split circuit's (psi, lambda), where rho is the
// product of k2 over the layer's rotations already un-applied and gam the
// product of g over those still applied; the sums scale by (rho gam)^2, and
// their X and Y parts flip sign when j itself is in cotangent form.
__device__ void split_layer_item(const SplitRot* rot, const int* undo, int l, int n, SplitLayer* lay,
                                 double* gfix) {
  const SplitRot* r = rot + (size_t)l * n;
  double gam = 1.0, rho = 1.0;
  uint32_t m = 0;
  for (int q = 0; q < n; ++q) {
    gam *= r[q].g;
    rho *= r[q].k2;
    if (r[q].cot) m |= 1u << q;
  }
  lay[l].gam = gam;
  lay[l].rho = rho;
  lay[l].cot_mask = m;
  lay[l].pad = 0;
  double undone_k2 = 1.0, applied_g = gam;
  for (int i = 0; i < n; ++i) {
    const int q = undo[(size_t)l * n + i];
    const double f = undone_k2 * applied_g;
    const double sc = (r[q].cot ? -1.0 : 1.0) / (f * f);
    gfix[((size_t)l * n + q) * 2 + 0] = sc;
    gfix[((size_t)l * n + q) * 2 + 1] = r[q].phi1;
    undone_k2 *= r[q].k2;
    applied_g /= r[q].g;
  }
}

__global__ void split_layer_kernel(const SplitRot* rot, const int* undo, int L, int n, SplitLayer* lay,
                                   double* gfix) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l < L) split_layer_item(rot, undo, l, n, lay, gfix);
}

// Factor of qubit q's bit b in the diagonal op after layer l (l = -1: before
// layer 0): Rz(phi1 of layer l + phi2 of layer l + 1), times -1 on b = 1 when
// q was rotated in cotangent form in layer l; conjugated for the backward.
__device__ __forceinline__ double2 diag_factor(const SplitRot* rot, const SplitLayer* lay, int L, int n, int l, int q,
                                               int b, bool bwd) {
  const double w = (l >= 0 ? rot[(size_t)l * n + q].phi1 : 0.0) + (l + 1 < L ? rot[(size_t)(l + 1) * n + q].phi2 : 0.0);
  double sn, cs;
  sincos(0.5 * w, &sn, &cs);
  double re = cs, im = b ? sn : -sn;
  if (bwd) im = -im;
  if (l >= 0 && b && ((lay[l].cot_mask >> q) & 1u)) re = -re, im = -im;
  return make_double2(re, im);
}

__device__ void split_diag_item(const SplitRot* rot, const SplitLayer* lay, int L, int n, int idx, float2* dq_f,
                                float2* dq_b) {
  // idx = ((l + 1) * n + q) * 2 + b
  const int b = idx & 1, q = (idx >> 1) % n, l = (idx >> 1) / n - 1;
  const double2 f = diag_factor(rot, lay, L, n, l, q, b, false);
  const double2 g = diag_factor(rot, lay, L, n, l, q, b, true);
  dq_f[idx] = make_float2((float)f.x, (float)f.y);
  dq_b[idx] = make_float2((float)g.x, (float)g.y);
}

__global__ void split_diag_kernel(const SplitRot* rot, const SplitLayer* lay, int L, int n, float2* dq_f,
                                  float2* dq_b) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < (L + 1) * n * 2) split_diag_item(rot, lay, L, n, idx, dq_f, dq_b);
}

// fp64 mode: the same factors in fp64.
__global__ void split_diag64_kernel(const SplitRot* rot, const SplitLayer* lay, int L, int n, double2* dq_f,
                                    double2* dq_b) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // ((l + 1) * n + q) * 2 + b
  if (idx >= (L + 1) * n * 2) return;
  const int b = idx & 1, q = (idx >> 1) % n, l = (idx >> 1) / n - 1;
  dq_f[idx] = diag_factor(rot, lay, L, n, l, q, b, false);
  dq_b[idx] = diag_factor(rot, lay, L, n, l, q, b, true);
}

// fp64 mode: the restore scale of every backward checkpoint pass (see the
// last item of split_pass_kernel).
__global__ void split_rscale64_kernel(const DevPass* passes, int n_passes, const SplitRot* rot, int n,
                                      double* rscale) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n_passes) return;
  const DevPass& P = passes[p];
  double rho = 1.0;
  if (P.ckpt >= 0 && P.rs_layer >= 0)
    for (int q = 0; q < n; ++q)
      if ((P.rs_mask >> q) & 1u) rho *= rot[(size_t)P.rs_layer * n + q].k2;
  rscale[p] = rho;
}

// Per pass: rotation slots, the register tables of its diagonal ops, and the
// restore scale.  Items per pass: kMaxSlots slots, kMaxDiag * kPos table
// entries, one scale.
constexpr int kSplitItems = kMaxSlots + kMaxDiag * kPos + 1;

__device__ void split_pass_item(const DevPass* passes, int idx, const SplitRot* rot, const SplitLayer* lay, int L,
                                int n, CoefRegion* cf, CoefRegion* ci, float* rscale) {
  const int p = idx / kSplitItems, it = idx % kSplitItems;
  const DevPass& P = passes[p];
  if (it < kMaxSlots) {
    if (it >= P.nslots) return;
    const SplitRot r = rot[P.slot_lq[it]];
    const float t = (float)r.tau;
    // forward: p = tau in both forms; backward: -tau in tangent form
    cf[p].rot[it][0] = make_float4(t, t, -t, -t);
    cf[p].rot[it][1] = make_float4((float)r.cot, 0.f, 0.f, 0.f);
    const float tb = r.cot ? t : -t;
    ci[p].rot[it][0] = make_float4(tb, tb, -tb, -tb);
    ci[p].rot[it][1] = make_float4((float)r.cot, 0.f, 0.f, 0.f);
    return;
  }
  if (it == kSplitItems - 1) {
    // backward checkpoint pass: the restored state takes the scale rho that
    // the un-applied rotations between the pass's end and the next diagonal
    // op have given the backward state
    double rho = 1.0;
    if (P.ckpt >= 0 && P.rs_layer >= 0)
      for (int q = 0; q < n; ++q)
        if ((P.rs_mask >> q) & 1u) rho *= rot[(size_t)P.rs_layer * n + q].k2;
    rscale[p] = (float)rho;
    return;
  }
  const int e = it - kMaxSlots, d = e / kPos, j = e % kPos;
  int ph = -1, l = 0;
  for (int o = 0; o < P.nops; ++o)
    if (P.ops[o].kind == OP_DIAG && P.ops[o].d == d) ph = P.ops[o].a, l = P.ops[o].c;
  if (ph < 0) return;
  // the global scale: forward 1 / gam(l); backward gam(l) / rho(l + 1)
  double fr = l >= 0 ? 1.0 / lay[l].gam : 1.0, fi = 0.0;
  double br = l >= 0 ? lay[l].gam / (l + 1 < L ? lay[l + 1].rho : 1.0) : 0.0, bi = 0.0;
  for (int k = 0; k < kRegBits; ++k) {
    const int tb = ph == 0 ? k : ph == 1 ? 5 + k : (k < 2 ? 10 + k : k - 2);  // reg_tbit
    const int q = P.tile_q[tb];
    if (q < 0) continue;  // a batch-unit bit
    const int b = (j >> k) & 1;
    const double2 f = diag_factor(rot, lay, L, n, l, q, b, false);
    const double2 g = diag_factor(rot, lay, L, n, l, q, b, true);
    double t = fr * f.x - fi * f.y;
    fi = fr * f.y + fi * f.x;
    fr = t;
    t = br * g.x - bi * g.y;
    bi = br * g.y + bi * g.x;
    br = t;
  }
  cf[p].diag[d][j] = make_float2((float)fr, (float)fi);
  ci[p].diag[d][j] = make_float2((float)br, (float)bi);
}

__global__ void split_pass_kernel(const DevPass* passes, int n_passes, const SplitRot* rot, const SplitLayer* lay,
                                  int L, int n, CoefRegion* cf, CoefRegion* ci, float* rscale) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < n_passes * kSplitItems) split_pass_item(passes, idx, rot, lay, L, n, cf, ci, rscale);
}

// Small circuits: the four stages above in one block, a barrier between
// stages that read what an earlier one wrote, one launch instead of four.
constexpr int kPrepSmallThreads = 1024;
constexpr int kPrepSmallItems = 4096;  // largest stage run by the one block

__global__ void __launch_bounds__(kPrepSmallThreads) split_prep_small_kernel(
    const DevPass* passes, int n_passes, const float* theta, int L, int n, const int* undo, SplitRot* rot,
    SplitLayer* lay, double* gfix, float2* dq_f, float2* dq_b, CoefRegion* cf, CoefRegion* ci, float* rscale) {
  const int t = threadIdx.x, T = blockDim.x;
  for (int i = t; i < L * n; i += T) split_rot_item(theta, i, rot);
  __syncthreads();
  for (int l = t; l < L; l += T) split_layer_item(rot, undo, l, n, lay, gfix);
  __syncthreads();
  for (int i = t; i < (L + 1) * n * 2; i += T) split_diag_item(rot, lay, L, n, i, dq_f, dq_b);
  for (int i = t; i < n_passes * kSplitItems; i += T) split_pass_item(passes, i, rot, lay, L, n, cf, ci, rscale);
}

// ---- split form of the fused CNOT schedule.  A segment (l, s) is the
// rotations of layer l on qubit set s (one pass); it sits between the
// diagonal D2 (its Rz(phi2) factors) and D1 (its Rz(phi1) factors and the
// segment's frame), global diagonal indices 4 l + 2 s + 0 / 1.  The state is
// exact at every pass boundary in both directions: forward D1 = D1_true Z^m
// / gam(l, s); backward D1 = gam Z^m D1_true^dagger (the forward frame after
// the segment's rotations), backward D2 = D2_true^dagger / rho(l, s) (the
// un-applied tangent forms left rho on the state).

// Per segment: its frame, and per rotation the scale of the backward sums
// (as split_layer_kernel, over the segment's qubits in the un-apply order).
__global__ void csplit_seg_kernel(const SplitRot* rot, const int* undo, int L, int n, uint32_t set0,
                                  SplitLayer* seg, double* gfix) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // 2 l + s
  if (idx >= 2 * L) return;
  const int l = idx >> 1, sid = idx & 1;
  const uint32_t mask = sid == 0 ? set0 : (((n >= 32) ? ~0u : ((1u << n) - 1u)) & ~set0);
  const SplitRot* r = rot + (size_t)l * n;
  double gam = 1.0, rho = 1.0;
  uint32_t m = 0;
  for (int q = 0; q < n; ++q)
    if ((mask >> q) & 1u) {
      gam *= r[q].g;
      rho *= r[q].k2;
      if (r[q].cot) m |= 1u << q;
    }
  seg[idx].gam = gam;
  seg[idx].rho = rho;
  seg[idx].cot_mask = m;
  seg[idx].pad = 0;
  double undone_k2 = 1.0, applied_g = gam;
  for (int i = 0; i < n; ++i) {
    const int q = undo[(size_t)l * n + i];
    if (!((mask >> q) & 1u)) continue;
    const double f = undone_k2 * applied_g;
    gfix[((size_t)l * n + q) * 2 + 0] = (r[q].cot ? -1.0 : 1.0) / (f * f);
    gfix[((size_t)l * n + q) * 2 + 1] = r[q].phi1;
    undone_k2 *= r[q].k2;
    applied_g /= r[q].g;
  }
}

// Factor of qubit q's bit b in diagonal d (forward; the backward's is its
// conjugate): Rz(phi2) of (l, q) for side 0, Rz(phi1) of (l, q) times -1 on
// b = 1 for a cotangent-form rotation for side 1; 1 for qubits outside the
// segment's set.
__device__ __forceinline__ double2 csplit_factor(const SplitRot* rot, const SplitLayer* seg, int n, uint32_t set0,
                                                 int d, int q, int b, bool bwd) {
  const int l = d >> 2, sid = (d >> 1) & 1, side = d & 1;
  const bool in0 = (set0 >> q) & 1u;
  if (in0 != (sid == 0)) return make_double2(1.0, 0.0);
  const SplitRot& r = rot[(size_t)l * n + q];
  double sn, cs;
  sincos(0.5 * (side ? r.phi1 : r.phi2), &sn, &cs);
  double re = cs, im = b ? sn : -sn;
  if (bwd) im = -im;
  if (side && b && ((seg[2 * l + sid].cot_mask >> q) & 1u)) re = -re, im = -im;
  return make_double2(re, im);
}

__global__ void csplit_diag_kernel(const SplitRot* rot, const SplitLayer* seg, int L, int n, uint32_t set0,
                                   float2* dq_f, float2* dq_b) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;  // ((d + 1) * n + q) * 2 + b
  if (idx >= (4 * L + 1) * n * 2) return;
  const int b = idx & 1, q = (idx >> 1) % n, d = (idx >> 1) / n - 1;
  if (d < 0) {  // (no diagonal -1 in this schedule)
    dq_f[idx] = dq_b[idx] = make_float2(1.f, 0.f);
    return;
  }
  const double2 f = csplit_factor(rot, seg, n, set0, d, q, b, false);
  const double2 g = csplit_factor(rot, seg, n, set0, d, q, b, true);
  dq_f[idx] = make_float2((float)f.x, (float)f.y);
  dq_b[idx] = make_float2((float)g.x, (float)g.y);
}

// Per pass: rotation slots, the register tables of its two diagonal ops (the
// global scales folded in) and the restore scale (1: exact boundaries).
__global__ void csplit_pass_kernel(const DevPass* passes, int n_passes, const SplitRot* rot, const SplitLayer* seg,
                                   int n, uint32_t set0, CoefRegion* cf, CoefRegion* ci, float* rscale) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_passes * kSplitItems) return;
  const int p = idx / kSplitItems, it = idx % kSplitItems;
  const DevPass& P = passes[p];
  if (it < kMaxSlots) {
    if (it >= P.nslots) return;
    const SplitRot r = rot[P.slot_lq[it]];
    const float t = (float)r.tau;
    cf[p].rot[it][0] = make_float4(t, t, -t, -t);
    cf[p].rot[it][1] = make_float4((float)r.cot, 0.f, 0.f, 0.f);
    const float tb = r.cot ? t : -t;
    ci[p].rot[it][0] = make_float4(tb, tb, -tb, -tb);
    ci[p].rot[it][1] = make_float4((float)r.cot, 0.f, 0.f, 0.f);
    return;
  }
  if (it == kSplitItems - 1) {
    rscale[p] = 1.f;
    return;
  }
  const int e = it - kMaxSlots, td = e / kPos, j = e % kPos;
  int ph = -1, d = 0;
  for (int o = 0; o < P.nops; ++o)
    if (P.ops[o].kind == OP_DIAG && P.ops[o].d == td) ph = P.ops[o].a, d = P.ops[o].c;
  if (ph < 0) return;
  const SplitLayer& S = seg[2 * (d >> 2) + ((d >> 1) & 1)];
  double fr = (d & 1) ? 1.0 / S.gam : 1.0, fi = 0.0;
  double br = (d & 1) ? S.gam : 1.0 / S.rho, bi = 0.0;
  for (int k = 0; k < kRegBits; ++k) {
    const int tb = ph == 0 ? k : ph == 1 ? 5 + k : (k < 2 ? 10 + k : k - 2);  // reg_tbit
    const int q = P.tile_q[tb];
    if (q < 0) continue;
    const int b = (j >> k) & 1;
    const double2 f = csplit_factor(rot, seg, n, set0, d, q, b, false);
    const double2 g = csplit_factor(rot, seg, n, set0, d, q, b, true);
    double t = fr * f.x - fi * f.y;
    fi = fr * f.y + fi * f.x;
    fr = t;
    t = br * g.x - bi * g.y;
    bi = br * g.y + bi * g.x;
    br = t;
  }
  cf[p].diag[td][j] = make_float2((float)fr, (float)fi);
  ci[p].diag[td][j] = make_float2((float)br, (float)bi);
}

}  // namespace

cudaError_t launch_prep_pass_coef(const DevPass* passes, int n_passes, const float* theta, CoefRegion* cf,
                                  CoefRegion* ci, cudaStream_t s) {
  const int tot = n_passes * kMaxSlots;
  prep_pass_coef_kernel<<<(tot + 127) / 128, 128, 0, s>>>(passes, n_passes, theta, cf, ci);
  return cudaGetLastError();
}

cudaError_t launch_prep_split(const DevPass* passes, int n_passes, const float* theta, int L, int n,
                              const int* undo, SplitRot* rot, SplitLayer* lay, double* gfix, float2* dq_f,
                              float2* dq_b, CoefRegion* cf, CoefRegion* ci, float* rscale, cudaStream_t s) {
  const int nr = L * n;
  if (nr <= kPrepSmallItems && (L + 1) * n * 2 <= kPrepSmallItems && n_passes * kSplitItems <= kPrepSmallItems) {
    split_prep_small_kernel<<<1, kPrepSmallThreads, 0, s>>>(passes, n_passes, theta, L, n, undo, rot, lay, gfix, dq_f,
                                                            dq_b, cf, ci, rscale);
    return cudaGetLastError();
  }
  split_rot_kernel<float><<<(nr + 127) / 128, 128, 0, s>>>(theta, nr, rot);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  split_layer_kernel<<<(L + 127) / 128, 128, 0, s>>>(rot, undo, L, n, lay, gfix);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nd = (L + 1) * n * 2;
  split_diag_kernel<<<(nd + 127) / 128, 128, 0, s>>>(rot, lay, L, n, dq_f, dq_b);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int np = n_passes * kSplitItems;
  split_pass_kernel<<<(np + 127) / 128, 128, 0, s>>>(passes, n_passes, rot, lay, L, n, cf, ci, rscale);
  return cudaGetLastError();
}

int prep_split_launches(int L, int n, int n_passes) {
  const bool small = L * n <= kPrepSmallItems && (L + 1) * n * 2 <= kPrepSmallItems &&
                     n_passes * kSplitItems <= kPrepSmallItems;
  return small ? 1 : 4;
}

cudaError_t launch_prep_split64(const DevPass* passes, int n_passes, const double* theta, int L, int n,
                                const int* undo, SplitRot* rot, SplitLayer* lay, double* gfix, double2* dq_f,
                                double2* dq_b, double* rscale, cudaStream_t s) {
  const int nr = L * n;
  split_rot_kernel<double><<<(nr + 127) / 128, 128, 0, s>>>(theta, nr, rot);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  split_layer_kernel<<<(L + 127) / 128, 128, 0, s>>>(rot, undo, L, n, lay, gfix);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nd = (L + 1) * n * 2;
  split_diag64_kernel<<<(nd + 127) / 128, 128, 0, s>>>(rot, lay, L, n, dq_f, dq_b);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  split_rscale64_kernel<<<(n_passes + 127) / 128, 128, 0, s>>>(passes, n_passes, rot, n, rscale);
  return cudaGetLastError();
}

cudaError_t launch_prep_split_cnot(const DevPass* passes, int n_passes, const float* theta, int L, int n,
                                   uint32_t set0, const int* undo, SplitRot* rot, SplitLayer* seg, double* gfix,
                                   float2* dq_f, float2* dq_b, CoefRegion* cf, CoefRegion* ci, float* rscale,
                                   cudaStream_t s) {
  const int nr = L * n;
  split_rot_kernel<float><<<(nr + 127) / 128, 128, 0, s>>>(theta, nr, rot);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  csplit_seg_kernel<<<(2 * L + 127) / 128, 128, 0, s>>>(rot, undo, L, n, set0, seg, gfix);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nd = (4 * L + 1) * n * 2;
  csplit_diag_kernel<<<(nd + 127) / 128, 128, 0, s>>>(rot, seg, L, n, set0, dq_f, dq_b);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int np = n_passes * kSplitItems;
  csplit_pass_kernel<<<(np + 127) / 128, 128, 0, s>>>(passes, n_passes, rot, seg, n, set0, cf, ci, rscale);
  return cudaGetLastError();
}

}  // namespace qml
