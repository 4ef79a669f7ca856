// kernels.cuh -- launch wrappers of the sm_100a kernels (host-callable).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "device_plan.h"

namespace qml {

// Gate coefficients of one pass, as copied into a context's constant-memory
// region before the pass is launched.
//   rot[s]: rotation slot s.  Full SU(2) (OP_ROT): four float4 of broadcast
//     pairs (ar, ai, -ai, br, bi, -bi, -br, 0).  Split form (OP_RY): rot[s][0]
//     = (p, p, -p, -p) with p the tangent-form coefficient, rot[s][1].x = 1
//     for the cotangent form (see ry_apply in kernels.cu).
//   diag[d][j]: split form, diagonal op d: the complex factor (re, im) of
//     the register part j of a position.
struct CoefRegion {
  float4 rot[kMaxSlots][4];
  float2 diag[kMaxDiag][1 << kRegBits];
};

// Split form, per (layer, qubit): U = Rz(g) Ry(b) Rx(a) = Rz(phi1) Ry(vt) Rz(phi2)
// with (c, s) = (cos, sin)(vt / 2) >= 0.  The kernels apply Ry(vt) as
// tangent form [[1, -t], [t, 1]] (t = s / c, when c >= s; the state is then
// scaled by 1 / c) or cotangent form [[-u, 1], [1, u]] (u = c / s; scale
// -1 / s and a sign on the qubit's 0 half); g is that scale, k2 = g^2.
struct SplitRot {
  double tau, g, k2, phi1, phi2;
  int cot, pad;
};
// Split form, per layer l: the product of the layer's scales, of its k2, and
// the qubits rotated in cotangent form.
struct SplitLayer {
  double gam, rho;
  uint32_t cot_mask, pad;
};

// Arguments of one pass launch (forward or backward).
struct PassArgs {
  int region;            // constant-memory coefficient region of the context
  int n, B, U;           // qubits, samples, batch units (forward: ceil(B/2); backward: B)
  long long N;           // 2^n
  int n_tiles;           // tiles in this pass
  float2* buf0;          // forward: psi; backward: psi (plane 0)
  float2* buf1;          // backward: lambda (plane 1)
  float2* dummy;         // forward: partner plane of the last unit when B is odd
  const float2* enc;     // [U][n][2] (cos, sin)(x/2) of the unit's two samples (lane pairs)
  const float* g;        // backward: dL/dE [B]
  void* ckpt;            // checkpoint slots
  int storage;           // 0 fp32, 1 bf16
  int bmax;              // samples per checkpoint slot (slot stride)
  float* partials;       // backward gradient partials
  unsigned* status;
  int reupload;          // every layer starts with the encoding Ry(x_q) again
  const float2* dq;      // split form: [L + 1][n][2] per-qubit factors of the diagonal ops (this direction)
  const float* rscale;   // split form, backward checkpoint pass: scale of the restored state (null: 1);
                         // with npass > 0: the scales of all passes, by pass index
  // split form, circuits that fit one tile: every pass in one launch
  int npass;                 // passes of the launch (0: one pass, the kernel's parameter)
  const DevPass* passes;     // [npass] device copy, forward order
  const CoefRegion* coef;    // [npass] coefficients of this direction
  int zf;                    // forward, npass > 0: one sample per batch unit, the amplitude (re, im) in a
                             // lane pair (form 5; U = B); the chain runs from the encoding to the standard order
  uint32_t cz_nb[kMaxQubits];    // CZ neighbours of each qubit (qubit mask)
  uint32_t cz_nbhi[kMaxQubits];  // CZ neighbours of each qubit above it (qubit mask)
  // Z0 observable, working state in the standard order (at most two qubit
  // sets), tiles without batch-unit bits:
  double* epart;         // forward, last pass (non-null): per tile and sample, the partial sum of
                         // |psi|^2 (1 - 2 b0) over the tile, at [sample][tile's out-of-tile index]
};

// Dynamic shared memory of a pass block (tma: tensor-copy passes).
size_t pass_smem_bytes(int max_slots, bool tma);
// The same for the one-launch split passes of single-tile circuits (they
// also stage each pass's ops and coefficients).
size_t pass_multi_smem_bytes();

// Register layouts for tests: per (phase, variant) the tile bit of each of the
// 7 thread-index bits and 5 register-index bits, then the 12 slot weights and
// the slot count of the 16-byte exchanges, then the same for the 8-byte
// exchanges of tensor-copy passes.  Returns the number of ints.
int debug_layouts(int* out, int cap);

// Tensor maps (CUtensorMap, 128 bytes each) of a pass whose tiles are loaded
// by tensor copies.  Backward: m0 over psi (plane 0), m1 over lambda (plane 1).
// Forward: m0 over psi (planes 0 and 1 of unit u at samples 2u, 2u+1), m1 over
// the one-sample partner buffer that holds plane 1 of an odd batch's last unit.
struct PassMaps {
  alignas(64) unsigned char m0[128];
  alignas(64) unsigned char m1[128];
};
// Encode the maps of pass p over (buf0, buf1) (no-op when !p.tma).
cudaError_t encode_pass_maps(const DevPass& p, int n, int B, bool backward, const void* buf0, const void* buf1,
                             PassMaps* maps);

// Launch one pass; the kernel instance follows the pass's layout variant,
// how its tiles are loaded (n < 5: generic; tensor copies when p.tma) and
// the rotation form.  coef (device memory, may be null): the pass's gate
// coefficients, first copied in stream order into the context's
// constant-memory region of the unit that holds the instance (the first
// p.nslots rotation slots, and the diagonal tables when the pass has any).
cudaError_t launch_pass(bool backward, const PassArgs& a, const DevPass& p, const PassMaps& maps, int grid,
                        size_t smem, cudaStream_t s, const CoefRegion* coef = nullptr);
// The units that instantiate the pass kernel (pass_split.cu: split form;
// pass_fused.cu: fused SU(2) form, CZ or CNOT; pass_reup.cu: re-uploading;
// pass_csplit.cu: split form of the fused CNOT schedule).
// form: 0 fused SU(2), 1 and 2 re-uploading (2: per register pair), 3 split,
// 4 split with CNOT permutations, 5 the split form's one-launch forward with
// one sample per batch unit (pass_single.cu).
#define QML_PASS_UNIT_DECL(NAME)                                                                        \
  cudaError_t NAME##_launch(bool backward, int mode, int variant, int form, const PassArgs& a,           \
                            const DevPass& p, const PassMaps& maps, int grid, size_t smem,               \
                            const CoefRegion* coef, cudaStream_t s);                                    \
  cudaError_t NAME##_attr(size_t smem_thr, size_t smem_tma);
QML_PASS_UNIT_DECL(pass_split)
QML_PASS_UNIT_DECL(pass_fused)
QML_PASS_UNIT_DECL(pass_reup)
QML_PASS_UNIT_DECL(pass_csplit)
QML_PASS_UNIT_DECL(pass_single)
#undef QML_PASS_UNIT_DECL
// Full SU(2) coefficients of every pass slot: cf forward, ci backward ([P] regions).
cudaError_t launch_prep_pass_coef(const DevPass* passes, int n_passes, const float* theta, CoefRegion* cf,
                                  CoefRegion* ci, cudaStream_t s);
// Split form: every table the split passes need, from theta (fp64):
//   rot [L][n], lay [L], gfix [L][n][2] (gradient scale and phi1 per rotation),
//   dq_f / dq_b [L + 1][n][2] per-qubit diagonal factors, cf / ci [P] regions,
//   rscale [P] (restore scale of the backward checkpoint passes).
// undo: [L][n] qubits of each layer in the backward pass's un-apply order.
// Kernel launches of launch_prep_split for these sizes (1: one block runs
// every stage, for small circuits; else 4).
int prep_split_launches(int L, int n, int n_passes);
cudaError_t launch_prep_split(const DevPass* passes, int n_passes, const float* theta, int L, int n,
                              const int* undo, SplitRot* rot, SplitLayer* lay, double* gfix, float2* dq_f,
                              float2* dq_b, CoefRegion* cf, CoefRegion* ci, float* rscale, cudaStream_t s);
// Split form of the fused CNOT schedule (two qubit sets; set0: the first
// set's qubit mask): one segment per layer and set between two diagonal ops
// (global index 4 l + 2 set + side), seg [2 L] frames, dq_f / dq_b
// [4 L + 1][n][2], the other tables as above (rscale: 1).
cudaError_t launch_prep_split_cnot(const DevPass* passes, int n_passes, const float* theta, int L, int n,
                                   uint32_t set0, const int* undo, SplitRot* rot, SplitLayer* seg, double* gfix,
                                   float2* dq_f, float2* dq_b, CoefRegion* cf, CoefRegion* ci, float* rscale,
                                   cudaStream_t s);
// fp64 mode (coef.cu): the same tables from an fp64 theta, with the per-qubit
// diagonal factors dq_f / dq_b in fp64 and the restore scale of every pass.
cudaError_t launch_prep_split64(const DevPass* passes, int n_passes, const double* theta, int L, int n,
                                const int* undo, SplitRot* rot, SplitLayer* lay, double* gfix, double2* dq_f,
                                double2* dq_b, double* rscale, cudaStream_t s);
cudaError_t set_pass_smem_attr(size_t smem_thr, size_t smem_tma);
// mode: 0 generic addressing (n < 5), 1 thread loads, 2 tensor copies.
cudaError_t pass_occupancy(bool backward, int mode, size_t smem, int* blocks_per_sm);

cudaError_t launch_prep_enc(const float* x, int B, int n, float2* enc, cudaStream_t s);
cudaError_t launch_expect(const float2* psi, int B, int n, double* partial, float* E,
                          unsigned* status, cudaStream_t s);
size_t expect_partial_count(int B, int n);
// E[b] = the fixed-order sum of partial[b][0 .. chunks - 1] (fp64).
cudaError_t launch_expect_final(const double* partial, int chunks, int B, float* E, unsigned* status,
                               cudaStream_t s);
// gfix: split form, [L][n][2] (scale of the sums, phi1) per rotation; null otherwise.
cudaError_t launch_grad_reduce(const DevPass* passes, const int* slot_pass, const int* slot_index,
                               const float* partials, int grid, const float* theta, const double* gfix, int L,
                               int n, float* grad, unsigned* status, cudaStream_t s);
cudaError_t launch_loss_seed(const float* E, const float* y, int B, float* g, float* loss,
                             cudaStream_t s);
cudaError_t launch_bwd_init(float2* psi, float2* lam, const float* g, int B, int n, cudaStream_t s);

// In place, for every aligned chunk of 2^cb elements of buf (count elements):
// element j moves to sum_b j_b << to[b] (a permutation of the low cb index
// bits, cb <= 12).  count must be a multiple of 4096 and buf 16-byte aligned
// (cudaErrorInvalidValue otherwise); the grid is sized from sms.
cudaError_t launch_permute_bits(float2* buf, long long count, int cb, const int* to, int sms, cudaStream_t s);

// Observables O = sum_k c_k i^ny X^x Z^z, terms grouped by x (see kernels.cu).
struct ObsTerm {
  uint32_t z;  // qubits carrying Z or Y
  int ny;      // number of Y factors
  double c;    // coefficient
};
struct ObsGroup {
  uint32_t x;  // qubits carrying X or Y, shared by the group's terms
  int first, count;
  int pad;
};
// E[b] = <psi_b|O|psi_b> (partial: expect_partial_count(B, n) doubles).
cudaError_t launch_obs_expect(const float2* psi, int B, int n, const ObsGroup* groups, int ngroups,
                              const ObsTerm* terms, double* partial, float* E, unsigned* status, cudaStream_t s);
// lambda = g_b O psi, then psi and lambda into the backward planes (in place).
cudaError_t launch_obs_bwd_init(float2* psi, float2* lam, const float* g, int B, int n, const ObsGroup* groups,
                                int ngroups, const ObsTerm* terms, cudaStream_t s);
cudaError_t launch_encode(const float* x, int B, int n, float2* psi, cudaStream_t s);
cudaError_t launch_ckpt_copy(bool save, const float2* psi_in, float2* psi_out, void* slot,
                             int storage, long long count, cudaStream_t s);

// ---------------------------------------------------------- CNOT entanglers
// A linear map of the index bits over GF(2): col[k] is the image of bit k.
struct LinMap {
  uint32_t col[kMaxQubits];
};
// dst[b][j] = src[b][m(j)] for b < B, j < 2^n (m linear: XOR of col over j's
// bits; m_inv its inverse, used when the scatter form is the more local one).
cudaError_t launch_gather_bits(const float2* src, float2* dst, int n, int B, const LinMap& m, const LinMap& m_inv,
                               int sms, cudaStream_t s);
// fp64 mode: the same permutation of complex128 states, and slot save / restore
// (storage 0 fp32, 1 bf16, 2 fp64) of standard-layout states.
cudaError_t launch_gather_bits64(const double2* src, double2* dst, int n, int B, const LinMap& m,
                                 const LinMap& m_inv, int sms, cudaStream_t s);
cudaError_t launch_slot_copy64(bool save, double2* psi, void* slot, int storage, long long count, int sms,
                               cudaStream_t s);
// Checkpoint slot (standard layout, storage 0 fp32 / 1 bf16) from the forward
// pass's working layout in buf (and partner: an odd batch's last unit).
cudaError_t launch_slot_from_planes(const float2* buf, const float2* partner, void* slot, int storage, int B, int n,
                                   int sms, cudaStream_t s);
// psi lanes of the backward planes from a checkpoint slot (storage 0 fp32, 1 bf16).
cudaError_t launch_restore_planes(float2* plane0, float2* plane1, const void* slot, int storage, long long count,
                                  int sms, cudaStream_t s);

// ---------------------------------------------------------------- fp64 mode
constexpr int kF64Threads = 256;  // threads of an fp64 pass block
constexpr int kF64Warps = kF64Threads / 32;

// Arguments of one fp64 pass launch (f64.cu).  One block keeps one sample's
// tile; the state is in the standard index order.
struct Pass64Args {
  int n, B, T;            // qubits, samples, tile qubits of this pass
  int tmax;               // largest T of the context's passes (shared-memory size)
  uint32_t tile_mask;     // this pass's tile qubits
  long long n_tiles;      // B << (n - T)
  const double* theta;    // [L][n][3]
  const double* x;        // [B][n]
  double2* psi;           // [B][2^n]
  double2* lam;           // backward: [B][2^n]
  void* ckpt;             // checkpoint slots
  int storage;            // 0 fp32, 1 bf16, 2 fp64 slots
  long long slot_elems;   // elements per slot (max_batch << n)
  double* partials;       // backward gradient partials
  unsigned* status;
  int reupload;           // every layer starts with the encoding Ry(x_q) again
  uint32_t nb[kMaxQubits];    // CZ neighbours of each qubit (qubit mask)
  uint32_t nbhi[kMaxQubits];  // CZ neighbours of each qubit above it
  // split form (OP_RY / OP_DIAG passes; null otherwise)
  int L;                      // layers
  const SplitRot* srot;       // [L][n]
  const SplitLayer* slay;     // [L]
  const double2* dq;          // [L + 1][n][2] per-qubit diagonal factors of this direction
  const double* rscale;       // backward checkpoint pass: scale of the restored state (null: 1)
  // fused CNOT layers (OP_PERM, factor g = op.c): the gather maps of the
  // layer's factors on qubit bits, as columns (images of single qubits):
  // forward M_g^-1, backward M_g
  uint32_t perm_fwd[2][kMaxQubits];
  uint32_t perm_bwd[2][kMaxQubits];
};

size_t pass64_smem_bytes(bool backward, int tmax);
// Shared-memory opt-in of the fp64 pass kernels and their resident blocks per
// SM for tiles of up to 2^tmax positions.
cudaError_t pass64_setup(int tmax, int* blocks_fwd, int* blocks_bwd);
cudaError_t launch_pass64(bool backward, const Pass64Args& a, const DevPass& p, int grid, cudaStream_t s);
cudaError_t launch_bwd_init64(const double2* psi, double2* lam, const double* g, int B, int n, cudaStream_t s);
size_t expect64_partial_count(int B, int n);
cudaError_t launch_expect64(const double2* psi, int B, int n, double* partial, double* E, unsigned* status,
                            cudaStream_t s);
// gfix: split form, [L][n][2] (scale of the sums, phi1) per rotation; null otherwise.
cudaError_t launch_grad_reduce64(const DevPass* passes, const int* slot_pass, const int* slot_index,
                                 const double* partials, int grid, const double* theta, const double* gfix, int L,
                                 int n, double* grad, unsigned* status, cudaStream_t s);
cudaError_t launch_loss_seed64(const double* E, const double* y, int B, double* g, double* loss, cudaStream_t s);
// Pauli-sum observables in fp64: E[b] = <psi_b|O|psi_b> (partial: expect64_partial_count(B, n) doubles), and
// lambda = g_b O psi (separate buffers).
cudaError_t launch_obs_expect64(const double2* psi, int B, int n, const ObsGroup* groups, int ngroups,
                                const ObsTerm* terms, double* partial, double* E, unsigned* status, cudaStream_t s);
cudaError_t launch_obs_bwd_init64(const double2* psi, double2* lam, const double* g, int B, int n,
                                  const ObsGroup* groups, int ngroups, const ObsTerm* terms, cudaStream_t s);

}  // namespace qml
