// plan.hpp -- host-side pass schedule for the fused HEA kernels.
//
// The circuit (angle encoding, then L layers of Rx Ry Rz on every qubit and a
// CZ ladder) is cut into "passes".  One pass reads the state from HBM once,
// applies as many gates as fit on chip, and writes it back once; this is the
// forward gate fusion of the Deep-dive blog (sec. 1.4, item 1) and of the
// gist.science Technical Summary (sec. 2, "Forward Path Gate Fusion").  The
// backward pass runs the same passes in reverse (sec. 1.4, item 2).
//
// Qubits are split into sets of at most ten that are rotated together.  A
// pass owns 12 tile bits: the rotated set plus enough of the lowest other
// qubits ("passive" bits) to keep HBM accesses contiguous; for n <= 12 the
// tile is the whole state plus batch-unit bits.  The rotated qubits sit on
// tile bits 0-9, so the two register groups of five (tile bits 0-4 and 5-9,
// see device_plan.h) hold them all; circuits of 11-12 qubits also use the
// third group (tile bits 10-11).
#pragma once

#include <cstdint>
#include <string>
#include <utility>
#include <vector>

#include "device_plan.h"

namespace qml {

struct HostOp {
  int kind, a, b, c, d;  // as DevOp
};

struct HostPass {
  int set_id;                 // which qubit set is rotated
  int tile_q[kTileBits];      // tile bit -> qubit, or -1 - k for batch-unit bit k
  std::vector<int> out_q;     // qubits outside the tile, increasing
  int unit_bits;              // batch-unit bits inside the tile (n < 12)
  std::vector<HostOp> ops;    // forward order
  int load_phase, store_phase;
  bool gen;                   // forward: encode instead of loading
  bool last;                  // forward: last pass (stores the standard layout)
  int ckpt;                   // checkpoint slot written after this pass, or -1
  std::vector<int> slot_lq;   // gradient slot -> layer * n + qubit
  bool slow;
  int variant;                // see DevPass::variant
};

// Fused CNOT layers (two qubit sets A = sets[0], B = sets[1]).  A layer's
// CNOT list is a linear map M of the index bits over GF(2) (the amplitude at
// x moves to M x).  When the block of M from A's bits to A's bits is
// invertible, M = M2 M1 exactly, where M1 changes only A's bits ((M1 x)_A =
// (M x)_A) and M2 = M M1^-1 changes only B's bits.  M1 acts inside the tile
// of A's passes (B's bits, in or out of that tile, are only read), M2 inside
// B's.  So each layer runs as two passes and the state is never gathered
// through HBM: [M2 of the layer before, rotations of B], [rotations of A,
// M1]; one more pass applies the last layer's M2.  fwd[g] / inv[g] hold the
// columns of M_g / M_g^-1 (g = 0: M1, 1: M2) as qubit masks: the image of
// the single qubit q.
struct CnotLayers {
  uint32_t fwd[2][kMaxQubits];
  uint32_t inv[2][kMaxQubits];
};

struct Plan {
  int n = 0, L = 0, ckpt_block = 0;
  bool cnot = false;  // fused CNOT layers (CnotLayers)
  CnotLayers cl{};
  int n_sets = 0;
  // Address bit of each qubit in the working state between passes (HBM
  // layout; the standard layout is addr_of[q] = q).  Multi-set plans put the
  // first two qubits of the second set at address bits 2 and 3, so that every
  // set's tile is a run of >= 4 consecutive addresses plus these.
  std::vector<int> addr_of;
  std::vector<std::vector<int>> sets;
  std::vector<HostPass> passes;
  std::vector<int> slot_pass;   // [L*n] -> pass of (layer, qubit)
  std::vector<int> slot_index;  // [L*n] -> slot within that pass
  int n_ckpt = 0;               // checkpoint slots used
  int max_slots = 0;
};

// Build the schedule.  Returns an empty string on success, else an error.
// With cl, the fused CNOT schedule (two qubit sets only).
std::string make_plan(int n, int L, int ckpt_block, Plan* out, const CnotLayers* cl = nullptr);

// Factor the map of a CNOT list (control, target; applied in list order)
// into M2 M1 for the fused schedule of an n-qubit circuit; false when n does
// not give two qubit sets or the A-to-A block of the map is singular.
bool factor_cnot_layer(int n, const std::vector<std::pair<int, int>>& pairs, CnotLayers* out);

// Columns of the map of a CNOT list on qubit bits: fwd[q] = M e_q and
// inv[q] = M^-1 e_q.
void cnot_list_map(int n, const std::vector<std::pair<int, int>>& pairs, uint32_t* fwd, uint32_t* inv);

// Entangler of every layer: CZ on each bond (a, b).  The default is the
// chain (q, q+1), q = 0 .. n-2.
using Bonds = std::vector<std::pair<int, int>>;
Bonds chain_bonds(int n);

// Flatten to the device representation.  split: rotations as OP_RY and
// entanglers as OP_DIAG (the split form, see device_plan.h), with one more
// OP_DIAG right after the encoding.
void flatten_plan(const Plan& p, std::vector<DevPass>* passes, bool split = false);

// Split form: the qubits of every layer in the order the backward pass
// un-applies their rotations ([L][n], layer-major).
std::vector<int> undo_order(const Plan& p, const std::vector<DevPass>& split_passes);

// Entangler tables of each pass (cz_reg, cz_nb) for the bond list.
void set_pass_entangler(const Plan& p, const Bonds& bonds, std::vector<DevPass>* passes);

// Layout of qml_debug_schedule (see qml.h).
std::vector<int> describe_plan(const Plan& p);

}  // namespace qml
