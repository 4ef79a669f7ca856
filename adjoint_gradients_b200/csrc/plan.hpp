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

struct Plan {
  int n = 0, L = 0, ckpt_block = 0;
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
std::string make_plan(int n, int L, int ckpt_block, Plan* out);

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
