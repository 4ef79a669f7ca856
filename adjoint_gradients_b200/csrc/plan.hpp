// plan.hpp -- host-side pass schedule for the fused HEA kernels.
//
// The circuit (angle encoding, then L layers of Rx Ry Rz on every qubit and a
// CZ ladder) is cut into "passes".  One pass reads the state from HBM once,
// applies as many gates as fit on chip, and writes it back once; this is the
// forward gate fusion of the Deep-dive blog (sec. 1.4, item 1) and of the
// gist.science Technical Summary (sec. 2, "Forward Path Gate Fusion").  The
// backward pass runs the same passes in reverse (sec. 1.4, item 2).
//
// A pass owns a 12-bit tile: 4096 amplitude positions of one batch unit whose
// out-of-tile index bits are fixed.  Qubits are split into sets of at most ten
// that are rotated together; a pass rotates one set and carries enough of the
// lowest remaining qubits as "passive" tile bits to keep HBM accesses
// contiguous.  Inside a pass, 128 threads hold 32 positions each in registers.
// A "phase" says which five tile bits index a thread's registers (the qubits a
// 2x2 gate can be applied to without communication) and which seven index the
// thread; changing phase is a shared-memory exchange.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "device_plan.h"

namespace qml {

struct HostPhase {
  int reg_tbit[kRegBits];  // tile bit addressed by register-index bit k
  int thr_tbit[kThrBits];  // tile bit addressed by thread-index bit k (0..4 = lane)
};

struct HostOp {
  int kind;   // OP_EXCH / OP_ROT / OP_CZ / OP_GEN
  int a, b, c;
  // OP_EXCH: a = from phase, b = to phase (local indices)
  // OP_ROT : a = layer, b = register-bit mask, c = first gradient slot
  // OP_CZ  : a = layer
};

struct HostPass {
  int set_id;                 // which qubit set is rotated (-1: none)
  int tile_q[kTileBits];      // tile bit -> qubit, or -1 - k for batch-unit bit k
  std::vector<int> out_q;     // qubits outside the tile, increasing
  int unit_bits;              // batch-unit bits inside the tile (n < 12)
  std::vector<HostPhase> phases;
  std::vector<HostOp> ops;    // forward order
  int load_phase, store_phase;
  bool gen;                   // forward: encode instead of loading
  bool last;                  // forward: last pass (stores the standard layout)
  int ckpt;                   // checkpoint slot written after this pass, or -1
  int nslots;                 // gradient slots (one per rotated (layer, qubit))
  uint32_t swz_col[kTileBits];  // shared-memory swizzle column of each tile bit
};

struct Plan {
  int n = 0, L = 0, ckpt_block = 0;
  int n_sets = 0;
  std::vector<std::vector<int>> sets;
  std::vector<HostPass> passes;
  std::vector<int> slot_pass;   // [L*n] -> pass of (layer, qubit)
  std::vector<int> slot_index;  // [L*n] -> slot within that pass
  int n_ckpt = 0;               // checkpoint slots used
  int max_slots = 0;
};

// Build the schedule.  Returns an empty string on success, else an error.
std::string make_plan(int n, int L, int ckpt_block, Plan* out);

// Flatten to the device representation (phases / ops / passes arrays).
void flatten_plan(const Plan& p, std::vector<DevPass>* passes, std::vector<DevPhase>* phases,
                  std::vector<DevOp>* ops);

// Layout of qml_debug_schedule (see qml.h).
std::vector<int> describe_plan(const Plan& p);

}  // namespace qml
