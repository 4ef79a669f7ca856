// device_plan.h -- plain-old-data schedule records shared by the host planner
// and the CUDA kernels.  No CUDA or C++ library types.
#pragma once

#include <stdint.h>

namespace qml {

constexpr int kTileBits = 12;  // positions per tile = 4096
constexpr int kRegBits = 4;    // positions per thread = 16
constexpr int kThrBits = 8;    // threads per block = 256
constexpr int kPos = 1 << kRegBits;
constexpr int kThreads = 1 << kThrBits;
constexpr int kTilePos = 1 << kTileBits;
constexpr int kMaxSet = 10;           // qubits rotated per pass when n > 12
constexpr int kMaxLayersPerPass = 16; // cap for circuits that fit one tile
constexpr int kMaxOut = 30;           // out-of-tile qubits

enum : int { OP_EXCH = 1, OP_ROT = 2, OP_CZ = 3, OP_GEN = 4 };

// Where the 12 tile bits sit for one register layout.
struct DevPhase {
  int reg_q[kRegBits];        // qubit addressed by register-index bit k, or -1
  int reg_u[kRegBits];        // batch-unit bit addressed by register bit k, or -1
  int thr_q[kThrBits];        // qubit addressed by thread-index bit k, or -1
  int thr_u[kThrBits];        // batch-unit bit addressed by thread bit k, or -1
  uint32_t reg_phys[kRegBits];  // swizzled shared-memory slot of register bit k
  uint32_t thr_phys[kThrBits];  // swizzled shared-memory slot of thread bit k
  uint32_t cz_reg;            // bit j: CZ-ladder parity of register part of position j
  uint32_t z0_reg;            // bit j: qubit-0 bit of register part of position j
  int has_reg_unit;           // some register bit is a batch-unit bit
  int pad_;
};

struct DevOp {
  int kind, a, b, c;
};

struct DevPass {
  int op0, nops;        // ops[op0 .. op0+nops) in forward order
  int phase0, nphases;  // phases[phase0 .. phase0+nphases)
  int load_phase, store_phase;
  int gen, last;
  int ckpt;             // checkpoint slot, or -1
  int nslots;           // gradient slots
  int n_out;            // qubits outside the tile
  int unit_bits;        // batch-unit bits inside the tile
  int out_q[kMaxOut];
  long long partial_off;  // float offset of this pass's gradient partials
};

}  // namespace qml
