// device_plan.h -- plain-old-data schedule records shared by the host planner
// and the CUDA kernels.  No CUDA or C++ library types.
//
// A tile is 4096 amplitude positions (12 "tile bits") of one batch unit.  Its
// 256 threads each keep 16 positions in registers.  The register layout is
// one of three fixed "phases": in phase p the four register-index bits of a
// thread are tile bits 4p .. 4p+3, and the eight thread-index bits are the
// other tile bits in increasing order.  A 2x2 gate on a qubit that sits in a
// phase's register bits needs no communication; changing phase is a
// shared-memory exchange.  The planner decides which qubit each tile bit is.
#pragma once

#include <stdint.h>

namespace qml {

constexpr int kTileBits = 12;  // positions per tile = 4096
constexpr int kRegBits = 4;    // positions per thread = 16
constexpr int kThrBits = 8;    // threads per block = 256
constexpr int kPhases = 3;     // register layouts
constexpr int kPos = 1 << kRegBits;
constexpr int kThreads = 1 << kThrBits;
constexpr int kTilePos = 1 << kTileBits;
constexpr int kSmemSlots = kTilePos + (kTilePos >> 4);  // one pad slot per 16
constexpr int kMaxSet = 10;           // qubits rotated per pass when n > 12
constexpr int kMaxLayersPerPass = 8;  // cap for circuits that fit one tile
constexpr int kMaxOut = 30;           // out-of-tile qubits
constexpr int kMaxOps = 64;
constexpr int kMaxSlots = kMaxLayersPerPass * kTileBits;

enum : int { OP_EXCH = 1, OP_ROT = 2, OP_CZ = 3, OP_GEN = 4 };

// OP_EXCH: a = from phase, b = to phase
// OP_ROT : a = phase, b = register-bit mask, c = layer, d = first slot
// OP_CZ  : a = phase, c = layer
// OP_GEN : a = phase
struct DevOp {
  int kind, a, b, c, d;
};

struct DevPass {
  int nops;
  int load_phase, store_phase;
  int gen, last;
  int ckpt;             // checkpoint slot written after / read before this pass, or -1
  int nslots;           // rotated (layer, qubit) pairs = gradient slots
  int n_out;            // qubits outside the tile
  int unit_bits;        // batch-unit bits inside the tile
  int slow;             // a load/store/encode phase has a batch-unit register bit
  int tile_q[kTileBits];  // tile bit -> qubit (>= 0) or -1 - (batch-unit bit)
  int out_q[kMaxOut];     // out-of-tile qubits, increasing
  uint32_t cz_reg[kPhases];  // bit j: CZ-ladder parity of the register part of position j
  int pad_[1];
  long long partial_off;     // float offset of this pass's gradient partials
  int slot_lq[kMaxSlots];    // slot -> layer * n + qubit
  DevOp ops[kMaxOps];        // forward order
};

}  // namespace qml
