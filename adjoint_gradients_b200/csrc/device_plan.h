// device_plan.h -- plain-old-data schedule records shared by the host planner
// and the CUDA kernels.  No CUDA or C++ library types.
//
// A tile is 4096 amplitude positions (12 "tile bits") of one batch unit.  Its
// 128 threads each keep 32 positions in registers.  The register layout is
// one of three fixed "phases"; in each phase the five register-index bits of
// a thread are five fixed tile bits:
//   phase 0: tile bits 0-4      phase 1: tile bits 5-9
//   phase 2: tile bits 10, 11, 0, 1, 2   (only for circuits of 11-12 qubits)
// and the seven thread-index bits are the remaining tile bits in a fixed
// order (phase 1 has two orders, the layout variants V0 and V1).  A 2x2 gate on a qubit that sits in a phase's register bits needs no
// communication; changing phase is a shared-memory exchange.  The planner
// decides which qubit each tile bit is.
#pragma once

#include <stdint.h>

namespace qml {

constexpr int kTileBits = 12;  // positions per tile = 4096
constexpr int kRegBits = 5;    // positions per thread = 32
constexpr int kThrBits = 7;    // threads per block = 128
constexpr int kPhases = 3;     // register layouts
constexpr int kPos = 1 << kRegBits;
constexpr int kThreads = 1 << kThrBits;
// Resident pass blocks per SM: 3 x 128 threads x 168 registers fill the
// register file, 3 x ~69 KB of tile buffer fit the shared memory.
constexpr int kBlocksPerSm = 3;
// Passes that load tiles by tensor copies keep a 64 KB landing buffer next to
// their exchange buffer: two blocks per SM (up to 255 registers a thread).
constexpr int kBlocksPerSmTma = 2;
constexpr int kTilePos = 1 << kTileBits;
constexpr int kSmemSlots = kTilePos + (kTilePos >> 5) + 8;  // exchange slots (see wbit in the kernels)
constexpr int kMaxSet = 10;           // qubits rotated per pass when n > 12
constexpr int kMaxLayersPerPass = 2;  // cap for circuits that fit one tile
constexpr int kMaxOut = 30;           // out-of-tile qubits
constexpr int kMaxQubits = 30;
constexpr int kMaxOps = 24;
constexpr int kMaxSlots = kMaxLayersPerPass * kTileBits;  // rotations per pass
constexpr int kCoefRegions = 16;      // per-context regions of constant memory
constexpr int kMaxDiag = kMaxLayersPerPass + 1;  // diagonal ops per pass (split rotations)

// Exchange slot of tile position x in a permuted exchange: linear over GF(2)
// (so a gather map and the slot map compose into one set of columns) and
// conflict-free for the 8-byte accesses of every layout's unpermuted side:
// the lanes of a half warp vary tile bits {5,6,7,8}, {0,1,2,3}, {10,11,0,1}
// or {5,6,7,3}, which this map sends to four independent low slot bits.
constexpr uint32_t perm_slot(uint32_t x) { return x ^ ((x >> 5) & 15u) ^ ((x >> 8) & 12u); }

// OP_RY and OP_DIAG are the split form of OP_ROT and OP_CZ: every fused
// rotation U = Rz(g) Ry(b) Rx(a) is rewritten exactly as Rz(phi1) Ry(vt)
// Rz(phi2).  The Rz factors of consecutive layers and the layer's CZ bonds
// are all diagonal and meet between the layers, so each layer boundary is one
// diagonal op, and each rotation is a real Ry applied in tangent form.
// OP_PERM: the part of a layer's CNOT list that changes only the bits of
// the pass's tile (fused CNOT layers, see plan.hpp), applied as a gather of
// the tile's positions: while reading the copied tile, or in a layout
// exchange whose reads are permuted.
enum : int { OP_EXCH = 1, OP_ROT = 2, OP_CZ = 3, OP_GEN = 4, OP_RY = 5, OP_DIAG = 6, OP_PERM = 7 };

// Tensor-copy (TMA) view of a pass's tile, used when n > 12: the state
// [B][2^n] (working-state address order) is seen as a rank-5 tensor whose
// dimensions are runs of address bits plus the sample index.  A run of in-tile qubits
// is copied whole (box = 2^bits, at most 8 bits per dimension); a run of
// out-of-tile qubits is fixed per tile (box 1, coordinate = those bits of the
// tile's out-of-tile index); the sample dimension has box 1, merged with the
// highest qubit run when that run is out of the tile.  Unused dimensions have
// size 1.
constexpr int kTmaRank = 5;
enum : int { TD_PAD = 0, TD_IN = 1, TD_OUT = 2, TD_SAMPLE = 3, TD_OUT_SAMPLE = 4 };

// OP_EXCH: a = from phase, b = to phase
// OP_ROT : a = phase, b = register-bit mask, c = layer, d = first slot
// OP_CZ  : a = phase, c = layer
// OP_GEN : a = phase
// OP_RY  : as OP_ROT (split form)
// OP_DIAG: a = phase, c = layer l (the diagonal between layers l and l+1;
//          -1: the one before layer 0), d = its table in the pass (0..kMaxDiag-1);
//          in passes of the fused CNOT schedule c is the diagonal's index
//          4 l + 2 set + side (side 0 before the set's rotations of layer l,
//          1 after them)
// OP_PERM: a = from phase, b = to phase, c = factor (0: M1, 1: M2), d = layer
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
  int slow;             // a memory phase has a batch-unit register bit (n < 5)
  int variant;          // 0: phase-1 lanes are tile bits 0-4; 1: tile bits 0,1,2,10,11
  int pf_fwd, pf_bwd;   // op index after which the next tile is prefetched (-1: right after loading)
  int tma;              // 1: tiles are loaded by tensor copies (see kTmaRank)
  int tma_kind[kTmaRank];
  int tma_qlo[kTmaRank];    // lowest address bit of the run (TD_IN, TD_OUT, TD_OUT_SAMPLE)
  int tma_bits[kTmaRank];   // address bits in the run
  int tma_shift[kTmaRank];  // TD_OUT, TD_OUT_SAMPLE: first bit of the run in the out-of-tile index
  int sstride[kTileBits];   // element offset in the copied tile of each tile bit (plane 1 at +4096)
  int tile_q[kTileBits];  // tile bit -> qubit (>= 0) or -1 - (batch-unit bit)
  int out_q[kMaxOut];     // out-of-tile qubits, in increasing address order
  uint32_t tile_abit[kTileBits];  // tile bit -> its address bit in the working state (0: unit bit)
  uint32_t out_abit[kMaxOut];     // out-of-tile qubit -> its address bit
  uint32_t cz_reg[kPhases];  // bit j: entangler parity of the register part of position j
  uint32_t cz_nb[kPhases][kRegBits];  // CZ neighbours (qubit mask) of each register bit's qubit
  // OP_PERM (at most one per pass).  In direction dir (0 forward, 1
  // backward) position y of the tile after the op holds the position
  // G y + G_o o of the tile before it (o: the tile's out-of-tile bits; GF(2)
  // products, i.e. the xor of the columns of the set bits).  perm_at[dir]:
  // 0 none, 1 applied while reading the copied tile (columns as element
  // offsets in the landing buffer), 2 in the op's layout exchange (columns
  // as exchange slots, perm_slot).
  int perm_at[2];
  uint16_t pcol[2][kTileBits];
  uint16_t pcol_o[2][kMaxOut];
  int ndiag;                 // OP_DIAG ops in the pass (split form)
  int cnot;                  // 1: a pass of the fused CNOT schedule (see plan.hpp)
  int rs_layer;              // split form, checkpoint pass: layer of the next diagonal op after the pass
  uint32_t rs_mask;          // ... and the qubits it rotates between the pass's end and that op
  long long partial_off;     // float offset of this pass's gradient partials
  int slot_lq[kMaxSlots];    // slot -> layer * n + qubit
  DevOp ops[kMaxOps];        // forward order
};

}  // namespace qml
