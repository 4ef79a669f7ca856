// plan.cpp -- host-side pass schedule (see plan.hpp).
#include "plan.hpp"

#include <algorithm>

namespace qml {
namespace {

enum TaskKind { T_GEN, T_ROT, T_CZ, T_PERM };
struct Task {
  TaskKind kind;
  int layer;
  int set;
  int group;  // T_PERM: factor of the layer's CNOT map (0: M1, 1: M2)
};

// Tile bit addressed by register-index bit k in phase p (mirrors the kernels).
int reg_tbit(int p, int k) {
  if (p == 0) return k;
  if (p == 1) return 5 + k;
  return k < 2 ? 10 + k : k - 2;
}

// Phase p's register bits are all qubits (no batch-unit bit).
bool phase_fast(const HostPass& ps, int p) {
  for (int k = 0; k < kRegBits; ++k)
    if (ps.tile_q[reg_tbit(p, k)] < 0) return false;
  return true;
}


// Tensor-copy view of the tile (see kTmaRank) over the address bits of the
// working-state layout (addr_of).  Multi-set plans only: their tiles hold no
// batch-unit bit, address bits 0 and 1 are always in the tile, so the
// innermost run is >= 32 B.
void set_tma_view(int n, const HostPass& ps, const std::vector<int>& addr_of, DevPass* d) {
  d->tma = 0;
  for (int i = 0; i < kTmaRank; ++i) d->tma_kind[i] = TD_PAD, d->tma_qlo[i] = d->tma_bits[i] = d->tma_shift[i] = 0;
  for (int b = 0; b < kTileBits; ++b) d->sstride[b] = 0;
  if (n <= kTileBits || ps.slow || ps.unit_bits != 0) return;
  std::vector<int> tbit_of_a(n, -1);  // address bit -> tile bit
  for (int b = 0; b < kTileBits; ++b)
    if (ps.tile_q[b] >= 0) tbit_of_a[addr_of[ps.tile_q[b]]] = b;
  if (tbit_of_a[0] < 0 || tbit_of_a[1] < 0) return;
  int rank = 0, out_seen = 0;
  long long box = 1;  // elements of the box below the current dimension
  int q = 0;
  while (q < n) {
    const bool in = tbit_of_a[q] >= 0;
    int e = q;
    while (e < n && (tbit_of_a[e] >= 0) == in) ++e;
    if (in) {
      for (int lo = q; lo < e; lo += 8) {
        const int bits = std::min(8, e - lo);
        if (rank == kTmaRank) return;
        d->tma_kind[rank] = TD_IN, d->tma_qlo[rank] = lo, d->tma_bits[rank] = bits;
        for (int k = 0; k < bits; ++k) d->sstride[tbit_of_a[lo + k]] = (int)(box << k);
        box <<= bits;
        ++rank;
      }
    } else {
      if (rank == kTmaRank) return;
      d->tma_kind[rank] = e == n ? TD_OUT_SAMPLE : TD_OUT;
      d->tma_qlo[rank] = q, d->tma_bits[rank] = e - q, d->tma_shift[rank] = out_seen;
      out_seen += e - q;
      ++rank;
    }
    q = e;
  }
  if (tbit_of_a[n - 1] >= 0) {  // highest address bit in the tile: a separate sample dimension
    if (rank == kTmaRank) return;
    d->tma_kind[rank] = TD_SAMPLE;
    ++rank;
  }
  if (box != kTilePos) return;
  d->tma = 1;
}

// Qubit sets rotated together: the whole register for n <= 12, else
// ceil(n / 10) runs of consecutive qubits of near-equal size.
std::vector<std::vector<int>> qubit_sets(int n) {
  std::vector<std::vector<int>> sets;
  if (n <= kTileBits) {
    sets.push_back({});
    for (int q = 0; q < n; ++q) sets[0].push_back(q);
    return sets;
  }
  const int s = (n + kMaxSet - 1) / kMaxSet;
  const int base = n / s, extra = n % s;
  int q = 0;
  for (int i = 0; i < s; ++i) {
    const int sz = base + (i < extra ? 1 : 0);
    std::vector<int> set;
    for (int k = 0; k < sz; ++k) set.push_back(q++);
    sets.push_back(set);
  }
  return sets;
}

// GF(2) linear maps on qubit bits, stored as columns (the image of each
// single qubit as a qubit mask).
uint32_t gf2_apply(const uint32_t* cols, int n, uint32_t x) {
  uint32_t y = 0;
  for (int q = 0; q < n; ++q)
    if ((x >> q) & 1u) y ^= cols[q];
  return y;
}

// Inverse by Gauss-Jordan elimination on the rows; false if singular.
bool gf2_inverse(const uint32_t* cols, int n, uint32_t* inv) {
  // row r of the matrix: bit c = bit r of column c; augmented with identity
  std::vector<uint32_t> row(n), aug(n);
  for (int r = 0; r < n; ++r) {
    row[r] = 0;
    for (int c = 0; c < n; ++c)
      if ((cols[c] >> r) & 1u) row[r] |= 1u << c;
    aug[r] = 1u << r;
  }
  for (int c = 0; c < n; ++c) {
    int piv = -1;
    for (int r = c; r < n; ++r)
      if ((row[r] >> c) & 1u) {
        piv = r;
        break;
      }
    if (piv < 0) return false;
    std::swap(row[c], row[piv]);
    std::swap(aug[c], aug[piv]);
    for (int r = 0; r < n; ++r)
      if (r != c && ((row[r] >> c) & 1u)) row[r] ^= row[c], aug[r] ^= aug[c];
  }
  // rows of the inverse are aug; back to columns
  for (int c = 0; c < n; ++c) {
    inv[c] = 0;
    for (int r = 0; r < n; ++r)
      if ((aug[r] >> c) & 1u) inv[c] |= 1u << r;
  }
  return true;
}

// Fused CNOT layers: the gather columns of the pass's OP_PERM in both
// directions (see DevPass::perm_at).  The forward gathers through M_g^-1,
// the backward through M_g.  M1 (M2) changes only the bits of the first
// (second) set, all inside this pass's tile, and reads the others: in-tile
// columns stay in the tile, an out-of-tile qubit's column is itself plus
// in-tile bits.
void set_pass_perm(const Plan& p, const HostPass& ps, const std::vector<HostOp>& ops, DevPass* d) {
  d->perm_at[0] = d->perm_at[1] = 0;
  for (int dir = 0; dir < 2; ++dir) {
    for (int b = 0; b < kTileBits; ++b) d->pcol[dir][b] = 0;
    for (int k = 0; k < kMaxOut; ++k) d->pcol_o[dir][k] = 0;
  }
  int oi = -1;
  for (int o = 0; o < (int)ops.size(); ++o)
    if (ops[o].kind == OP_PERM) oi = o;
  if (oi < 0 || !p.cnot || !d->tma) return;
  const HostOp& op = ops[oi];
  const int g = op.c;
  auto tile_pattern = [&](uint32_t qmask) {
    uint32_t t = 0;
    for (int b = 0; b < kTileBits; ++b)
      if (ps.tile_q[b] >= 0 && ((qmask >> ps.tile_q[b]) & 1u)) t |= 1u << b;
    return t;
  };
  auto offset = [&](uint32_t t) {  // element offset in the copied tile (a bit permutation of t)
    uint32_t e = 0;
    for (int b = 0; b < kTileBits; ++b)
      if ((t >> b) & 1u) e += (uint32_t)d->sstride[b];
    return e;
  };
  d->perm_at[0] = (oi == 0 && op.a == op.b && op.a == ps.load_phase && !ps.gen) ? 1 : 2;
  d->perm_at[1] = (oi + 1 == (int)ops.size() && op.a == op.b && op.a == ps.store_phase) ? 1 : 2;
  for (int dir = 0; dir < 2; ++dir) {
    const uint32_t* G = dir == 0 ? p.cl.inv[g] : p.cl.fwd[g];
    auto space = [&](uint32_t t) { return (uint16_t)(d->perm_at[dir] == 1 ? offset(t) : perm_slot(t)); };
    for (int b = 0; b < kTileBits; ++b)
      if (ps.tile_q[b] >= 0) d->pcol[dir][b] = space(tile_pattern(G[ps.tile_q[b]]));
    for (int k = 0; k < (int)ps.out_q.size(); ++k) d->pcol_o[dir][k] = space(tile_pattern(G[ps.out_q[k]]));
  }
}

}  // namespace

void cnot_list_map(int n, const std::vector<std::pair<int, int>>& pairs, uint32_t* fwd, uint32_t* inv) {
  for (int q = 0; q < n; ++q) {
    uint32_t f = 1u << q, b = 1u << q;
    for (const auto& e : pairs) f ^= ((f >> e.first) & 1u) << e.second;
    for (auto it = pairs.rbegin(); it != pairs.rend(); ++it) b ^= ((b >> it->first) & 1u) << it->second;
    fwd[q] = f;
    inv[q] = b;
  }
}

bool factor_cnot_layer(int n, const std::vector<std::pair<int, int>>& pairs, CnotLayers* out) {
  const auto sets = qubit_sets(n);
  if (sets.size() != 2) return false;
  uint32_t mA = 0;
  for (int q : sets[0]) mA |= 1u << q;
  const uint32_t mB = ((n >= 32) ? ~0u : ((1u << n) - 1u)) & ~mA;
  uint32_t M[kMaxQubits], Mi[kMaxQubits], M1[kMaxQubits], M1i[kMaxQubits], M2[kMaxQubits], M2i[kMaxQubits];
  cnot_list_map(n, pairs, M, Mi);
  // M1: A's bits as M leaves them, B's bits unchanged
  for (int q = 0; q < n; ++q) M1[q] = (M[q] & mA) | ((1u << q) & mB);
  if (!gf2_inverse(M1, n, M1i)) return false;
  for (int q = 0; q < n; ++q) {
    M2[q] = gf2_apply(M, n, M1i[q]);     // M M1^-1
    M2i[q] = gf2_apply(M1, n, Mi[q]);    // M1 M^-1
    if ((M2[q] & mA) != ((1u << q) & mA)) return false;  // M2 must leave A's bits alone
  }
  *out = CnotLayers{};
  for (int q = 0; q < n; ++q) {
    out->fwd[0][q] = M1[q], out->inv[0][q] = M1i[q];
    out->fwd[1][q] = M2[q], out->inv[1][q] = M2i[q];
  }
  return true;
}

std::string make_plan(int n, int L, int ckpt_block, Plan* out, const CnotLayers* cl) {
  if (n < 1 || n > 30) return "n_qubits must be in [1, 30]";
  if (L < 1 || L > 100000) return "n_layers must be in [1, 100000]";
  if (ckpt_block < 0) return "ckpt_block must be >= 0";
  Plan p;
  p.n = n;
  p.L = L;
  p.ckpt_block = ckpt_block;

  p.sets = qubit_sets(n);
  p.n_sets = (int)p.sets.size();
  const int S = p.n_sets;
  if (cl && S != 2) return "fused CNOT layers need two qubit sets";
  p.cnot = cl != nullptr;
  if (cl) p.cl = *cl;
  // ---- working-state address bits: identity, except that plans with three
  // or more sets move the second set's first two qubits to address bits 2
  // and 3 (every set's tile then covers address bits 0-3 or 0-2: HBM runs of
  // >= 64 B instead of 32 B); the layout is converted to and from the
  // standard one by a separate kernel at the ends of the pass chain
  p.addr_of.resize(n);
  {
    std::vector<int> order;
    if (S >= 3) {
      order = {0, 1, p.sets[1][0], p.sets[1][1]};
      for (int q = 0; q < n; ++q)
        if (std::find(order.begin(), order.end(), q) == order.end()) order.push_back(q);
    } else {
      for (int q = 0; q < n; ++q) order.push_back(q);
    }
    for (int a = 0; a < n; ++a) p.addr_of[order[a]] = a;
  }
  p.n_ckpt = (ckpt_block > 0) ? (L + ckpt_block - 1) / ckpt_block - 1 : 0;

  // ---- task list: encode, then per layer the sets in boustrophedon order, then CZ;
  // fused CNOT layers: per layer [M2 of the layer before] the second set, the
  // first set, M1; at the end the last layer's M2
  std::vector<Task> tasks;
  tasks.push_back({T_GEN, -1, -1, 0});
  for (int l = 0; l < L; ++l) {
    if (cl) {
      if (l > 0) tasks.push_back({T_PERM, l - 1, 1, 1});
      tasks.push_back({T_ROT, l, 1, 0});
      tasks.push_back({T_ROT, l, 0, 0});
      tasks.push_back({T_PERM, l, 0, 0});
      continue;
    }
    for (int i = 0; i < S; ++i) tasks.push_back({T_ROT, l, (l % 2 == 0) ? i : S - 1 - i, 0});
    tasks.push_back({T_CZ, l, -1, 0});
  }
  if (cl) tasks.push_back({T_PERM, L - 1, 1, 1});

  // ---- group tasks into passes: a new pass starts when the rotated set
  // changes, when a single-tile pass is full, or after a checkpoint boundary
  // of a single-tile circuit (so that its slot is a clean layer boundary)
  struct Proto {
    int set = -1;
    std::vector<Task> t;
    int rots = 0;
    int ckpt = -1;
  };
  std::vector<Proto> protos(1);
  for (const Task& tk : tasks) {
    Proto* cur = &protos.back();
    if (tk.kind == T_ROT || tk.kind == T_PERM) {
      bool need_new = (cur->set >= 0 && cur->set != tk.set) || (S == 1 && cur->rots >= kMaxLayersPerPass);
      if (need_new) {
        protos.emplace_back();
        cur = &protos.back();
      }
      cur->set = tk.set;
      if (tk.kind == T_ROT) cur->rots++;
    }
    cur->t.push_back(tk);
    if (((tk.kind == T_CZ && !cl) || (tk.kind == T_PERM && tk.group == 0)) && ckpt_block > 0) {
      const int l = tk.layer;
      if ((l + 1) % ckpt_block == 0 && l + 1 < L) {
        cur->ckpt = (l + 1) / ckpt_block - 1;  // slot m-1 holds the state after layer m*b-1
        if (S == 1) protos.emplace_back();
      }
    }
  }
  if (protos.back().t.empty()) protos.pop_back();

  p.slot_pass.assign((size_t)L * n, -1);
  p.slot_index.assign((size_t)L * n, -1);

  for (size_t pi = 0; pi < protos.size(); ++pi) {
    const Proto& pr = protos[pi];
    HostPass ps;
    ps.set_id = pr.set;
    ps.last = (pi + 1 == protos.size());
    ps.ckpt = pr.ckpt;
    ps.gen = false;
    for (const Task& tk : pr.t)
      if (tk.kind == T_GEN) ps.gen = true;

    // ---- tile bits
    std::vector<bool> rotated_q(n, false);
    if (S == 1) {
      for (int q = 0; q < n; ++q) rotated_q[q] = true;
      ps.variant = 0;
      ps.unit_bits = kTileBits - n;
      for (int t = 0; t < kTileBits; ++t) ps.tile_q[t] = t < n ? t : -1 - (t - n);
    } else {
      // The passive tile bits are the other qubits with the lowest address
      // bits; the out-of-tile qubits are listed in address order.
      const std::vector<int>& set = p.sets[pr.set];
      std::vector<bool> in(n, false);
      for (int q : set) in[q] = rotated_q[q] = true;
      std::vector<int> by_addr(n);
      for (int q = 0; q < n; ++q) by_addr[p.addr_of[q]] = q;
      std::vector<int> passive;
      for (int a = 0; a < n && (int)(set.size() + passive.size()) < kTileBits; ++a) {
        const int q = by_addr[a];
        if (!in[q]) {
          passive.push_back(q);
          in[q] = true;
        }
      }
      for (int a = 0; a < n; ++a)
        if (!in[by_addr[a]]) ps.out_q.push_back(by_addr[a]);
      ps.unit_bits = 0;
      const bool identity = S < 3;
      if (identity && set[0] == 0) {
        // variant 0: the set on tile bits 0 .. |R|-1, passive after; phase
        // 1's lanes (tile bits 0-4) are qubits 0-4
        ps.variant = 0;
        for (int t = 0; t < (int)set.size(); ++t) ps.tile_q[t] = set[t];
        for (size_t i = 0; i < passive.size(); ++i) ps.tile_q[set.size() + i] = passive[i];
      } else {
        // variant 1: the two lowest-address passive qubits on tile bits 10
        // and 11 (never rotated: register bits only in phase 2), the other
        // in-tile qubits on tile bits 0 .. 9 in address order.  Phase 1's
        // lanes are tile bits 10, 11, 0, 1, 2 in lane order, so a warp
        // covers the five lowest in-tile addresses (long HBM runs; a half
        // warp reads contiguous elements of a copied tile).
        ps.variant = 1;
        ps.tile_q[10] = passive[0];
        ps.tile_q[11] = passive[1];
        int t = 0;
        for (int a = 0; a < n; ++a) {
          const int q = by_addr[a];
          if (in[q] && q != passive[0] && q != passive[1]) ps.tile_q[t++] = q;
        }
      }
    }
    if ((int)ps.out_q.size() > kMaxOut) return "internal: too many out-of-tile qubits";

    // ---- rotated qubits per register group (tile bits 0-4, 5-9, 10-11), and
    // the phase that touches HBM: phase 1 when its register bits are all
    // qubits (its lanes are the contiguous tile bits), else phase 0
    int mask[kPhases];
    std::vector<int> active;
    for (int g = 0; g < kPhases; ++g) {
      mask[g] = 0;
      const int nk = g == 2 ? 2 : kRegBits;
      for (int k = 0; k < nk; ++k) {
        const int q = ps.tile_q[reg_tbit(g, k)];
        if (q >= 0 && rotated_q[q]) mask[g] |= 1 << k;
      }
      if (mask[g]) active.push_back(g);
    }
    int mem = phase_fast(ps, 1) ? 1 : 0;
    ps.slow = !phase_fast(ps, mem);
    ps.load_phase = mem;

    // group order of the first rotation: start in the memory phase when
    // loading; when encoding, choose the direction that ends in it
    std::vector<int> order;
    if (std::find(active.begin(), active.end(), mem) != active.end()) order.push_back(mem);
    for (int g : active)
      if (g != mem) order.push_back(g);
    const bool ends_at_mem_if_forward = (pr.rots % 2 == 0);
    bool dir = true;
    if (ps.gen) dir = ends_at_mem_if_forward;
    int cur = mem;
    if (ps.gen) {
      // encode directly in the first group's layout when that layout is fast
      std::vector<int> first = order;
      if (!dir) std::reverse(first.begin(), first.end());
      if (first[0] != 2 && phase_fast(ps, first[0])) cur = first[0];  // memory ops use phase 0 or 1
      ps.load_phase = cur;
      ps.ops.push_back({OP_GEN, cur, 0, 0, 0});
    }
    int rot_i = 0;
    for (const Task& tk : pr.t) {
      if (tk.kind == T_ROT) {
        std::vector<int> ord = order;
        const bool d = (rot_i++ % 2 == 0) ? dir : !dir;
        if (!d) std::reverse(ord.begin(), ord.end());
        for (int g : ord) {
          if (g != cur) ps.ops.push_back({OP_EXCH, cur, g, 0, 0});
          cur = g;
          const int slot0 = (int)ps.slot_lq.size();
          for (int k = 0; k < kRegBits; ++k)
            if (mask[g] & (1 << k)) {
              const int q = ps.tile_q[reg_tbit(g, k)];
              const size_t idx = (size_t)tk.layer * n + q;
              p.slot_pass[idx] = (int)pi;
              p.slot_index[idx] = (int)ps.slot_lq.size();
              ps.slot_lq.push_back(tk.layer * n + q);
            }
          ps.ops.push_back({OP_ROT, g, mask[g], tk.layer, slot0});
        }
      } else if (tk.kind == T_CZ) {
        ps.ops.push_back({OP_CZ, cur, 0, tk.layer, 0});
      } else if (tk.kind == T_PERM) {
        // M1 ends the pass: its permuted exchange goes to the memory phase;
        // M2 starts one, in the phase it is in (the memory phase)
        const int to = tk.group == 0 ? mem : cur;
        ps.ops.push_back({OP_PERM, cur, to, tk.group, tk.layer});
        cur = to;
      }
    }
    if (cur != mem) ps.ops.push_back({OP_EXCH, cur, mem, 0, 0});
    ps.store_phase = mem;
    // (the split form adds one op after the encoding)
    if ((int)ps.ops.size() + (ps.gen ? 1 : 0) > kMaxOps) return "internal: too many ops in a pass";
    if ((int)ps.slot_lq.size() > kMaxSlots) return "internal: too many gradient slots in a pass";
    p.max_slots = std::max(p.max_slots, (int)ps.slot_lq.size());
    p.passes.push_back(ps);
  }
  for (size_t i = 0; i < p.slot_pass.size(); ++i)
    if (p.slot_pass[i] < 0) return "internal: a rotation was not scheduled";
  *out = p;
  return "";
}

void flatten_plan(const Plan& p, std::vector<DevPass>* passes, bool split) {
  passes->clear();
  // qubit mask of a rotation op of pass ps
  auto op_qubits = [](const HostPass& ps, const HostOp& o) {
    uint32_t m = 0;
    for (int k = 0; k < kRegBits; ++k)
      if (o.b & (1 << k)) m |= 1u << ps.tile_q[reg_tbit(o.a, k)];
    return m;
  };
  for (size_t pi = 0; pi < p.passes.size(); ++pi) {
    const HostPass& ps = p.passes[pi];
    DevPass d{};
    // op list (the split form renames rotations and entanglers, and adds the
    // diagonal that precedes layer 0 right after the encoding)
    std::vector<HostOp> ops;
    int ndiag = 0;
    if (split && p.cnot) {
      // fused CNOT layers: the pass's rotations (one layer of one set) are a
      // segment of their own between two diagonal ops, D2 (the Rz(phi2)
      // factors) before and D1 (the Rz(phi1) factors and the segment's
      // frame) after; global diagonal index 4 l + 2 set + (0: D2, 1: D1)
      int first_rot = -1, last_rot = -1;
      for (int o = 0; o < (int)ps.ops.size(); ++o)
        if (ps.ops[o].kind == OP_ROT) {
          if (first_rot < 0) first_rot = o;
          last_rot = o;
        }
      for (int o = 0; o < (int)ps.ops.size(); ++o) {
        const HostOp& h = ps.ops[o];
        const int dbase = 4 * h.c + 2 * ps.set_id;
        if (o == first_rot) ops.push_back({OP_DIAG, h.a, 0, dbase, ndiag++});
        HostOp x = h;
        if (x.kind == OP_ROT) x.kind = OP_RY;
        ops.push_back(x);
        if (o == last_rot) ops.push_back({OP_DIAG, h.a, 0, dbase + 1, ndiag++});
      }
    } else {
      for (const HostOp& h : ps.ops) {
        HostOp o = h;
        if (split && o.kind == OP_ROT) o.kind = OP_RY;
        if (split && o.kind == OP_CZ) o = {OP_DIAG, h.a, 0, h.c, ndiag++};
        ops.push_back(o);
        if (split && h.kind == OP_GEN) ops.push_back({OP_DIAG, h.a, 0, -1, ndiag++});
      }
    }
    d.nops = (int)ops.size();
    d.ndiag = ndiag;
    d.cnot = p.cnot ? 1 : 0;
    d.load_phase = ps.load_phase;
    d.store_phase = ps.store_phase;
    d.gen = ps.gen ? 1 : 0;
    d.last = ps.last ? 1 : 0;
    d.ckpt = ps.ckpt;
    d.nslots = (int)ps.slot_lq.size();
    d.n_out = (int)ps.out_q.size();
    d.unit_bits = ps.unit_bits;
    d.slow = ps.slow ? 1 : 0;
    d.variant = ps.variant;
    // forward: after the last exchange; backward (ops run in reverse): after the first
    d.pf_fwd = d.pf_bwd = -1;
    for (int o = 0; o < (int)ops.size(); ++o)
      if (ops[o].kind == OP_EXCH) {
        d.pf_fwd = o;
        if (d.pf_bwd < 0) d.pf_bwd = o;
      }
    // split form, checkpoint pass: the rotations between the pass's end and
    // the next diagonal op (all of that op's layer)
    d.rs_layer = -1;
    d.rs_mask = 0;
    if (split && ps.ckpt >= 0 && !p.cnot) {  // (fused CNOT layers: exact state at every pass boundary)
      bool found = false;
      for (size_t pj = pi + 1; pj < p.passes.size() && !found; ++pj)
        for (const HostOp& h : p.passes[pj].ops) {
          if (h.kind == OP_CZ) {
            d.rs_layer = h.c;
            found = true;
            break;
          }
          if (h.kind == OP_ROT) d.rs_mask |= op_qubits(p.passes[pj], h);
        }
    }
    for (int t = 0; t < kTileBits; ++t) d.tile_q[t] = ps.tile_q[t];
    set_tma_view(p.n, ps, p.addr_of, &d);
    for (int b = 0; b < kTileBits; ++b) d.tile_abit[b] = ps.tile_q[b] >= 0 ? 1u << p.addr_of[ps.tile_q[b]] : 0u;
    for (int i = 0; i < kMaxOut; ++i) d.out_abit[i] = i < d.n_out ? 1u << p.addr_of[ps.out_q[i]] : 0u;
    for (int i = 0; i < kMaxOut; ++i) d.out_q[i] = i < d.n_out ? ps.out_q[i] : -1;
    d.partial_off = 0;
    for (int s = 0; s < kMaxSlots; ++s) d.slot_lq[s] = s < d.nslots ? ps.slot_lq[s] : 0;
    set_pass_perm(p, ps, ops, &d);
    for (int o = 0; o < kMaxOps; ++o) {
      if (o < d.nops) {
        const HostOp& h = ops[o];
        d.ops[o] = {h.kind, h.a, h.b, h.c, h.d};
      } else {
        d.ops[o] = {0, 0, 0, 0, 0};
      }
    }
    passes->push_back(d);
  }
}

std::vector<int> undo_order(const Plan& p, const std::vector<DevPass>& sp) {
  const int n = p.n;
  std::vector<int> order((size_t)p.L * n, -1);
  std::vector<int> fill(p.L, 0);
  for (int pi = (int)sp.size() - 1; pi >= 0; --pi) {
    const DevPass& d = sp[pi];
    for (int o = d.nops - 1; o >= 0; --o) {
      const DevOp& op = d.ops[o];
      if (op.kind != OP_RY && op.kind != OP_ROT) continue;
      for (int k = 0; k < kRegBits; ++k)  // the kernel un-applies one op's rotations in increasing k
        if (op.b & (1 << k)) order[(size_t)op.c * n + fill[op.c]++] = d.tile_q[reg_tbit(op.a, k)];
    }
  }
  return order;
}

Bonds chain_bonds(int n) {
  Bonds b;
  for (int q = 0; q + 1 < n; ++q) b.push_back({q, q + 1});
  return b;
}

void set_pass_entangler(const Plan& p, const Bonds& bonds, std::vector<DevPass>* passes) {
  uint32_t nb[32] = {0};
  for (const auto& e : bonds) {
    nb[e.first] ^= 1u << e.second;  // a bond listed twice cancels (CZ^2 = I)
    nb[e.second] ^= 1u << e.first;
  }
  for (size_t pi = 0; pi < p.passes.size(); ++pi) {
    const HostPass& ps = p.passes[pi];
    DevPass& d = (*passes)[pi];
    for (int g = 0; g < kPhases; ++g) {
      // parity of sum over bonds of i_a i_b for each register part j of a position
      uint32_t w = 0;
      for (int j = 0; j < kPos; ++j) {
        uint32_t b = 0;
        for (int k = 0; k < kRegBits; ++k) {
          const int q = ps.tile_q[reg_tbit(g, k)];
          if ((j >> k) & 1 && q >= 0) b |= 1u << q;
        }
        int s = 0;
        for (const auto& e : bonds) s ^= (int)((b >> e.first) & (b >> e.second) & 1u);
        if (s) w |= 1u << j;
      }
      d.cz_reg[g] = w;
      for (int k = 0; k < kRegBits; ++k) {
        const int q = ps.tile_q[reg_tbit(g, k)];
        d.cz_nb[g][k] = q >= 0 ? nb[q] : 0u;
      }
    }
  }
}

std::vector<int> describe_plan(const Plan& p) {
  std::vector<int> v;
  v.push_back((int)p.passes.size());
  for (const HostPass& ps : p.passes) {
    v.push_back(ps.set_id);
    v.push_back(ps.gen ? 1 : 0);
    v.push_back(ps.last ? 1 : 0);
    v.push_back(ps.ckpt);
    v.push_back((int)ps.ops.size());
    for (const HostOp& o : ps.ops) {
      int a = o.a, b = 0, c = 0;
      if (o.kind == OP_EXCH) {
        b = o.b;
      } else if (o.kind == OP_ROT) {
        a = o.c;  // layer
        uint32_t qm = 0;
        for (int k = 0; k < kRegBits; ++k)
          if (o.b & (1 << k)) qm |= 1u << ps.tile_q[reg_tbit(o.a, k)];
        b = (int)qm;
        c = o.d;
      } else if (o.kind == OP_CZ) {
        a = o.c;  // layer
      }
      v.push_back(o.kind);
      v.push_back(a);
      v.push_back(b);
      v.push_back(c);
    }
  }
  return v;
}

}  // namespace qml
