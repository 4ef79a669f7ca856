// plan.cpp -- host-side pass schedule (see plan.hpp).
#include "plan.hpp"

#include <algorithm>
#include <cstdio>

namespace qml {
namespace {

enum TaskKind { T_GEN, T_ROT, T_CZ };
struct Task {
  TaskKind kind;
  int layer;
  int set;
};

int popcount32(uint32_t v) { return __builtin_popcount(v); }

// GF(2)^3: are a, b, c a basis?
bool basis3(uint32_t a, uint32_t b, uint32_t c) {
  if (!a || !b || a == b) return false;
  return c && c != a && c != b && c != (a ^ b);
}

// Choose, per tile bit >= 3, the 3-bit column that is XORed into the low three
// bits of the shared-memory slot, so that in every phase the eight lanes of a
// quarter warp (thread bits 0..2) hit eight different 16-byte bank groups.
bool choose_swizzle(HostPass* ps) {
  uint32_t col[kTileBits];
  uint64_t rng = 0x9E3779B97F4A7C15ull;
  for (int attempt = 0; attempt < 4096; ++attempt) {
    for (int t = 0; t < kTileBits; ++t) col[t] = t < 3 ? (1u << t) : 0xFFu;  // 0xFF = unassigned
    bool ok = true;
    for (const HostPhase& ph : ps->phases) {
      uint32_t v[3];
      for (int k = 0; k < 3; ++k) {
        int t = ph.thr_tbit[k];
        if (col[t] == 0xFFu) {
          // pick a value; first attempt is greedy, later attempts random
          uint32_t pick = 0;
          for (uint32_t cand = 1; cand < 8; ++cand) {
            uint32_t c = attempt == 0 ? cand : (uint32_t)(1 + ((rng >> 33) % 7));
            rng = rng * 6364136223846793005ull + 1442695040888963407ull;
            bool clash = false;
            for (int m = 0; m < k; ++m)
              if (c == v[m] || (k == 2 && c == (v[0] ^ v[1]))) clash = true;
            if (!clash) { pick = c; break; }
          }
          if (!pick) pick = 1;
          col[t] = pick;
        }
        v[k] = col[t];
      }
      if (!basis3(v[0], v[1], v[2])) { ok = false; break; }
    }
    if (ok) {
      for (int t = 0; t < kTileBits; ++t) ps->swz_col[t] = (t < 3) ? 0u : (col[t] == 0xFFu ? 0u : col[t]);
      return true;
    }
    rng ^= (uint64_t)attempt * 0xD1B54A32D192ED03ull;
  }
  return false;
}

uint32_t phys_of_bit(const HostPass& ps, int t) { return (1u << t) ^ ps.swz_col[t]; }

// How many leading lanes address consecutive low qubits 0, 1, 2, ... (a
// measure of how contiguous a warp's global access is in this phase).
int coalesce_score(const HostPass& ps, const HostPhase& ph) {
  int s = 0;
  for (int k = 0; k < 5; ++k) {
    if (ps.tile_q[ph.thr_tbit[k]] != k) break;
    ++s;
  }
  return s;
}

}  // namespace

std::string make_plan(int n, int L, int ckpt_block, Plan* out) {
  if (n < 1 || n > 30) return "n_qubits must be in [1, 30]";
  if (L < 1 || L > 100000) return "n_layers must be in [1, 100000]";
  if (ckpt_block < 0) return "ckpt_block must be >= 0";
  Plan p;
  p.n = n;
  p.L = L;
  p.ckpt_block = ckpt_block;

  // ---- qubit sets rotated together
  if (n <= kTileBits) {
    p.sets.push_back({});
    for (int q = 0; q < n; ++q) p.sets[0].push_back(q);
  } else {
    int s = (n + kMaxSet - 1) / kMaxSet;
    int base = n / s, extra = n % s, q = 0;
    for (int i = 0; i < s; ++i) {
      int sz = base + (i < extra ? 1 : 0);
      std::vector<int> set;
      for (int k = 0; k < sz; ++k) set.push_back(q++);
      p.sets.push_back(set);
    }
  }
  p.n_sets = (int)p.sets.size();
  const int S = p.n_sets;

  int n_blocks = (ckpt_block > 0) ? (L + ckpt_block - 1) / ckpt_block : 1;
  p.n_ckpt = (ckpt_block > 0) ? n_blocks - 1 : 0;

  // ---- task list: encode, then per layer the sets in boustrophedon order, then CZ
  std::vector<Task> tasks;
  tasks.push_back({T_GEN, -1, -1});
  for (int l = 0; l < L; ++l) {
    for (int i = 0; i < S; ++i) tasks.push_back({T_ROT, l, (l % 2 == 0) ? i : S - 1 - i});
    tasks.push_back({T_CZ, l, -1});
  }

  // ---- group tasks into passes
  struct Proto {
    int set = -1;
    std::vector<Task> t;
    int rots = 0;
    int ckpt = -1;
  };
  std::vector<Proto> protos(1);
  for (const Task& tk : tasks) {
    Proto* cur = &protos.back();
    if (tk.kind == T_ROT) {
      bool need_new = false;
      if (cur->set >= 0 && cur->set != tk.set) need_new = true;
      if (S == 1 && cur->rots >= kMaxLayersPerPass) need_new = true;
      if (need_new) {
        protos.emplace_back();
        cur = &protos.back();
      }
      cur->set = tk.set;
      cur->rots++;
    }
    cur->t.push_back(tk);
    if (tk.kind == T_CZ && ckpt_block > 0) {
      int l = tk.layer;
      if ((l + 1) % ckpt_block == 0 && l + 1 < L) {
        int m = (l + 1) / ckpt_block;  // slot m-1 holds the state after layer m*b-1
        if (S == 1) {
          // single-tile circuits: cut the pass here so the slot is a layer boundary
          cur->ckpt = m - 1;
          protos.emplace_back();
        } else {
          cur->ckpt = m - 1;  // written after the pass that holds this CZ
        }
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
    ps.gen = false;
    ps.last = (pi + 1 == protos.size());
    ps.ckpt = pr.ckpt;
    ps.nslots = 0;

    // tile bits
    std::vector<int> tq;
    if (S == 1) {
      for (int q = 0; q < n; ++q) tq.push_back(q);
      ps.unit_bits = kTileBits - n;
      for (int t = 0; t < kTileBits; ++t) ps.tile_q[t] = t < n ? t : -1 - (t - n);
    } else {
      const std::vector<int>& set = p.sets[pr.set >= 0 ? pr.set : 0];
      std::vector<bool> in(n, false);
      for (int q : set) in[q] = true;
      tq = set;
      for (int q = 0; q < n && (int)tq.size() < kTileBits; ++q)
        if (!in[q]) { tq.push_back(q); in[q] = true; }
      std::sort(tq.begin(), tq.end());
      for (int q = 0; q < n; ++q)
        if (!in[q]) ps.out_q.push_back(q);
      ps.unit_bits = 0;
      for (int t = 0; t < kTileBits; ++t) ps.tile_q[t] = tq[t];
    }
    std::vector<int> q2t(n, -1);
    for (int t = 0; t < kTileBits; ++t)
      if (ps.tile_q[t] >= 0) q2t[ps.tile_q[t]] = t;

    // register groups: the rotated qubits in chunks of five
    std::vector<int> rot_q = (S == 1) ? p.sets[0] : p.sets[pr.set >= 0 ? pr.set : 0];
    std::vector<std::vector<int>> groups;  // tile bits
    for (size_t i = 0; i < rot_q.size(); i += kRegBits) {
      std::vector<int> g;
      for (size_t k = i; k < rot_q.size() && k < i + kRegBits; ++k) g.push_back(q2t[rot_q[k]]);
      groups.push_back(g);
    }
    std::vector<bool> rotated_tbit(kTileBits, false);
    for (auto& g : groups)
      for (int t : g) rotated_tbit[t] = true;
    for (auto& g : groups) {
      HostPhase ph;
      std::vector<bool> used(kTileBits, false);
      for (int t : g) used[t] = true;
      std::vector<int> regs = g;
      // pad: highest passive qubit bits, then highest other qubit bits, then unit bits
      for (int pass_kind = 0; pass_kind < 3 && (int)regs.size() < kRegBits; ++pass_kind) {
        for (int t = kTileBits - 1; t >= 0 && (int)regs.size() < kRegBits; --t) {
          if (used[t]) continue;
          bool is_q = ps.tile_q[t] >= 0;
          bool ok = (pass_kind == 0 && is_q && !rotated_tbit[t]) || (pass_kind == 1 && is_q) ||
                    (pass_kind == 2 && !is_q);
          if (ok) { regs.push_back(t); used[t] = true; }
        }
      }
      for (int k = 0; k < kRegBits; ++k) ph.reg_tbit[k] = regs[k];
      int h = 0;
      for (int t = 0; t < kTileBits; ++t)
        if (!used[t]) ph.thr_tbit[h++] = t;
      ps.phases.push_back(ph);
    }
    const int G = (int)groups.size();
    // best group for global access
    int best = 0, best_score = -1;
    for (int g = 0; g < G; ++g) {
      int sc = coalesce_score(ps, ps.phases[g]);
      if (sc > best_score) { best_score = sc; best = g; }
    }
    std::vector<int> order;
    order.push_back(best);
    for (int g = 0; g < G; ++g)
      if (g != best) order.push_back(g);

    bool has_gen = false;
    for (const Task& tk : pr.t)
      if (tk.kind == T_GEN) has_gen = true;
    ps.gen = has_gen;
    int nrot = pr.rots;
    // direction of the first rotation: loading passes start in the best
    // layout; encoding passes choose the direction that ends in it
    bool forward_dir = true;
    if (has_gen) forward_dir = (nrot % 2 == 0);

    int cur = -1;
    bool gen_emitted = false;
    int rot_i = 0;
    auto emit_exch = [&](int to) {
      if (cur >= 0 && cur != to) ps.ops.push_back({OP_EXCH, cur, to, 0});
      cur = to;
    };
    for (const Task& tk : pr.t) {
      if (tk.kind == T_GEN) continue;  // emitted lazily once the layout is known
      if (tk.kind == T_ROT) {
        bool dir = (rot_i % 2 == 0) ? forward_dir : !forward_dir;
        ++rot_i;
        std::vector<int> ord = order;
        if (!dir) std::reverse(ord.begin(), ord.end());
        for (int g : ord) {
          if (cur < 0) {
            cur = g;
            if (has_gen && !gen_emitted) {
              ps.ops.push_back({OP_GEN, 0, 0, 0});
              gen_emitted = true;
            }
            ps.load_phase = g;
          }
          emit_exch(g);
          uint32_t mask = 0;
          const HostPhase& ph = ps.phases[g];
          for (int k = 0; k < kRegBits; ++k)
            for (int t : groups[g])
              if (ph.reg_tbit[k] == t) mask |= 1u << k;
          int slot0 = ps.nslots;
          for (int k = 0; k < kRegBits; ++k)
            if (mask & (1u << k)) {
              int q = ps.tile_q[ph.reg_tbit[k]];
              size_t idx = (size_t)tk.layer * n + q;
              p.slot_pass[idx] = (int)pi;
              p.slot_index[idx] = ps.nslots++;
            }
          ps.ops.push_back({OP_ROT, tk.layer, (int)mask, slot0});
        }
      } else if (tk.kind == T_CZ) {
        if (cur < 0) return "internal: CZ before any rotation in a pass";
        ps.ops.push_back({OP_CZ, tk.layer, 0, 0});
      }
    }
    if (cur < 0) return "internal: pass without rotations";
    if (coalesce_score(ps, ps.phases[cur]) < best_score) emit_exch(best);
    ps.store_phase = cur;
    if (!choose_swizzle(&ps)) return "internal: no bank-conflict-free swizzle found";
    p.max_slots = std::max(p.max_slots, ps.nslots);
    p.passes.push_back(ps);
  }
  for (size_t i = 0; i < p.slot_pass.size(); ++i)
    if (p.slot_pass[i] < 0) return "internal: a rotation was not scheduled";
  *out = p;
  return "";
}

void flatten_plan(const Plan& p, std::vector<DevPass>* passes, std::vector<DevPhase>* phases,
                  std::vector<DevOp>* ops) {
  passes->clear();
  phases->clear();
  ops->clear();
  for (const HostPass& ps : p.passes) {
    DevPass d{};
    d.op0 = (int)ops->size();
    d.nops = (int)ps.ops.size();
    d.phase0 = (int)phases->size();
    d.nphases = (int)ps.phases.size();
    d.load_phase = ps.load_phase;
    d.store_phase = ps.store_phase;
    d.gen = ps.gen ? 1 : 0;
    d.last = ps.last ? 1 : 0;
    d.ckpt = ps.ckpt;
    d.nslots = ps.nslots;
    d.n_out = (int)ps.out_q.size();
    d.unit_bits = ps.unit_bits;
    for (int i = 0; i < kMaxOut; ++i) d.out_q[i] = i < d.n_out ? ps.out_q[i] : -1;
    d.partial_off = 0;
    passes->push_back(d);
    for (const HostOp& o : ps.ops) ops->push_back({o.kind, o.a, o.b, o.c});
    for (const HostPhase& ph : ps.phases) {
      DevPhase dp{};
      dp.has_reg_unit = 0;
      uint32_t qbit[kRegBits];
      for (int k = 0; k < kRegBits; ++k) {
        int t = ph.reg_tbit[k];
        int q = ps.tile_q[t];
        dp.reg_q[k] = q >= 0 ? q : -1;
        dp.reg_u[k] = q >= 0 ? -1 : (-1 - q);
        if (q < 0) dp.has_reg_unit = 1;
        dp.reg_phys[k] = phys_of_bit(ps, t);
        qbit[k] = q >= 0 ? (1u << q) : 0u;
      }
      for (int k = 0; k < kThrBits; ++k) {
        int t = ph.thr_tbit[k];
        int q = ps.tile_q[t];
        dp.thr_q[k] = q >= 0 ? q : -1;
        dp.thr_u[k] = q >= 0 ? -1 : (-1 - q);
        dp.thr_phys[k] = phys_of_bit(ps, t);
      }
      dp.cz_reg = 0;
      dp.z0_reg = 0;
      for (int j = 0; j < kPos; ++j) {
        uint32_t b = 0;
        for (int k = 0; k < kRegBits; ++k)
          if (j & (1 << k)) b |= qbit[k];
        if (popcount32(b & (b >> 1)) & 1) dp.cz_reg |= 1u << j;
        if (b & 1u) dp.z0_reg |= 1u << j;
      }
      phases->push_back(dp);
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
    int cur = ps.load_phase;  // the layout the first data op runs in
    for (const HostOp& o : ps.ops) {
      int b = o.b;
      if (o.kind == OP_EXCH) cur = o.b;
      if (o.kind == OP_ROT) {
        uint32_t qm = 0;
        for (int k = 0; k < kRegBits; ++k)
          if (o.b & (1 << k)) {
            const int q = ps.tile_q[ps.phases[cur].reg_tbit[k]];
            if (q >= 0) qm |= 1u << q;
          }
        b = (int)qm;
      }
      v.push_back(o.kind);
      v.push_back(o.a);
      v.push_back(b);
      v.push_back(o.c);
    }
  }
  return v;
}

}  // namespace qml
