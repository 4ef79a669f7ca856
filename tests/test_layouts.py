"""CPU checks of the kernels' register layouts and shared-memory maps (no GPU).

The tables come from the library itself (qml_debug_layouts, qml_debug_tile_view).
  * every layout is a bijection of thread bits and register bits onto the 12
    tile bits;
  * the exchange slot map (sum of per-bit weights) is injective and fits the
    shared buffer;
  * layout exchanges are free of bank conflicts: the eight lanes of each
    quarter warp (one 128-byte wavefront of 16-byte accesses) hit eight
    different 16-byte bank groups;
  * the 8-byte exchanges of tensor-copy passes (re pairs, then im pairs,
    through a buffer of their own) are injective, fit their buffer and are
    free of bank conflicts: the 16 lanes of each half warp hit 16 different
    8-byte bank pairs, for every layout and register;
  * reading a tile that arrived by tensor copy is free of bank conflicts: in
    the memory layout, the 16 lanes of each half warp (8-byte accesses) hit 16
    different 8-byte bank pairs.
"""
import pytest

from adjoint_gradients_b200 import qml


def test_layouts_are_bijections_and_slots_fit():
    d = qml.debug_layouts()
    w = d["weights"]
    for (P, V), (thr, reg) in d["layouts"].items():
        assert sorted(thr + reg) == list(range(12)), (P, V)
    slots = {sum(w[b] for b in range(12) if (t >> b) & 1) for t in range(4096)}
    assert len(slots) == 4096
    assert max(slots) < d["slots"]


def test_exchanges_have_no_bank_conflicts():
    d = qml.debug_layouts()
    w = d["weights"]
    for (P, V), (thr, _) in d["layouts"].items():
        for q in range(4):
            groups = set()
            for lane in range(8 * q, 8 * q + 8):
                s = sum(w[thr[m]] for m in range(5) if (lane >> m) & 1)
                groups.add(s % 8)
            assert len(groups) == 8, (P, V, q)


def test_8_byte_exchanges_fit_and_have_no_bank_conflicts():
    d = qml.debug_layouts()
    w = d["weights8"]
    slots = {sum(w[b] for b in range(12) if (t >> b) & 1) for t in range(4096)}
    assert len(slots) == 4096
    assert max(slots) < d["slots8"]
    for (P, V), (thr, reg) in d["layouts"].items():
        for j in range(32):
            r = sum(w[reg[k]] for k in range(5) if (j >> k) & 1)
            for h in range(2):
                pairs = set()
                for lane in range(16 * h, 16 * h + 16):
                    pairs.add((r + sum(w[thr[m]] for m in range(5) if (lane >> m) & 1)) % 16)
                assert len(pairs) == 16, (P, V, j, h)


@pytest.mark.parametrize("n", [13, 16, 17, 20, 21, 25, 26, 29, 30])
def test_copied_tile_reads_have_no_bank_conflicts(n):
    lay = qml.debug_layouts()["layouts"]
    ctx = qml.Context(n, 3, 4, workspace=False)
    for p in range(ctx.debug_schedule()[0]):
        v = ctx.debug_tile_view(p)
        assert v["tma"] == 1
        thr = lay[(1, v["variant"])][0]
        for h in range(2):
            banks = set()
            for lane in range(16 * h, 16 * h + 16):
                off = sum(v["sstride"][thr[m]] for m in range(5) if (lane >> m) & 1)
                banks.add(off % 16)
            assert len(banks) == 16, (n, p, h)
