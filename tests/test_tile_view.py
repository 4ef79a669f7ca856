"""CPU check of the tensor-copy view of each pass (no GPU).

For circuits above 12 qubits a pass loads each tile with bulk tensor copies:
the working state [B][2^n] (qubits stored at permuted address bits) is viewed
as a rank-5 tensor whose dimensions are runs of address bits and the sample
index.  For every such pass this test recomputes, from the view the library
reports, the element each copied box position comes from (the coordinate
rule the kernel uses, restated here) and checks that
  * the box is exactly the tile: position p of the tile (tile bits -> address
    bits, out-of-tile bits from the tile index) lands at box offset sum_b p_b *
    sstride[b], and that offset map is a bijection onto [0, 4096);
  * the address bits are a permutation of the qubits, and every set's tile
    covers address bits 0 and 1 (runs of >= 32 bytes);
  * the innermost dimension starts at qubit 0 and spans >= 16 bytes, and every
    other dimension's stride is a multiple of 16 bytes (tensor-copy rules).
"""
import numpy as np
import pytest

from adjoint_gradients_b200 import qml

TD_PAD, TD_IN, TD_OUT, TD_SAMPLE, TD_OUT_SAMPLE = range(5)


def box_elements(view, n, B, sample, o):
    """Global element index [sample][2^n] of every box position (box order)."""
    dims = view["dims"]
    N = 1 << n
    ranges, starts, strides = [], [], []
    for d in dims:
        k = d["kind"]
        ob = (o >> d["shift"]) & ((1 << d["bits"]) - 1)
        if k == TD_IN:
            ranges.append(1 << d["bits"]); starts.append(0); strides.append(1 << d["qlo"])
        elif k == TD_OUT:
            ranges.append(1); starts.append(ob); strides.append(1 << d["qlo"])
        elif k == TD_SAMPLE:
            ranges.append(1); starts.append(sample); strides.append(N)
        elif k == TD_OUT_SAMPLE:
            ranges.append(1); starts.append(ob | (sample << d["bits"])); strides.append(1 << d["qlo"])
        else:
            ranges.append(1); starts.append(0); strides.append(0)
    idx = np.zeros(1, dtype=np.int64)
    for r, s0, st in zip(ranges, starts, strides):  # dimension 0 is innermost
        idx = (idx[None, :] + ((s0 + np.arange(r)) * st)[:, None]).reshape(-1)
    return idx


@pytest.mark.parametrize("n,L", [(13, 3), (16, 3), (17, 4), (20, 4), (21, 3), (25, 3), (29, 4), (30, 3)])
def test_tensor_copy_view_is_the_tile(n, L):
    ctx = qml.Context(n, L, 4, workspace=False)
    n_pass = ctx.debug_schedule()[0]
    B, N = 5, 1 << n
    rng = np.random.default_rng(n * 100 + L)
    checked = 0
    for p in range(n_pass):
        v = ctx.debug_tile_view(p)
        assert v["tma"] == 1, f"pass {p} of n={n} has no tensor-copy view"
        tq, ss, out_q = v["tile_q"], v["sstride"], v["out_q"]
        ta, oa = v["tile_addr"], v["out_addr"]
        assert all(q >= 0 for q in tq) and sorted(tq + out_q) == list(range(n))
        assert sorted(ta + oa) == list(range(n)) and 0 in ta and 1 in ta
        assert oa == sorted(oa), "out-of-tile qubits must be listed in address order"
        d0 = v["dims"][0]
        assert d0["kind"] == TD_IN and d0["qlo"] == 0 and (8 << d0["bits"]) >= 16
        for d in v["dims"][1:]:
            if d["kind"] in (TD_IN, TD_OUT, TD_OUT_SAMPLE):
                assert (8 << d["qlo"]) % 16 == 0
        pos = np.arange(4096)
        off = np.zeros(4096, dtype=np.int64)
        amp = np.zeros(4096, dtype=np.int64)
        for b in range(12):
            bit = (pos >> b) & 1
            off += bit * ss[b]
            amp += bit << ta[b]
        assert sorted(off.tolist()) == list(range(4096)), "offsets are not a bijection"
        n_out = len(out_q)
        for t in rng.integers(0, (B << n_out), size=6):
            o, u = int(t) & ((1 << n_out) - 1), int(t) >> n_out
            base = sum(((o >> k) & 1) << a for k, a in enumerate(oa))
            sample = min(u, B - 1)
            got = box_elements(v, n, B, sample, o)
            want = np.empty(4096, dtype=np.int64)
            want[off] = sample * N + base + amp
            np.testing.assert_array_equal(got, want)
            checked += 1
    assert checked > 0


def test_small_circuits_load_with_threads():
    for n in (4, 9, 12):
        ctx = qml.Context(n, 3, 4, workspace=False)
        for p in range(ctx.debug_schedule()[0]):
            assert ctx.debug_tile_view(p)["tma"] == 0
