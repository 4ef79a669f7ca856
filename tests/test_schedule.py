"""CPU tests of the host pass scheduler and of the C-ABI surface (no GPU).

The schedule is replayed combinatorially: every (layer, qubit) rotation must
occur exactly once, each qubit's rotations in layer order, the CZ ladder of
layer l after every rotation of layer l and before any rotation of layer l+1,
and layout exchanges must chain (from = current layout).
"""
import ctypes
import os

import pytest

from adjoint_gradients_b200 import qml

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def parse(sched):
    P = sched[0]
    i = 1
    passes = []
    for _ in range(P):
        set_id, gen, last, ck, nops = sched[i:i + 5]
        i += 5
        ops = [tuple(sched[i + 4 * k:i + 4 * k + 4]) for k in range(nops)]
        i += 4 * nops
        passes.append(dict(set=set_id, gen=gen, last=last, ckpt=ck, ops=ops))
    assert i == len(sched)
    return passes


def replay(n, L, passes, ckpt_block):
    seen = {}
    order = 0
    cz_at = {}
    last_layer = [-1] * n
    for pi, ps in enumerate(passes):
        cur = None
        for kind, a, b, c in ps["ops"]:
            if kind == 4:
                assert pi == 0 and order == 0, "encoding must come first"
                cur = a
            elif kind == 1:
                assert cur is None or a == cur, "exchange must start from the current layout"
                cur = b
            elif kind == 2:
                for q in range(n):
                    if (b >> q) & 1:
                        assert (a, q) not in seen, f"rotation {(a, q)} scheduled twice"
                        assert last_layer[q] == a - 1, "rotations of a qubit out of layer order"
                        assert (a - 1) < 0 or (a - 1) in cz_at, "rotation before the previous CZ ladder"
                        last_layer[q] = a
                        seen[(a, q)] = order
                        order += 1
            elif kind == 3:
                assert all(last_layer[q] == a for q in range(n)), "CZ before all rotations of its layer"
                assert a not in cz_at
                cz_at[a] = order
                order += 1
    assert len(seen) == n * L
    assert sorted(cz_at) == list(range(L))
    assert passes[0]["gen"] == 1 and passes[-1]["last"] == 1
    assert sum(p["last"] for p in passes) == 1
    ck = [p["ckpt"] for p in passes if p["ckpt"] >= 0]
    nslots = (L + ckpt_block - 1) // ckpt_block - 1 if ckpt_block else 0
    assert ck == list(range(nslots))


@pytest.mark.parametrize("n,L,ck", [(1, 3, 0), (2, 5, 2), (3, 9, 4), (4, 2, 0), (5, 17, 3), (8, 12, 5),
                                    (11, 20, 0), (12, 10, 0), (12, 30, 7), (13, 4, 1), (16, 7, 2),
                                    (20, 100, 10), (20, 1000, 20), (21, 5, 0), (29, 20, 10), (30, 3, 1)])
def test_schedule_replays_the_circuit(n, L, ck):
    ctx = qml.Context(n, L, 4, ckpt_block=ck, workspace=False)
    passes = parse(ctx.debug_schedule())
    replay(n, L, passes, ck)
    assert ctx.num_ckpt_slots == ((L + ck - 1) // ck - 1 if ck else 0)


def test_pass_counts_match_the_design():
    # n <= 12: one pass per 2 layers; n = 20: L + 1 passes (two qubit sets);
    # n = 29: 2L + 1 passes (three sets, boustrophedon)
    assert len(parse(qml.Context(12, 10, 4, workspace=False).debug_schedule())) == 5
    assert len(parse(qml.Context(20, 100, 4, workspace=False).debug_schedule())) == 101
    assert len(parse(qml.Context(29, 20, 4, workspace=False).debug_schedule())) == 41


def test_library_exports_every_declared_symbol():
    lib = qml.load_library()
    header = open(os.path.join(ROOT, "include", "qml.h")).read()
    import re

    declared = set(re.findall(r"QML_API [^;(]*?\b(qml_\w+)\(", header))
    assert declared == set(qml.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_create_rejects_bad_configs():
    lib = qml.load_library()
    h = ctypes.c_void_p()
    for cfg in [(0, 3, 4, 0, 0), (31, 3, 4, 0, 0), (5, 0, 4, 0, 0), (5, 3, 0, 0, 0), (5, 3, 4, -1, 0),
                (5, 3, 4, 0, 7)]:
        c = qml._Config(*cfg)
        assert lib.qml_create(ctypes.byref(c), 0, ctypes.byref(h)) == 1
        assert not h.value
    assert lib.qml_create(None, 0, ctypes.byref(h)) == 1


def test_calls_without_workspace_fail_cleanly():
    ctx = qml.Context(6, 3, 4, workspace=False)
    lib = ctx.lib
    assert lib.qml_forward_expect(ctx._h, 16, 16, 2, 16, 16, None) == 3  # QML_ERR_WORKSPACE
    assert lib.qml_forward_expect(ctx._h, 16, 16, 9, 16, 16, None) == 1  # B > max_batch
    assert lib.qml_status_str(5) == b"checkpoint slot mismatch"
    assert lib.qml_abi_version() == 1
    assert ctx.workspace_bytes() > 0 and ctx.workspace_bytes(host_step=True) > ctx.workspace_bytes()


def test_set_observable_validates_and_counts():
    ctx = qml.Context(3, 2, 4, workspace=False)
    assert ctx.observable_terms == 0
    ctx.set_observable([(1.0, "XIZ"), (-0.5, "YYI"), (0.25, "XZZ")])
    assert ctx.observable_terms == 3
    lib = ctx.lib
    c = (ctypes.c_double * 2)(1.0, 2.0)
    assert lib.qml_set_observable(ctx._h, 2, b"XIZQII", c) == 1       # bad letter
    assert lib.qml_set_observable(ctx._h, -1, None, None) == 1
    assert lib.qml_set_observable(ctx._h, 4097, b"I" * 3 * 4097, (ctypes.c_double * 4097)()) == 1
    nan = (ctypes.c_double * 1)(float("nan"))
    assert lib.qml_set_observable(ctx._h, 1, b"ZII", nan) == 1
    assert ctx.observable_terms == 3   # a rejected call keeps the previous observable
    ctx.set_observable(None)
    assert ctx.observable_terms == 0


def test_set_entangler_validates_and_counts():
    ctx = qml.Context(5, 2, 4, workspace=False)
    assert ctx.entangler_bonds == 4  # the chain
    ctx.set_entangler([(0, 2), (4, 1), (3, 0)])
    assert ctx.entangler_bonds == 3
    lib = ctx.lib
    for bad in [[(0, 0)], [(0, 5)], [(-1, 2)]]:
        flat = (ctypes.c_int * 2)(*bad[0])
        assert lib.qml_set_entangler(ctx._h, 1, flat) == 1
    assert lib.qml_set_entangler(ctx._h, -1, None) == 1
    assert ctx.entangler_bonds == 3
    ctx.set_entangler([])
    assert ctx.entangler_bonds == 0
    ctx.set_entangler(None)
    assert ctx.entangler_bonds == 4


def test_set_reupload_flags():
    ctx = qml.Context(6, 2, 4, workspace=False)
    assert not ctx.reupload
    ctx.set_reupload(True)
    assert ctx.reupload
    ctx.set_reupload(False)
    assert not ctx.reupload
    small = qml.Context(3, 2, 4, workspace=False)
    assert small.lib.qml_set_reupload(small._h, 1) == 2  # QML_ERR_UNSUPPORTED below 5 qubits
