"""Host-side checks of the CNOT entangler's C ABI (no GPU needed)."""
import ctypes

from adjoint_gradients_b200 import qml


def _ctx(n, L, B, ck=0, f64=False):
    lib = qml.load_library()
    cfg = qml._Config(n, L, B, ck, 0)
    h = ctypes.c_void_p()
    create = lib.qml_create_f64 if f64 else lib.qml_create
    assert create(ctypes.byref(cfg), 0, ctypes.byref(h)) == qml.QML_OK
    return lib, h


def _pairs(p):
    flat = [v for e in p for v in e]
    return (ctypes.c_int * max(1, len(flat)))(*flat)


def test_cnot_setter_validates_and_switches_kind():
    lib, h = _ctx(10, 3, 4)
    assert lib.qml_entangler_kind(h) == 0
    assert lib.qml_set_entangler_cnot(h, 0, _pairs([])) == 1
    assert lib.qml_set_entangler_cnot(h, 1, _pairs([(3, 3)])) == 1
    assert lib.qml_set_entangler_cnot(h, 1, _pairs([(0, 10)])) == 1
    assert lib.qml_entangler_kind(h) == 0
    ladder = [(q, q + 1) for q in range(9)]
    assert lib.qml_set_entangler_cnot(h, len(ladder), _pairs(ladder)) == qml.QML_OK
    assert lib.qml_entangler_kind(h) == 1 and lib.qml_entangler_bonds(h) == 9
    assert lib.qml_set_entangler(h, 0, None) == qml.QML_OK
    assert lib.qml_entangler_kind(h) == 0 and lib.qml_entangler_bonds(h) == 0
    lib.qml_destroy(h)


def test_cnot_in_both_precisions_and_three_qubit_sets():
    lib, h = _ctx(8, 2, 2, f64=True)
    assert lib.qml_set_entangler_cnot(h, 1, _pairs([(0, 1)])) == qml.QML_OK
    assert lib.qml_entangler_kind(h) == 1
    lib.qml_destroy(h)
    lib, h = _ctx(23, 1, 1)  # three qubit sets: the map is taken to the working-state addresses
    assert lib.qml_set_entangler_cnot(h, 2, _pairs([(0, 22), (12, 3)])) == qml.QML_OK
    lib.qml_destroy(h)


def test_cnot_workspace_holds_a_second_state():
    n, B = 14, 6
    lib, h = _ctx(n, 4, B, 2)
    before = lib.qml_workspace_bytes(h, B)
    ladder = [(q, q + 1) for q in range(n - 1)]
    assert lib.qml_set_entangler_cnot(h, len(ladder), _pairs(ladder)) == qml.QML_OK
    after = lib.qml_workspace_bytes(h, B)
    assert after - before >= 8 * B * (1 << n) + 8 * (1 << n)
    lib.qml_destroy(h)


def _map(lib, h):
    need = lib.qml_debug_entangler_map(h, None, 0)
    buf = (ctypes.c_int * need)()
    lib.qml_debug_entangler_map(h, buf, need)
    v = list(buf)
    n = v[0]
    return n, v[1:1 + n], v[1 + n:1 + 2 * n], v[1 + 2 * n:1 + 3 * n], v[1 + 3 * n:1 + 4 * n]


def _apply(cols, b):
    out = 0
    for k, c in enumerate(cols):
        if (b >> k) & 1:
            out ^= c
    return out


def _simulate(pairs, b):
    """A basis index through the CNOT list, one gate at a time."""
    for c, t in pairs:
        if (b >> c) & 1:
            b ^= 1 << t
    return b


def test_ladder_map_is_the_prefix_xor():
    n = 9
    lib, h = _ctx(n, 2, 2)
    ladder = [(q, q + 1) for q in range(n - 1)]
    assert lib.qml_set_entangler_cnot(h, len(ladder), _pairs(ladder)) == qml.QML_OK
    _, M, Minv, _, _ = _map(lib, h)
    for k in range(n):
        assert M[k] == ((1 << n) - 1) & ~((1 << k) - 1)  # bit k reaches bits k..n-1
        assert Minv[k] == (1 << k) | ((1 << (k + 1)) if k + 1 < n else 0)
    lib.qml_destroy(h)


def test_map_matches_gate_by_gate_action_and_inverts():
    import numpy as np

    rng = np.random.default_rng(5)
    for n, L in [(6, 1), (14, 2), (23, 1)]:
        lib, h = _ctx(n, L, 1)
        allp = [(a, b) for a in range(n) for b in range(n) if a != b]
        pairs = [allp[i] for i in rng.choice(len(allp), size=n + 3, replace=False)]
        assert lib.qml_set_entangler_cnot(h, len(pairs), _pairs(pairs)) == qml.QML_OK
        _, M, Minv, Ma, Mainv = _map(lib, h)
        for b in rng.integers(0, 1 << n, size=64):
            b = int(b)
            assert _apply(M, b) == _simulate(pairs, b)
            assert _apply(Minv, _apply(M, b)) == b
            assert _apply(Mainv, _apply(Ma, b)) == b
        lib.qml_destroy(h)


def test_address_map_is_the_qubit_map_with_renamed_bits():
    """Three qubit sets: the working state sits at permuted addresses (qubit q at
    address bit addr[q], read from the pass view), and the layer map on
    addresses must send addr(b) to addr(M b)."""
    import numpy as np

    n = 23
    lib, h = _ctx(n, 1, 1)
    need = lib.qml_debug_tile_view(h, 0, None, 0)
    buf = (ctypes.c_int * need)()
    lib.qml_debug_tile_view(h, 0, buf, need)
    v = list(buf)
    tile_q = [v[21 + 2 * b] for b in range(12)]
    n_out = v[21 + 24]
    out_q = v[21 + 25:21 + 25 + n_out]
    j = 21 + 25 + n_out
    tile_a, out_a = v[j:j + 12], v[j + 12:j + 12 + n_out]
    addr = {}
    for q, a in list(zip(tile_q, tile_a)) + list(zip(out_q, out_a)):
        if q >= 0:
            addr[q] = a
    assert sorted(addr) == list(range(n)) and sorted(addr.values()) == list(range(n))
    assert any(addr[q] != q for q in range(n))  # the permuted layout is in force

    def to_addr(b):
        return sum(1 << addr[q] for q in range(n) if (b >> q) & 1)

    ladder = [(q, q + 1) for q in range(n - 1)] + [(n - 1, 0)]
    assert lib.qml_set_entangler_cnot(h, len(ladder), _pairs(ladder)) == qml.QML_OK
    _, M, _, Ma, Mainv = _map(lib, h)
    rng = np.random.default_rng(9)
    for b in rng.integers(0, 1 << n, size=128):
        b = int(b)
        assert _apply(Ma, to_addr(b)) == to_addr(_apply(M, b))
        assert _apply(Mainv, _apply(Ma, to_addr(b))) == to_addr(b)
    lib.qml_destroy(h)


def _fused(lib, h):
    need = lib.qml_debug_entangler_map(h, None, 0)
    buf = (ctypes.c_int * need)()
    lib.qml_debug_entangler_map(h, buf, need)
    v = list(buf)
    n = v[0]
    j = 1 + 4 * n
    return v[j], v[j + 1:j + 1 + n], v[j + 1 + n:j + 1 + 2 * n]


def _sets(n):
    """The two qubit sets of a 13..20-qubit circuit: consecutive runs, the first one longer when n is odd."""
    a = (n + 1) // 2
    return list(range(a)), list(range(a, n))


def test_fused_factors_recompose_the_layer_and_touch_one_set_each():
    """M = M2 M1 with M1 changing only the first set's bits and M2 only the second's, checked on
    basis states pushed through the list gate by gate (an independent simulation of the list)."""
    import numpy as np

    rng = np.random.default_rng(11)
    for n in (13, 16, 20):
        A, Bq = _sets(n)
        mA = sum(1 << q for q in A)
        allp = [(a, b) for a in range(n) for b in range(n) if a != b]
        lists = [[(q, q + 1) for q in range(n - 1)], [(q, (q + 1) % n) for q in range(n)]]
        lists += [[allp[i] for i in rng.choice(len(allp), size=n + 2, replace=False)] for _ in range(4)]
        n_fused = 0
        for pairs in lists:
            lib, h = _ctx(n, 3, 2, 1)
            assert lib.qml_set_entangler_cnot(h, len(pairs), _pairs(pairs)) == qml.QML_OK
            fused, M1, M2 = _fused(lib, h)
            if fused:
                n_fused += 1
                for b in [int(v) for v in rng.integers(0, 1 << n, size=48)] + [1 << q for q in range(n)]:
                    y1 = _apply(M1, b)
                    assert (y1 ^ b) & ~mA == 0  # M1 leaves the second set alone
                    y2 = _apply(M2, y1)
                    assert (y2 ^ y1) & mA == 0  # M2 leaves the first set alone
                    assert y2 == _simulate(pairs, b)
            lib.qml_destroy(h)
        assert n_fused >= 2  # the ladder and the ring always factor


def test_fused_schedule_has_two_passes_per_layer():
    n, L = 16, 5
    lib, h = _ctx(n, L, 2, 2)
    ladder = [(q, q + 1) for q in range(n - 1)]
    assert lib.qml_set_entangler_cnot(h, len(ladder), _pairs(ladder)) == qml.QML_OK
    need = lib.qml_debug_schedule(h, None, 0)
    buf = (ctypes.c_int * need)()
    lib.qml_debug_schedule(h, buf, need)
    v = list(buf)
    assert v[0] == 2 * L + 1  # [M2 of the layer before, second set], [first set, M1]; then the last M2
    # every pass holds at most one permutation op (kind 7)
    i, perms = 1, []
    for _ in range(v[0]):
        nops = v[i + 4]
        kinds = [v[i + 5 + 4 * k] for k in range(nops)]
        perms.append(kinds.count(7))
        i += 5 + 4 * nops
    assert perms[0] == 0 and all(p == 1 for p in perms[1:])
    lib.qml_destroy(h)


def test_unfactorable_maps_and_other_sizes_stay_on_the_gather_path():
    """Maps whose first-set block is singular, and circuits of one or three qubit sets."""
    # SWAP(0, 9) from three CNOTs at n = 16 (sets 0-7 and 8-15): the first set's block of the map is
    # singular (qubit 0's new value comes from the second set only)
    lib, h = _ctx(16, 2, 2)
    swap = [(0, 9), (9, 0), (0, 9)]
    assert lib.qml_set_entangler_cnot(h, 3, _pairs(swap)) == qml.QML_OK
    assert _fused(lib, h)[0] == 0
    lib.qml_destroy(h)
    for n, f64, fused in [(12, False, 0), (21, False, 0), (21, True, 0), (16, True, 1)]:
        lib, h = _ctx(n, 2, 2, f64=f64)
        ladder = [(q, q + 1) for q in range(n - 1)]
        assert lib.qml_set_entangler_cnot(h, len(ladder), _pairs(ladder)) == qml.QML_OK
        assert _fused(lib, h)[0] == fused  # two qubit sets fuse in both precisions
        lib.qml_destroy(h)
