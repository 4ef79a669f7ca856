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
