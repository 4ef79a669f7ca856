"""Host-side checks of the fp64 compute mode's C ABI (no GPU needed: context
creation, precision, argument and precision checks, workspace sizing)."""
import ctypes

import pytest

from adjoint_gradients_b200 import qml


def _ctx(n, L, B, ck=0, storage="fp64", f64=True):
    lib = qml.load_library()
    cfg = qml._Config(n, L, B, ck, qml.STORAGE[storage])
    h = ctypes.c_void_p()
    create = lib.qml_create_f64 if f64 else lib.qml_create
    return lib, create(ctypes.byref(cfg), 0, ctypes.byref(h)), h


def test_create_f64_and_precision():
    lib, st, h = _ctx(10, 4, 3, 2)
    assert st == qml.QML_OK
    assert lib.qml_precision(h) == 64
    lib.qml_destroy(h)
    lib, st, h = _ctx(10, 4, 3, 2, storage="fp32", f64=False)
    assert st == qml.QML_OK and lib.qml_precision(h) == 32
    lib.qml_destroy(h)
    assert lib.qml_precision(None) == -1


def test_fp64_slots_only_for_fp64_contexts():
    lib, st, h = _ctx(10, 4, 3, 2, storage="fp64", f64=False)
    assert st == 1 and not h.value  # QML_ERR_INVALID_ARG
    for storage in ("fp32", "bf16", "fp64"):
        lib, st, h = _ctx(10, 4, 3, 2, storage=storage)
        assert st == qml.QML_OK
        lib.qml_destroy(h)


def test_calls_of_the_other_precision_are_unsupported():
    lib, st, h = _ctx(8, 3, 2, 1)
    assert st == qml.QML_OK
    vp = ctypes.c_void_p(16)  # never dereferenced: the precision check comes first
    assert lib.qml_forward_expect(h, vp, vp, 2, vp, vp, None) == 2
    assert lib.qml_backward_adjoint(h, vp, vp, 2, vp, vp, vp, vp, None) == 2
    assert lib.qml_loss_seed(h, vp, vp, 2, vp, vp, None) == 2
    assert lib.qml_expect_z0(h, vp, 2, vp, None) == 2
    assert lib.qml_step_host(h, vp, vp, vp, 2, vp, vp, vp, None) == 2
    lib.qml_destroy(h)
    lib, st, h = _ctx(8, 3, 2, 1, storage="fp32", f64=False)
    assert lib.qml_forward_expect_f64(h, vp, vp, 2, vp, vp, None) == 2
    assert lib.qml_backward_adjoint_f64(h, vp, vp, 2, vp, vp, vp, vp, None) == 2
    assert lib.qml_loss_seed_f64(h, vp, vp, 2, vp, vp, None) == 2
    assert lib.qml_step_host_f64(h, vp, vp, vp, 2, vp, vp, vp, None) == 2
    lib.qml_destroy(h)


def test_reupload_allowed_below_five_qubits_in_fp64():
    lib, st, h = _ctx(3, 2, 2)
    assert lib.qml_set_reupload(h, 1) == qml.QML_OK
    lib.qml_destroy(h)
    lib, st, h = _ctx(3, 2, 2, storage="fp32", f64=False)
    assert lib.qml_set_reupload(h, 1) == 2
    lib.qml_destroy(h)


@pytest.mark.parametrize("n,L,B,ck", [(12, 10, 4, 2), (20, 6, 2, 3)])
def test_workspace_holds_fp64_slots(n, L, B, ck):
    sizes = {}
    for storage in ("fp32", "fp64", "bf16"):
        lib, st, h = _ctx(n, L, B, ck, storage=storage)
        slots = lib.qml_num_ckpt_slots(h)
        sizes[storage] = lib.qml_workspace_bytes(h, B)
        lib.qml_destroy(h)
    assert slots > 0
    amps = slots * B * (1 << n)
    # slot bytes per amplitude: 16 (fp64), 8 (fp32), 4 (bf16); the rest of the layout is shared
    assert sizes["fp64"] - sizes["fp32"] >= 8 * amps - 512
    assert sizes["fp64"] - sizes["fp32"] <= 8 * amps + 512
    assert sizes["fp32"] - sizes["bf16"] >= 4 * amps - 512
