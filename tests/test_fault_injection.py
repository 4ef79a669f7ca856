"""Error paths, driven from the host (no GPU fault is provoked).

QML_FAULT (read when a context is created) injects a workspace failure, lost
checkpoint slots or NaN gate coefficients; a NaN angle in theta is a real
host-made fault.  Each must surface as its status code, not as a wrong result.
"""
import ctypes

import numpy as np
import pytest

from adjoint_gradients_b200 import qml
from adjoint_gradients_b200.inputs import random_case


def _create(n, L, B, ck=0):
    lib = qml.load_library()
    cfg = qml._Config(n, L, B, ck, 0)
    h = ctypes.c_void_p()
    assert lib.qml_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == qml.QML_OK
    return lib, h


def test_injected_workspace_failure(monkeypatch):
    monkeypatch.setenv("QML_FAULT", "alloc")
    lib, h = _create(8, 2, 2)
    assert lib.qml_set_workspace(h, ctypes.c_void_p(256), 1 << 20, None) == 3  # QML_ERR_WORKSPACE
    lib.qml_destroy(h)


def test_unknown_fault_is_ignored(monkeypatch):
    monkeypatch.setenv("QML_FAULT", "something-else")
    lib, h = _create(8, 2, 2)
    lib.qml_destroy(h)


torch = pytest.importorskip("torch")


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


@pytest.mark.gpu
def test_nan_angle_reports_numeric_error():
    n, L, B = 10, 3, 2
    x, theta, _ = random_case(8100, B, n, L)
    theta[1, 4, 0] = np.nan
    ctx = qml.Context(n, L, B)
    psi, E = ctx.forward(dev(theta), dev(x))
    with pytest.raises(qml.QmlError) as ei:
        ctx.sync()
    assert ei.value.code == 6  # QML_ERR_NUMERIC
    ctx.sync()  # the status word was cleared by the read
    x2, theta2, _ = random_case(8101, B, n, L)
    ctx.forward(dev(theta2), dev(x2))
    ctx.sync()  # the context stays usable


@pytest.mark.gpu
def test_injected_nan_coefficients(monkeypatch):
    monkeypatch.setenv("QML_FAULT", "nan_theta")
    n, L, B = 14, 2, 2
    x, theta, _ = random_case(8200, B, n, L)
    ctx = qml.Context(n, L, B)
    ctx.forward(dev(theta), dev(x))
    with pytest.raises(qml.QmlError) as ei:
        ctx.sync()
    assert ei.value.code == 6


@pytest.mark.gpu
def test_injected_nan_coefficients_cnot(monkeypatch):
    monkeypatch.setenv("QML_FAULT", "nan_theta")
    n, L, B = 9, 2, 3
    x, theta, _ = random_case(8210, B, n, L)
    ctx = qml.Context(n, L, B)
    ctx.set_entangler([(q, q + 1) for q in range(n - 1)], kind="cnot")
    ctx.forward(dev(theta), dev(x))
    with pytest.raises(qml.QmlError) as ei:
        ctx.sync()
    assert ei.value.code == 6


@pytest.mark.gpu
def test_injected_nan_angle_fp64(monkeypatch):
    monkeypatch.setenv("QML_FAULT", "nan_theta")
    n, L, B = 9, 2, 2
    x, theta, _ = random_case(8220, B, n, L)
    ctx = qml.Context(n, L, B, precision="fp64")
    d64 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).cuda()
    ctx.forward(d64(theta), d64(x))
    with pytest.raises(qml.QmlError) as ei:
        ctx.sync()
    assert ei.value.code == 6


@pytest.mark.gpu
def test_injected_lost_checkpoints(monkeypatch):
    monkeypatch.setenv("QML_FAULT", "ckpt_corrupt")
    n, L, B = 14, 4, 2
    x, theta, y = random_case(8300, B, n, L)
    ctx = qml.Context(n, L, B, ckpt_block=2)
    td, xd = dev(theta), dev(x)
    psi, E = ctx.forward(td, xd)
    g, _ = ctx.loss_seed(E, dev(y))
    with pytest.raises(qml.QmlError) as ei:
        ctx.backward(td, xd, psi, ctx.new_state(B), g)
    assert ei.value.code == 5  # QML_ERR_CKPT_MISMATCH
    ctx.sync()
