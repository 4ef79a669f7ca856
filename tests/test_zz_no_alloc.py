"""GPU test of qml_expect_z0_static, the allocation-free Z0 expectation.

Callers that may not allocate device memory (a plugin inside a framework that
owns all device memory, a loop where a possibly synchronising cudaMalloc is
forbidden) use this entry point: it needs no context and no workspace, its
scratch is an array compiled into the library.  It is called directly through
the C ABI on states the CPU oracle produced, and must agree with the oracle's
<Z0> and with the workspace-based qml_expect_z0 within the tolerance of the
other expectation tests (1e-5 on unit-norm states), for calls in a row with
different shapes, so that later calls run over scratch an earlier call left
behind.  This file is collected last on purpose; it passes alone in a fresh
process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest

import oracle
from adjoint_gradients_b200.inputs import random_case

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def static_expect(lib, psi, n, B):
    out = torch.full((B,), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.qml_expect_z0_static(ctypes.c_void_p(psi.data_ptr()), n, B, ctypes.c_void_p(out.data_ptr()),
                                  ctypes.c_void_p(stream))
    torch.cuda.synchronize()
    return rc, out.cpu().numpy().astype(np.float64)


def test_static_scratch_expectation_matches_oracle_and_workspace_version():
    from adjoint_gradients_b200 import qml

    lib = qml.load_library()
    # (B, n): 20 partials, then 6 (over the first call's leftovers), then 8
    for seed, (B, n) in enumerate([(5, 18), (3, 17), (2, 20)]):
        x, theta, _ = random_case(9000 + seed, B, n, 2)
        Eo, psio = oracle.forward(x, theta, want_state=True)
        psi = torch.from_numpy(np.stack([psio.real, psio.imag], axis=-1).astype(np.float32)).cuda()
        rc, E = static_expect(lib, psi, n, B)
        assert rc == 0, qml.STATUS_NAMES.get(rc, rc)
        np.testing.assert_allclose(E, Eo, atol=1e-5, rtol=0)
        ctx = qml.Context(n, 2, B)
        ref = ctx.expect_z0(psi).cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(E, ref, atol=1e-5, rtol=0)


def test_static_scratch_passes_non_finite_values_through():
    from adjoint_gradients_b200 import qml

    lib = qml.load_library()
    n, B = 12, 2
    x, theta, _ = random_case(9100, B, n, 1)
    Eo, psio = oracle.forward(x, theta, want_state=True)
    st = np.stack([psio.real, psio.imag], axis=-1).astype(np.float32)
    st[1, 7, 0] = np.nan
    rc, E = static_expect(lib, torch.from_numpy(st).cuda(), n, B)
    assert rc == 0  # no status word: the NaN reaches the output, nothing is latched
    np.testing.assert_allclose(E[0], Eo[0], atol=1e-5)
    assert np.isnan(E[1])


def test_static_scratch_rejects_oversized_calls():
    from adjoint_gradients_b200 import qml

    lib = qml.load_library()
    x = torch.zeros(16, device="cuda")
    # 2^29 amplitudes per state -> 8192 partials per sample: 5 samples exceed 32768
    rc = lib.qml_expect_z0_static(ctypes.c_void_p(x.data_ptr()), 29, 5, ctypes.c_void_p(x.data_ptr()), None)
    assert rc == 3  # QML_ERR_WORKSPACE, nothing launched
    rc = lib.qml_expect_z0_static(None, 10, 1, ctypes.c_void_p(x.data_ptr()), None)
    assert rc == 1
