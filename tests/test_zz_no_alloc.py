"""GPU test of qml_expect_z0_static, the allocation-free Z0 expectation.

It is called directly through the C ABI (no context, no workspace) and must
agree with the workspace-based qml_expect_z0 on the same states, for two calls
in a row with different shapes, so that the second call runs over scratch the
first one left behind.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def random_states(seed, B, n):
    g = torch.Generator(device="cpu").manual_seed(seed)
    st = torch.randn((B, 1 << n, 2), generator=g, dtype=torch.float32)
    st /= torch.sqrt((st ** 2).sum(dim=(1, 2), keepdim=True))
    return st.cuda()


def test_static_scratch_expectation_matches_workspace_version():
    from adjoint_gradients_b200 import qml

    lib = qml.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    for seed, (B, n) in enumerate([(6, 18), (3, 21)]):
        psi = random_states(100 + seed, B, n)
        ctx = qml.Context(n, 1, B)
        ref = ctx.expect_z0(psi)
        out = torch.full((B,), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.qml_expect_z0_static(ctypes.c_void_p(psi.data_ptr()), n, B, ctypes.c_void_p(out.data_ptr()),
                                      ctypes.c_void_p(stream))
        assert rc == 0, qml.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        np.testing.assert_allclose(out.cpu().numpy(), ref.cpu().numpy(), atol=1e-5, rtol=0)
        assert np.all(np.abs(out.cpu().numpy()) <= 1.0 + 1e-5)


def test_static_scratch_rejects_oversized_calls():
    from adjoint_gradients_b200 import qml

    lib = qml.load_library()
    x = torch.zeros(16, device="cuda")
    # 2^29 amplitudes per state -> 8192 partials per sample: 5 samples exceed 32768
    rc = lib.qml_expect_z0_static(ctypes.c_void_p(x.data_ptr()), 29, 5, ctypes.c_void_p(x.data_ptr()), None)
    assert rc == 3  # QML_ERR_WORKSPACE, nothing launched
    rc = lib.qml_expect_z0_static(None, 10, 1, ctypes.c_void_p(x.data_ptr()), None)
    assert rc == 1
