"""GPU parity for data re-uploading (the encoding Ry(x_q) again at the start of
every layer) against the oracle.  Same tolerances as the default circuit."""
import numpy as np
import pytest

import oracle
from adjoint_gradients_b200.inputs import random_case

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def qml():
    from adjoint_gradients_b200 import qml as m

    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


@pytest.mark.parametrize("n,L,B,ck,st", [(5, 3, 5, 0, "fp32"), (7, 4, 3, 2, "fp32"), (11, 3, 4, 0, "fp32"),
                                         (12, 4, 6, 3, "bf16"), (13, 3, 3, 1, "fp32"), (17, 2, 3, 0, "fp32"),
                                         (20, 3, 2, 2, "fp32"), (23, 2, 1, 0, "fp32")])
def test_reupload_parity(n, L, B, ck, st):
    x, theta, y = random_case(1200 + n, B, n, L)
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st)
    ctx.set_reupload(True)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    E = E.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(E, oracle.forward(x, theta, reupload=True), atol=1e-4)
    g = oracle.loss_seed(E, y)
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g)).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    ctx.sync()
    gref, _ = oracle.adjoint(x, theta, g, reupload=True)
    tol = 2e-2 if st == "bf16" else 1e-4
    err = np.abs(grad - gref)
    assert np.all(err <= tol + 1e-3 * np.abs(gref)), float(err.max())


def test_reupload_with_ring_and_pauli_sum():
    n, L, B = 14, 3, 3
    x, theta, y = random_case(1300, B, n, L)
    bonds = [(q, (q + 1) % n) for q in range(n)]
    obs = [(0.8, "X" + "I" * (n - 1)), (-0.4, "ZZ" + "I" * (n - 2))]
    ctx = qml().Context(n, L, B, ckpt_block=1)
    ctx.set_reupload(True)
    ctx.set_entangler(bonds)
    ctx.set_observable(obs)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    E = E.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(E, oracle.forward(x, theta, observable=obs, bonds=bonds, reupload=True), atol=2e-4)
    g = oracle.loss_seed(E, y)
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g)).cpu().numpy().astype(np.float64)
    ctx.sync()
    gref, _ = oracle.adjoint(x, theta, g, observable=obs, bonds=bonds, reupload=True)
    assert np.all(np.abs(grad - gref) <= 2e-4 + 1e-3 * np.abs(gref)), float(np.abs(grad - gref).max())
