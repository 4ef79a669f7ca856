"""GPU parity: the CUDA path (through the C ABI) against the complex128 oracle.

Tolerances (fp32 compute): forward <Z0> abs error <= 1e-4; gradient abs error
<= 1e-4 + 1e-3 |g| for L <= 100, <= 1e-3 + 1e-3 |g| for deeper circuits, and
<= 2e-2 + 1e-3 |g| when checkpoints are stored in bf16.  State vectors are
compared element by element with abs error <= 2e-5 (unit-norm states; fp32
rounding over the gate sequence stays far below this at these depths).
"""
import numpy as np
import pytest

import oracle
from adjoint_gradients_b200.inputs import WORKLOADS, make_inputs, random_case

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def qml():
    from adjoint_gradients_b200 import qml as m

    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def grad_tol(L, storage):
    if storage == "bf16":
        return 2e-2
    return 1e-4 if L <= 100 else 1e-3


def run_gpu(n, L, x, theta, g, ckpt_block=0, storage="fp32", want_state=False):
    B = x.shape[0]
    ctx = qml().Context(n, L, B, ckpt_block=ckpt_block, storage=storage)
    xd, td, gd = dev(x), dev(theta), dev(g)
    psi, E = ctx.forward(td, xd)
    psi_final = psi.clone() if want_state else None
    lam = ctx.new_state(B)
    grad = ctx.backward(td, xd, psi, lam, gd)
    torch.cuda.synchronize()
    ctx.sync()
    return E.cpu().numpy().astype(np.float64), grad.cpu().numpy().astype(np.float64), psi_final


CASES = [
    # n, L, B, ckpt_block, storage
    (1, 3, 3, 0, "fp32"),
    (2, 5, 5, 2, "fp32"),
    (4, 2, 8, 0, "fp32"),
    (5, 7, 4, 3, "bf16"),
    (7, 4, 9, 0, "fp32"),
    (10, 3, 9, 1, "fp32"),  # one sample per batch unit in the one-launch forward (3 tiles, not 2)
    (11, 3, 6, 1, "fp32"),
    (12, 5, 7, 2, "fp32"),
    (12, 4, 5, 2, "bf16"),
    (13, 3, 5, 0, "fp32"),
    (14, 4, 3, 2, "fp32"),
    (16, 3, 2, 1, "bf16"),
    (17, 2, 3, 0, "fp32"),
    (21, 2, 2, 1, "fp32"),
    (23, 3, 1, 0, "fp32"),
]


@pytest.mark.parametrize("n,L,B,ck,st", CASES)
def test_forward_state_and_expectation(n, L, B, ck, st):
    x, theta, y = random_case(1000 + 17 * n + L, B, n, L)
    Eo, psio = oracle.forward(x, theta, want_state=True)
    g = oracle.loss_seed(Eo, y)
    E, grad, psi = run_gpu(n, L, x, theta, g, ck, st, want_state=True)
    np.testing.assert_allclose(E, Eo, atol=1e-4)
    got = psi.cpu().numpy().astype(np.float64)
    got = got[..., 0] + 1j * got[..., 1]
    assert np.max(np.abs(got - psio)) < 2e-5
    gref, _ = oracle.adjoint(x, theta, g)
    tol = grad_tol(L, st)
    assert np.all(np.abs(grad - gref) <= tol + 1e-3 * np.abs(gref)), np.max(np.abs(grad - gref))


def test_tiny_workload_parity_and_parameter_shift():
    w = WORKLOADS["tiny_4q_L2"]
    x, theta, y = make_inputs(w)
    Eo = oracle.forward(x, theta)
    g = oracle.loss_seed(Eo, y)
    E, grad, _ = run_gpu(w.n, w.L, x, theta, g)
    np.testing.assert_allclose(E, Eo, atol=1e-4)
    gref, _ = oracle.adjoint(x, theta, g)
    assert np.all(np.abs(grad - gref) <= 1e-4 + 1e-3 * np.abs(gref))
    # parameter shift through the GPU forward pass itself
    ctx = qml().Context(w.n, w.L, w.B)
    xd = dev(x)
    shift = np.zeros_like(theta)
    for idx in np.ndindex(theta.shape):
        tp, tm = theta.copy(), theta.copy()
        tp[idx] += np.pi / 2
        tm[idx] -= np.pi / 2
        Ep = ctx.forward(dev(tp), xd)[1].cpu().numpy().astype(np.float64)
        Em = ctx.forward(dev(tm), xd)[1].cpu().numpy().astype(np.float64)
        shift[idx] = np.dot(g, 0.5 * (Ep - Em))
    assert np.all(np.abs(grad - shift) <= 2e-4 + 1e-3 * np.abs(shift))


def test_12q_workload_parity():
    w = WORKLOADS["hea_12q_L10"]
    x, theta, y = make_inputs(w)
    Eo = oracle.forward(x, theta)
    g = oracle.loss_seed(Eo, y)
    E, grad, _ = run_gpu(w.n, w.L, x, theta, g)
    np.testing.assert_allclose(E, Eo, atol=1e-4)
    gref, _ = oracle.adjoint(x, theta, g)
    assert np.all(np.abs(grad - gref) <= 1e-4 + 1e-3 * np.abs(gref)), np.max(np.abs(grad - gref))


def test_encode_matches_oracle_product_state():
    n, B = 9, 5
    x, _, _ = random_case(3, B, n, 1)
    ctx = qml().Context(n, 1, B)
    psi = ctx.encode(dev(x))
    _, ref = oracle.forward(x, np.zeros((0, n, 3)), want_state=True)
    got = psi.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got[..., 0] + 1j * got[..., 1] - ref)) < 1e-6


def test_expect_z0_standalone():
    n, B = 15, 3
    x, theta, _ = random_case(5, B, n, 2)
    Eo, psio = oracle.forward(x, theta, want_state=True)
    ctx = qml().Context(n, 2, B)
    st = np.stack([psio.real, psio.imag], axis=-1)
    E = ctx.expect_z0(dev(st)).cpu().numpy()
    np.testing.assert_allclose(E, Eo, atol=1e-5)


def test_loss_seed():
    B = 37
    rng = np.random.default_rng(0)
    E = rng.uniform(-1, 1, B)
    y = rng.choice([-1.0, 1.0], B)
    ctx = qml().Context(3, 1, B)
    g, loss = ctx.loss_seed(dev(E), dev(y))
    np.testing.assert_allclose(g.cpu().numpy(), 2 * (E - y) / B, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(loss.cpu().numpy()[0], np.mean((E - y) ** 2), rtol=1e-6)


@pytest.mark.parametrize("storage", ["fp32", "bf16"])
def test_ckpt_save_restore_bits(storage):
    n, B = 10, 3
    ctx = qml().Context(n, 4, B, ckpt_block=2, storage=storage)
    rng = np.random.default_rng(1)
    st = rng.standard_normal((B, 1 << n, 2)).astype(np.float32)
    ctx.ckpt_save(0, dev(st))
    out = ctx.new_state(B)
    ctx.ckpt_restore(0, out)
    got = out.cpu().numpy()
    if storage == "fp32":
        np.testing.assert_array_equal(got, st)
    else:
        np.testing.assert_array_equal(got, oracle.bf16_widen(oracle.bf16_round(st)))


def test_ckpt_restore_mismatch_is_reported():
    ctx = qml().Context(6, 4, 4, ckpt_block=2)
    out = ctx.new_state(4)
    with pytest.raises(qml().QmlError) as e:
        ctx.ckpt_restore(0, out)
    assert e.value.code == 5


def test_deterministic_gradients():
    n, L, B = 14, 3, 3
    x, theta, y = random_case(8, B, n, L)
    g = np.array([0.3, -0.2, 0.9])
    _, g1, _ = run_gpu(n, L, x, theta, g, 1)
    _, g2, _ = run_gpu(n, L, x, theta, g, 1)
    np.testing.assert_array_equal(g1, g2)


def test_bad_arguments_rejected():
    m = qml()
    ctx = m.Context(5, 2, 4)
    x = dev(np.zeros((5, 5)))
    th = dev(np.zeros((2, 5, 3)))
    with pytest.raises(m.QmlError) as e:
        ctx.forward(th, x)  # B = 5 > max_batch = 4
    assert e.value.code == 1
