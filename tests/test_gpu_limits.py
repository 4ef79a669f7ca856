"""GPU checks at the size limits and on degenerate circuits, against closed
forms that hold for any number of qubits (no oracle state is needed, so they
run at n = 30, the largest supported register: 8 GiB per state).

One layer (derived with Bloch vectors; the CZ ladder after the last layer
commutes with Z0, and the other qubits never reach qubit 0 before it):
    E = cos x0 cos a cos b - sin x0 sin b,  a = theta[0][0][0], b = theta[0][0][1]
    dE/da = -sin a cos b cos x0,  dE/db = -cos a sin b cos x0 - cos b sin x0,
    every other derivative (Rz of qubit 0, all other qubits) = 0.
theta = 0 (any depth): E = cos x0; the only non-zero derivatives are those of
the Ry angles on qubit 0: layer l's Ry meets qubit 0's Bloch x component
sin x0, dephased by <Z1> = cos x1 once for every CZ(0, 1) before it (two CZ
cancel), so dE/dtheta[l][0][1] = -sin x0 cos(x1)^(l mod 2).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def qml():
    from adjoint_gradients_b200 import qml as m

    return m


def run(n, L, x, theta, ck=0, st="fp32"):
    B = x.shape[0]
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st)
    xd = torch.tensor(x, dtype=torch.float32, device="cuda")
    td = torch.tensor(theta, dtype=torch.float32, device="cuda")
    psi, E = ctx.forward(td, xd)
    g = torch.ones(B, dtype=torch.float32, device="cuda")
    lam = ctx.new_state(B)
    grad = ctx.backward(td, xd, psi, lam, g)
    torch.cuda.synchronize()
    ctx.sync()
    out = E.cpu().numpy().astype(np.float64), grad.cpu().numpy().astype(np.float64)
    del psi, lam, ctx
    torch.cuda.empty_cache()
    return out


def one_layer_reference(x, theta):
    a, b = theta[0, 0, 0], theta[0, 0, 1]
    E = np.cos(x[:, 0]) * np.cos(a) * np.cos(b) - np.sin(x[:, 0]) * np.sin(b)
    g = np.zeros_like(theta)
    g[0, 0, 0] = np.sum(-np.sin(a) * np.cos(b) * np.cos(x[:, 0]))
    g[0, 0, 1] = np.sum(-np.cos(a) * np.sin(b) * np.cos(x[:, 0]) - np.cos(b) * np.sin(x[:, 0]))
    return E, g


@pytest.mark.parametrize("n,B", [(30, 1), (29, 2), (25, 3), (21, 1)])
def test_one_layer_closed_form_at_large_n(n, B):
    rng = np.random.default_rng(n)
    x = rng.uniform(0, np.pi, (B, n))
    theta = rng.uniform(0, 2 * np.pi, (1, n, 3))
    E, grad = run(n, 1, x, theta)
    Er, gr = one_layer_reference(x, theta)
    np.testing.assert_allclose(E, Er, atol=1e-5)
    np.testing.assert_allclose(grad, gr, atol=1e-5)


@pytest.mark.parametrize("n,L,ck,st", [(30, 2, 1, "bf16"), (20, 7, 3, "fp32"), (13, 5, 2, "bf16"), (3, 4, 1, "fp32")])
def test_zero_angles_closed_form(n, L, ck, st):
    B = 1 if n >= 29 else 3
    rng = np.random.default_rng(7 + n)
    x = rng.uniform(0, np.pi, (B, n))
    E, grad = run(n, L, x, np.zeros((L, n, 3)), ck, st)
    want = np.zeros((L, n, 3))
    for l in range(L):
        f = np.cos(x[:, 1]) ** (l % 2) if n > 1 else 1.0
        want[l, 0, 1] = np.sum(-np.sin(x[:, 0]) * f)
    tol = 2e-3 if st == "bf16" else 1e-5
    np.testing.assert_allclose(E, np.cos(x[:, 0]), atol=1e-5)
    np.testing.assert_allclose(grad, want, atol=tol)


def test_single_qubit_single_sample():
    x = np.array([[0.9]])
    theta = np.array([[[0.4, -1.3, 2.2]]])
    E, grad = run(1, 1, x, theta)
    Er, gr = one_layer_reference(x, theta)
    np.testing.assert_allclose(E, Er, atol=1e-6)
    np.testing.assert_allclose(grad, gr, atol=1e-6)
