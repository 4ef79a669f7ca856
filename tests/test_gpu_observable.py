"""GPU parity for general observables (sums of Pauli strings) against the oracle.

O = sum_k c_k P_k with letter q of each string acting on qubit q.  The oracle
applies the strings as explicit one-qubit matrices; the CUDA path evaluates
them matrix-free by bit flips.  Tolerances scale with ||c||_1 (a bound on
|<O>|): E abs error <= 1e-4 ||c||_1; gradient abs error <= (1e-4 + 1e-3 |g|)
||c||_1 in fp32, 2e-2 ||c||_1 with bf16 checkpoints.
"""
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


def random_observable(rng, n, terms):
    obs = [(float(rng.normal()), "".join(rng.choice(list("IXYZ"), size=n))) for _ in range(terms)]
    # a term that flips the highest qubit (crosses tiles) and one that is the identity
    obs.append((0.7, "I" * (n - 1) + "X"))
    obs.append((-0.3, "I" * n))
    return obs


def tfim(n, h=0.9):
    """Transverse-field Ising chain: sum_q Z_q Z_{q+1} + h sum_q X_q."""
    out = []
    for q in range(n - 1):
        w = ["I"] * n
        w[q] = w[q + 1] = "Z"
        out.append((1.0, "".join(w)))
    for q in range(n):
        w = ["I"] * n
        w[q] = "X"
        out.append((h, "".join(w)))
    return out


def run(n, L, x, theta, y, obs, ck=0, st="fp32"):
    B = x.shape[0]
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st)
    ctx.set_observable(obs)
    assert ctx.observable_terms == len(obs)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    g = dev(oracle.loss_seed(E.cpu().numpy().astype(np.float64), y))
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), g)
    torch.cuda.synchronize()
    ctx.sync()
    return E.cpu().numpy().astype(np.float64), g.cpu().numpy().astype(np.float64), grad.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("n,L,B,ck,st,terms", [
    (4, 3, 5, 0, "fp32", 6),
    (9, 4, 3, 2, "fp32", 10),
    (12, 3, 6, 0, "fp32", 8),
    (13, 3, 3, 1, "bf16", 8),
    (17, 2, 3, 0, "fp32", 12),
    (20, 2, 2, 1, "fp32", 5),
])
def test_random_observable_parity(n, L, B, ck, st, terms):
    rng = np.random.default_rng(500 + n)
    x, theta, y = random_case(600 + n, B, n, L)
    obs = random_observable(rng, n, terms)
    scale = sum(abs(c) for c, _ in obs)
    E, g, grad = run(n, L, x, theta, y, obs, ck, st)
    Eo = oracle.forward(x, theta, observable=obs)
    np.testing.assert_allclose(E, Eo, atol=1e-4 * scale)
    gref, _ = oracle.adjoint(x, theta, g, observable=obs)
    tol = (2e-2 if st == "bf16" else 1e-4) * scale
    err = np.abs(grad - gref)
    assert np.all(err <= tol + 1e-3 * scale * np.abs(gref)), float(err.max())


def test_tfim_20_qubits():
    n, L, B = 20, 3, 2
    x, theta, y = random_case(777, B, n, L)
    obs = tfim(n)
    E, g, grad = run(n, L, x, theta, y, obs, ck=2)
    scale = sum(abs(c) for c, _ in obs)
    Eo = oracle.forward(x, theta, observable=obs)
    np.testing.assert_allclose(E, Eo, atol=1e-4 * scale)
    gref, _ = oracle.adjoint(x, theta, g, observable=obs)
    assert np.all(np.abs(grad - gref) <= 1e-4 * scale + 1e-3 * np.abs(gref)), float(np.abs(grad - gref).max())


def test_expect_observable_on_oracle_states_and_reset():
    rng = np.random.default_rng(3)
    n, L, B = 14, 2, 4
    x, theta, _ = random_case(31, B, n, L)
    obs = random_observable(rng, n, 9)
    _, psi = oracle.forward(x, theta, want_state=True)
    st = torch.from_numpy(np.stack([psi.real, psi.imag], -1).astype(np.float32)).cuda()
    ctx = qml().Context(n, L, B)
    ctx.set_observable(obs)
    E = ctx.expect_observable(st).cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(E, oracle.forward(x, theta, observable=obs), atol=1e-5 * sum(abs(c) for c, _ in obs))
    ctx.set_observable(None)
    assert ctx.observable_terms == 0
    E0 = ctx.expect_observable(st).cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(E0, oracle.forward(x, theta), atol=1e-5)
    ctx.sync()


def test_z0_as_an_observable_matches_the_default_path():
    n, L, B = 13, 3, 3
    x, theta, y = random_case(88, B, n, L)
    obs = [(1.0, "Z" + "I" * (n - 1))]
    E1, g1, G1 = run(n, L, x, theta, y, obs)
    ctx = qml().Context(n, L, B)
    xd, td = dev(x), dev(theta)
    psi, E2 = ctx.forward(td, xd)
    G2 = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g1))
    np.testing.assert_allclose(E1, E2.cpu().numpy(), atol=1e-6)
    np.testing.assert_allclose(G1, G2.cpu().numpy(), atol=1e-6)
