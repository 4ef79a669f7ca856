"""GPU parity for CZ entanglers on arbitrary bond lists against the oracle.

Every layer ends with CZ on each listed bond.  Same tolerances as the chain
(E abs <= 1e-4; gradient abs <= 1e-4 + 1e-3 |g| in fp32, 2e-2 + 1e-3 |g| with
bf16 checkpoints).
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


def random_bonds(rng, n, count):
    pairs = [(a, b) for a in range(n) for b in range(a + 1, n)]
    idx = rng.choice(len(pairs), size=min(count, len(pairs)), replace=False)
    return [tuple(int(v) for v in pairs[i]) for i in idx]


def run(n, L, x, theta, y, bonds, ck=0, st="fp32", obs=None):
    B = x.shape[0]
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st)
    ctx.set_entangler(bonds)
    ctx.set_observable(obs)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    g = oracle.loss_seed(E.cpu().numpy().astype(np.float64), y)
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g))
    torch.cuda.synchronize()
    ctx.sync()
    return E.cpu().numpy().astype(np.float64), g, grad.cpu().numpy().astype(np.float64)


def check(n, L, B, bonds, ck=0, st="fp32", obs=None, seed=0):
    x, theta, y = random_case(seed, B, n, L)
    E, g, grad = run(n, L, x, theta, y, bonds, ck, st, obs)
    Eo = oracle.forward(x, theta, observable=obs, bonds=bonds)
    scale = 1.0 if obs is None else sum(abs(c) for c, _ in obs)
    np.testing.assert_allclose(E, Eo, atol=1e-4 * scale)
    gref, _ = oracle.adjoint(x, theta, g, observable=obs, bonds=bonds)
    tol = (2e-2 if st == "bf16" else 1e-4) * scale
    err = np.abs(grad - gref)
    assert np.all(err <= tol + 1e-3 * np.abs(gref)), float(err.max())


@pytest.mark.parametrize("n,L,B,ck,st", [(4, 3, 5, 0, "fp32"), (9, 4, 3, 2, "fp32"), (12, 3, 4, 0, "fp32"),
                                         (13, 3, 3, 1, "bf16"), (17, 2, 3, 0, "fp32"), (20, 2, 2, 1, "fp32")])
def test_random_bond_graph(n, L, B, ck, st):
    rng = np.random.default_rng(900 + n)
    check(n, L, B, random_bonds(rng, n, n + 3), ck, st, seed=910 + n)


@pytest.mark.parametrize("n", [6, 20, 23])
def test_ring(n):
    check(n, 3, 2, [(q, q + 1) for q in range(n - 1)] + [(n - 1, 0)], seed=920 + n)


@pytest.mark.parametrize("n", [5, 14])
def test_no_entangler_and_all_to_all(n):
    check(n, 3, 3, [], seed=930 + n)
    check(n, 2, 2, [(a, b) for a in range(n) for b in range(a + 1, n)][:60], seed=940 + n)


def test_ring_with_a_pauli_sum():
    n = 13
    obs = [(1.0, "XZ" + "I" * (n - 2)), (0.5, "I" * (n - 1) + "Y"), (-0.7, "Z" * n)]
    check(n, 2, 3, [(q, (q + 1) % n) for q in range(n)], obs=obs, seed=950)
