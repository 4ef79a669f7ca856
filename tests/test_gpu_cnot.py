"""GPU parity for CNOT entanglers (through the C ABI) against the oracle.

Every layer ends with CNOT(control, target) on each listed pair in list order.
Tolerances as for the CZ chain in fp32: E abs <= 1e-4, states element by
element <= 2e-5, gradients <= 1e-4 + 1e-3 |g| (2e-2 + 1e-3 |g| with bf16
checkpoints).  Odd batches exercise the partner plane of the last sample pair.
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


def pairs_of(kind, n, rng):
    if kind == "ladder":
        return [(q, q + 1) for q in range(n - 1)]
    if kind == "ring":
        return [(q, (q + 1) % n) for q in range(n)]
    allp = [(a, b) for a in range(n) for b in range(n) if a != b]
    return [allp[i] for i in rng.choice(len(allp), size=n + 2, replace=False)]


CASES = [
    # n, L, B, ckpt_block, storage, pairs
    (2, 3, 3, 0, "fp32", "ladder"),
    (4, 2, 5, 1, "fp32", "ladder"),
    (7, 3, 4, 2, "fp32", "ring"),
    (11, 2, 3, 0, "fp32", "ladder"),
    (12, 3, 5, 1, "bf16", "ladder"),
    (14, 2, 3, 1, "fp32", "ladder"),
    (17, 3, 2, 0, "fp32", "random"),
    (20, 2, 3, 1, "fp32", "ladder"),
    # two qubit sets, fp32: the layer maps are applied inside the rotation passes (fused schedule)
    (13, 3, 5, 1, "bf16", "ladder"),
    (15, 4, 3, 2, "fp32", "ring"),
    (16, 3, 2, 1, "fp32", "random"),
    (19, 3, 1, 1, "fp32", "random"),
    (20, 3, 2, 1, "bf16", "ring"),
    (20, 4, 3, 0, "fp32", "ladder"),
    (21, 2, 3, 1, "fp32", "ladder"),  # three qubit sets: permuted working-state addresses
    (22, 3, 3, 1, "bf16", "ladder"),  # three sets with bf16 checkpoints on the working-state layout
    (23, 2, 1, 0, "fp32", "random"),
]


@pytest.mark.parametrize("n,L,B,ck,st,kind", CASES)
def test_cnot_state_expectation_gradient(n, L, B, ck, st, kind):
    rng = np.random.default_rng(7000 + n)
    pairs = pairs_of(kind, n, rng)
    x, theta, y = random_case(7100 + n + L, B, n, L)
    Eo, psio = oracle.forward(x, theta, want_state=True, bonds=pairs, entangler="cnot")
    g = oracle.loss_seed(Eo, y)
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st)
    ctx.set_entangler(pairs, kind="cnot")
    assert ctx.entangler_kind == "cnot"
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    got = psi.cpu().numpy().astype(np.float64)
    got = got[..., 0] + 1j * got[..., 1]
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g)).cpu().numpy().astype(np.float64)
    ctx.sync()
    np.testing.assert_allclose(E.cpu().numpy().astype(np.float64), Eo, atol=1e-4)
    assert np.max(np.abs(got - psio)) < 2e-5
    gref, _ = oracle.adjoint(x, theta, g, bonds=pairs, entangler="cnot")
    tol = 2e-2 if st == "bf16" else 1e-4
    assert np.all(np.abs(grad - gref) <= tol + 1e-3 * np.abs(gref)), np.max(np.abs(grad - gref))


def test_cnot_with_reupload_and_pauli_sum():
    n, L, B = 13, 3, 3
    pairs = [(q, q + 1) for q in range(n - 1)]
    obs = [(0.7, "X" + "I" * (n - 1)), (-0.5, "ZZ" + "I" * (n - 2)), (0.3, "I" * (n - 1) + "Y")]
    x, theta, y = random_case(7300, B, n, L)
    Eo = oracle.forward(x, theta, observable=obs, bonds=pairs, reupload=True, entangler="cnot")
    g = oracle.loss_seed(Eo, y)
    ctx = qml().Context(n, L, B, ckpt_block=1)
    ctx.set_entangler(pairs, kind="cnot")
    ctx.set_reupload(True)
    ctx.set_observable(obs)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g)).cpu().numpy().astype(np.float64)
    ctx.sync()
    np.testing.assert_allclose(E.cpu().numpy().astype(np.float64), Eo, atol=1e-4)
    gref, _ = oracle.adjoint(x, theta, g, observable=obs, bonds=pairs, reupload=True, entangler="cnot")
    assert np.all(np.abs(grad - gref) <= 1e-4 + 1e-3 * np.abs(gref)), np.max(np.abs(grad - gref))


def test_switching_back_to_cz_restores_the_chain():
    n, L, B = 9, 2, 4
    x, theta, _ = random_case(7400, B, n, L)
    ctx = qml().Context(n, L, B)
    ctx.set_entangler([(q, q + 1) for q in range(n - 1)], kind="cnot")
    ctx.forward(dev(theta), dev(x))
    ctx.set_entangler(None)
    assert ctx.entangler_kind == "cz"
    E = ctx.forward(dev(theta), dev(x))[1].cpu().numpy().astype(np.float64)
    ctx.sync()
    np.testing.assert_allclose(E, oracle.forward(x, theta), atol=1e-4)


@pytest.mark.parametrize("n,L,B,ck,st,kind", [(5, 3, 3, 1, "fp64", "ladder"), (13, 3, 2, 1, "fp64", "ring"),
                                              (14, 2, 3, 1, "bf16", "ladder"), (21, 2, 2, 1, "fp64", "ladder"),
                                              # two qubit sets: the layer maps inside the fp64 passes
                                              (16, 4, 3, 2, "fp64", "ladder"), (19, 3, 2, 0, "fp32", "random"),
                                              (20, 3, 1, 1, "bf16", "ring")])
def test_cnot_fp64(n, L, B, ck, st, kind):
    """fp64 mode with CNOT lists: tolerances of the fp64 parity tests (1e-10 + 1e-9 |g| with fp64 or no
    slots; bf16 slots round the restarted state to 2^-8: 2e-2 + 1e-3 |g|)."""
    rng = np.random.default_rng(7500 + n)
    pairs = pairs_of(kind, n, rng)
    x, theta, y = random_case(7600 + n, B, n, L)
    Eo, psio = oracle.forward(x, theta, want_state=True, bonds=pairs, entangler="cnot")
    g = oracle.loss_seed(Eo, y)
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st, precision="fp64")
    ctx.set_entangler(pairs, kind="cnot")
    d64 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).cuda()
    xd, td = d64(x), d64(theta)
    psi, E = ctx.forward(td, xd)
    got = psi.cpu().numpy()
    got = got[..., 0] + 1j * got[..., 1]
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), d64(g)).cpu().numpy()
    ctx.sync()
    assert np.max(np.abs(E.cpu().numpy() - Eo)) <= 1e-11
    assert np.max(np.abs(got - psio)) <= 1e-12
    gref, _ = oracle.adjoint(x, theta, g, bonds=pairs, entangler="cnot")
    a, r = (2e-2, 1e-3) if st == "bf16" else (1e-10, 1e-9)
    assert np.all(np.abs(grad - gref) <= a + r * np.abs(gref)), np.max(np.abs(grad - gref))
