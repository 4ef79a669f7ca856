"""GPU parity of the fp64 compute mode (through the C ABI) against the complex128 oracle.

Tolerances.  With fp64 checkpoint slots, or none, the CUDA path and the oracle
differ only in rounding order: each 2x2 gate adds a relative error of a few
2^-53 per amplitude, and at most a few thousand gates act on an amplitude
here, so |dE| <= 1e-11, the state agrees element by element to 1e-12 and the
gradients (sums over every amplitude and sample) to 1e-10 + 1e-9 |g|.  fp32
slots restart the backward pass from a state rounded to 2^-24 relative:
1e-5 + 1e-4 |g|.  bf16 slots round to 2^-8: 2e-2 + 1e-3 |g| (as in fp32 mode).
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
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).cuda()


GRAD_TOL = {"fp64": (1e-10, 1e-9), "fp32": (1e-5, 1e-4), "bf16": (2e-2, 1e-3)}


def run_f64(n, L, x, theta, g, ckpt_block=0, storage="fp64", bonds=None, reupload=False, want_state=False):
    B = x.shape[0]
    ctx = qml().Context(n, L, B, ckpt_block=ckpt_block, storage=storage, precision="fp64")
    assert ctx.precision_bits == 64
    if bonds is not None:
        ctx.set_entangler(bonds)
    if reupload:
        ctx.set_reupload(True)
    xd, td, gd = dev(x), dev(theta), dev(g)
    psi, E = ctx.forward(td, xd)
    psi_final = psi.clone() if want_state else None
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), gd)
    torch.cuda.synchronize()
    ctx.sync()
    return E.cpu().numpy(), grad.cpu().numpy(), psi_final


CASES = [
    # n, L, B, ckpt_block, slot storage
    (1, 3, 3, 0, "fp64"),
    (2, 5, 5, 2, "fp64"),
    (4, 2, 8, 0, "fp64"),
    (5, 7, 4, 3, "fp64"),
    (7, 4, 9, 0, "fp64"),
    (11, 3, 6, 1, "fp64"),
    (12, 5, 7, 2, "fp64"),
    (13, 3, 5, 0, "fp64"),
    (14, 4, 3, 2, "fp64"),
    (16, 3, 2, 1, "fp32"),
    (17, 2, 3, 0, "fp64"),
    (10, 6, 3, 2, "bf16"),
    (21, 2, 2, 1, "fp64"),
    (23, 3, 1, 0, "fp64"),
]


@pytest.mark.parametrize("n,L,B,ck,st", CASES)
def test_f64_state_expectation_and_gradient(n, L, B, ck, st):
    x, theta, y = random_case(5000 + 31 * n + L, B, n, L)
    Eo, psio = oracle.forward(x, theta, want_state=True)
    g = oracle.loss_seed(Eo, y)
    E, grad, psi = run_f64(n, L, x, theta, g, ck, st, want_state=True)
    assert np.max(np.abs(E - Eo)) <= 1e-11, np.max(np.abs(E - Eo))
    got = psi.cpu().numpy()
    got = got[..., 0] + 1j * got[..., 1]
    assert np.max(np.abs(got - psio)) <= 1e-12, np.max(np.abs(got - psio))
    gref, _ = oracle.adjoint(x, theta, g)
    a, r = GRAD_TOL[st]
    assert np.all(np.abs(grad - gref) <= a + r * np.abs(gref)), np.max(np.abs(grad - gref))


@pytest.mark.parametrize("n,L,B,ck", [(5, 3, 4, 0), (9, 4, 3, 2), (13, 3, 2, 1), (20, 2, 2, 1)])
def test_f64_reupload(n, L, B, ck):
    x, theta, y = random_case(6100 + n, B, n, L)
    Eo = oracle.forward(x, theta, reupload=True)
    g = oracle.loss_seed(Eo, y)
    E, grad, _ = run_f64(n, L, x, theta, g, ck, reupload=True)
    assert np.max(np.abs(E - Eo)) <= 1e-11
    gref, _ = oracle.adjoint(x, theta, g, reupload=True)
    assert np.all(np.abs(grad - gref) <= 1e-10 + 1e-9 * np.abs(gref)), np.max(np.abs(grad - gref))


@pytest.mark.parametrize("n,L,B,kind", [(6, 3, 3, "ring"), (14, 3, 2, "ring"), (13, 2, 2, "random"),
                                        (8, 2, 3, "none")])
def test_f64_entanglers(n, L, B, kind):
    rng = np.random.default_rng(6200 + n)
    if kind == "ring":
        bonds = [(q, (q + 1) % n) for q in range(n)]
    elif kind == "none":
        bonds = []
    else:
        pairs = [(a, b) for a in range(n) for b in range(a + 1, n)]
        bonds = [pairs[i] for i in rng.choice(len(pairs), size=2 * n, replace=False)]
    x, theta, y = random_case(6300 + n, B, n, L)
    Eo = oracle.forward(x, theta, bonds=bonds)
    g = oracle.loss_seed(Eo, y)
    E, grad, _ = run_f64(n, L, x, theta, g, 1, bonds=bonds)
    assert np.max(np.abs(E - Eo)) <= 1e-11
    gref, _ = oracle.adjoint(x, theta, g, bonds=bonds)
    assert np.all(np.abs(grad - gref) <= 1e-10 + 1e-9 * np.abs(gref)), np.max(np.abs(grad - gref))


def test_f64_parameter_shift_tiny_workload():
    """The gradient against the parameter-shift rule through the fp64 forward pass itself."""
    w = WORKLOADS["tiny_4q_L2"]
    x, theta, y = make_inputs(w)
    ctx = qml().Context(w.n, w.L, w.B, precision="fp64")
    xd = dev(x)
    E = ctx.forward(dev(theta), xd)[1]
    g, _ = ctx.loss_seed(E, dev(y))
    psi = ctx.forward(dev(theta), xd)[0]
    grad = ctx.backward(dev(theta), xd, psi, ctx.new_state(w.B), g).cpu().numpy()
    gh = g.cpu().numpy()
    shift = np.zeros_like(theta)
    for idx in np.ndindex(theta.shape):
        tp, tm = theta.copy(), theta.copy()
        tp[idx] += np.pi / 2
        tm[idx] -= np.pi / 2
        Ep = ctx.forward(dev(tp), xd)[1].cpu().numpy()
        Em = ctx.forward(dev(tm), xd)[1].cpu().numpy()
        shift[idx] = np.dot(gh, 0.5 * (Ep - Em))
    assert np.max(np.abs(grad - shift)) <= 1e-12


def test_f64_deterministic_and_loss_seed():
    n, L, B = 14, 4, 5
    x, theta, y = random_case(6400, B, n, L)
    ctx = qml().Context(n, L, B, ckpt_block=2, storage="fp64", precision="fp64")
    xd, td = dev(x), dev(theta)
    out = []
    for _ in range(2):
        psi, E = ctx.forward(td, xd)
        g, loss = ctx.loss_seed(E, dev(y))
        out.append(ctx.backward(td, xd, psi, ctx.new_state(B), g).cpu().numpy())
    assert np.array_equal(out[0], out[1])
    Eo = oracle.forward(x, theta)
    assert abs(loss.item() - np.mean((Eo - y) ** 2)) <= 1e-12
    np.testing.assert_allclose(g.cpu().numpy(), oracle.loss_seed(Eo, y), rtol=0, atol=1e-12)


def test_f64_step_host_matches_device_calls():
    n, L, B = 12, 3, 4
    x, theta, y = random_case(6500, B, n, L)
    ctx = qml().Context(n, L, B, ckpt_block=1, storage="fp64", precision="fp64", host_step=True)
    r = ctx.step_host(np.ascontiguousarray(x), np.ascontiguousarray(theta), np.ascontiguousarray(y))
    ctx.sync()
    Eo = oracle.forward(x, theta)
    g = oracle.loss_seed(Eo, y)
    gref, _ = oracle.adjoint(x, theta, g)
    assert np.max(np.abs(r.expect - Eo)) <= 1e-11
    assert abs(r.loss[0] - np.mean((Eo - y) ** 2)) <= 1e-12
    assert np.all(np.abs(r.grad - gref) <= 1e-10 + 1e-9 * np.abs(gref))


def test_f64_large_sampled_state():
    """24 qubits (three qubit sets), one sample: sampled amplitudes, Z0 and the
    gradient against the oracle at the same size."""
    n, L, B = 24, 2, 1
    x, theta, y = random_case(6600, B, n, L)
    Eo, psio = oracle.forward(x, theta, want_state=True)
    g = oracle.loss_seed(Eo, y)
    E, grad, psi = run_f64(n, L, x, theta, g, 1, want_state=True)
    assert abs(E[0] - Eo[0]) <= 1e-11
    rng = np.random.default_rng(1)
    idx = rng.integers(0, 1 << n, size=4096)
    got = psi.cpu().numpy()[0, idx]
    assert np.max(np.abs(got[:, 0] + 1j * got[:, 1] - psio[0, idx])) <= 1e-12
    gref, _ = oracle.adjoint(x, theta, g)
    assert np.all(np.abs(grad - gref) <= 1e-10 + 1e-9 * np.abs(gref))


@pytest.mark.parametrize("n,L,B,ck", [(6, 3, 3, 1), (14, 2, 3, 1)])
def test_f64_pauli_sum_observable(n, L, B, ck):
    """O = a transverse-field Ising sum with a Y term, evaluated and seeded in fp64."""
    obs = [(1.0, "".join("Z" if k in (q, q + 1) else "I" for k in range(n))) for q in range(n - 1)]
    obs += [(0.9, "".join("X" if k == q else "I" for k in range(n))) for q in range(n)]
    obs += [(-0.4, "Y" + "I" * (n - 2) + "X")]
    x, theta, y = random_case(6700 + n, B, n, L)
    Eo = oracle.forward(x, theta, observable=obs)
    g = oracle.loss_seed(Eo, y)
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage="fp64", precision="fp64")
    ctx.set_observable(obs)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g)).cpu().numpy()
    ctx.sync()
    assert np.max(np.abs(E.cpu().numpy() - Eo)) <= 1e-10
    gref, _ = oracle.adjoint(x, theta, g, observable=obs)
    assert np.all(np.abs(grad - gref) <= 1e-9 + 1e-9 * np.abs(gref)), np.max(np.abs(grad - gref))
