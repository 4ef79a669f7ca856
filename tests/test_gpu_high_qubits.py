"""GPU parity above 20 qubits with non-zero gradients on every qubit.

Circuits of 21 or more qubits have three qubit sets, and their state sits at
permuted working-state addresses between passes.  With the Z0 observable and
few layers, Z0's backward light cone makes every gradient beyond qubit L-1
exactly zero, so those cases cannot see a wrong gradient slot or a lost
partial sum of the third set.  Here the observable is a sum of one- and
two-qubit Pauli strings that covers every qubit (Z_q Z_{q+1} on each bond, X
or Y on each qubit), which gives O(1) gradients on all qubits, the highest
included; each gradient is compared with the complex128 oracle.

Tolerances: with ||c||_1 the sum of |coefficients| (a bound on |<O>|), E abs
<= 1e-4 ||c||_1 and gradient abs <= 1e-4 ||c||_1 + 1e-3 |g| in fp32; 2e-2
||c||_1 + 1e-3 |g| with bf16 checkpoints (the workload statement's bounds,
with the absolute part scaled by the observable's norm).
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


def covering_observable(n):
    """Z_q Z_{q+1} on every bond, then X on even and Y on odd qubits."""
    out = []
    for q in range(n - 1):
        w = ["I"] * n
        w[q] = w[q + 1] = "Z"
        out.append((1.0, "".join(w)))
    for q in range(n):
        w = ["I"] * n
        w[q] = "XY"[q % 2]
        out.append((0.9 if q % 2 == 0 else -0.6, "".join(w)))
    return out


def run(n, L, x, theta, y, obs, ck, st, entangler=None, reupload=False):
    B = x.shape[0]
    ctx = qml().Context(n, L, B, ckpt_block=ck, storage=st)
    ctx.set_observable(obs)
    if entangler is not None:
        ctx.set_entangler(entangler, kind="cnot")
    if reupload:
        ctx.set_reupload(True)
    xd, td = dev(x), dev(theta)
    psi, E = ctx.forward(td, xd)
    E = E.cpu().numpy().astype(np.float64)
    g = oracle.loss_seed(E, y)
    grad = ctx.backward(td, xd, psi, ctx.new_state(B), dev(g))
    torch.cuda.synchronize()
    ctx.sync()
    out = E, g.astype(np.float32).astype(np.float64), grad.cpu().numpy().astype(np.float64)
    del psi, ctx
    torch.cuda.empty_cache()
    return out


def check(n, L, B, ck, st, seed, entangler=None, reupload=False):
    x, theta, y = random_case(seed, B, n, L)
    obs = covering_observable(n)
    scale = sum(abs(c) for c, _ in obs)
    kw = dict(observable=obs, reupload=reupload)
    if entangler is not None:
        kw.update(bonds=entangler, entangler="cnot")
    E, g, grad = run(n, L, x, theta, y, obs, ck, st, entangler, reupload)
    Eo = oracle.forward(x, theta, **kw)
    np.testing.assert_allclose(E, Eo, atol=1e-4 * scale, rtol=0)
    gref, _ = oracle.adjoint(x, theta, g, **kw)
    # the case must reach the highest qubits: every qubit has an O(1e-2) gradient
    per_qubit = np.abs(gref).max(axis=(0, 2))
    assert np.all(per_qubit > 1e-2), per_qubit
    tol = (2e-2 if st == "bf16" else 1e-4) * scale
    err = np.abs(grad - gref)
    assert np.all(err <= tol + 1e-3 * np.abs(gref)), (float(err.max()), np.unravel_index(err.argmax(), err.shape))
    return err


@pytest.mark.parametrize("n,L,B,ck,st", [
    (21, 3, 3, 1, "fp32"),   # odd batch: the forward's partner plane
    (23, 3, 2, 1, "fp32"),
    (22, 3, 1, 1, "bf16"),
    (25, 2, 1, 0, "fp32"),
])
def test_every_qubit_gradient_above_20_qubits(n, L, B, ck, st):
    check(n, L, B, ck, st, seed=8000 + n + L)


def test_reupload_above_20_qubits():
    check(22, 2, 2, 1, "fp32", seed=8101, reupload=True)


def test_cnot_ladder_bf16_checkpoints_above_20_qubits():
    n = 21
    check(n, 3, 3, 1, "bf16", seed=8202, entangler=[(q, q + 1) for q in range(n - 1)])
