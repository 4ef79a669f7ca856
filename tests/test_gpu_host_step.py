"""qml_step_host in a row: the first call runs eagerly, the second captures the
step into a CUDA graph and later calls replay it.  Every call must match the
oracle (E abs <= 1e-4, gradients <= 1e-4 + 1e-3 |g|), replays must agree bit
for bit with the eager call, new values written into the same host buffers
must be picked up by a replay, and a setter must send the next call back to the
eager path (with the new setting in force)."""
import numpy as np
import pytest

import oracle
from adjoint_gradients_b200.inputs import random_case

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def pinned(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).pin_memory()


def check(out, x, theta, y, **kw):
    Eo = oracle.forward(x, theta, **kw)
    go, _ = oracle.adjoint(x, theta, oracle.loss_seed(Eo, y), **kw)
    E = out.expect.numpy().astype(np.float64)
    g = out.grad.numpy().astype(np.float64)
    np.testing.assert_allclose(E, Eo, atol=1e-4)
    assert np.all(np.abs(g - go) <= 1e-4 + 1e-3 * np.abs(go)), np.max(np.abs(g - go))
    np.testing.assert_allclose(out.loss.numpy()[0], np.mean((Eo - y) ** 2), atol=1e-4)


@pytest.mark.parametrize("n,L,B,ck,kind", [(12, 3, 5, 1, "cz"), (16, 3, 3, 1, "cnot")])
def test_host_step_replays_a_graph(n, L, B, ck, kind):
    from adjoint_gradients_b200 import qml

    x, theta, y = random_case(8800 + n, B, n, L)
    ctx = qml.Context(n, L, B, ckpt_block=ck, host_step=True)
    pairs = [(q, q + 1) for q in range(n - 1)]
    kw = {}
    if kind == "cnot":
        ctx.set_entangler(pairs, kind="cnot")
        kw = {"bonds": pairs, "entangler": "cnot"}
    xh, th, yh = pinned(x), pinned(theta), pinned(y)
    out = qml.StepResult(pinned(np.zeros(B)), pinned(np.zeros(1)), pinned(np.zeros((L, n, 3))))
    first = None
    counts = []
    for _ in range(4):
        c0 = ctx.launch_count
        ctx.step_host(xh, th, yh, out)
        counts.append(ctx.launch_count - c0)
        check(out, x, theta, y, **kw)
        snap = (out.expect.numpy().copy(), out.grad.numpy().copy())
        if first is None:
            first = snap
        else:
            assert np.array_equal(snap[0], first[0]) and np.array_equal(snap[1], first[1])
    assert len(set(counts)) == 1 and counts[0] > 0  # replays account for the kernels they launch
    # new angles in the same host buffer: the replay reads them
    theta2 = np.random.default_rng(8900 + n).uniform(0, 2 * np.pi, theta.shape)
    th.copy_(torch.from_numpy(theta2.astype(np.float32)))
    ctx.step_host(xh, th, yh, out)
    check(out, x, theta2.astype(np.float32).astype(np.float64), y, **kw)
    # a setter in between: back to the eager path with the new observable
    obs = [(0.6, "X" + "I" * (n - 1)), (-0.4, "ZZ" + "I" * (n - 2))]
    ctx.set_observable(obs)
    for _ in range(3):
        ctx.step_host(xh, th, yh, out)
        check(out, x, theta2.astype(np.float32).astype(np.float64), y, observable=obs, **kw)
    ctx.sync()
