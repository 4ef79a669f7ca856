"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself:
  * closed forms derived independently with SO(3) Bloch-vector rotations
    (L = 0, theta = 0, Rz-only, L = 1, L = 2);
  * a dense brute-force simulator built here from scipy's matrix exponential and
    numpy kron products (n <= 5), with gradients by the exact parameter-shift rule;
  * parameter shift and central finite differences of the oracle's own forward
    pass against its adjoint gradient (the adjoint code path is separate);
  * invariants: norm, |E| <= 1, the backward walk returning |0...0>, and the
    exact zeros of the light cone of Z0;
  * bf16 rounding against torch's float32 -> bfloat16 conversion.

The method: Kawase, "Fast and memory-efficient classical simulation of quantum
machine learning via forward and backward gate fusion" -- Deep-dive blog §1.2
(E(theta), adjoint gradient, lambda recursion) and §2.1 (HEA of Rx, Ry, Rz + CZ).
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from adjoint_gradients_b200.inputs import WORKLOADS, make_inputs, random_case

# ----------------------------------------------------------------------------- helpers

PAULI = {
    0: np.array([[0, 1], [1, 0]], dtype=complex),
    1: np.array([[0, -1j], [1j, 0]], dtype=complex),
    2: np.array([[1, 0], [0, -1]], dtype=complex),
}


def dense_rot(p, t):
    return scipy.linalg.expm(-0.5j * t * PAULI[p])


def dense_on(u, q, n):
    """Full 2^n operator of a one-qubit u on qubit q (qubit 0 = least significant bit)."""
    return np.kron(np.eye(1 << (n - 1 - q)), np.kron(u, np.eye(1 << q)))


def dense_cz(q1, q2, n):
    idx = np.arange(1 << n)
    both = ((idx >> q1) & 1) & ((idx >> q2) & 1)
    return np.diag(np.where(both == 1, -1.0, 1.0)).astype(complex)


def dense_state(x, theta):
    n = x.shape[0]
    psi = np.zeros(1 << n, dtype=complex)
    psi[0] = 1
    for q in range(n):
        psi = dense_on(dense_rot(1, x[q]), q, n) @ psi
    for l in range(theta.shape[0]):
        for q in range(n):
            for a in range(3):
                psi = dense_on(dense_rot(a, theta[l, q, a]), q, n) @ psi
        for q in range(n - 1):
            psi = dense_cz(q, q + 1, n) @ psi
    return psi


def dense_E(x, theta):
    n = x.shape[0]
    psi = dense_state(x, theta)
    return float(np.real(np.conj(psi) @ (dense_on(PAULI[2], 0, n) @ psi)))


def bloch_rx(v, a):
    x, y, z = v
    return np.array([x, y * np.cos(a) - z * np.sin(a), y * np.sin(a) + z * np.cos(a)])


def bloch_ry(v, b):
    x, y, z = v
    return np.array([x * np.cos(b) + z * np.sin(b), y, -x * np.sin(b) + z * np.cos(b)])


def bloch_rz(v, c):
    x, y, z = v
    return np.array([x * np.cos(c) - y * np.sin(c), x * np.sin(c) + y * np.cos(c), z])


def bloch_layer(v, ang):
    return bloch_rz(bloch_ry(bloch_rx(v, ang[0]), ang[1]), ang[2])


def closed_form_E(x, theta):
    """<Z0> for L <= 2 by Bloch vectors: the CZ(0,1) of layer 0 dephases qubit 0's
    x and y components by <Z1>; no other CZ changes qubit 0's reduced state, and
    the last CZ ladder commutes with Z0."""
    L = theta.shape[0]
    v0 = np.array([np.sin(x[0]), 0.0, np.cos(x[0])])
    if L == 0:
        return v0[2]
    v0 = bloch_layer(v0, theta[0, 0])
    if L == 1:
        return v0[2]
    assert L == 2
    z1 = 1.0
    if x.shape[0] > 1:
        z1 = bloch_layer(np.array([np.sin(x[1]), 0.0, np.cos(x[1])]), theta[0, 1])[2]
    v0 = np.array([v0[0] * z1, v0[1] * z1, v0[2]])
    return bloch_layer(v0, theta[1, 0])[2]


def shift_grad_E(fwd, x, theta):
    """Parameter-shift dE_b/dtheta for every parameter: [B][L][n][3] (exact for exp(-itP/2))."""
    B = x.shape[0]
    out = np.zeros((B,) + theta.shape)
    for idx in np.ndindex(theta.shape):
        tp = theta.copy()
        tm = theta.copy()
        tp[idx] += np.pi / 2
        tm[idx] -= np.pi / 2
        out[(slice(None),) + idx] = 0.5 * (fwd(x, tp) - fwd(x, tm))
    return out


# ----------------------------------------------------------------------------- closed forms


@pytest.mark.parametrize("n", [1, 2, 5, 9])
def test_no_layers_is_cos_x0(n):
    x, _, _ = random_case(11 + n, 6, n, 0)
    E = oracle.forward(x, np.zeros((0, n, 3)))
    np.testing.assert_allclose(E, np.cos(x[:, 0]), atol=1e-14)


@pytest.mark.parametrize("n,L", [(3, 1), (6, 4), (10, 3)])
def test_zero_angles_is_cos_x0(n, L):
    x, _, _ = random_case(21 + n, 5, n, L)
    E = oracle.forward(x, np.zeros((L, n, 3)))
    np.testing.assert_allclose(E, np.cos(x[:, 0]), atol=1e-13)


@pytest.mark.parametrize("n,L", [(4, 2), (7, 5)])
def test_rz_only_is_cos_x0_and_rz_grads_vanish(n, L):
    x, theta, _ = random_case(31 + n, 4, n, L)
    theta[..., 0] = 0.0
    theta[..., 1] = 0.0
    E = oracle.forward(x, theta)
    np.testing.assert_allclose(E, np.cos(x[:, 0]), atol=1e-13)
    grad, _ = oracle.adjoint(x, theta, np.ones(4))
    np.testing.assert_allclose(grad[..., 2], 0.0, atol=1e-13)


@pytest.mark.parametrize("n", [1, 2, 3, 8])
def test_one_layer_closed_form(n):
    x, theta, _ = random_case(41 + n, 5, n, 1)
    E = oracle.forward(x, theta)
    a, b = theta[0, 0, 0], theta[0, 0, 1]
    x0 = x[:, 0]
    np.testing.assert_allclose(E, np.cos(x0) * np.cos(a) * np.cos(b) - np.sin(x0) * np.sin(b), atol=1e-13)
    # gradient seeded with g_b = 1 for one sample at a time
    for bi in range(x.shape[0]):
        g = np.zeros(x.shape[0])
        g[bi] = 1.0
        grad, _ = oracle.adjoint(x, theta, g)
        want = np.zeros_like(theta)
        want[0, 0, 0] = -np.sin(a) * np.cos(b) * np.cos(x0[bi])
        want[0, 0, 1] = -np.cos(a) * np.sin(b) * np.cos(x0[bi]) - np.cos(b) * np.sin(x0[bi])
        np.testing.assert_allclose(grad, want, atol=1e-13)


@pytest.mark.parametrize("n", [1, 2, 3, 6])
def test_two_layer_closed_form(n):
    x, theta, _ = random_case(51 + n, 6, n, 2)
    E = oracle.forward(x, theta)
    want = np.array([closed_form_E(x[b], theta) for b in range(x.shape[0])])
    np.testing.assert_allclose(E, want, atol=1e-13)


def test_rotation_conventions():
    # Ry(t)|0>: <Z> = cos t (encoding with one qubit, no layers) ...
    t = np.array([[0.3], [1.1], [2.9]])
    np.testing.assert_allclose(oracle.forward(t, np.zeros((0, 1, 3))), np.cos(t[:, 0]), atol=1e-15)
    # ... and Rx(a) after encoding x=0 gives <Z> = cos a; Ry(b) gives cos b.
    th = np.zeros((1, 1, 3))
    th[0, 0, 0] = 0.7
    np.testing.assert_allclose(oracle.forward(np.zeros((1, 1)), th), [np.cos(0.7)], atol=1e-15)
    # Ry(pi/2)|0> then Ry(b): <Z> = cos(pi/2 + b) = -sin b pins the sign of Ry.
    th = np.zeros((1, 1, 3))
    th[0, 0, 1] = 0.4
    np.testing.assert_allclose(oracle.forward(np.full((1, 1), np.pi / 2), th), [-np.sin(0.4)], atol=1e-15)
    # Rx(a) on Ry(pi/2)|0> = |+>: X axis is invariant under Rx, so <Z> = 0 for any a.
    th = np.zeros((1, 1, 3))
    th[0, 0, 0] = 1.3
    np.testing.assert_allclose(oracle.forward(np.full((1, 1), np.pi / 2), th), [0.0], atol=1e-15)


# ----------------------------------------------------------------------------- brute force


@pytest.mark.parametrize("n,L,seed", [(1, 2, 1), (2, 3, 2), (3, 2, 3), (4, 2, 4), (5, 3, 5)])
def test_dense_brute_force_state_energy_gradient(n, L, seed):
    x, theta, y = random_case(seed, 3, n, L)
    E, psi = oracle.forward(x, theta, want_state=True)
    for b in range(3):
        ref = dense_state(x[b], theta)
        np.testing.assert_allclose(psi[b], ref, atol=1e-12)
        assert abs(E[b] - dense_E(x[b], theta)) < 1e-12
    g = oracle.loss_seed(E, y)
    grad, E2 = oracle.adjoint(x, theta, g)
    np.testing.assert_allclose(E2, E, atol=1e-14)
    dense_fwd = lambda xx, tt: np.array([dense_E(xx[b], tt) for b in range(xx.shape[0])])
    want = np.einsum("b,b...->...", g, shift_grad_E(dense_fwd, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-12)


# ----------------------------------------------------------------------------- parameter shift / FD


def test_parameter_shift_tiny_workload():
    w = WORKLOADS["tiny_4q_L2"]
    x, theta, y = make_inputs(w)
    grad, E = oracle.adjoint(x, theta, np.zeros(w.B))
    g = oracle.loss_seed(E, y)
    grad, _ = oracle.adjoint(x, theta, g)
    want = np.einsum("b,b...->...", g, shift_grad_E(oracle.forward, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-10)
    assert w.params == 24 and grad.size == 24


def test_parameter_shift_12q_workload_all_params():
    w = WORKLOADS["hea_12q_L10"]
    x, theta, y = make_inputs(w)
    x = x[:2]  # two samples, every one of the 360 parameters
    E = oracle.forward(x, theta)
    g = oracle.loss_seed(E, y[:2])
    grad, _ = oracle.adjoint(x, theta, g)
    want = np.einsum("b,b...->...", g, shift_grad_E(oracle.forward, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-10)


def test_central_finite_difference_of_mean_loss():
    x, theta, y = random_case(77, 4, 6, 4)

    def loss(t):
        return np.mean((oracle.forward(x, t) - y) ** 2)

    E = oracle.forward(x, theta)
    grad, _ = oracle.adjoint(x, theta, oracle.loss_seed(E, y))
    h = 1e-5
    rng = np.random.default_rng(5)
    for _ in range(20):
        idx = tuple(rng.integers(0, s) for s in theta.shape)
        tp, tm = theta.copy(), theta.copy()
        tp[idx] += h
        tm[idx] -= h
        fd = (loss(tp) - loss(tm)) / (2 * h)
        assert abs(fd - grad[idx]) < 1e-8, (idx, fd, grad[idx])


# ----------------------------------------------------------------------------- invariants


def test_norm_bounds_and_return_to_zero_state():
    x, theta, _ = random_case(91, 3, 9, 6)
    E, psi = oracle.forward(x, theta, want_state=True)
    np.testing.assert_allclose(np.sum(np.abs(psi) ** 2, axis=1), 1.0, atol=1e-13)
    assert np.all(np.abs(E) <= 1.0 + 1e-14)
    _, _, psi0 = oracle.adjoint(x, theta, np.ones(3), want_state=True)
    ref = np.zeros_like(psi0)
    ref[:, 0] = 1.0
    np.testing.assert_allclose(psi0, ref, atol=1e-12)


@pytest.mark.parametrize("n,L", [(6, 3), (8, 5), (5, 9)])
def test_light_cone_zeros(n, L):
    """A rotation in layer l (0-based) on qubit q cannot reach Z0 if q > L-1-l, and
    the Rz on the edge qubit q = L-1-l only meets Z from the CZ spread.  These
    gradients are zero in exact arithmetic; the fp64 walk leaves ~1e-17."""
    x, theta, _ = random_case(101 + n, 3, n, L)
    grad, _ = oracle.adjoint(x, theta, np.array([0.3, -1.0, 0.7]))
    for l in range(L):
        edge = L - 1 - l
        for q in range(n):
            if q > edge:
                np.testing.assert_allclose(grad[l, q], 0.0, atol=1e-14)
            elif q == edge:
                assert abs(grad[l, q, 2]) < 1e-14
                assert np.max(np.abs(grad[l, q, :2])) > 1e-6


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.4028235e38, -3.4028235e38,
                  1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9, 1.0 - 2.0 ** -9], dtype=np.float32),
    ])
    # exact halfway cases: low 16 bits == 0x8000
    halves = (rng.integers(0, 2 ** 15, 500, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32).view(np.float32)
    vals = np.concatenate([vals, halves[np.isfinite(halves)]])
    ours = oracle.bf16_round(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    nan = oracle.bf16_round(np.array([np.nan], dtype=np.float32))
    assert (nan[0] & 0x7F80) == 0x7F80 and (nan[0] & 0x7F) != 0
    back = oracle.bf16_widen(ours)
    np.testing.assert_array_equal(oracle.bf16_round(back), ours)


# ----------------------------------------------------------------------------- Pauli-sum observables
#
# E = <psi|O|psi> for a general observable O (Deep-dive blog §1.2) taken as a sum
# of Pauli strings; lambda_M = dL/dE * O psi_M.  Letter q of a string acts on
# qubit q.

PAULI_OF = {"X": PAULI[0], "Y": PAULI[1], "Z": PAULI[2]}


def dense_observable(obs, n):
    H = np.zeros((1 << n, 1 << n), dtype=complex)
    for c, word in obs:
        M = np.eye(1 << n, dtype=complex)
        for q, ch in enumerate(word):
            if ch != "I":
                M = dense_on(PAULI_OF[ch], q, n) @ M
        H += c * M
    return H


def random_observable(rng, n, terms):
    obs = []
    for _ in range(terms):
        word = "".join(rng.choice(list("IXYZ"), size=n))
        obs.append((float(rng.normal()), word))
    return obs


def test_observable_z0_reproduces_the_default():
    x, theta, y = random_case(11, 3, 5, 3)
    obs = [(1.0, "ZIIII")]
    np.testing.assert_allclose(oracle.forward(x, theta, observable=obs), oracle.forward(x, theta), atol=1e-14)
    g = np.array([0.4, -1.1, 0.25])
    ga, Ea = oracle.adjoint(x, theta, g, observable=obs)
    gb, Eb = oracle.adjoint(x, theta, g)
    np.testing.assert_allclose(ga, gb, atol=1e-14)
    np.testing.assert_allclose(Ea, Eb, atol=1e-14)


def test_observable_product_state_closed_forms():
    """L = 0: qubit q is Ry(x_q)|0>, Bloch vector (sin x_q, 0, cos x_q), and the
    qubits are uncorrelated, so a Pauli string's value is the product of the
    per-qubit components."""
    x = np.array([[0.3, 1.1, 2.0, 0.7]])
    th = np.zeros((0, 4, 3))
    bloch = {"I": np.ones(4), "X": np.sin(x[0]), "Y": np.zeros(4), "Z": np.cos(x[0])}
    for word in ["XIII", "IYII", "IIZI", "ZZII", "XIZI", "IXXZ", "YIIX", "ZXZX", "IIII"]:
        want = np.prod([bloch[ch][q] for q, ch in enumerate(word)])
        got = oracle.forward(x, th, observable=[(1.0, word)])[0]
        assert abs(got - want) < 1e-14, word


@pytest.mark.parametrize("n,L,seed", [(1, 2, 21), (2, 2, 22), (3, 3, 23), (4, 2, 24), (5, 2, 25)])
def test_observable_dense_brute_force(n, L, seed):
    rng = np.random.default_rng(seed)
    x, theta, y = random_case(seed, 2, n, L)
    obs = random_observable(rng, n, 4)
    H = dense_observable(obs, n)
    assert np.allclose(H, H.conj().T)

    def dense_fwd(xx, tt):
        out = []
        for b in range(xx.shape[0]):
            psi = dense_state(xx[b], tt)
            out.append(float(np.real(np.conj(psi) @ (H @ psi))))
        return np.array(out)

    E = oracle.forward(x, theta, observable=obs)
    np.testing.assert_allclose(E, dense_fwd(x, theta), atol=1e-12)
    g = oracle.loss_seed(E, y)
    grad, E2 = oracle.adjoint(x, theta, g, observable=obs)
    np.testing.assert_allclose(E2, E, atol=1e-13)
    want = np.einsum("b,b...->...", g, shift_grad_E(dense_fwd, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-11)


def test_observable_is_linear():
    rng = np.random.default_rng(31)
    x, theta, _ = random_case(31, 3, 6, 3)
    o1, o2 = random_observable(rng, 6, 3), random_observable(rng, 6, 2)
    both = o1 + [(2.0 * c, w) for c, w in o2]
    E1, E2, E12 = (oracle.forward(x, theta, observable=o) for o in (o1, o2, both))
    np.testing.assert_allclose(E12, E1 + 2.0 * E2, atol=1e-13)
    g = np.array([0.3, -0.8, 1.2])
    G1, G2, G12 = (oracle.adjoint(x, theta, g, observable=o)[0] for o in (o1, o2, both))
    np.testing.assert_allclose(G12, G1 + 2.0 * G2, atol=1e-12)


def test_observable_parameter_shift():
    rng = np.random.default_rng(41)
    x, theta, y = random_case(41, 2, 7, 2)
    obs = random_observable(rng, 7, 6) + [(0.5, "XXIIIIZ")]
    E = oracle.forward(x, theta, observable=obs)
    g = oracle.loss_seed(E, y)
    grad, _ = oracle.adjoint(x, theta, g, observable=obs)
    fwd = lambda xx, tt: oracle.forward(xx, tt, observable=obs)
    want = np.einsum("b,b...->...", g, shift_grad_E(fwd, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-10)


def test_observable_rejects_bad_words():
    x, theta, _ = random_case(1, 1, 3, 1)
    for bad in [[(1.0, "ZZ")], [(1.0, "ZQI")]]:
        with pytest.raises(ValueError):
            oracle.forward(x, theta, observable=bad)


@pytest.mark.parametrize("n,L", [(1, 3), (2, 4), (6, 5)])
def test_zero_angles_gradient_closed_form(n, L):
    """theta = 0: only layer l's Ry on qubit 0 has a derivative, -sin x0 dephased
    by <Z1> = cos x1 for an odd number of preceding CZ(0, 1) (CZ^2 = I)."""
    x, _, _ = random_case(60 + n, 3, n, 1)
    grad, E = oracle.adjoint(x, np.zeros((L, n, 3)), np.ones(3))
    want = np.zeros((L, n, 3))
    for l in range(L):
        f = np.cos(x[:, 1]) ** (l % 2) if n > 1 else 1.0
        want[l, 0, 1] = np.sum(-np.sin(x[:, 0]) * f)
    np.testing.assert_allclose(grad, want, atol=1e-13)
    np.testing.assert_allclose(E, np.cos(x[:, 0]), atol=1e-14)


# ----------------------------------------------------------------------------- entanglers
#
# Every layer ends with CZ on each bond of a list (the default is the chain
# (q, q+1)); CZ gates are diagonal, so any bond graph keeps the fused-pass
# structure.


def dense_state_bonds(x, theta, bonds):
    n = x.shape[0]
    psi = np.zeros(1 << n, dtype=complex)
    psi[0] = 1
    for q in range(n):
        psi = dense_on(dense_rot(1, x[q]), q, n) @ psi
    for l in range(theta.shape[0]):
        for q in range(n):
            for a in range(3):
                psi = dense_on(dense_rot(a, theta[l, q, a]), q, n) @ psi
        for a, b in bonds:
            psi = dense_cz(a, b, n) @ psi
    return psi


def random_bonds(rng, n, count):
    pairs = [(a, b) for a in range(n) for b in range(a + 1, n)]
    idx = rng.choice(len(pairs), size=min(count, len(pairs)), replace=False)
    return [tuple(int(v) for v in (pairs[i] if rng.random() < 0.5 else pairs[i][::-1])) for i in idx]


def test_explicit_chain_equals_the_default():
    x, theta, _ = random_case(5, 3, 6, 3)
    chain = [(q, q + 1) for q in range(5)]
    np.testing.assert_allclose(oracle.forward(x, theta, bonds=chain), oracle.forward(x, theta), atol=1e-15)
    g = np.array([0.2, 0.5, -0.9])
    np.testing.assert_allclose(oracle.adjoint(x, theta, g, bonds=chain)[0], oracle.adjoint(x, theta, g)[0],
                               atol=1e-15)


@pytest.mark.parametrize("n,L,seed", [(2, 3, 71), (3, 2, 72), (4, 3, 73), (5, 2, 74)])
def test_random_bond_graph_dense_brute_force(n, L, seed):
    rng = np.random.default_rng(seed)
    bonds = random_bonds(rng, n, n + 1)
    x, theta, y = random_case(seed, 2, n, L)
    Z0 = dense_on(PAULI[2], 0, n)

    def dense_fwd(xx, tt):
        return np.array([float(np.real(np.conj(p) @ (Z0 @ p)))
                         for p in (dense_state_bonds(xx[b], tt, bonds) for b in range(xx.shape[0]))])

    E = oracle.forward(x, theta, bonds=bonds)
    np.testing.assert_allclose(E, dense_fwd(x, theta), atol=1e-12)
    g = oracle.loss_seed(E, y)
    grad, _ = oracle.adjoint(x, theta, g, bonds=bonds)
    want = np.einsum("b,b...->...", g, shift_grad_E(dense_fwd, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-11)


def test_no_entangler_is_a_product_of_bloch_rotations():
    x, theta, _ = random_case(9, 2, 4, 5)
    E = oracle.forward(x, theta, bonds=[])
    for b in range(2):
        v = np.array([np.sin(x[b, 0]), 0.0, np.cos(x[b, 0])])
        for l in range(5):
            v = bloch_layer(v, theta[l, 0])
        assert abs(E[b] - v[2]) < 1e-13


@pytest.mark.parametrize("n,L", [(4, 3), (6, 4)])
def test_ring_zero_angle_gradient_closed_form(n, L):
    """theta = 0 with a ring (chain plus CZ(n-1, 0)): qubit 0's Bloch x component
    is dephased by cos x1 cos x_{n-1} once per odd number of preceding layers."""
    ring = [(q, q + 1) for q in range(n - 1)] + [(n - 1, 0)]
    x, _, _ = random_case(80 + n, 3, n, 1)
    grad, E = oracle.adjoint(x, np.zeros((L, n, 3)), np.ones(3), bonds=ring)
    want = np.zeros((L, n, 3))
    for l in range(L):
        f = (np.cos(x[:, 1]) * np.cos(x[:, n - 1])) ** (l % 2)
        want[l, 0, 1] = np.sum(-np.sin(x[:, 0]) * f)
    np.testing.assert_allclose(grad, want, atol=1e-13)
    np.testing.assert_allclose(E, np.cos(x[:, 0]), atol=1e-14)


# ----------------------------------------------------------------------------- data re-uploading
#
# Every layer starts with the angle encoding Ry(x_q) on every qubit again.


def dense_state_reupload(x, theta):
    n = x.shape[0]
    psi = np.zeros(1 << n, dtype=complex)
    psi[0] = 1
    enc = lambda p: [p := dense_on(dense_rot(1, x[q]), q, n) @ p for q in range(n)][-1]
    psi = enc(psi)
    for l in range(theta.shape[0]):
        psi = enc(psi)
        for q in range(n):
            for a in range(3):
                psi = dense_on(dense_rot(a, theta[l, q, a]), q, n) @ psi
        for q in range(n - 1):
            psi = dense_cz(q, q + 1, n) @ psi
    return psi


def test_reupload_one_layer_closed_form():
    """One layer: qubit 0 sees Ry(x0) twice = Ry(2 x0), then Rx(a) Ry(b)."""
    x, theta, _ = random_case(17, 4, 5, 1)
    a, b = theta[0, 0, 0], theta[0, 0, 1]
    want = np.cos(2 * x[:, 0]) * np.cos(a) * np.cos(b) - np.sin(2 * x[:, 0]) * np.sin(b)
    np.testing.assert_allclose(oracle.forward(x, theta, reupload=True), want, atol=1e-14)


@pytest.mark.parametrize("n,L,seed", [(1, 3, 91), (3, 2, 92), (4, 3, 93)])
def test_reupload_dense_brute_force(n, L, seed):
    x, theta, y = random_case(seed, 2, n, L)
    Z0 = dense_on(PAULI[2], 0, n)

    def dense_fwd(xx, tt):
        return np.array([float(np.real(np.conj(p) @ (Z0 @ p)))
                         for p in (dense_state_reupload(xx[b], tt) for b in range(xx.shape[0]))])

    E = oracle.forward(x, theta, reupload=True)
    np.testing.assert_allclose(E, dense_fwd(x, theta), atol=1e-12)
    g = oracle.loss_seed(E, y)
    grad, _ = oracle.adjoint(x, theta, g, reupload=True)
    want = np.einsum("b,b...->...", g, shift_grad_E(dense_fwd, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-11)


def test_reupload_returns_to_the_zero_state():
    x, theta, _ = random_case(19, 2, 7, 4)
    _, _, psi0 = oracle.adjoint(x, theta, np.ones(2), want_state=True, reupload=True)
    ref = np.zeros_like(psi0)
    ref[:, 0] = 1.0
    np.testing.assert_allclose(psi0, ref, atol=1e-12)


# ---------------------------------------------------------------------------
# CNOT entanglers: every layer ends with CNOT(control, target) on each pair of
# a list, in list order (the pages name CNOT gates as the other entangler their
# kernels fuse).  Pinned by a dense CNOT built from projectors, by the exact
# action on computational basis states (a CNOT ladder maps bit k to the XOR of
# bits 0..k) and by the parameter-shift rule.


def dense_cnot(c, t, n):
    """|0><0|_c (x) I + |1><1|_c (x) X_t, as a 2^n matrix."""
    p0 = np.array([[1, 0], [0, 0]], dtype=complex)
    p1 = np.array([[0, 0], [0, 1]], dtype=complex)
    return dense_on(p0, c, n) + dense_on(p1, c, n) @ dense_on(PAULI[0], t, n)


def dense_state_cnot(x, theta, pairs):
    n = x.shape[0]
    psi = np.zeros(1 << n, dtype=complex)
    psi[0] = 1
    for q in range(n):
        psi = dense_on(dense_rot(1, x[q]), q, n) @ psi
    for l in range(theta.shape[0]):
        for q in range(n):
            for a in range(3):
                psi = dense_on(dense_rot(a, theta[l, q, a]), q, n) @ psi
        for c, t in pairs:
            psi = dense_cnot(c, t, n) @ psi
    return psi


@pytest.mark.parametrize("n,L,seed,kind", [(2, 3, 81, "ladder"), (3, 2, 82, "ladder"), (4, 3, 83, "ring"),
                                           (5, 2, 84, "random")])
def test_cnot_dense_brute_force(n, L, seed, kind):
    rng = np.random.default_rng(seed)
    if kind == "ladder":
        pairs = [(q, q + 1) for q in range(n - 1)]
    elif kind == "ring":
        pairs = [(q, (q + 1) % n) for q in range(n)]
    else:
        pairs = random_bonds(rng, n, n + 1)
    x, theta, y = random_case(seed, 2, n, L)
    Z0 = dense_on(PAULI[2], 0, n)

    def dense_fwd(xx, tt):
        return np.array([float(np.real(np.conj(p) @ (Z0 @ p)))
                         for p in (dense_state_cnot(xx[b], tt, pairs) for b in range(xx.shape[0]))])

    E, psi = oracle.forward(x, theta, want_state=True, bonds=pairs, entangler="cnot")
    np.testing.assert_allclose(psi[0], dense_state_cnot(x[0], theta, pairs), atol=1e-12)
    np.testing.assert_allclose(E, dense_fwd(x, theta), atol=1e-12)
    g = oracle.loss_seed(E, y)
    grad, _ = oracle.adjoint(x, theta, g, bonds=pairs, entangler="cnot")
    want = np.einsum("b,b...->...", g, shift_grad_E(dense_fwd, x, theta))
    np.testing.assert_allclose(grad, want, atol=1e-11)


@pytest.mark.parametrize("n,L", [(3, 1), (5, 2), (7, 3)])
def test_cnot_ladder_on_basis_states(n, L):
    """x in {0, pi} encodes a basis state (Ry(pi)|0> = |1>); with theta = 0 each
    ladder layer replaces bit k by the XOR of bits 0..k."""
    rng = np.random.default_rng(90 + n)
    bits = rng.integers(0, 2, size=(4, n))
    x = bits * np.pi
    theta = np.zeros((L, n, 3))
    pairs = [(q, q + 1) for q in range(n - 1)]
    _, psi = oracle.forward(x, theta, want_state=True, bonds=pairs, entangler="cnot")
    for b in range(4):
        v = list(bits[b])
        for _ in range(L):
            v = [int(np.bitwise_xor.reduce(v[:k + 1])) for k in range(n)]
        want = sum(bit << k for k, bit in enumerate(v))
        assert abs(abs(psi[b, want]) - 1.0) < 1e-12
        assert np.sum(np.abs(psi[b]) ** 2) - abs(psi[b, want]) ** 2 < 1e-24


def test_cnot_control_and_target_are_not_interchangeable():
    """CNOT(0, 1) on |01> (qubit 0 set) gives |11>; CNOT(1, 0) leaves it."""
    x = np.array([[np.pi, 0.0]])
    theta = np.zeros((1, 2, 3))
    _, a = oracle.forward(x, theta, want_state=True, bonds=[(0, 1)], entangler="cnot")
    _, b = oracle.forward(x, theta, want_state=True, bonds=[(1, 0)], entangler="cnot")
    assert abs(abs(a[0, 3]) - 1) < 1e-12 and abs(abs(b[0, 1]) - 1) < 1e-12


def test_cnot_returns_to_the_zero_state():
    x, theta, y = random_case(95, 3, 6, 4)
    pairs = [(q, q + 1) for q in range(5)]
    E = oracle.forward(x, theta, bonds=pairs, entangler="cnot")
    _, _, psi0 = oracle.adjoint(x, theta, oracle.loss_seed(E, y), want_state=True, bonds=pairs, entangler="cnot")
    assert np.max(np.abs(psi0[:, 0] - 1)) < 1e-12 and np.max(np.abs(psi0[:, 1:])) < 1e-12
