"""CPU checks of the algebra and layout facts behind the flip-tracked rotations
of the split-form tensor-copy passes (no GPU).

The split form applies every rotation Ry as the tangent form T(t) = [[1, -t],
[t, 1]] = Ry / cos, or as the cotangent form C(u) = [[-u, 1], [1, u]].  The
tensor-copy passes apply C(u) as T(-u) followed by a flip X of the qubit's
register bit that is not carried out (register j then holds position j ^ f),
and rely on:
  * C(u) = X T(-u);
  * X T(t) X = T(-t): a later rotation of a flipped bit negates its
    coefficient;
  * X Y X = -Y and X Z X = -Z, X X X = X: the backward sums of a flipped bit's
    qubit, Im<l|P|p> taken on the flipped state, negate their y and z parts;
  * the in-place update x <- x - t y, then y <- t x' + (1 + t^2) y, is T(t);
  * a diagonal op on the flipped state reads its factor at j ^ f;
  * in the layouts the tensor-copy passes exchange between (phases 0 and 1),
    every register bit of one layout is a thread bit of the other, so an
    exchange resolves every pending flip by moving the reading thread's slot
    base; in the warp-local exchanges those thread bits are lane bits.
"""
import numpy as np
import pytest

from adjoint_gradients_b200 import qml

X = np.array([[0, 1], [1, 0]], dtype=complex)
Y = np.array([[0, -1j], [1j, 0]], dtype=complex)
Z = np.array([[1, 0], [0, -1]], dtype=complex)


def T(t):
    return np.array([[1, -t], [t, 1]], dtype=complex)


def C(u):
    return np.array([[-u, 1], [1, u]], dtype=complex)


@pytest.mark.parametrize("u", [0.0, 0.3, -0.7, 1.0])
def test_cotangent_form_is_flip_after_tangent_form(u):
    assert np.allclose(C(u), X @ T(-u))


@pytest.mark.parametrize("t", [0.0, 0.25, -0.9, 1.0])
def test_flip_negates_the_tangent_coefficient(t):
    assert np.allclose(X @ T(t) @ X, T(-t))


def test_flip_conjugation_of_the_generators():
    assert np.allclose(X @ X @ X, X)
    assert np.allclose(X @ Y @ X, -Y)
    assert np.allclose(X @ Z @ X, -Z)


def test_sums_on_a_flipped_state():
    """Im<l|P|p> on the flipped pair (X l, X p): s_x kept, s_y and s_z negated."""
    rng = np.random.default_rng(7)
    p = rng.normal(size=2) + 1j * rng.normal(size=2)
    lam = rng.normal(size=2) + 1j * rng.normal(size=2)
    s = [np.imag(np.vdot(lam, P @ p)) for P in (X, Y, Z)]
    sf = [np.imag(np.vdot(X @ lam, P @ (X @ p))) for P in (X, Y, Z)]
    assert np.allclose(sf, [s[0], -s[1], -s[2]])


@pytest.mark.parametrize("t", [0.0, 0.5, -0.8, 1.0])
def test_in_place_update_is_the_tangent_form(t):
    rng = np.random.default_rng(3)
    x, y = rng.normal(size=2) + 1j * rng.normal(size=2)
    x2 = x - t * y
    y2 = t * x2 + (1 + t * t) * y
    assert np.allclose([x2, y2], T(t) @ np.array([x, y]))


def test_diagonal_on_a_flipped_register_index():
    """D X^f = X^f D' with D'(j) = D(j ^ f) on a 5-bit register index."""
    rng = np.random.default_rng(5)
    d = np.exp(1j * rng.uniform(0, 2 * np.pi, 32))
    psi = rng.normal(size=32) + 1j * rng.normal(size=32)
    for f in (0, 1, 6, 19, 31):
        stored = psi[np.arange(32) ^ f]  # register j holds position j ^ f
        applied = d[np.arange(32) ^ f] * stored
        assert np.allclose(applied, (d * psi)[np.arange(32) ^ f])


def test_register_bits_of_phase_0_and_1_are_thread_bits_of_the_other():
    d = qml.debug_layouts()
    lay = d["layouts"]
    for V in (0, 1):
        for x, y in ((0, 1), (1, 0)):
            if (x, V) not in lay or (y, V) not in lay:
                continue
            thr_y, reg_y = lay[(y, V)]
            _, reg_x = lay[(x, V)]
            for t in reg_x:
                assert t in thr_y and t not in reg_y, (x, y, V, t)


def test_warp_local_exchange_flips_stay_in_the_warp():
    """Where both layouts take the warp index from tile bits 10 and 11, the
    other layout's register bits are lane bits of the reading layout."""
    d = qml.debug_layouts()
    lay = d["layouts"]
    for V in (0, 1):
        for x, y in ((0, 1), (1, 0)):
            if (x, V) not in lay or (y, V) not in lay:
                continue
            thr_x, reg_x = lay[(x, V)]
            thr_y, _ = lay[(y, V)]
            if thr_x[5:7] == [10, 11] and thr_y[5:7] == [10, 11]:
                for t in reg_x:
                    assert thr_y.index(t) < 5, (x, y, V, t)
