"""Oracle -- TEST INFRASTRUCTURE, not part of the product.

A plain complex128 CPU simulator of the hardware-efficient ansatz and its adjoint
gradient (``qml_oracle.c``), loaded through ctypes.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
package.  The CUDA library never calls it and shares no code with it.

Every function follows the definitions printed on the summaries of Kawase,
"Fast and memory-efficient classical simulation of quantum machine learning via
forward and backward gate fusion" (arXiv 2603.02804):

* ``forward``  -- E(theta) = <psi_M|O|psi_M>  (Deep-dive blog, §1.2, the E(theta) equation)
  with O = Z0, or a sum of Pauli strings (``observable``)
* ``adjoint``  -- dL/dtheta_j = 2 Re<lambda_j|dU_j/dtheta_j|psi_{j-1}>,
  lambda_{j-1} = U_j^dagger lambda_j  (Deep-dive blog, §1.2, adjoint-gradient equation
  and the lambda recursion; the factor 2 is the derivative of <psi|O|psi>)
* ``bf16_round`` -- IEEE round-to-nearest-even narrowing of fp32 to bfloat16, the
  storage format of the memory-save mode (Gist-EN Technical Summary §2).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qml_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqml_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, IEEE semantics: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=gnu11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.oracle_forward.argtypes = [ctypes.c_int] * 3 + [_dp] * 4
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_adjoint.argtypes = [ctypes.c_int] * 3 + [_dp] * 6
        lib.oracle_adjoint.restype = ctypes.c_int
        lib.oracle_forward_obs.argtypes = [ctypes.c_int] * 3 + [_dp] * 2 + [ctypes.c_int, ctypes.c_char_p] + [_dp] * 3
        lib.oracle_forward_obs.restype = ctypes.c_int
        lib.oracle_adjoint_obs.argtypes = [ctypes.c_int] * 3 + [_dp] * 2 + [ctypes.c_int, ctypes.c_char_p] + [_dp] * 5
        lib.oracle_adjoint_obs.restype = ctypes.c_int
        _ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_forward_gen.argtypes = ([ctypes.c_int] * 3 + [_dp] * 2 + [ctypes.c_int, ctypes.c_int, _ip,
                                           ctypes.c_int, ctypes.c_char_p] + [_dp] * 3)
        lib.oracle_forward_gen.restype = ctypes.c_int
        lib.oracle_adjoint_gen.argtypes = ([ctypes.c_int] * 3 + [_dp] * 2 + [ctypes.c_int, ctypes.c_int, _ip,
                                           ctypes.c_int, ctypes.c_char_p] + [_dp] * 5)
        lib.oracle_adjoint_gen.restype = ctypes.c_int
        lib.oracle_forward_ent.argtypes = ([ctypes.c_int] * 3 + [_dp] * 2 + [ctypes.c_int] * 3 + [_ip,
                                           ctypes.c_int, ctypes.c_char_p] + [_dp] * 3)
        lib.oracle_forward_ent.restype = ctypes.c_int
        lib.oracle_adjoint_ent.argtypes = ([ctypes.c_int] * 3 + [_dp] * 2 + [ctypes.c_int] * 3 + [_ip,
                                           ctypes.c_int, ctypes.c_char_p] + [_dp] * 5)
        lib.oracle_adjoint_ent.restype = ctypes.c_int
        lib.oracle_bf16_round.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t]
        lib.oracle_bf16_widen.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _prep(x, theta):
    x = np.ascontiguousarray(x, dtype=np.float64)
    theta = np.ascontiguousarray(theta, dtype=np.float64)
    if x.ndim != 2 or theta.ndim != 3 or theta.shape[2] != 3:
        raise ValueError("x must be [B][n] and theta [L][n][3]")
    B, n = x.shape
    L = theta.shape[0]
    if L > 0 and theta.shape[1] != n:
        raise ValueError("theta must be [L][n][3] with the same n as x")
    return x, theta, B, n, L


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _observable(observable, n):
    """(term count, Pauli letters, coefficients) of [(coef, "XIZ...")]: letter q of a
    string acts on qubit q."""
    if observable is None:
        return 0, None, None
    letters, coef = [], []
    for c, word in observable:
        if len(word) != n or any(ch not in "IXYZ" for ch in word):
            raise ValueError(f"Pauli string {word!r} must have {n} letters from IXYZ")
        letters.append(word)
        coef.append(float(c))
    return len(coef), "".join(letters).encode(), np.ascontiguousarray(coef, dtype=np.float64)


def _bonds(bonds):
    """(count, int pointer) of an entangler [(a, b), ...] (None: the CZ chain)."""
    if bonds is None:
        return 0, None, None
    arr = np.ascontiguousarray(np.asarray(bonds, dtype=np.int32).reshape(-1, 2))
    return arr.shape[0], arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


_ENTANGLERS = {"cz": 0, "cnot": 1}


def forward(x, theta, want_state: bool = False, observable=None, bonds=None, reupload: bool = False,
            entangler: str = "cz"):
    """<O> per sample (O = Z0, or the Pauli sum ``observable`` = [(coef, word)]), and
    optionally the final states ``[B][2^n]`` complex128.  ``bonds``: the pairs
    of every layer's entangler, applied in list order (None: the chain q, q+1);
    ``entangler``: "cz", or "cnot" (each pair is (control, target)).
    ``reupload``: every layer starts with the encoding Ry(x_q) again."""
    x, theta, B, n, L = _prep(x, theta)
    E = np.zeros(B, dtype=np.float64)
    psi = np.zeros((B, 1 << n, 2), dtype=np.float64) if want_state else None
    k, words, coef = _observable(observable, n)
    nb, keep, bp = _bonds(bonds)
    rc = _load().oracle_forward_ent(n, L, B, _ptr(x), _ptr(theta), int(reupload), _ENTANGLERS[entangler], nb, bp,
                                    k, words, _ptr(coef), _ptr(E), _ptr(psi))
    if rc != 0:
        raise RuntimeError("oracle_forward_ent failed")
    if want_state:
        return E, psi[..., 0] + 1j * psi[..., 1]
    return E


def adjoint(x, theta, g, want_state: bool = False, observable=None, bonds=None, reupload: bool = False,
            entangler: str = "cz"):
    """sum_b g_b dE_b/dtheta as ``[L][n][3]``, <O> per sample, and optionally the
    state after walking the circuit back to its start (must be |0...0>)."""
    x, theta, B, n, L = _prep(x, theta)
    g = np.ascontiguousarray(g, dtype=np.float64)
    if g.shape != (B,):
        raise ValueError("g must be [B]")
    grad = np.zeros((L, n, 3), dtype=np.float64)
    E = np.zeros(B, dtype=np.float64)
    psi0 = np.zeros((B, 1 << n, 2), dtype=np.float64) if want_state else None
    k, words, coef = _observable(observable, n)
    nb, keep, bp = _bonds(bonds)
    rc = _load().oracle_adjoint_ent(n, L, B, _ptr(x), _ptr(theta), int(reupload), _ENTANGLERS[entangler], nb, bp,
                                    k, words, _ptr(coef), _ptr(g), _ptr(grad), _ptr(E), _ptr(psi0))
    if rc != 0:
        raise RuntimeError("oracle_adjoint_ent failed")
    if want_state:
        return grad, E, psi0[..., 0] + 1j * psi0[..., 1]
    return grad, E


def loss_seed(E, y):
    """g_b = dL/dE_b for L = mean_b (E_b - y_b)^2."""
    E = np.asarray(E, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return 2.0 * (E - y) / E.shape[0]


def bf16_round(a) -> np.ndarray:
    """fp32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_bf16_round(a.ctypes.data, out.ctypes.data, a.size)
    return out


def bf16_widen(u) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> fp32 (exact)."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    out = np.empty(u.shape, dtype=np.float32)
    _load().oracle_bf16_widen(u.ctypes.data, out.ctypes.data, u.size)
    return out
