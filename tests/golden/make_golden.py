"""Write the stored expected values used by the full-size GPU parity tests.

Every number here comes from the CPU oracle (oracle/) on the seeded workload
inputs (adjoint_gradients_b200/inputs.py); nothing comes from the CUDA path.

    python tests/golden/make_golden.py [name ...]

Files (numpy .npz, float64):
  hea_20q_L100.npz      E of samples 0-3 and dE_0/dtheta (100 x 20 x 3)
  deep_20q_L1000.npz    E of sample 0 and dE_0/dtheta (1000 x 20 x 3); samples
                        0 of the batch-60 and batch-85 workloads are the same
                        draw, so one file serves both storage modes
  wide_29q_L20.npz      E of samples 0-3 and dE_0/dtheta (20 x 29 x 3) of the
                        29-qubit circuit, computed on its first 20 qubits: after
                        L layers the Heisenberg-evolved Z0 is supported on
                        qubits 0 .. L-1 (each CZ ladder widens the support by one
                        qubit and CZ(L-1, L) never meets it), so the 29-qubit
                        <Z0> and gradients equal those of the truncated circuit,
                        and the gradients on qubits >= L are exactly zero.
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from adjoint_gradients_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def one_hot(B, i=0):
    g = np.zeros(B)
    g[i] = 1.0
    return g


def hea_20q_L100():
    w = WORKLOADS["hea_20q_L100"]
    x, theta, _ = make_inputs(w)
    E = oracle.forward(x[:4], theta)
    grad, E0 = oracle.adjoint(x[:1], theta, one_hot(1))
    assert abs(E0[0] - E[0]) < 1e-12
    return dict(E=E, grad0=grad, n=w.n, L=w.L, samples=np.arange(4))


def deep_20q_L1000():
    w = WORKLOADS["deep_20q_L1000_fp32"]
    x, theta, _ = make_inputs(w)
    x85, theta85, _ = make_inputs(WORKLOADS["deep_20q_L1000_bf16"])
    assert np.array_equal(x85[:60], x) and np.array_equal(theta85, theta)
    grad, E = oracle.adjoint(x[:1], theta, one_hot(1))
    return dict(E=E, grad0=grad, n=w.n, L=w.L, samples=np.arange(1))


def wide_29q_L20():
    w = WORKLOADS["wide_29q_L20"]
    x, theta, _ = make_inputs(w)
    keep = w.L  # qubits 0 .. L-1 carry the light cone of Z0
    E = oracle.forward(x[:, :keep], theta[:, :keep, :])
    g_small, _ = oracle.adjoint(x[:1, :keep], theta[:, :keep, :], one_hot(1))
    grad = np.zeros((w.L, w.n, 3))
    grad[:, :keep, :] = g_small
    return dict(E=E, grad0=grad, n=w.n, L=w.L, samples=np.arange(w.B))


JOBS = {"hea_20q_L100": hea_20q_L100, "deep_20q_L1000": deep_20q_L1000, "wide_29q_L20": wide_29q_L20}


def main(names):
    for name in names or JOBS:
        t0 = time.time()
        data = JOBS[name]()
        np.savez_compressed(os.path.join(HERE, name + ".npz"), **data)
        print(f"{name}: {time.time() - t0:.0f} s, E={np.array2string(data['E'], precision=6)}", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
