"""Seeded synthetic inputs for the HEA workloads.

This module only draws random numbers and names the workload sizes; it holds none
of the simulation's arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from it.

Recipe (one numpy PCG64 generator per array, seeded per workload index ``c``):
  x     ~ U[0, pi)   shape [B][n]      seed 1000 + c   (angle-encoding features)
  theta ~ U[0, 2pi)  shape [L][n][3]   seed 2000 + c   (Rx, Ry, Rz angles per qubit per layer)
  y     ~ {-1, +1}   shape [B]         seed 3000 + c   (uniform labels)
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    n: int          # qubits
    L: int          # layers
    B: int          # samples per call (mini-batch)
    ckpt_block: int  # layers per checkpoint block (0 = no checkpoints)
    storage: str    # "fp32" or "bf16" checkpoint storage
    samples_per_epoch: int = 0

    @property
    def params(self) -> int:
        return self.L * self.n * 3


# The five HEA workloads: tiny, 12-qubit, 20-qubit/100-layer (headline),
# 20-qubit/1000-layer (two storage modes), 29-qubit/20-layer.
WORKLOADS = {
    "tiny_4q_L2": Workload(0, "tiny_4q_L2", 4, 2, 8, 0, "fp32"),
    "hea_12q_L10": Workload(1, "hea_12q_L10", 12, 10, 256, 0, "fp32"),
    "hea_20q_L100": Workload(2, "hea_20q_L100", 20, 100, 64, 10, "fp32"),
    "deep_20q_L1000_fp32": Workload(3, "deep_20q_L1000_fp32", 20, 1000, 60, 20, "fp32", 1000),
    "deep_20q_L1000_bf16": Workload(3, "deep_20q_L1000_bf16", 20, 1000, 85, 20, "bf16", 1000),
    "wide_29q_L20": Workload(4, "wide_29q_L20", 29, 20, 4, 10, "bf16"),
}


def draw_x(c: int, B: int, n: int) -> np.ndarray:
    return np.random.default_rng(1000 + c).uniform(0.0, np.pi, size=(B, n))


def draw_theta(c: int, L: int, n: int) -> np.ndarray:
    return np.random.default_rng(2000 + c).uniform(0.0, 2.0 * np.pi, size=(L, n, 3))


def draw_y(c: int, B: int) -> np.ndarray:
    return np.random.default_rng(3000 + c).integers(0, 2, size=B).astype(np.float64) * 2.0 - 1.0


def make_inputs(w: Workload, B: int | None = None):
    """(x [B][n], theta [L][n][3], y [B]) in float64 for workload ``w``."""
    B = w.B if B is None else B
    return draw_x(w.index, B, w.n), draw_theta(w.index, w.L, w.n), draw_y(w.index, B)


def random_case(seed: int, B: int, n: int, L: int):
    """A free-form seeded case (for tests): x, theta, y as above from one seed."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(0.0, np.pi, size=(B, n))
    theta = rng.uniform(0.0, 2.0 * np.pi, size=(L, n, 3))
    y = rng.integers(0, 2, size=B).astype(np.float64) * 2.0 - 1.0
    return x, theta, y
