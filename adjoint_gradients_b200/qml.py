"""ctypes binding of libqml (include/qml.h).

Argument marshalling only: torch tensors provide device memory and streams, every
step of the simulation runs in the library's CUDA kernels.  If the compiled
library is missing this module raises immediately; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# QML_LIBRARY: the path of another build of the library (e.g. one made with other
# compile flags); the in-tree build by default
LIB_PATH = os.environ.get("QML_LIBRARY") or os.path.join(_HERE, "libqml.so")

QML_OK = 0
STATUS_NAMES = {
    0: "QML_OK", 1: "QML_ERR_INVALID_ARG", 2: "QML_ERR_UNSUPPORTED", 3: "QML_ERR_WORKSPACE",
    4: "QML_ERR_CUDA", 5: "QML_ERR_CKPT_MISMATCH", 6: "QML_ERR_NUMERIC", 7: "QML_ERR_BOUNDS",
    8: "QML_ERR_TIMEOUT",
}
STORAGE = {"fp32": 0, "bf16": 1, "fp64": 2}
PRECISION = ("fp32", "fp64")

# every function include/qml.h declares
EXPORTS = [
    "qml_abi_version", "qml_status_str", "qml_create", "qml_destroy", "qml_workspace_bytes",
    "qml_set_workspace", "qml_init_state_encode", "qml_forward_expect", "qml_backward_adjoint",
    "qml_loss_seed", "qml_ckpt_save", "qml_ckpt_restore", "qml_num_ckpt_slots", "qml_expect_z0",
    "qml_host_workspace_bytes", "qml_step_host", "qml_sync", "qml_debug_schedule",
    "qml_enable_timing", "qml_read_timing", "qml_launch_count", "qml_expect_z0_static",
    "qml_debug_tile_view", "qml_debug_layouts", "qml_set_observable", "qml_observable_terms",
    "qml_expect_observable", "qml_set_entangler", "qml_entangler_bonds", "qml_set_reupload", "qml_reupload",
    "qml_create_f64", "qml_precision", "qml_forward_expect_f64", "qml_backward_adjoint_f64", "qml_loss_seed_f64",
    "qml_step_host_f64", "qml_set_entangler_cnot", "qml_entangler_kind", "qml_debug_entangler_map",
    "qml_split_form", "qml_measure_fma_peak",
]


def measure_fma_peak(fp64: bool, iters: int = 200000, stream=None) -> tuple[float, float]:
    """(TFLOP/s, launch ms) of independent FMA chains on the current device
    (qml_measure_fma_peak): DFMA when fp64, else the packed f32x2 FMA."""
    lib = load_library()
    tf = ctypes.c_double()
    ms = ctypes.c_float()
    _check(lib.qml_measure_fma_peak(1 if fp64 else 0, iters, _stream_handle(stream), ctypes.byref(tf),
                                    ctypes.byref(ms)), "qml_measure_fma_peak")
    return tf.value, ms.value


def debug_layouts() -> dict:
    """The kernels' register layouts (see qml_debug_layouts in include/qml.h)."""
    lib = load_library()
    need = lib.qml_debug_layouts(None, 0)
    buf = (ctypes.c_int * need)()
    lib.qml_debug_layouts(buf, need)
    v = list(buf)
    lay = {}
    k = 0
    for P in range(3):
        for V in range(2):
            lay[(P, V)] = (v[k:k + 7], v[k + 7:k + 12])
            k += 12
    return dict(layouts=lay, weights=v[k:k + 12], slots=v[k + 12], weights8=v[k + 13:k + 25], slots8=v[k + 25])


class QmlError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")


class _Config(ctypes.Structure):
    _fields_ = [("n_qubits", ctypes.c_int), ("n_layers", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("ckpt_block", ctypes.c_int), ("storage", ctypes.c_int)]


_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int


def load_library(path: str = LIB_PATH):
    """Load libqml.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libqml.so not found at {path}: run `python -m adjoint_gradients_b200.build`")
    lib = ctypes.CDLL(path)
    sig = {
        "qml_abi_version": ([], _i),
        "qml_status_str": ([_i], ctypes.c_char_p),
        "qml_create": ([ctypes.POINTER(_Config), _i, ctypes.POINTER(_vp)], _i),
        "qml_destroy": ([_vp], _i),
        "qml_workspace_bytes": ([_vp, _i], ctypes.c_size_t),
        "qml_host_workspace_bytes": ([_vp, _i], ctypes.c_size_t),
        "qml_set_workspace": ([_vp, _vp, ctypes.c_size_t, _vp], _i),
        "qml_init_state_encode": ([_vp, _vp, _i, _vp, _vp], _i),
        "qml_forward_expect": ([_vp, _vp, _vp, _i, _vp, _vp, _vp], _i),
        "qml_backward_adjoint": ([_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp], _i),
        "qml_loss_seed": ([_vp, _vp, _vp, _i, _vp, _vp, _vp], _i),
        "qml_ckpt_save": ([_vp, _i, _vp, _i, _vp], _i),
        "qml_ckpt_restore": ([_vp, _i, _vp, _i, _vp], _i),
        "qml_num_ckpt_slots": ([_vp], _i),
        "qml_expect_z0": ([_vp, _vp, _i, _vp, _vp], _i),
        "qml_step_host": ([_vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp], _i),
        "qml_sync": ([_vp, _vp], _i),
        "qml_debug_schedule": ([_vp, ctypes.POINTER(_i), _i], _i),
        "qml_enable_timing": ([_vp, _i], _i),
        "qml_read_timing": ([_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong),
                             ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)], _i),
        "qml_launch_count": ([_vp], ctypes.c_longlong),
        "qml_expect_z0_static": ([_vp, _i, _i, _vp, _vp], _i),
        "qml_debug_tile_view": ([_vp, _i, ctypes.POINTER(_i), _i], _i),
        "qml_debug_layouts": ([ctypes.POINTER(_i), _i], _i),
        "qml_set_observable": ([_vp, _i, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)], _i),
        "qml_observable_terms": ([_vp], _i),
        "qml_expect_observable": ([_vp, _vp, _i, _vp, _vp], _i),
        "qml_set_entangler": ([_vp, _i, ctypes.POINTER(_i)], _i),
        "qml_entangler_bonds": ([_vp], _i),
        "qml_set_reupload": ([_vp, _i], _i),
        "qml_reupload": ([_vp], _i),
        "qml_split_form": ([_vp], _i),
        "qml_measure_fma_peak": ([_i, _i, _vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_float)], _i),
        "qml_create_f64": ([ctypes.POINTER(_Config), _i, ctypes.POINTER(_vp)], _i),
        "qml_precision": ([_vp], _i),
        "qml_forward_expect_f64": ([_vp, _vp, _vp, _i, _vp, _vp, _vp], _i),
        "qml_backward_adjoint_f64": ([_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp], _i),
        "qml_loss_seed_f64": ([_vp, _vp, _vp, _i, _vp, _vp, _vp], _i),
        "qml_step_host_f64": ([_vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp], _i),
        "qml_set_entangler_cnot": ([_vp, _i, ctypes.POINTER(_i)], _i),
        "qml_entangler_kind": ([_vp], _i),
        "qml_debug_entangler_map": ([_vp, ctypes.POINTER(_i), _i], _i),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _check(code: int, what: str):
    if code != QML_OK:
        raise QmlError(code, what)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


@dataclass
class StepResult:
    expect: object
    loss: object
    grad: object


class Context:
    """One circuit shape (n qubits, L layers) on one CUDA device.

    Complex states are torch float32 tensors of shape [B, 2^n, 2] (re, im), or
    complex64 tensors of shape [B, 2^n]; with precision="fp64" float64
    [B, 2^n, 2] or complex128 [B, 2^n], and float64 inputs and outputs.
    """

    def __init__(self, n_qubits: int, n_layers: int, max_batch: int, ckpt_block: int = 0,
                 storage: str = "fp32", device: int = 0, host_step: bool = False, workspace=True,
                 precision: str = "fp32"):
        if precision not in PRECISION:
            raise ValueError(f"precision must be one of {PRECISION}")
        self.lib = load_library()
        self.n, self.L, self.max_batch = n_qubits, n_layers, max_batch
        self.ckpt_block, self.storage, self.device = ckpt_block, storage, device
        self.precision = precision
        self.f64 = precision == "fp64"
        cfg = _Config(n_qubits, n_layers, max_batch, ckpt_block, STORAGE[storage])
        h = _vp()
        create = self.lib.qml_create_f64 if self.f64 else self.lib.qml_create
        _check(create(ctypes.byref(cfg), device, ctypes.byref(h)), "qml_create_f64" if self.f64 else "qml_create")
        self._h = h
        self.ws = None
        self._host_step = host_step
        if workspace:
            self.allocate_workspace(host_step=host_step)

    # ----------------------------------------------------------------- admin
    def close(self):
        if getattr(self, "_h", None):
            self.lib.qml_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, host_step: bool = False) -> int:
        f = self.lib.qml_host_workspace_bytes if host_step else self.lib.qml_workspace_bytes
        return int(f(self._h, self.max_batch))

    def allocate_workspace(self, host_step: bool = False, stream=None):
        import torch

        self._host_step = host_step
        nbytes = self.workspace_bytes(host_step)
        self.ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=f"cuda:{self.device}")
        base = self.ws.data_ptr()
        aligned = (base + 255) // 256 * 256
        _check(self.lib.qml_set_workspace(self._h, aligned, nbytes, _stream_handle(stream)), "qml_set_workspace")

    @property
    def num_ckpt_slots(self) -> int:
        return int(self.lib.qml_num_ckpt_slots(self._h))

    def debug_schedule(self) -> list[int]:
        need = self.lib.qml_debug_schedule(self._h, None, 0)
        buf = (ctypes.c_int * need)()
        self.lib.qml_debug_schedule(self._h, buf, need)
        return list(buf)

    def set_observable(self, observable=None):
        """Observable for the following calls: None (Z0) or [(coef, word)], where
        letter q of `word` (one of I, X, Y, Z) acts on qubit q."""
        if not observable:
            _check(self.lib.qml_set_observable(self._h, 0, None, None), "qml_set_observable")
            return
        words = "".join(w for _, w in observable).encode()
        coef = (ctypes.c_double * len(observable))(*[float(c) for c, _ in observable])
        _check(self.lib.qml_set_observable(self._h, len(observable), words, coef), "qml_set_observable")

    def set_entangler(self, bonds=None, kind: str = "cz"):
        """Pairs [(a, b), ...] ending every layer; None means the chain (q, q+1).
        kind "cz": CZ on each pair; "cnot": CNOT(control a, target b) on each
        pair in list order (needs a second state buffer: the workspace is
        re-allocated when it is too small)."""
        if bonds is None:
            bonds = [(q, q + 1) for q in range(self.n - 1)]
        flat = [int(v) for e in bonds for v in e]
        arr = (ctypes.c_int * max(1, len(flat)))(*flat)
        if kind == "cz":
            _check(self.lib.qml_set_entangler(self._h, len(bonds), arr), "qml_set_entangler")
        elif kind == "cnot":
            _check(self.lib.qml_set_entangler_cnot(self._h, len(bonds), arr), "qml_set_entangler_cnot")
        else:
            raise ValueError("kind must be 'cz' or 'cnot'")
        self._reset_workspace()

    def _reset_workspace(self):
        """Set the workspace again after a change of entangler (the schedule's
        device copies and the layout may change with it); a larger one is
        allocated when the current buffer is too small."""
        if self.ws is None:
            return
        nbytes = self.workspace_bytes(self._host_step)
        if self.ws.numel() - 256 < nbytes:
            self.allocate_workspace(host_step=self._host_step)
            return
        aligned = (self.ws.data_ptr() + 255) // 256 * 256
        _check(self.lib.qml_set_workspace(self._h, aligned, nbytes, _stream_handle(None)), "qml_set_workspace")

    @property
    def entangler_kind(self) -> str:
        return "cnot" if self.lib.qml_entangler_kind(self._h) == 1 else "cz"

    def set_reupload(self, on: bool = True):
        """Data re-uploading: every layer starts with the encoding Ry(x_q) again."""
        _check(self.lib.qml_set_reupload(self._h, 1 if on else 0), "qml_set_reupload")

    @property
    def reupload(self) -> bool:
        return bool(self.lib.qml_reupload(self._h))

    @property
    def split_form(self) -> bool:
        """True when the passes run in split form (see qml_split_form)."""
        return bool(self.lib.qml_split_form(self._h))

    @property
    def cnot_fused(self) -> bool:
        """True when CNOT layers run through the fused schedule (their maps applied
        inside the rotation passes; see qml_set_entangler_cnot)."""
        if self.lib.qml_entangler_kind(self._h) != 1:
            return False
        need = self.lib.qml_debug_entangler_map(self._h, None, 0)
        buf = (ctypes.c_int * need)()
        self.lib.qml_debug_entangler_map(self._h, buf, need)
        return bool(buf[1 + 4 * self.n]) and not self.reupload

    @property
    def entangler_bonds(self) -> int:
        return int(self.lib.qml_entangler_bonds(self._h))

    @property
    def observable_terms(self) -> int:
        return int(self.lib.qml_observable_terms(self._h))

    def expect_observable(self, psi, expect=None, stream=None):
        import torch

        B = psi.shape[0]
        expect = torch.empty(B, dtype=torch.float32, device=psi.device) if expect is None else expect
        _check(self.lib.qml_expect_observable(self._h, self._state_ptr(psi), B, _ptr(expect),
                                              _stream_handle(stream)), "qml_expect_observable")
        return expect

    def debug_tile_view(self, pass_index: int) -> dict:
        """Memory view of one pass (see qml_debug_tile_view in include/qml.h)."""
        need = self.lib.qml_debug_tile_view(self._h, pass_index, None, 0)
        if need < 0:
            raise IndexError(pass_index)
        buf = (ctypes.c_int * need)()
        self.lib.qml_debug_tile_view(self._h, pass_index, buf, need)
        v = list(buf)
        dims = [dict(kind=v[1 + 4 * d], qlo=v[2 + 4 * d], bits=v[3 + 4 * d], shift=v[4 + 4 * d]) for d in range(5)]
        i = 21
        tile_q = [v[i + 2 * b] for b in range(12)]
        sstride = [v[i + 2 * b + 1] for b in range(12)]
        n_out = v[i + 24]
        j = i + 25 + n_out
        return dict(tma=v[0], dims=dims, tile_q=tile_q, sstride=sstride, out_q=v[i + 25:j],
                    tile_addr=v[j:j + 12], out_addr=v[j + 12:j + 12 + n_out], variant=v[j + 12 + n_out])

    def enable_timing(self, on: bool = True):
        _check(self.lib.qml_enable_timing(self._h, 1 if on else 0), "qml_enable_timing")

    def read_timing(self):
        """(fwd pass ms, fwd pass launches, bwd pass ms, bwd pass launches) since the last read."""
        fm, bm = ctypes.c_double(), ctypes.c_double()
        fn, bn = ctypes.c_longlong(), ctypes.c_longlong()
        _check(self.lib.qml_read_timing(self._h, ctypes.byref(fm), ctypes.byref(fn), ctypes.byref(bm),
                                        ctypes.byref(bn)), "qml_read_timing")
        return fm.value, fn.value, bm.value, bn.value

    @property
    def launch_count(self) -> int:
        return int(self.lib.qml_launch_count(self._h))

    def sync(self, stream=None):
        _check(self.lib.qml_sync(self._h, _stream_handle(stream)), "qml_sync (device status)")

    # ------------------------------------------------------------- compute
    @property
    def real_dtype(self):
        import torch

        return torch.float64 if self.f64 else torch.float32

    def new_state(self, B: int):
        import torch

        return torch.empty((B, 1 << self.n, 2), dtype=self.real_dtype, device=f"cuda:{self.device}")

    def _state_ptr(self, t):
        import torch

        if t.dtype in (torch.complex64, torch.complex128):
            t = torch.view_as_real(t)
        if t.dtype != self.real_dtype or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"state must be a contiguous CUDA {self.real_dtype} [B, 2^n, 2] tensor "
                             "(or its complex view)")
        return t.data_ptr()

    def encode(self, x, psi=None, stream=None):
        B = x.shape[0]
        psi = self.new_state(B) if psi is None else psi
        _check(self.lib.qml_init_state_encode(self._h, _ptr(x), B, self._state_ptr(psi), _stream_handle(stream)),
               "qml_init_state_encode")
        return psi

    def forward(self, theta, x, psi=None, expect=None, stream=None):
        import torch

        B = x.shape[0]
        psi = self.new_state(B) if psi is None else psi
        expect = torch.empty(B, dtype=self.real_dtype, device=x.device) if expect is None else expect
        f = self.lib.qml_forward_expect_f64 if self.f64 else self.lib.qml_forward_expect
        _check(f(self._h, _ptr(theta), _ptr(x), B, self._state_ptr(psi), _ptr(expect), _stream_handle(stream)),
               "qml_forward_expect")
        return psi, expect

    def backward(self, theta, x, psi, lam, dLdE, grad=None, stream=None):
        import torch

        B = x.shape[0]
        grad = torch.empty((self.L, self.n, 3), dtype=self.real_dtype, device=x.device) if grad is None else grad
        f = self.lib.qml_backward_adjoint_f64 if self.f64 else self.lib.qml_backward_adjoint
        _check(f(self._h, _ptr(theta), _ptr(x), B, self._state_ptr(psi), self._state_ptr(lam), _ptr(dLdE),
                 _ptr(grad), _stream_handle(stream)), "qml_backward_adjoint")
        return grad

    def loss_seed(self, expect, y, stream=None):
        import torch

        B = expect.shape[0]
        g = torch.empty(B, dtype=self.real_dtype, device=expect.device)
        loss = torch.empty(1, dtype=self.real_dtype, device=expect.device)
        f = self.lib.qml_loss_seed_f64 if self.f64 else self.lib.qml_loss_seed
        _check(f(self._h, _ptr(expect), _ptr(y), B, _ptr(g), _ptr(loss), _stream_handle(stream)), "qml_loss_seed")
        return g, loss

    def expect_z0(self, psi, expect=None, stream=None):
        import torch

        B = psi.shape[0]
        expect = torch.empty(B, dtype=torch.float32, device=psi.device) if expect is None else expect
        _check(self.lib.qml_expect_z0(self._h, self._state_ptr(psi), B, _ptr(expect), _stream_handle(stream)),
               "qml_expect_z0")
        return expect

    def ckpt_save(self, slot: int, psi, stream=None):
        _check(self.lib.qml_ckpt_save(self._h, slot, self._state_ptr(psi), psi.shape[0], _stream_handle(stream)),
               "qml_ckpt_save")

    def ckpt_restore(self, slot: int, psi, stream=None):
        _check(self.lib.qml_ckpt_restore(self._h, slot, self._state_ptr(psi), psi.shape[0], _stream_handle(stream)),
               "qml_ckpt_restore")

    def step_host(self, x: np.ndarray, theta: np.ndarray, y: np.ndarray, out: StepResult | None = None,
                  stream=None) -> StepResult:
        """Forward + loss + backward from (preferably pinned) host arrays."""
        B = x.shape[0]
        dt = np.float64 if self.f64 else np.float32
        if out is None:
            out = StepResult(np.empty(B, dt), np.empty(1, dt), np.empty((self.L, self.n, 3), dt))

        def hp(a):
            if hasattr(a, "data_ptr"):
                return a.data_ptr()
            assert a.dtype == dt and a.flags.c_contiguous
            return a.ctypes.data

        f = self.lib.qml_step_host_f64 if self.f64 else self.lib.qml_step_host
        _check(f(self._h, hp(x), hp(theta), hp(y), B, hp(out.expect), hp(out.loss), hp(out.grad),
                 _stream_handle(stream)), "qml_step_host")
        return out

    @property
    def precision_bits(self) -> int:
        return int(self.lib.qml_precision(self._h))
