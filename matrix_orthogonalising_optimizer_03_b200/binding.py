"""ctypes binding of libmuon.so (C ABI in include/muon.h).

Argument marshalling only: every step of the Muon update runs in the library's
CUDA kernels. PyTorch supplies device memory and streams. The functions here
raise `MuonError` when the library is missing or a call fails; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_int32, c_int64, c_size_t, c_uint32, c_void_p
from typing import List, Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmuon.so")

MUON_OK = 0
STATUS_NAMES = {
    0: "MUON_OK", 1: "MUON_ERR_INVALID_ARG", 2: "MUON_ERR_SHAPE", 3: "MUON_ERR_DTYPE",
    4: "MUON_ERR_ALIAS", 5: "MUON_ERR_WORKSPACE", 6: "MUON_ERR_CUDA", 7: "MUON_ERR_TIMEOUT",
    8: "MUON_ERR_UNSUPPORTED",
}
MUON_F32, MUON_BF16 = 0, 1
MUON_MODE_MUON, MUON_MODE_MUONGS, MUON_MODE_MUONH, MUON_MODE_TWOSIDED = 0, 1, 2, 3
MUON_SCALE_MOONLIGHT, MUON_SCALE_KELLER, MUON_SCALE_NONE = 0, 1, 2
MUON_NESTEROV, MUON_EQUILIBRATE, MUON_NS_FP32, MUON_WANT_STATS = 1, 2, 4, 8

MODES = {"muon": MUON_MODE_MUON, "muongs": MUON_MODE_MUONGS, "muonh": MUON_MODE_MUONH,
         "twosided": MUON_MODE_TWOSIDED}
SCALES = {"moonlight": MUON_SCALE_MOONLIGHT, "keller": MUON_SCALE_KELLER, "none": MUON_SCALE_NONE}


class MuonError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}" if what else
                         STATUS_NAMES.get(status, str(status)))


class MuonMatrix(ctypes.Structure):
    _fields_ = [("W", c_void_p), ("grad", c_void_p), ("momentum", c_void_p),
                ("rows", c_int64), ("cols", c_int64),
                ("ld_w", c_int64), ("ld_g", c_int64), ("ld_m", c_int64),
                ("w_dtype", c_int32), ("g_dtype", c_int32)]


class MuonHParams(ctypes.Structure):
    _fields_ = [("lr", c_float), ("momentum", c_float), ("weight_decay", c_float),
                ("ns_coeffs", c_float * 3), ("ns_steps", c_int32), ("eps", c_float),
                ("mode", c_int32), ("scale", c_int32), ("scale_k", c_float), ("flags", c_uint32)]


class MuonStats(ctypes.Structure):
    _fields_ = [("w_norm", c_float), ("w_dot_o", c_float), ("o_norm", c_float),
                ("update_rms", c_float), ("equil_axis", c_int32), ("reserved", c_int32)]


class MuonQkSlice(ctypes.Structure):
    _fields_ = [("W", c_void_p), ("row0", c_int64), ("rows", c_int64), ("cols", c_int64),
                ("ld", c_int64), ("head", c_int32), ("power", c_float)]


class MuonNSMatrix(ctypes.Structure):
    _fields_ = [("X", c_void_p), ("O", c_void_p), ("rows", c_int64), ("cols", c_int64),
                ("ld_x", c_int64), ("ld_o", c_int64), ("dtype", c_int32), ("reserved", c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Loads libmuon.so and declares its signatures. Raises if the library is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise MuonError(-1, f"libmuon.so not found at {path}; build it with "
                            "`python -m matrix_orthogonalising_optimizer_03_b200.build`")
    lib = ctypes.CDLL(path)
    P = POINTER
    sig = {
        "muon_abi_version": (c_int, []),
        "muon_status_string": (ctypes.c_char_p, [c_int]),
        "muon_hparams_default": (c_int, [P(MuonHParams)]),
        "muon_validate": (c_int, [P(MuonMatrix), c_int, P(MuonHParams)]),
        "muon_workspace_size": (c_size_t, [P(MuonMatrix), c_int, P(MuonHParams)]),
        "muon_step_batched": (c_int, [P(MuonMatrix), c_int, P(MuonHParams), c_void_p, c_size_t,
                                      c_void_p, c_void_p]),
        "muon_plan_create": (c_int, [P(MuonMatrix), c_int, P(MuonHParams), P(c_void_p)]),
        "muon_plan_workspace_size": (c_size_t, [c_void_p]),
        "muon_plan_set_hparams": (c_int, [c_void_p, P(MuonHParams)]),
        "muon_plan_step": (c_int, [c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
        "muon_plan_destroy": (None, [c_void_p]),
        "muon_ns_workspace_size": (c_size_t, [P(MuonNSMatrix), c_int, P(MuonHParams)]),
        "muon_newton_schulz_batched": (c_int, [P(MuonNSMatrix), c_int, P(MuonHParams), c_void_p,
                                               c_size_t, c_void_p]),
        "muon_query_device_status": (c_int, [c_void_p, c_void_p]),
        "muon_newton_schulz_noalloc": (c_int, [P(MuonNSMatrix), P(MuonHParams), c_void_p, c_void_p]),
        "muon_plan_profile_enable": (c_int, [c_void_p, c_int]),
        "muon_wait_probe": (c_int, [c_void_p, c_int64, c_void_p]),
        "muon_qk_clip": (c_int, [P(MuonQkSlice), c_int, c_void_p, c_int, c_float, c_void_p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if lib.muon_abi_version() != 1:
        raise MuonError(-1, "unexpected libmuon ABI version")
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != MUON_OK:
        raise MuonError(status, what)


def hparams(lr: float = 0.02, momentum: float = 0.95, weight_decay: float = 0.0,
            ns_coeffs: Sequence[float] = (3.4445, -4.7750, 2.0315), ns_steps: int = 5,
            eps: float = 1e-7, mode: str = "muon", scale: str = "moonlight", scale_k: float = 0.2,
            nesterov: bool = True, equilibrate: bool = False, ns_fp32: bool = False) -> MuonHParams:
    hp = MuonHParams()
    _check(load().muon_hparams_default(ctypes.byref(hp)), "muon_hparams_default")
    hp.lr, hp.momentum, hp.weight_decay = lr, momentum, weight_decay
    hp.ns_coeffs[0], hp.ns_coeffs[1], hp.ns_coeffs[2] = ns_coeffs
    hp.ns_steps, hp.eps = ns_steps, eps
    hp.mode, hp.scale, hp.scale_k = MODES[mode], SCALES[scale], scale_k
    hp.flags = ((MUON_NESTEROV if nesterov else 0) | (MUON_EQUILIBRATE if equilibrate else 0) |
                (MUON_NS_FP32 if ns_fp32 else 0))
    return hp


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return MUON_F32
    if t.dtype == torch.bfloat16:
        return MUON_BF16
    raise MuonError(3, f"unsupported dtype {t.dtype}")


def _check_2d(t, name: str):
    if t.dim() != 2:
        raise MuonError(2, f"{name} must be 2-D (got {t.dim()}-D)")
    if t.stride(1) != 1 and t.size(1) > 1:
        raise MuonError(2, f"{name} must be row-major with unit column stride")
    if not t.is_cuda:
        raise MuonError(1, f"{name} must be a CUDA tensor")


def matrix_array(params, grads, momenta):
    """The muon_matrix_t array for lists of W (fp32), G (fp32/bf16), M (fp32) tensors."""
    n = len(params)
    if len(grads) != n or len(momenta) != n:
        raise MuonError(1, "params, grads and momenta must have the same length")
    arr = (MuonMatrix * n)()
    for i, (w, g, m) in enumerate(zip(params, grads, momenta)):
        for t, nm in ((w, "W"), (g, "grad"), (m, "momentum")):
            _check_2d(t, nm)
        if tuple(g.shape) != tuple(w.shape) or tuple(m.shape) != tuple(w.shape):
            raise MuonError(2, "W, grad and momentum shapes differ")
        arr[i] = MuonMatrix(w.data_ptr(), g.data_ptr(), m.data_ptr(), w.size(0), w.size(1),
                            max(w.stride(0), w.size(1)), max(g.stride(0), g.size(1)),
                            max(m.stride(0), m.size(1)), _dtype_code(w), _dtype_code(g))
    return arr


def _device_of(tensors):
    """The CUDA device of the first tensor (the library runs on the current device, so
    every call switches to the device that holds its matrices); None for empty lists."""
    return tensors[0].device if len(tensors) else None


def _on(device):
    """Context that makes `device` current for one library call."""
    import contextlib
    return _torch().cuda.device(device) if device is not None else contextlib.nullcontext()


def _stream_ptr(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _stats_ptr(stats) -> Optional[int]:
    if stats is None:
        return None
    torch = _torch()
    if stats.dtype != torch.int32 or stats.numel() % 6 != 0 or not stats.is_cuda:
        raise MuonError(1, "stats must be a CUDA int32 tensor of n*6 elements")
    return stats.data_ptr()


def _status_ptr(status) -> Optional[int]:
    """Device address of a one-word status tensor (int32 or uint32, at least one
    element, on a CUDA device), or None. Anything else raises before any launch."""
    if status is None:
        return None
    torch = _torch()
    ok_dtypes = [torch.int32] + ([torch.uint32] if hasattr(torch, "uint32") else [])
    if not status.is_cuda:
        raise MuonError(1, "status must be a CUDA tensor")
    if status.dtype not in ok_dtypes:
        raise MuonError(1, f"status must be int32 or uint32 (got {status.dtype})")
    if status.numel() < 1:
        raise MuonError(1, "status must have at least one element")
    return status.data_ptr()


def new_stats(n: int, device="cuda"):
    """A device buffer for n muon_stats_t (int32 storage; see `decode_stats`)."""
    return _torch().zeros((n, 6), dtype=_torch().int32, device=device)


def decode_stats(stats) -> List[dict]:
    torch = _torch()
    s = stats.detach().cpu()
    f = s.view(torch.float32)
    return [dict(w_norm=float(f[i, 0]), w_dot_o=float(f[i, 1]), o_norm=float(f[i, 2]),
                 update_rms=float(f[i, 3]), equil_axis=int(s[i, 4])) for i in range(s.shape[0])]


def new_workspace(nbytes: int, device="cuda"):
    """A 256-byte aligned device workspace (torch allocations are 512-byte aligned)."""
    ws = _torch().empty(max(int(nbytes), 1), dtype=_torch().uint8, device=device)
    if ws.data_ptr() % 256:
        raise MuonError(5, "workspace allocation is not 256-byte aligned")
    return ws


def workspace_size(params, grads, momenta, hp: MuonHParams) -> int:
    arr = matrix_array(params, grads, momenta)
    return int(load().muon_workspace_size(arr, len(arr), ctypes.byref(hp)))


def step_batched(params, grads, momenta, hp: MuonHParams, workspace=None, stats=None,
                 stream=None):
    """One Muon step over the lists (muon_step_batched). Returns the workspace used."""
    lib = load()
    arr = matrix_array(params, grads, momenta)
    n = len(arr)
    if workspace is None:
        size = lib.muon_workspace_size(arr, n, ctypes.byref(hp))
        if n and size == 0:
            _check(lib.muon_validate(arr, n, ctypes.byref(hp)), "muon_validate")
        workspace = new_workspace(size, params[0].device if n else "cuda")
    with _on(_device_of(params)):
        _check(lib.muon_step_batched(arr, n, ctypes.byref(hp), workspace.data_ptr(),
                                     workspace.numel(), _stats_ptr(stats), _stream_ptr(stream)),
               "muon_step_batched")
    return workspace


class Plan:
    """A cached plan (muon_plan_*) over a fixed list of matrices, owning its workspace."""

    def __init__(self, params, grads, momenta, hp: MuonHParams, workspace=None):
        self._lib = load()
        self._arr = matrix_array(params, grads, momenta)
        self._keep = (list(params), list(grads), list(momenta))
        self.n = len(self._arr)
        self.hp = hp
        h = c_void_p()
        _check(self._lib.muon_plan_create(self._arr, self.n, ctypes.byref(hp), ctypes.byref(h)),
               "muon_plan_create")
        self._plan = h
        self.workspace_bytes = int(self._lib.muon_plan_workspace_size(h))
        self.device = _device_of(params)
        self.workspace = (workspace if workspace is not None
                          else new_workspace(self.workspace_bytes, self.device or "cuda"))

    def set_hparams(self, hp: MuonHParams):
        _check(self._lib.muon_plan_set_hparams(self._plan, ctypes.byref(hp)), "muon_plan_set_hparams")
        self.hp = hp

    def step(self, stats=None, stream=None):
        with _on(self.device):
            _check(self._lib.muon_plan_step(self._plan, self.workspace.data_ptr(),
                                            self.workspace.numel(), _stats_ptr(stats),
                                            _stream_ptr(stream)), "muon_plan_step")

    def query_device_status(self, stream=None) -> int:
        with _on(self.device):
            return int(self._lib.muon_query_device_status(self.workspace.data_ptr(),
                                                          _stream_ptr(stream)))

    def close(self):
        if getattr(self, "_plan", None):
            self._lib.muon_plan_destroy(self._plan)
            self._plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def newton_schulz(xs, outs, hp: MuonHParams, workspace=None, stream=None):
    """O_i = NS(X_i / (||X_i||_F + eps)) for lists of 2-D CUDA tensors (fp32 or bf16)."""
    lib = load()
    n = len(xs)
    arr = (MuonNSMatrix * n)()
    for i, (x, o) in enumerate(zip(xs, outs)):
        _check_2d(x, "X")
        _check_2d(o, "O")
        if x.dtype != o.dtype or tuple(x.shape) != tuple(o.shape):
            raise MuonError(3, "X and O must have the same dtype and shape")
        arr[i] = MuonNSMatrix(x.data_ptr(), o.data_ptr(), x.size(0), x.size(1),
                              max(x.stride(0), x.size(1)), max(o.stride(0), o.size(1)),
                              _dtype_code(x), 0)
    if workspace is None:
        size = lib.muon_ns_workspace_size(arr, n, ctypes.byref(hp))
        workspace = new_workspace(size, xs[0].device if n else "cuda")
    with _on(_device_of(xs)):
        _check(lib.muon_newton_schulz_batched(arr, n, ctypes.byref(hp), workspace.data_ptr(),
                                              workspace.numel(), _stream_ptr(stream)),
               "muon_newton_schulz_batched")
    return workspace


def newton_schulz_noalloc(x, o, hp: MuonHParams, status=None, stream=None):
    """O = NS(X / (||X||_F + eps)) for one matrix, using the library's static scratch
    instead of a workspace (for callers that cannot allocate device memory).
    status: optional CUDA int32/uint32 one-element tensor for the device error word."""
    lib = load()
    status_ptr = _status_ptr(status)
    _check_2d(x, "X")
    _check_2d(o, "O")
    if x.dtype != o.dtype or tuple(x.shape) != tuple(o.shape):
        raise MuonError(3, "X and O must have the same dtype and shape")
    if o.device != x.device:
        raise MuonError(1, "X and O must be on the same device")
    if status is not None and status.device != x.device:
        raise MuonError(1, "status must be on the device of X")
    m = MuonNSMatrix(x.data_ptr(), o.data_ptr(), x.size(0), x.size(1), max(x.stride(0), x.size(1)),
                     max(o.stride(0), o.size(1)), _dtype_code(x), 0)
    with _on(x.device):
        _check(lib.muon_newton_schulz_noalloc(ctypes.byref(m), ctypes.byref(hp), status_ptr,
                                              _stream_ptr(stream)), "muon_newton_schulz_noalloc")


class QkClipPlan:
    """QK-Clip over a fixed set of slices: the slice descriptors are marshalled once, and
    every `apply()` rescales the heads whose current S_max (read on the device from the
    same `s_max` tensor) exceeds tau. slices: list of (W tensor fp32 2-D CUDA, row0, rows,
    head, power); s_max: CUDA float32 tensor with one entry per head. The weights and
    s_max must stay alive while the plan is used."""

    def __init__(self, slices, s_max, tau: float = 100.0):
        self._lib = load()
        arr = (MuonQkSlice * len(slices))()
        for i, (w, r0, nr, h, pw) in enumerate(slices):
            _check_2d(w, "W")
            if w.dtype != _torch().float32:
                raise MuonError(3, "QK-Clip weights must be float32")
            if w.device != s_max.device:
                raise MuonError(1, "QK-Clip weights and s_max must be on the same GPU")
            arr[i] = MuonQkSlice(w.data_ptr(), r0, nr, w.size(1), max(w.stride(0), w.size(1)), h, pw)
        if s_max.dtype != _torch().float32 or not s_max.is_cuda:
            raise MuonError(1, "s_max must be a CUDA float32 tensor")
        self._arr, self._n, self.s_max, self.tau = arr, len(slices), s_max, float(tau)

    def apply(self, stream=None):
        with _on(self.s_max.device):
            _check(self._lib.muon_qk_clip(self._arr, self._n, self.s_max.data_ptr(),
                                          self.s_max.numel(), self.tau, _stream_ptr(stream)),
                   "muon_qk_clip")


def qk_clip(slices, s_max, tau: float = 100.0, stream=None):
    """QK-Clip, one call. slices: list of (W tensor fp32 2-D CUDA, row0, rows, head, power);
    s_max: CUDA float32 tensor with one entry per head."""
    QkClipPlan(slices, s_max, tau).apply(stream)


class StreamedSteps:
    """Optimizer steps fed with gradients that arrive from pinned host memory.

    Two device gradient buffers alternate: while step t runs on the compute stream
    from buffer t % 2, the gradients of step t + 1 are copied into the other buffer
    on a copy stream, so the host-to-device transfer overlaps the step. Each buffer
    has its own plan over the same weights and momenta. `step(host_flat)` enqueues
    the copy of `host_flat` (a pinned tensor holding all gradients back to back, in
    the order of `params`) and the step that consumes it; the per-matrix statistics
    of the step are copied back to pinned host memory (`stats_host`).
    """

    def __init__(self, params, momenta, hp: MuonHParams, grad_dtype=None):
        torch = _torch()
        self.params, self.momenta = list(params), list(momenta)
        dev = self.params[0].device
        gdt = grad_dtype or torch.bfloat16
        self.numel = sum(p.numel() for p in self.params)
        self.bufs, self.plans = [], []
        for _ in range(2):
            flat = torch.empty(self.numel, dtype=gdt, device=dev)
            views, off = [], 0
            for p in self.params:
                views.append(flat[off:off + p.numel()].view(p.shape))
                off += p.numel()
            self.bufs.append(flat)
            self.plans.append(Plan(self.params, views, self.momenta, hp))
        self.stats = new_stats(len(self.params), dev)
        self.stats_host = torch.empty_like(self.stats, device="cpu").pin_memory()
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.copied = [torch.cuda.Event(), torch.cuda.Event()]
        self.consumed = [torch.cuda.Event(), torch.cuda.Event()]
        self.t = 0

    def step(self, host_flat, stream=None):
        torch = _torch()
        comp = stream or torch.cuda.current_stream()
        b = self.t % 2
        with torch.cuda.stream(self.copy_stream):
            self.copy_stream.wait_event(self.consumed[b])   # buffer b free again
            self.bufs[b].copy_(host_flat, non_blocking=True)
            self.copied[b].record(self.copy_stream)
        comp.wait_event(self.copied[b])
        self.plans[b].step(stats=self.stats, stream=comp)
        self.consumed[b].record(comp)
        with torch.cuda.stream(comp):   # the read-back follows the step on its stream
            self.stats_host.copy_(self.stats, non_blocking=True)
        self.t += 1

    def close(self):
        for p in self.plans:
            p.close()
