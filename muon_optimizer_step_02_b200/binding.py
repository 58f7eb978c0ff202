"""ctypes binding of libmuonb200.so (include/muon_b200.h).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: if the library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_double, c_float, c_int32,
                    c_int64, c_size_t, c_void_p)
from typing import List, Optional, Sequence, Tuple

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libmuonb200.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = -1
MUON_ERR_UNSUPPORTED = -2
MUON_ERR_ALIGNMENT = -3
MUON_ERR_CUDA = -4
MUON_ERR_TIMEOUT = -5
MUON_ERR_WORKSPACE = -6

KIND_NAMES = ("prologue", "gram", "poly", "apply", "final", "ns")


class muon_matrix_t(Structure):
    _fields_ = [("w", c_void_p), ("momentum", c_void_p),
                ("grad_bf16", c_void_p), ("update_out", c_void_p),
                ("rows", c_int32), ("cols", c_int32),
                ("update_scale", c_float)]


class muon_hyper_t(Structure):
    _fields_ = [("momentum", c_float), ("lr", c_float),
                ("weight_decay", c_float), ("eps_row", c_float),
                ("eps_frob", c_float), ("nesterov", c_int32),
                ("eq_r", c_int32)]


class MuonError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib():
    """Loads the library once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m muon_optimizer_step_02_b200._build` (no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    L.muon_plan_create.argtypes = [POINTER(c_int32), POINTER(c_int32), c_int32,
                                   c_int32, POINTER(c_void_p)]
    L.muon_plan_create.restype = c_int32
    L.muon_plan_workspace_bytes.argtypes = [c_void_p]
    L.muon_plan_workspace_bytes.restype = c_size_t
    L.muon_step_batched.argtypes = [c_void_p, POINTER(muon_matrix_t),
                                    POINTER(muon_hyper_t), POINTER(c_float),
                                    c_int32, c_void_p, c_size_t, c_void_p]
    L.muon_step_batched.restype = c_int32
    L.ema_update_batched.argtypes = [POINTER(c_void_p), POINTER(c_void_p),
                                     POINTER(c_int64), c_int32, c_float,
                                     c_void_p]
    L.ema_update_batched.restype = c_int32
    L.muon_get_last_error.argtypes = [c_void_p, c_void_p]
    L.muon_get_last_error.restype = c_int32
    L.muon_status_string.argtypes = [c_int32]
    L.muon_status_string.restype = c_char_p
    L.muon_plan_destroy.argtypes = [c_void_p]
    L.muon_plan_destroy.restype = None
    L.muon_plan_set_timing.argtypes = [c_void_p, c_int32]
    L.muon_plan_set_timing.restype = c_int32
    L.muon_plan_timing_read.argtypes = [c_void_p, POINTER(c_int32),
                                        POINTER(c_double), c_int32]
    L.muon_plan_timing_read.restype = c_int32
    L.muon_step_launches.argtypes = [c_int32]
    L.muon_step_launches.restype = c_int32
    L.muon_plan_step_launches.argtypes = [c_void_p, c_int32]
    L.muon_plan_step_launches.restype = c_int32
    L.ema_update_launches.argtypes = [c_int32]
    L.ema_update_launches.restype = c_int32
    L.muon_plan_set_fault.argtypes = [c_void_p, c_int32]
    L.muon_plan_set_fault.restype = c_int32
    L.muon_abi_version.argtypes = []
    L.muon_abi_version.restype = c_int32
    L.muon_step_batched_noalloc.argtypes = [POINTER(muon_matrix_t), c_int32,
                                            POINTER(muon_hyper_t),
                                            POINTER(c_float), c_int32,
                                            c_void_p]
    L.muon_step_batched_noalloc.restype = c_int32
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().muon_status_string(status).decode()


def _check(status: int, what: str):
    if status != MUON_OK:
        raise MuonError(status, what)


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") \
        else int(stream)


def _check_tensor(t, dtype, shape, what):
    import torch
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} must have shape {tuple(shape)}, got "
                         f"{tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")


class MuonPlan:
    """A plan for a fixed list of matrix shapes (rows, cols)."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], max_ns_steps: int = 5):
        L = lib()
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        n = len(self.shapes)
        rows = (c_int32 * n)(*[r for r, _ in self.shapes])
        cols = (c_int32 * n)(*[c for _, c in self.shapes])
        h = c_void_p()
        _check(L.muon_plan_create(rows, cols, n, int(max_ns_steps),
                                  ctypes.byref(h)), "muon_plan_create")
        self._h = h
        self.max_ns_steps = int(max_ns_steps)
        self.workspace_bytes = int(L.muon_plan_workspace_bytes(h))

    @property
    def handle(self):
        return self._h

    def alloc_workspace(self, device=None):
        import torch
        return torch.empty(max(self.workspace_bytes, 1), dtype=torch.uint8,
                           device=device or "cuda")

    def step(self, weights, momenta, grads, hyper, coeffs, workspace,
             update_scales: Optional[Sequence[float]] = None,
             update_out=None, stream=None):
        """One batched Muon step (muon_step_batched).  weights/momenta: fp32
        CUDA tensors (updated in place); grads: bf16 CUDA tensors; hyper: an
        object with momentum, lr, weight_decay, eps_row, eps_frob, nesterov,
        eq_r; coeffs: ns_steps rows of (a, b, c)."""
        self.bind(weights, momenta, grads, hyper, coeffs, workspace,
                  update_scales, update_out)(stream)

    def bind(self, weights, momenta, grads, hyper, coeffs, workspace,
             update_scales: Optional[Sequence[float]] = None,
             update_out=None):
        """Checks and marshals the arguments once; returns a callable
        `run(stream=None)` that enqueues muon_step_batched with them.  The
        tensors must stay alive and in place while the callable is used."""
        import torch
        n = len(self.shapes)
        if not (len(weights) == len(momenta) == len(grads) == n):
            raise ValueError("one weight, momentum and gradient per matrix")
        if update_out is not None and len(update_out) != n:
            raise ValueError("update_out must list one tensor (or None) per "
                             "matrix")
        mats = (muon_matrix_t * n)()
        for i, (r, c) in enumerate(self.shapes):
            _check_tensor(weights[i], torch.float32, (r, c), f"weights[{i}]")
            _check_tensor(momenta[i], torch.float32, (r, c), f"momenta[{i}]")
            _check_tensor(grads[i], torch.bfloat16, (r, c), f"grads[{i}]")
            o = update_out[i] if update_out is not None else None
            if o is not None:
                _check_tensor(o, torch.float32, (r, c), f"update_out[{i}]")
            s = (update_scales[i] if update_scales is not None
                 else max(1.0, r / c) ** 0.5)
            mats[i] = muon_matrix_t(weights[i].data_ptr(),
                                    momenta[i].data_ptr(),
                                    grads[i].data_ptr(),
                                    o.data_ptr() if o is not None else None,
                                    r, c, float(s))
        hp = muon_hyper_t(float(hyper.momentum), float(hyper.lr),
                          float(hyper.weight_decay), float(hyper.eps_row),
                          float(hyper.eps_frob), int(bool(hyper.nesterov)),
                          int(bool(hyper.eq_r)))
        flat = [float(v) for row in coeffs for v in row]
        k = len(flat) // 3
        carr = (c_float * max(len(flat), 1))(*flat)
        _check_tensor(workspace, torch.uint8, (workspace.numel(),),
                      "workspace")
        fn = lib().muon_step_batched
        h, hp_ref = self._h, ctypes.byref(hp)
        ws_ptr, ws_n = workspace.data_ptr(), workspace.numel()
        keep = (mats, hp, carr, weights, momenta, grads, update_out, workspace)

        def run(stream=None):
            _ = keep
            _check(fn(h, mats, hp_ref, carr, k, ws_ptr, ws_n,
                      _stream_handle(stream)), "muon_step_batched")
        return run

    def last_error(self, stream=None) -> int:
        return int(lib().muon_get_last_error(self._h, _stream_handle(stream)))

    def step_launches(self, ns_steps: int) -> int:
        return int(lib().muon_plan_step_launches(self._h, int(ns_steps)))

    def set_timing(self, enable: bool):
        _check(lib().muon_plan_set_timing(self._h, int(enable)),
               "muon_plan_set_timing")

    def timing_read(self):
        n = len(KIND_NAMES)
        launches = (c_int32 * n)()
        ms = (c_double * n)()
        _check(lib().muon_plan_timing_read(self._h, launches, ms, n),
               "muon_plan_timing_read")
        return {KIND_NAMES[k]: (int(launches[k]), float(ms[k]))
                for k in range(n)}

    def set_fault(self, fault: int):
        _check(lib().muon_plan_set_fault(self._h, int(fault)),
               "muon_plan_set_fault")

    def close(self):
        if getattr(self, "_h", None):
            lib().muon_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def muon_step_batched(plan: MuonPlan, *args, **kw):
    plan.step(*args, **kw)


def ema_update_batched(emas: Sequence, params: Sequence, decay: float,
                       stream=None):
    """E <- decay E + (1 - decay) P for every (E, P) pair (fp32 CUDA
    tensors, contiguous, same numel)."""
    ema_bind(emas, params, decay)(stream)


def ema_bind(emas: Sequence, params: Sequence, decay: float):
    """Checks and marshals the arguments of ema_update_batched once; returns
    a callable `run(stream=None)`."""
    import torch
    n = len(emas)
    if len(params) != n:
        raise ValueError("one parameter tensor per EMA tensor")
    e_arr = (c_void_p * max(n, 1))()
    p_arr = (c_void_p * max(n, 1))()
    num = (c_int64 * max(n, 1))()
    for i in range(n):
        e, p = emas[i], params[i]
        for t, what in ((e, f"emas[{i}]"), (p, f"params[{i}]")):
            if not t.is_cuda or t.dtype != torch.float32 or \
                    not t.is_contiguous():
                raise ValueError(f"{what} must be a contiguous fp32 CUDA "
                                 "tensor")
        if e.numel() != p.numel():
            raise ValueError(f"emas[{i}] and params[{i}] differ in size")
        e_arr[i] = e.data_ptr()
        p_arr[i] = p.data_ptr()
        num[i] = e.numel()
    fn = lib().ema_update_batched
    keep = (e_arr, p_arr, num, list(emas), list(params))
    d = float(decay)

    def run(stream=None):
        _ = keep
        _check(fn(e_arr, p_arr, num, n, d, _stream_handle(stream)),
               "ema_update_batched")
    return run


def step_launches(ns_steps: int) -> int:
    return int(lib().muon_step_launches(int(ns_steps)))


def ema_launches(n_tensors: int) -> int:
    return int(lib().ema_update_launches(int(n_tensors)))


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024
NOALLOC_MAX_MATS = 64


def muon_step_batched_noalloc(weights, momenta, grads, hyper, coeffs,
                              update_scales: Optional[Sequence[float]] = None,
                              update_out=None, stream=None):
    """One batched Muon step through muon_step_batched_noalloc: no plan and
    no workspace; the library's fixed device scratch array is used instead
    (for callers that cannot allocate device memory).  Same tensor rules as
    MuonPlan.step."""
    import torch
    n = len(weights)
    if not (len(momenta) == len(grads) == n):
        raise ValueError("one weight, momentum and gradient per matrix")
    mats = (muon_matrix_t * max(n, 1))()
    for i in range(n):
        r, c = (int(v) for v in weights[i].shape)
        _check_tensor(weights[i], torch.float32, (r, c), f"weights[{i}]")
        _check_tensor(momenta[i], torch.float32, (r, c), f"momenta[{i}]")
        _check_tensor(grads[i], torch.bfloat16, (r, c), f"grads[{i}]")
        o = update_out[i] if update_out is not None else None
        if o is not None:
            _check_tensor(o, torch.float32, (r, c), f"update_out[{i}]")
        s = (update_scales[i] if update_scales is not None
             else max(1.0, r / c) ** 0.5)
        mats[i] = muon_matrix_t(weights[i].data_ptr(), momenta[i].data_ptr(),
                                grads[i].data_ptr(),
                                o.data_ptr() if o is not None else None,
                                r, c, float(s))
    hp = muon_hyper_t(float(hyper.momentum), float(hyper.lr),
                      float(hyper.weight_decay), float(hyper.eps_row),
                      float(hyper.eps_frob), int(bool(hyper.nesterov)),
                      int(bool(hyper.eq_r)))
    flat = [float(v) for row in coeffs for v in row]
    carr = (c_float * max(len(flat), 1))(*flat)
    _check(lib().muon_step_batched_noalloc(mats, n, ctypes.byref(hp), carr,
                                           len(flat) // 3,
                                           _stream_handle(stream)),
           "muon_step_batched_noalloc")
