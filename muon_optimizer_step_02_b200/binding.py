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

_PKG = os.path.dirname(os.path.abspath(__file__))
# MUONB200_LIB selects another build of the library, e.g. the device-checked
# one (CHECKED_LIB_PATH), for a whole process.
LIB_PATH = os.environ.get("MUONB200_LIB") or os.path.join(_PKG, "libmuonb200.so")
CHECKED_LIB_PATH = os.path.join(_PKG, "libmuonb200_checked.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = -1
MUON_ERR_UNSUPPORTED = -2
MUON_ERR_ALIGNMENT = -3
MUON_ERR_CUDA = -4
MUON_ERR_TIMEOUT = -5
MUON_ERR_WORKSPACE = -6
MUON_ERR_DEVICE_CHECK = -7

KIND_NAMES = ("prologue", "gram", "poly", "apply", "final", "ns", "scale")


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


class muon_ramp_t(Structure):
    _fields_ = [("v0", c_float), ("v1", c_float), ("t0", c_int32),
                ("t1", c_int32)]


class muon_schedule_t(Structure):
    _fields_ = [("momentum", muon_ramp_t), ("lr", muon_ramp_t)]


def make_schedule(momentum_ramp, lr_ramp) -> muon_schedule_t:
    """(v0, v1, t0, t1) ramps for the momentum and the learning rate."""
    m, l = momentum_ramp, lr_ramp
    return muon_schedule_t(muon_ramp_t(float(m[0]), float(m[1]), int(m[2]), int(m[3])),
                           muon_ramp_t(float(l[0]), float(l[1]), int(l[2]), int(l[3])))


class adamw_hyper_t(Structure):
    _fields_ = [("lr", c_float), ("beta1", c_float), ("beta2", c_float),
                ("eps", c_float), ("weight_decay", c_float)]


class adamw_tensor_t(Structure):
    _fields_ = [("param", c_void_p), ("grad", c_void_p), ("exp_avg", c_void_p),
                ("exp_avg_sq", c_void_p), ("ema", c_void_p), ("numel", c_int64)]


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
    L.muon_step_batched_sched.argtypes = [c_void_p, POINTER(muon_matrix_t),
                                          POINTER(muon_hyper_t),
                                          POINTER(muon_schedule_t), c_void_p,
                                          POINTER(c_float), c_int32, c_void_p,
                                          c_size_t, c_void_p]
    L.muon_step_batched_sched.restype = c_int32
    L.adamw_ema_batched.argtypes = [POINTER(adamw_tensor_t), c_int32,
                                    POINTER(adamw_hyper_t), c_int32, c_void_p,
                                    c_float, c_void_p]
    L.adamw_ema_batched.restype = c_int32
    L.adamw_ema_launches.argtypes = [c_int32, c_int32]
    L.adamw_ema_launches.restype = c_int32
    L.muon_plan_error_async.argtypes = [c_void_p, c_void_p, c_void_p]
    L.muon_plan_error_async.restype = c_int32
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
    L.muon_noalloc_error_async.argtypes = [c_void_p, c_void_p]
    L.muon_noalloc_error_async.restype = c_int32
    L.muon_noalloc_set_fault.argtypes = [c_int32]
    L.muon_noalloc_set_fault.restype = c_int32
    L.muon_f32_to_bf16.argtypes = [c_void_p, c_void_p, c_int64, c_void_p]
    L.muon_f32_to_bf16.restype = c_int32
    L.muon_device_checks.argtypes = []
    L.muon_device_checks.restype = c_int32
    L.muon_device_allocation_count.argtypes = []
    L.muon_device_allocation_count.restype = c_int64
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
             update_out=None, stream=None, schedule=None, step_dev=None):
        """One batched Muon step (muon_step_batched, or with `schedule` and
        `step_dev` muon_step_batched_sched).  weights/momenta: fp32 CUDA
        tensors (updated in place); grads: bf16 CUDA tensors; hyper: an
        object with momentum, lr, weight_decay, eps_row, eps_frob, nesterov,
        eq_r; coeffs: ns_steps rows of (a, b, c)."""
        self.bind(weights, momenta, grads, hyper, coeffs, workspace,
                  update_scales, update_out, schedule, step_dev)(stream)

    def bind(self, weights, momenta, grads, hyper, coeffs, workspace,
             update_scales: Optional[Sequence[float]] = None,
             update_out=None, schedule=None, step_dev=None):
        """Checks and marshals the arguments once; returns a callable
        `run(stream=None)` that enqueues muon_step_batched with them (or
        muon_step_batched_sched when `schedule`, a pair of (v0, v1, t0, t1)
        ramps for momentum and lr, and `step_dev`, a one-element int32 CUDA
        tensor holding the step number, are given).  The tensors must stay
        alive and in place while the callable is used."""
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
        if any(len(row) != 3 for row in coeffs):
            raise ValueError("coeffs: one (a, b, c) row per Newton-Schulz step")
        flat = [float(v) for row in coeffs for v in row]
        k = len(flat) // 3
        carr = (c_float * max(len(flat), 1))(*flat)
        _check_tensor(workspace, torch.uint8, (workspace.numel(),),
                      "workspace")
        hp_ref = ctypes.byref(hp)
        ws_ptr, ws_n = workspace.data_ptr(), workspace.numel()
        # The callable holds the plan (so that it outlives every bound call)
        # and reads its handle at call time (so that a closed plan raises
        # instead of handing a freed handle to the library).
        plan = self
        keep = (mats, hp, carr, weights, momenta, grads, update_out, workspace)
        if schedule is not None:
            if step_dev is None:
                raise ValueError("a schedule needs step_dev")
            _check_tensor(step_dev, torch.int32, (1,), "step_dev")
            sch = make_schedule(*schedule)
            fn_s = lib().muon_step_batched_sched
            sch_ref, sp = ctypes.byref(sch), step_dev.data_ptr()
            keep = keep + (sch, step_dev)

            def run_sched(stream=None):
                _ = keep
                _check(fn_s(plan._live_handle(), mats, hp_ref, sch_ref, sp, carr,
                            k, ws_ptr, ws_n, _stream_handle(stream)),
                       "muon_step_batched_sched")
            return run_sched
        fn = lib().muon_step_batched

        def run(stream=None):
            _ = keep
            _check(fn(plan._live_handle(), mats, hp_ref, carr, k, ws_ptr, ws_n,
                      _stream_handle(stream)), "muon_step_batched")
        return run

    def _live_handle(self):
        if self._h is None:
            raise MuonError(MUON_ERR_INVALID_ARG, "the plan has been closed")
        return self._h

    def last_error(self, stream=None) -> int:
        return int(lib().muon_get_last_error(self._h, _stream_handle(stream)))

    def error_async(self, host_word, stream=None):
        """Enqueues a copy of the device error word into `host_word` (a
        one-element int32 CPU tensor, pinned for the copy to be asynchronous);
        read it after the stream has passed this point."""
        import torch
        if host_word.dtype != torch.int32 or host_word.device.type != "cpu" or \
                host_word.numel() < 1:
            raise ValueError("host_word must be an int32 CPU tensor")
        _check(lib().muon_plan_error_async(self._h, host_word.data_ptr(),
                                           _stream_handle(stream)),
               "muon_plan_error_async")

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


def adamw_ema_bind(params: Sequence, grads: Sequence, exp_avgs: Sequence,
                   exp_avg_sqs: Sequence, emas: Sequence, hyper, ema_decay: float,
                   step: int = 1, step_dev=None):
    """Marshals adamw_ema_batched once and returns `run(step_now=None,
    stream=None)`.  All tensors fp32 CUDA, contiguous, same numel per index;
    emas[i] may be None.  hyper: an object with lr, beta1, beta2, eps,
    weight_decay.  With step_dev (one-element int32 CUDA tensor) the device
    counter gives the step; otherwise `step`, or run's `step_now`."""
    import torch
    n = len(params)
    if not (len(grads) == len(exp_avgs) == len(exp_avg_sqs) == len(emas) == n):
        raise ValueError("one grad, exp_avg, exp_avg_sq and ema entry per param")
    arr = (adamw_tensor_t * max(n, 1))()
    for i in range(n):
        k = params[i].numel()
        for t, what in ((params[i], "params"), (grads[i], "grads"),
                        (exp_avgs[i], "exp_avgs"), (exp_avg_sqs[i], "exp_avg_sqs")):
            _check_tensor(t, torch.float32, (t.numel(),) if t.dim() == 1 else tuple(t.shape),
                          f"{what}[{i}]")
            if t.numel() != k:
                raise ValueError(f"{what}[{i}] has {t.numel()} elements, expected {k}")
        e = emas[i]
        if e is not None:
            _check_tensor(e, torch.float32, tuple(e.shape), f"emas[{i}]")
            if e.numel() != k:
                raise ValueError(f"emas[{i}] has {e.numel()} elements, expected {k}")
        arr[i] = adamw_tensor_t(params[i].data_ptr(), grads[i].data_ptr(),
                                exp_avgs[i].data_ptr(), exp_avg_sqs[i].data_ptr(),
                                e.data_ptr() if e is not None else None, k)
    hp = adamw_hyper_t(float(hyper.lr), float(hyper.beta1), float(hyper.beta2),
                       float(hyper.eps), float(hyper.weight_decay))
    sp = None
    if step_dev is not None:
        _check_tensor(step_dev, torch.int32, (1,), "step_dev")
        sp = step_dev.data_ptr()
    fn = lib().adamw_ema_batched
    keep = (arr, hp, list(params), list(grads), list(exp_avgs), list(exp_avg_sqs),
            list(emas), step_dev)
    hp_ref = ctypes.byref(hp)

    def run(step_now: Optional[int] = None, stream=None):
        _ = keep
        _check(fn(arr, n, hp_ref, int(step if step_now is None else step_now), sp,
                  float(ema_decay), _stream_handle(stream)), "adamw_ema_batched")
    return run


def adamw_ema_batched(params, grads, exp_avgs, exp_avg_sqs, emas, hyper,
                      ema_decay: float, step: int = 1, step_dev=None, stream=None):
    adamw_ema_bind(params, grads, exp_avgs, exp_avg_sqs, emas, hyper, ema_decay,
                   step, step_dev)(stream=stream)


def adamw_ema_launches(n_tensors: int, with_step_dev: bool = False) -> int:
    return int(lib().adamw_ema_launches(int(n_tensors), int(bool(with_step_dev))))


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
        if weights[i].dim() != 2:
            raise ValueError(f"weights[{i}] must be a matrix")
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
    if any(len(row) != 3 for row in coeffs):
        raise ValueError("coeffs: one (a, b, c) row per Newton-Schulz step")
    flat = [float(v) for row in coeffs for v in row]
    carr = (c_float * max(len(flat), 1))(*flat)
    _check(lib().muon_step_batched_noalloc(mats, n, ctypes.byref(hp), carr,
                                           len(flat) // 3,
                                           _stream_handle(stream)),
           "muon_step_batched_noalloc")


def noalloc_error_async(host_word, stream=None):
    """Enqueues a copy of the allocation-free path's error word into
    `host_word` (a one-element int32 CPU tensor, pinned for the copy to be
    asynchronous); non-zero once the stream has passed this point means the
    last muon_step_batched_noalloc call gave up on a bounded wait."""
    import torch
    if host_word.dtype != torch.int32 or host_word.device.type != "cpu" or \
            host_word.numel() < 1:
        raise ValueError("host_word must be an int32 CPU tensor")
    _check(lib().muon_noalloc_error_async(host_word.data_ptr(),
                                          _stream_handle(stream)),
           "muon_noalloc_error_async")


def noalloc_set_fault(fault: int):
    """Test hook of the allocation-free path (see muon_plan_set_fault)."""
    _check(lib().muon_noalloc_set_fault(int(fault)), "muon_noalloc_set_fault")


def device_allocation_count() -> int:
    """Device allocations the library has made in this process so far."""
    return int(lib().muon_device_allocation_count())


def f32_to_bf16(dst, src, stream=None):
    """dst (bf16 CUDA tensor) <- src (fp32 CUDA tensor, same numel) rounded to
    nearest even, by the library's conversion kernel."""
    import torch
    if not (src.is_cuda and dst.is_cuda) or src.dtype != torch.float32 or \
            dst.dtype != torch.bfloat16 or src.numel() != dst.numel() or \
            not (src.is_contiguous() and dst.is_contiguous()):
        raise ValueError("f32_to_bf16: contiguous fp32 src and bf16 dst CUDA "
                         "tensors of one size")
    _check(lib().muon_f32_to_bf16(dst.data_ptr(), src.data_ptr(), src.numel(),
                                  _stream_handle(stream)), "muon_f32_to_bf16")
