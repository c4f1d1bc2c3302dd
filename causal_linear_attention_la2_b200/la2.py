"""ctypes binding of libla2.so -- argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
only turns torch tensors into device pointers and sizes, passes the caller's
current CUDA stream, and raises on a non-OK status.  There is no fallback: if
the library is missing or a shape is unsupported, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libla2.so")

LA2_OK = 0
LA2_ERR_INVALID_ARG = 1
LA2_ERR_UNSUPPORTED = 2
LA2_ERR_WORKSPACE = 3
LA2_ERR_CUDA = 4
LA2_ERR_TIMEOUT = 5

LA2_DTYPE_F32 = 0
LA2_DTYPE_BF16 = 1

# Every entry point include/la2.h declares.
EXPORTS = ("la2_workspace_bytes", "la2_fwd", "la2_fwd_state", "la2_fwd_ex", "la2_bwd", "la2_bwd_ex",
           "la2_decode", "la2_status_str", "la2_device_status", "la2_last_launch_count",
           "la2_fwd_noalloc", "la2_set_schedule", "la2_plan_info", "la2_selftest_timeout",
           "la2_bwd_state", "la2_dlambda", "la2_dlambda_workspace_bytes",
           "la2_norm_workspace_bytes", "la2_fwd_norm", "la2_bwd_norm")

LA2_LAYOUT_BHTD = 0
LA2_LAYOUT_BTHD = 1
_LAYOUTS = {"bhtd": LA2_LAYOUT_BHTD, "bthd": LA2_LAYOUT_BTHD}

LA2_SCHEDULE_AUTO = 0
LA2_SCHEDULE_UNIFORM = 1
LA2_SCHEDULE_BALANCED = 2
_SCHEDULES = {"auto": LA2_SCHEDULE_AUTO, "uniform": LA2_SCHEDULE_UNIFORM, "balanced": LA2_SCHEDULE_BALANCED}


class LA2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {la2_status_str(status)} ({status})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libla2.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libla2.so not found at {path}; build it with "
                           "`python -m causal_linear_attention_la2_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.la2_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.la2_workspace_bytes.restype = sz
    lib.la2_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.la2_fwd.restype = i
    lib.la2_fwd_state.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.la2_fwd_state.restype = i
    lib.la2_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.la2_bwd.restype = i
    lib.la2_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, sz, vp]
    lib.la2_fwd_ex.restype = i
    lib.la2_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, sz,
                               vp]
    lib.la2_bwd_ex.restype = i
    lib.la2_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.la2_decode.restype = i
    lib.la2_status_str.argtypes = [i]
    lib.la2_status_str.restype = ctypes.c_char_p
    lib.la2_device_status.argtypes = [ctypes.POINTER(ctypes.c_int), i]
    lib.la2_device_status.restype = i
    lib.la2_last_launch_count.argtypes = []
    lib.la2_last_launch_count.restype = i
    lib.la2_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.la2_fwd_noalloc.restype = i
    lib.la2_set_schedule.argtypes = [i]
    lib.la2_set_schedule.restype = i
    lib.la2_plan_info.argtypes = [i, i, i, i, i, i, i, i, ctypes.POINTER(LA2Plan), i]
    lib.la2_plan_info.restype = i
    lib.la2_selftest_timeout.argtypes = [vp, vp, vp, vp, vp, i, i, i, ctypes.c_uint, vp]
    lib.la2_selftest_timeout.restype = i
    lib.la2_bwd_state.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i,
                                  i, i, vp, sz, vp]
    lib.la2_bwd_state.restype = i
    lib.la2_dlambda_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.la2_dlambda_workspace_bytes.restype = sz
    lib.la2_dlambda.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.la2_dlambda.restype = i
    lib.la2_norm_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
    lib.la2_norm_workspace_bytes.restype = sz
    lib.la2_fwd_norm.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
    lib.la2_fwd_norm.restype = i
    lib.la2_bwd_norm.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                 vp, sz, vp]
    lib.la2_bwd_norm.restype = i
    _lib = lib
    return lib


def la2_status_str(status: int) -> str:
    return load().la2_status_str(int(status)).decode()


def la2_workspace_bytes(B, H, T, d, e, block, dtype, is_bwd) -> int:
    return int(load().la2_workspace_bytes(B, H, T, d, e, block, dtype, int(is_bwd)))


def la2_device_status(reset: bool = True) -> int:
    code = ctypes.c_int(0)
    st = load().la2_device_status(ctypes.byref(code), int(reset))
    if st != LA2_OK:
        raise LA2Error(st, "la2_device_status")
    return code.value


def la2_last_launch_count() -> int:
    return int(load().la2_last_launch_count())


class LA2Plan(ctypes.Structure):
    """la2_plan of include/la2.h."""
    _fields_ = [("d", ctypes.c_int), ("e", ctypes.c_int), ("schedule", ctypes.c_int),
                ("units", ctypes.c_longlong), ("segments", ctypes.c_int), ("tiles_per_cta", ctypes.c_int),
                ("ctas", ctypes.c_longlong), ("prepass_ctas", ctypes.c_longlong)]


def la2_plan_info(B, H, T, d, e, block=128, dtype=LA2_DTYPE_BF16, is_bwd=False) -> list:
    """The launch plan(s) of a bf16 call of these sizes, as dicts (one per
    launch group); [] for an empty problem or fp32 inputs."""
    plans = (LA2Plan * 2)()
    n = int(load().la2_plan_info(B, H, T, d, e, block, dtype, int(is_bwd), plans, 2))
    if n < 0:
        raise LA2Error(LA2_ERR_INVALID_ARG, "la2_plan_info")
    names = {LA2_SCHEDULE_UNIFORM: "uniform", LA2_SCHEDULE_BALANCED: "balanced"}
    return [{"d": p.d, "e": p.e, "schedule": names[p.schedule], "units": p.units, "segments": p.segments,
             "tiles_per_cta": p.tiles_per_cta, "ctas": p.ctas, "prepass_ctas": p.prepass_ctas}
            for p in plans[:n]]


def la2_set_schedule(schedule: str) -> str:
    """Sets how the bf16 kernels spread their work over CTAs ("auto",
    "uniform" or "balanced"); returns the previous setting."""
    prev = int(load().la2_set_schedule(_SCHEDULES[schedule]))
    return {v: k for k, v in _SCHEDULES.items()}[prev]


# ---------------------------------------------------------------- raw C calls

def la2_selftest_timeout_raw(q, k, v, decay, out, T, d, e, limit_us, stream=0) -> int:
    """Failure-path self-test: the bf16 forward kernel waits, bounded by
    limit_us, on a flag nothing sets and records LA2_ERR_TIMEOUT; returns the
    launch status (read the recorded code with la2_device_status)."""
    return int(load().la2_selftest_timeout(q, k, v, decay, out, T, d, e, limit_us, stream))


def la2_fwd_raw(q, k, v, decay, out, B, H, T, d, e, block, dtype, workspace=0, ws_bytes=0,
                stream=0) -> int:
    """The C call with integer pointers; returns the status code."""
    return int(load().la2_fwd(q, k, v, decay, out, B, H, T, d, e, block, dtype, workspace,
                              ws_bytes, stream))


def la2_fwd_noalloc_raw(q, k, v, decay, out, B, H, T, d, e, block, dtype, stream=0) -> int:
    """The allocation-free forward (scratch built into the library); returns the status."""
    return int(load().la2_fwd_noalloc(q, k, v, decay, out, B, H, T, d, e, block, dtype, stream))


def la2_bwd_raw(q, k, v, decay, dout, dq, dk, dv, B, H, T, d, e, block, dtype, workspace=0,
                ws_bytes=0, stream=0) -> int:
    return int(load().la2_bwd(q, k, v, decay, dout, dq, dk, dv, B, H, T, d, e, block, dtype,
                              workspace, ws_bytes, stream))


# ------------------------------------------------------------- torch wrappers

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LA2_DTYPE_BF16
    if t.dtype == torch.float32:
        return LA2_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float32")


def _out_dtype(out_dtype) -> tuple:
    """(torch dtype, la2_dtype code) of the outputs: fp32 (None) or bf16."""
    if out_dtype is None or out_dtype == torch.float32:
        return torch.float32, LA2_DTYPE_F32
    if out_dtype == torch.bfloat16:
        return torch.bfloat16, LA2_DTYPE_BF16
    raise TypeError(f"unsupported out_dtype {out_dtype}; expected torch.float32 or torch.bfloat16")


def _check(t: torch.Tensor, name: str, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


_ws_cache: dict = {}


def _workspace(nbytes: int, device, workspace=None):
    """(pointer, size) of a device workspace of at least nbytes (256-byte aligned).

    A caller-provided uint8 tensor is used as is; otherwise one buffer per
    device is kept and grown on demand (torch's allocator, plumbing only).
    """
    if nbytes <= 0:
        return 0, 0
    if workspace is not None:
        if not workspace.is_cuda or workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace must be a CUDA buffer of at least {nbytes} bytes")
        return workspace.data_ptr(), workspace.numel() * workspace.element_size()
    key = torch.device(device).index
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf.data_ptr(), buf.numel()


def la2_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, decay: torch.Tensor,
            out: torch.Tensor | None = None, block: int = 128, stream=None,
            workspace: torch.Tensor | None = None) -> torch.Tensor:
    """o[b,h,t] = sum_{s<=t} decay[h]^(t-s) (q[b,h,t] . k[b,h,s]) v[b,h,s], on q's device.

    q, k, v: bf16 or fp32; the output is fp32 (la2_fwd_ex also writes bf16)."""
    B, H, T, d = q.shape
    e = v.shape[-1]
    dt = _dtype_code(q)
    _check(q, "q", (B, H, T, d), q.dtype)
    _check(k, "k", (B, H, T, d), q.dtype)
    _check(v, "v", (B, H, T, e), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    if out is None:
        out = torch.empty((B, H, T, e), dtype=torch.float32, device=q.device)
    _check(out, "out", (B, H, T, e), torch.float32)
    wp, wn = _workspace(la2_workspace_bytes(B, H, T, d, e, block, dt, 0), q.device, workspace)
    st = la2_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(), out.data_ptr(),
                     B, H, T, d, e, block, dt, wp, wn, _stream_ptr(stream))
    if st != LA2_OK:
        raise LA2Error(st, "la2_fwd")
    return out


def la2_fwd_state_raw(q, k, v, decay, out, init_state, final_state, B, H, T, d, e, block, dtype,
                      workspace=0, ws_bytes=0, stream=0) -> int:
    """The C call with integer pointers (0 = NULL for the states); returns the status."""
    return int(load().la2_fwd_state(q, k, v, decay, out, init_state, final_state, B, H, T, d, e,
                                    block, dtype, workspace, ws_bytes, stream))


def la2_fwd_state(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, decay: torch.Tensor,
                  init_state: torch.Tensor | None = None, out: torch.Tensor | None = None,
                  final_state: torch.Tensor | None = None, block: int = 128, stream=None,
                  workspace: torch.Tensor | None = None):
    """(out, final_state): la2_fwd started from init_state ([B, H, d, e] fp32, None = 0),
    returning the state after the last position as well."""
    B, H, T, d = q.shape
    e = v.shape[-1]
    dt = _dtype_code(q)
    _check(q, "q", (B, H, T, d), q.dtype)
    _check(k, "k", (B, H, T, d), q.dtype)
    _check(v, "v", (B, H, T, e), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    out = torch.empty((B, H, T, e), **f32) if out is None else out
    final_state = torch.empty((B, H, d, e), **f32) if final_state is None else final_state
    _check(out, "out", (B, H, T, e), torch.float32)
    _check(final_state, "final_state", (B, H, d, e), torch.float32)
    ip = 0
    if init_state is not None:
        _check(init_state, "init_state", (B, H, d, e), torch.float32)
        ip = init_state.data_ptr()
    wp, wn = _workspace(la2_workspace_bytes(B, H, T, d, e, block, dt, 0), q.device, workspace)
    st = la2_fwd_state_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                           out.data_ptr(), ip, final_state.data_ptr(), B, H, T, d, e, block, dt,
                           wp, wn, _stream_ptr(stream))
    if st != LA2_OK:
        raise LA2Error(st, "la2_fwd_state")
    return out, final_state


def _dims(q, v, layout):
    """(B, H, T, d, e) from q's and v's shapes in the given layout."""
    if layout == "bhtd":
        B, H, T, d = q.shape
    elif layout == "bthd":
        B, T, H, d = q.shape
    else:
        raise ValueError(f"unknown layout {layout!r}; expected 'bhtd' or 'bthd'")
    return B, H, T, d, v.shape[-1]


def _shape(layout, B, H, T, D):
    return (B, H, T, D) if layout == "bhtd" else (B, T, H, D)


def la2_fwd_ex(q, k, v, decay, layout: str = "bhtd", init_state=None, out=None, final_state=None,
               want_final: bool = False, block: int = 128, stream=None, workspace=None,
               out_dtype=None):
    """la2_fwd_state for q, k, v (and out) laid out [B, H, T, D] ('bhtd') or
    [B, T, H, D] ('bthd'), out of type out_dtype (torch.float32, the default, or
    torch.bfloat16).  Returns out, or (out, final_state) with want_final or a
    final_state buffer given."""
    B, H, T, d, e = _dims(q, v, layout)
    dt = _dtype_code(q)
    odt, oc = _out_dtype(out_dtype)
    _check(q, "q", _shape(layout, B, H, T, d), q.dtype)
    _check(k, "k", _shape(layout, B, H, T, d), q.dtype)
    _check(v, "v", _shape(layout, B, H, T, e), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    out = torch.empty(_shape(layout, B, H, T, e), dtype=odt, device=q.device) if out is None else out
    _check(out, "out", _shape(layout, B, H, T, e), odt)
    if final_state is None and want_final:
        final_state = torch.empty((B, H, d, e), **f32)
    fp = 0
    if final_state is not None:
        _check(final_state, "final_state", (B, H, d, e), torch.float32)
        fp = final_state.data_ptr()
    ip = 0
    if init_state is not None:
        _check(init_state, "init_state", (B, H, d, e), torch.float32)
        ip = init_state.data_ptr()
    wp, wn = _workspace(la2_workspace_bytes(B, H, T, d, e, block, dt, 0), q.device, workspace)
    st = int(load().la2_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                               out.data_ptr(), ip, fp, B, H, T, d, e, block, dt, oc,
                               _LAYOUTS[layout], wp, wn, _stream_ptr(stream)))
    if st != LA2_OK:
        raise LA2Error(st, "la2_fwd_ex")
    return (out, final_state) if final_state is not None else out


def la2_bwd_ex(q, k, v, decay, dout, layout: str = "bhtd", dq=None, dk=None, dv=None,
               block: int = 128, stream=None, workspace=None, out_dtype=None):
    """la2_bwd for tensors laid out [B, H, T, D] ('bhtd') or [B, T, H, D] ('bthd'),
    dq, dk, dv of type out_dtype (torch.float32, the default, or torch.bfloat16)."""
    B, H, T, d, e = _dims(q, v, layout)
    dt = _dtype_code(q)
    odt, oc = _out_dtype(out_dtype)
    for t, n, D in ((q, "q", d), (k, "k", d), (v, "v", e), (dout, "dout", e)):
        _check(t, n, _shape(layout, B, H, T, D), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    o = dict(dtype=odt, device=q.device)
    dq = torch.empty(_shape(layout, B, H, T, d), **o) if dq is None else dq
    dk = torch.empty(_shape(layout, B, H, T, d), **o) if dk is None else dk
    dv = torch.empty(_shape(layout, B, H, T, e), **o) if dv is None else dv
    for t, n, D in ((dq, "dq", d), (dk, "dk", d), (dv, "dv", e)):
        _check(t, n, _shape(layout, B, H, T, D), odt)
    wp, wn = _workspace(la2_workspace_bytes(B, H, T, d, e, block, dt, 1), q.device, workspace)
    st = int(load().la2_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                               dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, T,
                               d, e, block, dt, oc, _LAYOUTS[layout], wp, wn, _stream_ptr(stream)))
    if st != LA2_OK:
        raise LA2Error(st, "la2_bwd_ex")
    return dq, dk, dv


def la2_bwd_state(q, k, v, decay, dout, init_state=None, d_final_state=None, layout: str = "bhtd",
                  dq=None, dk=None, dv=None, d_init_state=None, want_d_init: bool = True,
                  block: int = 128, stream=None, workspace=None, out_dtype=None):
    """(dq, dk, dv, d_init_state) of sum(dout * out) + sum(d_final_state * final_state) for
    the forward la2_fwd_ex(q, k, v, decay, layout, init_state); states [B, H, d, e] fp32
    (None = zero), dq, dk, dv of type out_dtype (torch.float32 or torch.bfloat16).
    d_init_state is None unless want_d_init or a buffer is given."""
    B, H, T, d, e = _dims(q, v, layout)
    dt = _dtype_code(q)
    odt, oc = _out_dtype(out_dtype)
    for t, n, D in ((q, "q", d), (k, "k", d), (v, "v", e), (dout, "dout", e)):
        _check(t, n, _shape(layout, B, H, T, D), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    o = dict(dtype=odt, device=q.device)
    dq = torch.empty(_shape(layout, B, H, T, d), **o) if dq is None else dq
    dk = torch.empty(_shape(layout, B, H, T, d), **o) if dk is None else dk
    dv = torch.empty(_shape(layout, B, H, T, e), **o) if dv is None else dv
    for t, n, D in ((dq, "dq", d), (dk, "dk", d), (dv, "dv", e)):
        _check(t, n, _shape(layout, B, H, T, D), odt)
    if d_init_state is None and want_d_init:
        d_init_state = torch.empty((B, H, d, e), **f32)
    ptrs = []
    for t, n in ((init_state, "init_state"), (d_final_state, "d_final_state"),
                 (d_init_state, "d_init_state")):
        if t is not None:
            _check(t, n, (B, H, d, e), torch.float32)
        ptrs.append(0 if t is None else t.data_ptr())
    wp, wn = _workspace(la2_workspace_bytes(B, H, T, d, e, block, dt, 1), q.device, workspace)
    st = int(load().la2_bwd_state(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                                  dout.data_ptr(), ptrs[0], ptrs[1], dq.data_ptr(), dk.data_ptr(),
                                  dv.data_ptr(), ptrs[2], B, H, T, d, e, block, dt, oc,
                                  _LAYOUTS[layout], wp, wn, _stream_ptr(stream)))
    if st != LA2_OK:
        raise LA2Error(st, "la2_bwd_state")
    return dq, dk, dv, d_init_state


def la2_dlambda_workspace_bytes(B, H, T, d, e, dtype) -> int:
    return int(load().la2_dlambda_workspace_bytes(B, H, T, d, e, dtype))


def la2_dlambda(q, k, v, decay, dout, init_state=None, d_final_state=None, layout: str = "bhtd",
                d_decay=None, stream=None, workspace=None):
    """dL/d(decay) [H] (summed over the batch) for L = sum(dout * out) + sum(d_final_state *
    final_state), the forward la2_fwd_ex(q, k, v, decay, layout, init_state)."""
    B, H, T, d, e = _dims(q, v, layout)
    dt = _dtype_code(q)
    for t, n, D in ((q, "q", d), (k, "k", d), (v, "v", e), (dout, "dout", e)):
        _check(t, n, _shape(layout, B, H, T, D), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    d_decay = torch.empty((H,), dtype=torch.float32, device=q.device) if d_decay is None else d_decay
    _check(d_decay, "d_decay", (H,), torch.float32)
    ptrs = []
    for t, n in ((init_state, "init_state"), (d_final_state, "d_final_state")):
        if t is not None:
            _check(t, n, (B, H, d, e), torch.float32)
        ptrs.append(0 if t is None else t.data_ptr())
    wp, wn = _workspace(la2_dlambda_workspace_bytes(B, H, T, d, e, dt), q.device, workspace)
    st = int(load().la2_dlambda(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                                dout.data_ptr(), ptrs[0], ptrs[1], d_decay.data_ptr(), B, H, T, d, e,
                                dt, _LAYOUTS[layout], wp, wn, _stream_ptr(stream)))
    if st != LA2_OK:
        raise LA2Error(st, "la2_dlambda")
    return d_decay


def la2_norm_workspace_bytes(B, H, T, d, e, block, dtype, is_bwd) -> int:
    return int(load().la2_norm_workspace_bytes(B, H, T, d, e, block, dtype, int(is_bwd)))


def la2_fwd_norm(q, k, v, decay, layout: str = "bhtd", y=None, den=None, block: int = 128,
                 stream=None, workspace=None):
    """(y, den): the normalised form y_t = num_t / (q_t . z_t), z_t = decay z_{t-1} + k_t."""
    B, H, T, d, e = _dims(q, v, layout)
    dt = _dtype_code(q)
    for t, n, D in ((q, "q", d), (k, "k", d), (v, "v", e)):
        _check(t, n, _shape(layout, B, H, T, D), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    y = torch.empty(_shape(layout, B, H, T, e), **f32) if y is None else y
    den = torch.empty((B, H, T), **f32) if den is None else den
    _check(y, "y", _shape(layout, B, H, T, e), torch.float32)
    _check(den, "den", (B, H, T), torch.float32)
    wp, wn = _workspace(la2_norm_workspace_bytes(B, H, T, d, e, block, dt, 0), q.device, workspace)
    st = int(load().la2_fwd_norm(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                                 y.data_ptr(), den.data_ptr(), B, H, T, d, e, block, dt,
                                 _LAYOUTS[layout], wp, wn, _stream_ptr(stream)))
    if st != LA2_OK:
        raise LA2Error(st, "la2_fwd_norm")
    return y, den


def la2_bwd_norm(q, k, v, decay, y, den, dy, layout: str = "bhtd", dq=None, dk=None, dv=None,
                 block: int = 128, stream=None, workspace=None):
    """(dq, dk, dv) of sum(dy * y) for (y, den) = la2_fwd_norm(q, k, v, decay)."""
    B, H, T, d, e = _dims(q, v, layout)
    dt = _dtype_code(q)
    for t, n, D in ((q, "q", d), (k, "k", d), (v, "v", e), (dy, "dy", e)):
        _check(t, n, _shape(layout, B, H, T, D), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    _check(y, "y", _shape(layout, B, H, T, e), torch.float32)
    _check(den, "den", (B, H, T), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty(_shape(layout, B, H, T, d), **f32) if dq is None else dq
    dk = torch.empty(_shape(layout, B, H, T, d), **f32) if dk is None else dk
    dv = torch.empty(_shape(layout, B, H, T, e), **f32) if dv is None else dv
    wp, wn = _workspace(la2_norm_workspace_bytes(B, H, T, d, e, block, dt, 1), q.device, workspace)
    st = int(load().la2_bwd_norm(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                                 y.data_ptr(), den.data_ptr(), dy.data_ptr(), dq.data_ptr(),
                                 dk.data_ptr(), dv.data_ptr(), B, H, T, d, e, block, dt,
                                 _LAYOUTS[layout], wp, wn, _stream_ptr(stream)))
    if st != LA2_OK:
        raise LA2Error(st, "la2_bwd_norm")
    return dq, dk, dv


def la2_decode_raw(q, k, v, decay, state, out, B, H, d, e, dtype, stream=0) -> int:
    return int(load().la2_decode(q, k, v, decay, state, out, B, H, d, e, dtype, stream))


def la2_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, decay: torch.Tensor,
               state: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One token per sequence: state <- decay state + k v^T (in place), returns state^T q.

    q, k: [B, H, d], v: [B, H, e] (bf16 or fp32); state: [B, H, d, e] fp32."""
    B, H, d = q.shape
    e = v.shape[-1]
    dt = _dtype_code(q)
    _check(q, "q", (B, H, d), q.dtype)
    _check(k, "k", (B, H, d), q.dtype)
    _check(v, "v", (B, H, e), q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    _check(state, "state", (B, H, d, e), torch.float32)
    out = torch.empty((B, H, e), dtype=torch.float32, device=q.device) if out is None else out
    _check(out, "out", (B, H, e), torch.float32)
    st = la2_decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(),
                        state.data_ptr(), out.data_ptr(), B, H, d, e, dt, _stream_ptr(stream))
    if st != LA2_OK:
        raise LA2Error(st, "la2_decode")
    return out


def la2_bwd(q, k, v, decay, dout, dq=None, dk=None, dv=None, block: int = 128, stream=None,
            workspace: torch.Tensor | None = None):
    """(dq, dk, dv) of sum(dout * la2_fwd(q, k, v, decay)); decay is not differentiated."""
    B, H, T, d = q.shape
    e = v.shape[-1]
    dt = _dtype_code(q)
    for t, n, shp in ((q, "q", (B, H, T, d)), (k, "k", (B, H, T, d)), (v, "v", (B, H, T, e)),
                      (dout, "dout", (B, H, T, e))):
        _check(t, n, shp, q.dtype)
    _check(decay, "decay", (H,), torch.float32)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty((B, H, T, d), **f32) if dq is None else dq
    dk = torch.empty((B, H, T, d), **f32) if dk is None else dk
    dv = torch.empty((B, H, T, e), **f32) if dv is None else dv
    for t, n, shp in ((dq, "dq", (B, H, T, d)), (dk, "dk", (B, H, T, d)), (dv, "dv", (B, H, T, e))):
        _check(t, n, shp, torch.float32)
    wp, wn = _workspace(la2_workspace_bytes(B, H, T, d, e, block, dt, 1), q.device, workspace)
    st = la2_bwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), decay.data_ptr(), dout.data_ptr(),
                     dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, T, d, e, block, dt, wp, wn,
                     _stream_ptr(stream))
    if st != LA2_OK:
        raise LA2Error(st, "la2_bwd")
    return dq, dk, dv
