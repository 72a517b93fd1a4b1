"""Python binding of the KDA C ABI (include/kda.h): argument marshalling only.

Every computation runs in the CUDA library ``libkda_b200.so`` built in-tree by
``gated_delta_rule_122_b200.build``.  If the library is missing, calls raise;
there is no fallback of any kind.  Tensors must be contiguous; device tensors
are passed as raw pointers together with the current CUDA stream.  Host
(CPU) tensors are accepted too: they are copied to the current device, the same
C entry point runs, and the results are copied back (the end-to-end path).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["KDAError", "forward", "forward_varlen", "forward_varlen_raw", "forward_varlen_gdn2", "forward_scalar_gate", "forward_gdn2",
           "forward_raw", "forward_sequential", "decode_step", "decode_step_raw",
           "decode_step_scalar_gate", "decode_step_gdn2", "decode_tokens", "state_copy",
           "selftest_bounded_wait", "set_schedule", "get_schedule", "schedule", "library",
           "library_path", "status_string", "version", "EXPORTED_SYMBOLS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkda_b200.so")
_lib = None
_lock = threading.Lock()

EXPORTED_SYMBOLS = ("kda_forward", "kda_forward_workspace_bytes", "kda_workspace_status",
                    "kda_forward_noalloc", "kda_noalloc_status", "kda_forward_varlen", "kda_forward_varlen_raw",
                    "kda_forward_varlen_gdn2", "kda_forward_scalar_gate",
                    "kda_forward_gdn2", "kda_forward_raw", "kda_forward_sequential", "kda_decode_step",
                    "kda_decode_step_gdn2", "kda_decode_step_raw", "kda_decode_step_scalar_gate",
                    "kda_decode_tokens", "kda_state_copy", "kda_selftest_bounded_wait", "kda_status_string",
                    "kda_version", "kda_forward_host", "kda_forward_host_workspace_bytes", "kda_decode_step_host",
                    "kda_decode_step_host_workspace_bytes", "kda_set_schedule", "kda_get_schedule")

_DT = {torch.float32: 0, torch.bfloat16: 1}
_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float


class KDAError(RuntimeError):
    """A non-OK status returned by the KDA C library."""

    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} (status {code})")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """Load libkda_b200.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError("the KDA CUDA library is not built (expected "
                                   f"{_LIB_PATH}); run: python -m gated_delta_rule_122_b200.build")
            lib = ctypes.CDLL(_LIB_PATH)
            fwd_args = [_vp] * 8 + [_i] * 5 + [_f] + [_i] * 3
            lib.kda_forward.argtypes = fwd_args + [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward.restype = _i
            lib.kda_forward_sequential.argtypes = fwd_args + [_vp]
            lib.kda_forward_sequential.restype = _i
            lib.kda_forward_noalloc.argtypes = fwd_args + [_vp]
            lib.kda_forward_noalloc.restype = _i
            lib.kda_noalloc_status.argtypes = [_vp]
            lib.kda_noalloc_status.restype = _i
            lib.kda_forward_varlen.argtypes = [_vp] * 9 + [_i] * 5 + [_f] + [_i] * 3 + \
                [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward_varlen.restype = _i
            lib.kda_forward_varlen_raw.argtypes = lib.kda_forward_varlen.argtypes
            lib.kda_forward_varlen_raw.restype = _i
            lib.kda_forward_varlen_gdn2.argtypes = [_vp] * 10 + [_i] * 5 + [_f] + [_i] * 3 + \
                [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward_varlen_gdn2.restype = _i
            lib.kda_forward_scalar_gate.argtypes = fwd_args + [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward_scalar_gate.restype = _i
            lib.kda_forward_raw.argtypes = fwd_args + [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward_raw.restype = _i
            lib.kda_decode_step_raw.argtypes = [_vp] * 7 + [_i] * 4 + [_f] + [_i] * 3 + [_vp]
            lib.kda_decode_step_raw.restype = _i
            lib.kda_decode_step_scalar_gate.argtypes = [_vp] * 7 + [_i] * 4 + [_f] + [_i] * 3 + [_vp]
            lib.kda_decode_step_scalar_gate.restype = _i
            lib.kda_forward_gdn2.argtypes = [_vp] * 9 + [_i] * 5 + [_f] + [_i] * 3 + \
                [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward_gdn2.restype = _i
            lib.kda_decode_step_gdn2.argtypes = [_vp] * 8 + [_i] * 4 + [_f] + [_i] * 3 + [_vp]
            lib.kda_decode_step_gdn2.restype = _i
            lib.kda_decode_tokens.argtypes = [_vp] * 6 + [_vp, _i, _i, _vp, _vp] + [_i] * 5 + [_f] + \
                [_i] * 3 + [_vp, _vp]
            lib.kda_decode_tokens.restype = _i
            lib.kda_state_copy.argtypes = [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp]
            lib.kda_state_copy.restype = _i
            lib.kda_selftest_bounded_wait.argtypes = [_i, ctypes.c_uint, _vp, _vp]
            lib.kda_selftest_bounded_wait.restype = _i
            lib.kda_forward_workspace_bytes.argtypes = [_i] * 5
            lib.kda_forward_workspace_bytes.restype = ctypes.c_size_t
            lib.kda_workspace_status.argtypes = [_vp, _vp]
            lib.kda_workspace_status.restype = _i
            lib.kda_decode_step.argtypes = [_vp] * 7 + [_i] * 4 + [_f] + [_i] * 3 + [_vp]
            lib.kda_decode_step.restype = _i
            lib.kda_status_string.argtypes = [_i]
            lib.kda_status_string.restype = ctypes.c_char_p
            lib.kda_version.argtypes = []
            lib.kda_version.restype = _i
            lib.kda_forward_host.argtypes = [_i] + fwd_args + [_vp, ctypes.c_size_t, _vp]
            lib.kda_forward_host.restype = _i
            lib.kda_forward_host_workspace_bytes.argtypes = [_i] * 9
            lib.kda_forward_host_workspace_bytes.restype = ctypes.c_size_t
            lib.kda_decode_step_host.argtypes = [_vp] * 7 + [_i] * 4 + [_f] + [_i] * 3 + [_vp, ctypes.c_size_t, _vp]
            lib.kda_decode_step_host.restype = _i
            lib.kda_decode_step_host_workspace_bytes.argtypes = [_i] * 7
            lib.kda_decode_step_host_workspace_bytes.restype = ctypes.c_size_t
            lib.kda_set_schedule.argtypes = [_i]
            lib.kda_set_schedule.restype = _i
            lib.kda_get_schedule.argtypes = []
            lib.kda_get_schedule.restype = _i
            _lib = lib
    return _lib


def status_string(code: int) -> str:
    return library().kda_status_string(int(code)).decode()


def version() -> int:
    return library().kda_version()


_SCHEDULES = {"auto": 0, "chunked": 1, "scan": 2}


def set_schedule(name: str) -> None:
    """Process-wide prefill schedule (kda_set_schedule): "auto" (the tensor-core chunk
    kernel where it applies, the column scan otherwise), "chunked" or "scan"."""
    if name not in _SCHEDULES:
        raise ValueError(f"unknown schedule {name!r}; expected one of {sorted(_SCHEDULES)}")
    code = library().kda_set_schedule(_SCHEDULES[name])
    if code != 0:
        raise KDAError("kda_set_schedule", code)


def get_schedule() -> str:
    code = library().kda_get_schedule()
    return {v: k for k, v in _SCHEDULES.items()}[code]


class schedule:
    """Context manager: ``with schedule("chunked"): ...`` sets the prefill schedule for
    the block and restores the previous one after it."""

    def __init__(self, name: str):
        self.name = name
        self.prev = None

    def __enter__(self):
        self.prev = get_schedule()
        set_schedule(self.name)
        return self

    def __exit__(self, *exc):
        set_schedule(self.prev)
        return False


def _ptr(t):
    return None if t is None else _vp(t.data_ptr())


def _dt(t: torch.Tensor, name: str) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"{name}: dtype {t.dtype} not supported (float32 or bfloat16)")
    return _DT[t.dtype]


def _check(name, t, device):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _stream_handle(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _to_device(tensors, device):
    return [None if t is None else t.to(device, non_blocking=True) for t in tensors]


# Host-buffer prefills go through the library's host-buffer entry point, which moves the
# inputs in and the results out itself (pipelined over token segments).
_HOST_KIND = {"kda_forward": 0, "kda_forward_scalar_gate": 1, "kda_forward_raw": 2}


def _prefill_host(fn_name, q, k, v, alpha, beta, initial_state, scale, output_final_state,
                  out_dtype, out, final_state, check_status, gate_per_head):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    a_shape = (B, T, H) if gate_per_head else (B, T, H, dk)
    if tuple(k.shape) != (B, T, H, dk) or tuple(v.shape[:3]) != (B, T, H) or tuple(alpha.shape) != a_shape \
            or tuple(beta.shape) != (B, T, H):
        raise ValueError("shapes: q,k [B,T,H,dk], alpha " + ("[B,T,H]" if gate_per_head else "[B,T,H,dk]")
                         + ", v [B,T,H,dv], beta [B,T,H]")
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("initial_state", initial_state), ("out", out), ("final_state", final_state)):
        if t is not None:
            if t.device.type != "cpu":
                raise ValueError(f"{name} must be a host tensor like q")
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
    if k.dtype != q.dtype or v.dtype != q.dtype or alpha.dtype != beta.dtype:
        raise TypeError("q/k/v and alpha/beta must each share a dtype")
    if initial_state is not None and (initial_state.dtype != torch.float32
                                      or tuple(initial_state.shape) != (B, H, dk, dv)):
        raise ValueError("initial_state must be float32 [B,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=out_dtype, pin_memory=True)
    if tuple(out.shape) != (B, T, H, dv):
        raise ValueError("out must be [B,T,H,dv]")
    if final_state is None and output_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=True)
    dev = torch.device("cuda", torch.cuda.current_device())
    lib = library()
    kind = _HOST_KIND[fn_name]
    qd, gd, od = _DT[q.dtype], _dt(alpha, "alpha"), _dt(out, "out")
    ws_bytes = lib.kda_forward_host_workspace_bytes(B, T, H, dk, dv, qd, gd, od, kind)
    with torch.cuda.device(dev):
        ws = torch.empty(max(ws_bytes, 256), device=dev, dtype=torch.uint8)
        stream = _vp(_stream_handle(dev))
        code = lib.kda_forward_host(kind, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(initial_state),
                                    _ptr(out), _ptr(final_state), B, T, H, dk, dv, float(scale), qd, gd, od,
                                    _ptr(ws), ws.numel(), stream)
        if code == 0 and check_status:
            code = lib.kda_workspace_status(_ptr(ws), stream)
        torch.cuda.current_stream(dev).synchronize()
    if code != 0:
        raise KDAError("kda_forward_host", code)
    return out, final_state


def _prefill(fn_name, q, k, v, alpha, beta, initial_state, scale, output_final_state,
             out_dtype, out, final_state, workspace=None, check_status=False, gate_per_head=False):
    host = q.device.type == "cpu"
    if host and fn_name in _HOST_KIND:
        return _prefill_host(fn_name, q, k, v, alpha, beta, initial_state, scale, output_final_state,
                             out_dtype, out, final_state, check_status, gate_per_head)
    host_out = host_state = None
    if host:
        # end-to-end path: host inputs are copied in (asynchronously when pinned),
        # results are copied back into host tensors before returning
        dev = torch.device("cuda", torch.cuda.current_device())
        q, k, v, alpha, beta, initial_state = _to_device(
            [q, k, v, alpha, beta, initial_state], dev)
        host_out, host_state = out, final_state
        out = None if out is None else torch.empty(out.shape, device=dev, dtype=out.dtype)
        final_state = None if final_state is None else torch.empty(final_state.shape, device=dev,
                                                                    dtype=final_state.dtype)
    device = q.device
    if device.type != "cuda":
        raise ValueError("KDA runs on CUDA devices only")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta)):
        _check(name, t, device)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share a dtype")
    if alpha.dtype != beta.dtype:
        raise TypeError("alpha and beta must share a dtype")
    a_shape = (B, T, H) if gate_per_head else (B, T, H, dk)
    if tuple(k.shape) != (B, T, H, dk) or tuple(alpha.shape) != a_shape \
            or tuple(v.shape) != (B, T, H, dv) or tuple(beta.shape) != (B, T, H):
        raise ValueError("shapes: q,k [B,T,H,dk], alpha " + ("[B,T,H]" if gate_per_head else "[B,T,H,dk]")
                         + ", v [B,T,H,dv], beta [B,T,H]")
    if initial_state is not None:
        _check("initial_state", initial_state, device)
        if initial_state.dtype != torch.float32 or tuple(initial_state.shape) != (B, H, dk, dv):
            raise ValueError("initial_state must be float32 [B,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((B, T, H, dv), device=device, dtype=out_dtype)
    _check("out", out, device)
    if final_state is None and output_final_state:
        final_state = torch.empty((B, H, dk, dv), device=device, dtype=torch.float32)
    if final_state is not None:
        _check("final_state", final_state, device)
    lib = library()
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(initial_state), _ptr(out),
            _ptr(final_state), B, T, H, dk, dv, float(scale), _DT[q.dtype], _dt(alpha, "alpha"),
            _dt(out, "out")]
    with torch.cuda.device(device):
        stream = _vp(_stream_handle(device))
        if fn_name in ("kda_forward", "kda_forward_scalar_gate", "kda_forward_raw"):
            ws_bytes = lib.kda_forward_workspace_bytes(B, T, H, dk, dv)
            ws = workspace
            if ws is None or ws.numel() * ws.element_size() < ws_bytes:
                ws = torch.empty(max(ws_bytes, 16), device=device, dtype=torch.uint8)
            code = getattr(lib, fn_name)(*args, _ptr(ws), ws.numel() * ws.element_size(), stream)
            if code == 0 and check_status:
                code = lib.kda_workspace_status(_ptr(ws), stream)
        else:
            code = lib.kda_forward_sequential(*args, stream)
    if code != 0:
        raise KDAError(fn_name, code)
    if host:
        with torch.cuda.device(device):
            if host_out is None:
                host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
            host_out.copy_(out, non_blocking=True)
            if final_state is not None:
                if host_state is None:
                    host_state = torch.empty(final_state.shape, dtype=final_state.dtype,
                                             pin_memory=True)
                host_state.copy_(final_state, non_blocking=True)
            torch.cuda.current_stream(device).synchronize()
        return host_out, (host_state if final_state is not None else None)
    return out, final_state


def forward(q, k, v, alpha, beta, initial_state=None, scale=None, output_final_state=True,
            out_dtype=torch.float32, out=None, final_state=None, workspace=None,
            check_status=False):
    """Chunkwise KDA prefill (C entry point ``kda_forward``).

    q, k, alpha: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H] (q/k/v share a dtype,
    alpha/beta share a dtype; float32 or bfloat16).  initial_state: float32
    [B,H,dk,dv] or None.  workspace: optional device uint8 tensor of at least
    ``kda_forward_workspace_bytes`` bytes (allocated per call when omitted).
    check_status=True synchronizes and raises KDAError if a bounded device wait
    timed out.  Returns (o [B,T,H,dv] of out_dtype, final_state or None).
    """
    return _prefill("kda_forward", q, k, v, alpha, beta, initial_state, scale,
                    output_final_state, out_dtype, out, final_state, workspace, check_status)


def forward_scalar_gate(q, k, v, alpha, beta, initial_state=None, scale=None, output_final_state=True,
                        out_dtype=torch.float32, out=None, final_state=None, workspace=None,
                        check_status=False):
    """Gated DeltaNet prefill: one retention factor per (token, head), alpha [B,T,H]
    (C entry point ``kda_forward_scalar_gate``); otherwise the contract of ``forward``."""
    return _prefill("kda_forward_scalar_gate", q, k, v, alpha, beta, initial_state, scale,
                    output_final_state, out_dtype, out, final_state, workspace, check_status,
                    gate_per_head=True)


def forward_raw(q, k, v, gate_logit, beta_logit, initial_state=None, scale=None, output_final_state=True,
                out_dtype=torch.float32, out=None, final_state=None, workspace=None, check_status=False):
    """Prefill with the input preprocessing fused into the kernels (C entry point
    ``kda_forward_raw``): q, k un-normalised (each row divided by its L2 norm in the
    kernel), gate_logit [B,T,H,dk] with alpha = exp(-softplus(x)), beta_logit [B,T,H]
    with beta = sigmoid(y); otherwise the contract of ``forward``."""
    return _prefill("kda_forward_raw", q, k, v, gate_logit, beta_logit, initial_state, scale,
                    output_final_state, out_dtype, out, final_state, workspace, check_status)


def forward_sequential(q, k, v, alpha, beta, initial_state=None, scale=None,
                       output_final_state=True, out_dtype=torch.float32, out=None,
                       final_state=None):
    """The token-by-token schedule (C entry point ``kda_forward_sequential``); same contract."""
    return _prefill("kda_forward_sequential", q, k, v, alpha, beta, initial_state, scale,
                    output_final_state, out_dtype, out, final_state)


def _decode(fn, q, k, v, alpha, beta, state, scale, out_dtype, out, gate_per_head=False):
    """Shared marshalling of the one-token decode entry points (C function ``fn``)."""
    device = state.device
    if device.type != "cuda":
        raise ValueError("the decode step needs the state on a CUDA device")
    N, H, dk, dv = state.shape
    if fn == "kda_decode_step" and q.device.type == "cpu":
        return _decode_host(q, k, v, alpha, beta, state, scale, out_dtype, out)
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("state", state)):
        _check(name, t, device)
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    a_shape = (N, H) if gate_per_head else (N, H, dk)
    if tuple(q.shape) != (N, H, dk) or tuple(k.shape) != (N, H, dk) or \
            tuple(alpha.shape) != a_shape or tuple(v.shape) != (N, H, dv) or \
            tuple(beta.shape) != (N, H):
        raise ValueError("shapes: q,k [N,H,dk], alpha " + ("[N,H]" if gate_per_head else "[N,H,dk]")
                         + ", v [N,H,dv], beta [N,H], state [N,H,dk,dv]")
    if k.dtype != q.dtype or v.dtype != q.dtype or alpha.dtype != beta.dtype:
        raise TypeError("q/k/v and alpha/beta must each share a dtype")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((N, H, dv), device=device, dtype=out_dtype)
    _check("out", out, device)
    with torch.cuda.device(device):
        code = getattr(library(), fn)(
            _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(out),
            N, H, dk, dv, float(scale), _DT[q.dtype], _dt(alpha, "alpha"), _dt(out, "out"),
            _vp(_stream_handle(device)))
    if code != 0:
        raise KDAError(fn, code)
    return out


def _decode_host(q, k, v, alpha, beta, state, scale, out_dtype, out):
    """Decode step with host token vectors and host o, the state resident on the device
    (C entry point ``kda_decode_step_host``)."""
    device = state.device
    N, H, dk, dv = state.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor like q")
    _check("state", state, device)
    if tuple(q.shape) != (N, H, dk) or tuple(k.shape) != (N, H, dk) or tuple(alpha.shape) != (N, H, dk) \
            or tuple(v.shape) != (N, H, dv) or tuple(beta.shape) != (N, H):
        raise ValueError("shapes: q,k,alpha [N,H,dk], v [N,H,dv], beta [N,H], state [N,H,dk,dv]")
    if k.dtype != q.dtype or v.dtype != q.dtype or alpha.dtype != beta.dtype or state.dtype != torch.float32:
        raise TypeError("q/k/v and alpha/beta must each share a dtype; the state is float32")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((N, H, dv), dtype=out_dtype, pin_memory=True)
    if out.device.type != "cpu" or tuple(out.shape) != (N, H, dv):
        raise ValueError("out must be a host tensor [N,H,dv]")
    lib = library()
    qd, gd, od = _DT[q.dtype], _dt(alpha, "alpha"), _dt(out, "out")
    with torch.cuda.device(device):
        nb = lib.kda_decode_step_host_workspace_bytes(N, H, dk, dv, qd, gd, od)
        ws = torch.empty(max(nb, 256), device=device, dtype=torch.uint8)
        code = lib.kda_decode_step_host(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(out),
                                        N, H, dk, dv, float(scale), qd, gd, od, _ptr(ws), ws.numel(),
                                        _vp(_stream_handle(device)))
        torch.cuda.current_stream(device).synchronize()
    if code != 0:
        raise KDAError("kda_decode_step_host", code)
    return out


def decode_step(q, k, v, alpha, beta, state, scale=None, out_dtype=torch.float32, out=None):
    """One token per sequence (C entry point ``kda_decode_step``); ``state`` [N,H,dk,dv]
    float32 is updated in place.

    q, k, alpha: [N,H,dk]; v: [N,H,dv]; beta: [N,H].  Returns o [N,H,dv].
    """
    return _decode("kda_decode_step", q, k, v, alpha, beta, state, scale, out_dtype, out)


def decode_step_scalar_gate(q, k, v, alpha, beta, state, scale=None, out_dtype=torch.float32, out=None):
    """Gated DeltaNet decode step: alpha [N,H], one retention factor per (sequence, head)
    (C entry point ``kda_decode_step_scalar_gate``); otherwise the contract of ``decode_step``."""
    return _decode("kda_decode_step_scalar_gate", q, k, v, alpha, beta, state, scale, out_dtype, out,
                   gate_per_head=True)


def decode_step_raw(q, k, v, gate_logit, beta_logit, state, scale=None, out_dtype=torch.float32, out=None):
    """Decode step on raw inputs (C entry point ``kda_decode_step_raw``): the preprocessing
    of ``forward_raw``; otherwise the contract of ``decode_step``."""
    return _decode("kda_decode_step_raw", q, k, v, gate_logit, beta_logit, state, scale, out_dtype, out)


def _varlen(fn, q, k, v, alpha, beta, write, cu_seqlens, initial_state, scale, output_final_state, out_dtype,
            out, final_state, workspace, check_status):
    """Shared marshalling of the packed-sequence prefills (C function ``fn``); for GDN-2
    ``beta`` is the erase gate and ``write`` the write gate."""
    device = q.device
    if device.type != "cuda":
        raise ValueError("KDA runs on CUDA devices only")
    gdn2 = write is not None
    squeeze = q.dim() == 4
    if squeeze:
        if q.shape[0] != 1:
            raise ValueError("packed tensors are [total_T,H,d] or [1,total_T,H,d]")
        q, k, v, alpha, beta = (t[0] for t in (q, k, v, alpha, beta))
        if gdn2:
            write = write[0]
    total_T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta),
                    ("cu_seqlens", cu_seqlens)) + ((("write", write),) if gdn2 else ()):
        _check(name, t, device)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor [N+1]")
    N = cu_seqlens.numel() - 1
    b_shape = (total_T, H, dk) if gdn2 else (total_T, H)
    if tuple(k.shape) != (total_T, H, dk) or tuple(alpha.shape) != (total_T, H, dk) or \
            tuple(v.shape) != (total_T, H, dv) or tuple(beta.shape) != b_shape or \
            (gdn2 and tuple(write.shape) != (total_T, H, dv)):
        raise ValueError("shapes: q,k,alpha [total_T,H,dk], v [total_T,H,dv], " +
                         ("erase [total_T,H,dk], write [total_T,H,dv]" if gdn2 else "beta [total_T,H]"))
    if k.dtype != q.dtype or v.dtype != q.dtype or alpha.dtype != beta.dtype or \
            (gdn2 and write.dtype != alpha.dtype):
        raise TypeError("q/k/v and the gates must each share a dtype")
    if initial_state is not None:
        _check("initial_state", initial_state, device)
        if initial_state.dtype != torch.float32 or tuple(initial_state.shape) != (N, H, dk, dv):
            raise ValueError("initial_state must be float32 [N,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((total_T, H, dv), device=device, dtype=out_dtype)
    _check("out", out, device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), device=device, dtype=torch.float32)
    if final_state is not None:
        _check("final_state", final_state, device)
    lib = library()
    with torch.cuda.device(device):
        stream = _vp(_stream_handle(device))
        ws_bytes = lib.kda_forward_workspace_bytes(N, total_T, H, dk, dv)
        ws = workspace
        if ws is None or ws.numel() * ws.element_size() < ws_bytes:
            ws = torch.empty(max(ws_bytes, 16), device=device, dtype=torch.uint8)
        gates = (_ptr(alpha), _ptr(beta), _ptr(write)) if gdn2 else (_ptr(alpha), _ptr(beta))
        code = getattr(lib, fn)(
            _ptr(q), _ptr(k), _ptr(v), *gates, _ptr(cu_seqlens),
            _ptr(initial_state), _ptr(out), _ptr(final_state), N, total_T, H, dk, dv,
            float(scale), _DT[q.dtype], _dt(alpha, "alpha"), _dt(out, "out"), _ptr(ws),
            ws.numel() * ws.element_size(), stream)
        if code == 0 and check_status:
            code = lib.kda_workspace_status(_ptr(ws), stream)
    if code != 0:
        raise KDAError(fn, code)
    return (out.unsqueeze(0) if squeeze else out), final_state


def forward_varlen(q, k, v, alpha, beta, cu_seqlens, initial_state=None, scale=None,
                   output_final_state=True, out_dtype=torch.float32, out=None, final_state=None,
                   workspace=None, check_status=False):
    """Prefill over packed sequences of different lengths (C entry point ``kda_forward_varlen``).

    q, k, alpha: [total_T,H,dk] (or [1,total_T,H,dk]); v: [total_T,H,dv]; beta: [total_T,H];
    cu_seqlens: int32 [N+1] on the same device (0, then cumulative lengths).  initial_state:
    float32 [N,H,dk,dv] or None.  check_status=True synchronizes and raises KDAError on
    invalid offsets or a timed-out device wait.  Returns (o [total_T,H,dv], final_state or None).
    """
    return _varlen("kda_forward_varlen", q, k, v, alpha, beta, None, cu_seqlens, initial_state, scale,
                   output_final_state, out_dtype, out, final_state, workspace, check_status)


def forward_varlen_raw(q, k, v, gate_logit, beta_logit, cu_seqlens, initial_state=None, scale=None,
                       output_final_state=True, out_dtype=torch.float32, out=None, final_state=None,
                       workspace=None, check_status=False):
    """Packed-sequence prefill on raw inputs (C entry point ``kda_forward_varlen_raw``): the
    preprocessing of ``forward_raw`` with the layouts of ``forward_varlen``."""
    return _varlen("kda_forward_varlen_raw", q, k, v, gate_logit, beta_logit, None, cu_seqlens, initial_state,
                   scale, output_final_state, out_dtype, out, final_state, workspace, check_status)


def forward_varlen_gdn2(q, k, v, alpha, erase, write, cu_seqlens, initial_state=None, scale=None,
                        output_final_state=True, out_dtype=torch.float32, out=None, final_state=None,
                        workspace=None, check_status=False):
    """Packed-sequence GDN-2 prefill (C entry point ``kda_forward_varlen_gdn2``): erase
    [total_T,H,dk] and write [total_T,H,dv] gates in place of beta; otherwise ``forward_varlen``."""
    return _varlen("kda_forward_varlen_gdn2", q, k, v, alpha, erase, write, cu_seqlens, initial_state, scale,
                   output_final_state, out_dtype, out, final_state, workspace, check_status)


def forward_gdn2(q, k, v, alpha, erase, write, initial_state=None, scale=None, output_final_state=True,
                 out_dtype=torch.float32, out=None, final_state=None, workspace=None, check_status=False):
    """GDN-2 prefill (C entry point ``kda_forward_gdn2``): erase [B,T,H,dk] and write
    [B,T,H,dv] gates (alpha's dtype) in place of beta; otherwise the contract of ``forward``."""
    device = q.device
    if device.type != "cuda":
        raise ValueError("KDA runs on CUDA devices only")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("erase", erase), ("write", write)):
        _check(name, t, device)
    if tuple(k.shape) != (B, T, H, dk) or tuple(alpha.shape) != (B, T, H, dk) or \
            tuple(erase.shape) != (B, T, H, dk) or tuple(v.shape) != (B, T, H, dv) or \
            tuple(write.shape) != (B, T, H, dv):
        raise ValueError("shapes: q,k,alpha,erase [B,T,H,dk], v,write [B,T,H,dv]")
    if k.dtype != q.dtype or v.dtype != q.dtype or erase.dtype != alpha.dtype or write.dtype != alpha.dtype:
        raise TypeError("q/k/v and alpha/erase/write must each share a dtype")
    if initial_state is not None:
        _check("initial_state", initial_state, device)
        if initial_state.dtype != torch.float32 or tuple(initial_state.shape) != (B, H, dk, dv):
            raise ValueError("initial_state must be float32 [B,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((B, T, H, dv), device=device, dtype=out_dtype)
    _check("out", out, device)
    if final_state is None and output_final_state:
        final_state = torch.empty((B, H, dk, dv), device=device, dtype=torch.float32)
    if final_state is not None:
        _check("final_state", final_state, device)
    lib = library()
    with torch.cuda.device(device):
        stream = _vp(_stream_handle(device))
        ws_bytes = lib.kda_forward_workspace_bytes(B, T, H, dk, dv)
        ws = workspace
        if ws is None or ws.numel() * ws.element_size() < ws_bytes:
            ws = torch.empty(max(ws_bytes, 16), device=device, dtype=torch.uint8)
        code = lib.kda_forward_gdn2(
            _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(erase), _ptr(write), _ptr(initial_state),
            _ptr(out), _ptr(final_state), B, T, H, dk, dv, float(scale), _DT[q.dtype],
            _dt(alpha, "alpha"), _dt(out, "out"), _ptr(ws), ws.numel() * ws.element_size(), stream)
        if code == 0 and check_status:
            code = lib.kda_workspace_status(_ptr(ws), stream)
    if code != 0:
        raise KDAError("kda_forward_gdn2", code)
    return out, final_state


def decode_step_gdn2(q, k, v, alpha, erase, write, state, scale=None, out_dtype=torch.float32, out=None):
    """GDN-2 decode step (C entry point ``kda_decode_step_gdn2``): erase [N,H,dk] and write
    [N,H,dv] in place of beta; ``state`` [N,H,dk,dv] float32 is updated in place."""
    device = state.device
    N, H, dk, dv = state.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("erase", erase), ("write", write),
                    ("state", state)):
        _check(name, t, device)
    if tuple(q.shape) != (N, H, dk) or tuple(k.shape) != (N, H, dk) or tuple(alpha.shape) != (N, H, dk) \
            or tuple(erase.shape) != (N, H, dk) or tuple(v.shape) != (N, H, dv) or tuple(write.shape) != (N, H, dv):
        raise ValueError("shapes: q,k,alpha,erase [N,H,dk], v,write [N,H,dv], state [N,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((N, H, dv), device=device, dtype=out_dtype)
    _check("out", out, device)
    with torch.cuda.device(device):
        code = library().kda_decode_step_gdn2(
            _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(erase), _ptr(write), _ptr(state), _ptr(out),
            N, H, dk, dv, float(scale), _DT[q.dtype], _dt(alpha, "alpha"), _dt(out, "out"),
            _vp(_stream_handle(device)))
    if code != 0:
        raise KDAError("kda_decode_step_gdn2", code)
    return out


def _status_word(device):
    return torch.zeros(16, device=device, dtype=torch.uint8)


def decode_tokens(q, k, v, alpha, beta, state, state_slots=None, commit=True, token_states=None,
                  scale=None, out_dtype=torch.float32, out=None, check_status=False):
    """T tokens per sequence through the decode recurrence (C entry point ``kda_decode_tokens``).

    q, k, alpha [N,T,H,dk]; v [N,T,H,dv]; beta [N,T,H]; ``state`` is a pool
    [slots,H,dk,dv] float32; sequence n uses slot ``state_slots[n]`` (int32 [N] on the
    device; None: slot n; negative: skipped).  ``commit`` writes the state after the
    T tokens back to the slot; ``token_states`` ([N,T,H,dk,dv] float32, or True to
    allocate one) receives the state after every token.  Returns (o [N,T,H,dv],
    token_states or None).
    """
    device = state.device
    if device.type != "cuda":
        raise ValueError("decode_tokens needs the state pool on a CUDA device")
    slots, H, dk, dv = state.shape
    N, T = q.shape[0], q.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta), ("state", state)):
        _check(name, t, device)
    if state.dtype != torch.float32:
        raise TypeError("state must be float32")
    if tuple(q.shape) != (N, T, H, dk) or tuple(k.shape) != (N, T, H, dk) or \
            tuple(alpha.shape) != (N, T, H, dk) or tuple(v.shape) != (N, T, H, dv) or \
            tuple(beta.shape) != (N, T, H):
        raise ValueError("shapes: q,k,alpha [N,T,H,dk], v [N,T,H,dv], beta [N,T,H], state [slots,H,dk,dv]")
    if k.dtype != q.dtype or v.dtype != q.dtype or alpha.dtype != beta.dtype:
        raise TypeError("q/k/v and alpha/beta must each share a dtype")
    if state_slots is not None:
        _check("state_slots", state_slots, device)
        if state_slots.dtype != torch.int32 or tuple(state_slots.shape) != (N,):
            raise ValueError("state_slots must be int32 [N]")
    if token_states is True:
        token_states = torch.empty((N, T, H, dk, dv), device=device, dtype=torch.float32)
    if token_states is not None:
        _check("token_states", token_states, device)
        if token_states.dtype != torch.float32 or tuple(token_states.shape) != (N, T, H, dk, dv):
            raise ValueError("token_states must be float32 [N,T,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((N, T, H, dv), device=device, dtype=out_dtype)
    _check("out", out, device)
    status = _status_word(device) if check_status else None
    lib = library()
    with torch.cuda.device(device):
        stream = _vp(_stream_handle(device))
        code = lib.kda_decode_tokens(
            _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(state), _ptr(state_slots), slots,
            int(bool(commit)), _ptr(token_states), _ptr(out), N, T, H, dk, dv, float(scale), _DT[q.dtype],
            _dt(alpha, "alpha"), _dt(out, "out"), _ptr(status), stream)
        if code == 0 and status is not None:
            code = lib.kda_workspace_status(_ptr(status), stream)
    if code != 0:
        raise KDAError("kda_decode_tokens", code)
    return out, token_states


def state_copy(src, dst, src_index=None, dst_index=None, count=None, check_status=False):
    """Copy whole states between pools (C entry point ``kda_state_copy``): entry i copies
    ``src[src_index[i]]`` to ``dst[dst_index[i]]`` (int32 [count] on the device; None:
    identity; negative: skipped).  ``src`` and ``dst`` are float32 [slots,H,dk,dv] and
    may be the same tensor (a fork inside one pool)."""
    device = dst.device
    if device.type != "cuda":
        raise ValueError("state_copy needs CUDA tensors")
    _check("src", src, device)
    _check("dst", dst, device)
    if src.dtype != torch.float32 or dst.dtype != torch.float32 or src.dim() != 4 or \
            tuple(src.shape[1:]) != tuple(dst.shape[1:]):
        raise ValueError("src and dst must be float32 [slots,H,dk,dv] with equal H, dk, dv")
    for name, t in (("src_index", src_index), ("dst_index", dst_index)):
        if t is not None:
            _check(name, t, device)
            if t.dtype != torch.int32 or t.dim() != 1:
                raise ValueError(name + " must be int32 [count]")
    if count is None:
        idx = src_index if src_index is not None else dst_index
        count = idx.numel() if idx is not None else min(src.shape[0], dst.shape[0])
    _, H, dk, dv = dst.shape
    status = _status_word(device) if check_status else None
    lib = library()
    with torch.cuda.device(device):
        stream = _vp(_stream_handle(device))
        code = lib.kda_state_copy(_ptr(src), _ptr(src_index), src.shape[0], _ptr(dst), _ptr(dst_index),
                                  dst.shape[0], int(count), H, dk, dv, _ptr(status), stream)
        if code == 0 and status is not None:
            code = lib.kda_workspace_status(_ptr(status), stream)
    if code != 0:
        raise KDAError("kda_state_copy", code)
    return dst


def selftest_bounded_wait(arrive, limit_us=20000, device=None):
    """Run the device-side bounded-wait check (C entry point ``kda_selftest_bounded_wait``)
    and return the status code that ``kda_workspace_status`` reads back: 0 when the
    barrier was completed (arrive=True), KDA_ERR_TIMEOUT (8) after a wait that gave up."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    status = _status_word(device)
    lib = library()
    with torch.cuda.device(device):
        stream = _vp(_stream_handle(device))
        code = lib.kda_selftest_bounded_wait(int(bool(arrive)), int(limit_us), _ptr(status), stream)
        if code != 0:
            raise KDAError("kda_selftest_bounded_wait", code)
        return lib.kda_workspace_status(_ptr(status), stream)
