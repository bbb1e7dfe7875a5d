"""Python binding of the B200 MoDA library (``libmoda_b200.so``, C ABI in include/moda.h).

Argument marshalling only: every step of the operator runs in the library's sm_100a
kernels.  PyTorch supplies device memory and the current CUDA stream.  There is no CPU
or PyTorch fallback: if the compiled library is missing, importing the binding raises.

Low-level names mirror the C ABI (``moda_forward``, ``moda_backward``,
``moda_backward_workspace_size``, ``moda_check_device_errors``, ``moda_status_string``);
``forward`` / ``backward`` allocate outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoda_b200.so")

MODA_OK = 0
MODA_ERR_INVALID_ARGUMENT = 1
MODA_ERR_UNSUPPORTED = 2
MODA_ERR_CUDA = 3
MODA_ERR_TIMEOUT = 4
MODA_ERR_INTERNAL = 5

# Kernel launches one moda_backward call makes (row terms + depth, sequence, dQ convert),
# one per stage of moda_backward_stages.
BACKWARD_LAUNCHES = 3

# Every symbol include/moda.h declares (checked by the ABI tests).
EXPORTED = ("moda_forward", "moda_forward_depth_path", "moda_depth_attention_forward",
            "moda_depth_attention_backward", "moda_decode", "moda_decode_workspace_size",
            "moda_depth_kv_write",
            "moda_backward", "moda_backward_workspace_size",
            "moda_backward_stages", "moda_backward_noalloc", "moda_check_device_errors",
            "moda_test_set_device_fault", "moda_test_exp2_fma", "moda_status_string",
            "moda_last_error_message")


class ModaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({message})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python depth_aware_attention_b200/build.py`"
            " (or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.moda_forward.argtypes = [P] * 7 + [I] * 6 + [F, I, P]
    lib.moda_forward.restype = I
    lib.moda_forward_depth_path.argtypes = [P] * 7 + [I] * 6 + [F, I, I, P]
    lib.moda_forward_depth_path.restype = I
    lib.moda_depth_attention_forward.argtypes = [P] * 5 + [I] * 6 + [F, P]
    lib.moda_depth_attention_forward.restype = I
    lib.moda_depth_attention_backward.argtypes = [P] * 10 + [S] + [I] * 6 + [F, P]
    lib.moda_depth_attention_backward.restype = I
    lib.moda_decode_workspace_size.argtypes = [I] * 6
    lib.moda_decode_workspace_size.restype = S
    lib.moda_decode.argtypes = [P] * 8 + [S] + [I] * 6 + [F, P]
    lib.moda_decode.restype = I
    lib.moda_depth_kv_write.argtypes = [P] * 4 + [I] * 7 + [P]
    lib.moda_depth_kv_write.restype = I
    lib.moda_backward_workspace_size.argtypes = [I] * 6
    lib.moda_backward_workspace_size.restype = S
    lib.moda_backward.argtypes = [P] * 14 + [S] + [I] * 6 + [F, I, P]
    lib.moda_backward.restype = I
    lib.moda_backward_stages.argtypes = [P] * 14 + [S] + [I] * 6 + [F, I, ctypes.c_uint, P]
    lib.moda_backward_stages.restype = I
    lib.moda_backward_noalloc.argtypes = [P] * 13 + [I] * 6 + [F, I, P]
    lib.moda_backward_noalloc.restype = I
    lib.moda_test_set_device_fault.argtypes = [I, ctypes.c_uint64]
    lib.moda_test_set_device_fault.restype = I
    lib.moda_test_exp2_fma.argtypes = [P, P, I, P]
    lib.moda_test_exp2_fma.restype = I
    lib.moda_check_device_errors.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.moda_check_device_errors.restype = I
    lib.moda_status_string.argtypes = [I]
    lib.moda_status_string.restype = ctypes.c_char_p
    lib.moda_last_error_message.argtypes = []
    lib.moda_last_error_message.restype = ctypes.c_char_p
    return lib


lib = _load()


def _msg(status):
    detail = lib.moda_last_error_message().decode()
    base = lib.moda_status_string(status).decode()
    return f"{base}: {detail}" if detail else base


def _check(status, where):
    if status != MODA_OK:
        raise ModaError(status, where, _msg(status))


# ---------------------------------------------------------------- C-ABI mirrors
def moda_forward(q, k, v, kd, vd, out, lse, B, Hq, Hkv, T, L, d, scale, causal, stream):
    """Direct call of the C entry point with raw pointers (ints) and a stream handle."""
    return lib.moda_forward(q, k, v, kd, vd, out, lse, B, Hq, Hkv, T, L, d, float(scale),
                            int(causal), stream)


def moda_forward_depth_path(q, k, v, kd, vd, out, lse, B, Hq, Hkv, T, L, d, scale, causal,
                            depth_path, stream):
    """Direct call of moda_forward_depth_path with raw pointers (ints) and a stream handle."""
    return lib.moda_forward_depth_path(q, k, v, kd, vd, out, lse, B, Hq, Hkv, T, L, d,
                                       float(scale), int(causal), int(depth_path), stream)


def moda_depth_attention_forward(q, kd, vd, out, lse, B, Hq, Hkv, T, L, d, scale, stream):
    """Direct call of moda_depth_attention_forward with raw pointers (ints)."""
    return lib.moda_depth_attention_forward(q, kd, vd, out, lse, B, Hq, Hkv, T, L, d,
                                            float(scale), stream)


def moda_depth_attention_backward(q, kd, vd, out, lse, dout, dq, dkd, dvd, workspace,
                                  workspace_bytes, B, Hq, Hkv, T, L, d, scale, stream):
    """Direct call of moda_depth_attention_backward with raw pointers (ints)."""
    return lib.moda_depth_attention_backward(q, kd, vd, out, lse, dout, dq, dkd, dvd,
                                             workspace, workspace_bytes, B, Hq, Hkv, T, L, d,
                                             float(scale), stream)


def moda_decode_workspace_size(B, Hq, Hkv, S, L, d):
    return lib.moda_decode_workspace_size(B, Hq, Hkv, S, L, d)


def moda_decode(q, k, v, kd, vd, out, lse, workspace, workspace_bytes, B, Hq, Hkv, S, L, d,
                scale, stream):
    """Direct call of moda_decode with raw pointers (ints)."""
    return lib.moda_decode(q, k, v, kd, vd, out, lse, workspace, workspace_bytes, B, Hq, Hkv,
                           S, L, d, float(scale), stream)


def moda_depth_kv_write(x, w, kd, vd, B, T, hidden, Hkv, d, L, slot, stream):
    """Direct call of moda_depth_kv_write with raw pointers (ints)."""
    return lib.moda_depth_kv_write(x, w, kd, vd, B, T, hidden, Hkv, d, L, slot, stream)


def moda_backward(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, workspace,
                  workspace_bytes, B, Hq, Hkv, T, L, d, scale, causal, stream):
    return lib.moda_backward(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd,
                             workspace, workspace_bytes, B, Hq, Hkv, T, L, d, float(scale),
                             int(causal), stream)


def moda_backward_noalloc(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, B, Hq, Hkv,
                          T, L, d, scale, causal, stream):
    """The backward with library-owned static scratch (no workspace argument)."""
    return lib.moda_backward_noalloc(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, B,
                                     Hq, Hkv, T, L, d, float(scale), int(causal), stream)


def moda_backward_stages(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, workspace,
                         workspace_bytes, B, Hq, Hkv, T, L, d, scale, causal, stages, stream):
    return lib.moda_backward_stages(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd,
                                    workspace, workspace_bytes, B, Hq, Hkv, T, L, d,
                                    float(scale), int(causal), int(stages), stream)


def moda_backward_workspace_size(B, Hq, Hkv, T, L, d):
    return int(lib.moda_backward_workspace_size(B, Hq, Hkv, T, L, d))


def moda_check_device_errors(stream=None):
    """Synchronise `stream`; returns (status, flags) and clears the device error word."""
    flags = ctypes.c_uint32(0)
    st = lib.moda_check_device_errors(stream, ctypes.byref(flags))
    return st, int(flags.value)


def moda_test_set_device_fault(fault, wait_limit_ns=0):
    """TEST ONLY: set the kernels' injected fault and bounded-wait limit on the current
    device (0, 0 restores the normal state).  Returns the status."""
    return lib.moda_test_set_device_fault(int(fault), int(wait_limit_ns))


def moda_test_exp2_fma(x_ptr, y_ptr, n, stream=None):
    """TEST ONLY: raw call of the forward's FMA-pipe exp2 over n fp32 values; returns the
    status."""
    return lib.moda_test_exp2_fma(x_ptr, y_ptr, int(n), stream)


def test_exp2_fma(x):
    """TEST ONLY: 2^x for a contiguous fp32 CUDA tensor, by the forward kernel's FMA-pipe
    exponential, on the current stream."""
    import torch
    if not (x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    st = lib.moda_test_exp2_fma(x.data_ptr(), y.data_ptr(), x.numel(),
                                torch.cuda.current_stream(x.device).cuda_stream)
    _check(st, "moda_test_exp2_fma")
    return y


def moda_status_string(status):
    return lib.moda_status_string(status).decode()


def moda_last_error_message():
    """The message the calling thread's last failed call left (empty after a success)."""
    return lib.moda_last_error_message().decode()


# ---------------------------------------------------------------- torch conveniences
def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ndim(name, t, n):
    if t is None or t.dim() != n:
        raise ValueError(f"{name} must be a {n}-D tensor")


def _dims(q, k, kd):
    _ndim("q", q, 4)
    _ndim("k", k, 4)
    if kd is not None:
        _ndim("kd", kd, 5)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    L = 0 if kd is None else kd.shape[3]
    return B, Hq, Hkv, T, L, d


def _validate(device, specs, workspace=None):
    """Check each tensor's shape, dtype, contiguity and device before its pointer goes to
    the library, which sees only pointers and sizes: a tensor smaller than the sizes say,
    a strided view or another dtype would make a kernel read or write outside it.
    ``specs`` maps a name to (tensor, expected shape, expected dtype)."""
    for name, (t, shape, dtype) in specs.items():
        if t is None:
            raise ValueError(f"{name} is required")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {tuple(shape)}")
        if t.dtype != dtype:
            raise TypeError(f"{name} has dtype {t.dtype}; expected {dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}; expected {device}")
    if workspace is not None and (not workspace.is_contiguous() or workspace.device != device):
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    if device.type != "cuda":
        raise ValueError(f"the library runs on CUDA tensors, not on {device}")


def _nbytes(t):
    return t.numel() * t.element_size()


def forward(q, k, v, kd=None, vd=None, scale=None, causal=True, out=None, lse=None,
            depth_path=0):
    """MoDA forward on the current CUDA stream.  Returns (out bf16, lse fp32).

    q [B,Hq,T,d], k/v [B,Hkv,T,d], kd/vd [B,Hkv,T,L,d] (or None for L = 0): contiguous
    bf16 CUDA tensors.  scale defaults to 1/sqrt(d).  ``depth_path`` 0 lets the library
    choose; 1 forces the CUDA-core depth fold, 2 dense depth blocks on the tensor cores
    (moda_forward_depth_path).
    """
    import torch
    B, Hq, Hkv, T, L, d = _dims(q, k, kd)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    bf, kv = torch.bfloat16, (B, Hkv, T, d)
    spec = dict(q=(q, (B, Hq, T, d), bf), k=(k, kv, bf), v=(v, kv, bf),
                out=(out, (B, Hq, T, d), bf), lse=(lse, (B, Hq, T), torch.float32))
    if L:
        spec.update(kd=(kd, (B, Hkv, T, L, d), bf), vd=(vd, (B, Hkv, T, L, d), bf))
    _validate(q.device, spec)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(kd) if L else None, _ptr(vd) if L else None,
            _ptr(out), _ptr(lse), B, Hq, Hkv, T, L, d, float(scale), int(bool(causal)))
    if depth_path == 0:
        st = lib.moda_forward(*args, _stream_handle(q.device))
        _check(st, "moda_forward")
    else:
        st = lib.moda_forward_depth_path(*args, int(depth_path), _stream_handle(q.device))
        _check(st, "moda_forward_depth_path")
    return out, lse


def backward(q, k, v, kd, vd, out, lse, dout, scale=None, causal=True, workspace=None,
             grads=None, stages=7):
    """MoDA backward on the current CUDA stream.  Returns dict(dq, dk, dv, dkd, dvd).

    ``out``/``lse`` are the forward's results for the same inputs.  ``workspace`` (uint8
    CUDA tensor of at least moda_backward_workspace_size bytes) and ``grads`` (a dict of
    preallocated gradient tensors) are optional; missing ones are allocated with torch.
    ``stages`` (bit mask 1 | 2 | 4, see moda_backward_stages) runs part of the backward;
    the default runs all of it (moda_backward).
    """
    import torch
    B, Hq, Hkv, T, L, d = _dims(q, k, kd)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws = moda_backward_workspace_size(B, Hq, Hkv, T, L, d)
    if workspace is None:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    g = dict(grads or {})
    if g.get("dq") is None:
        g["dq"] = torch.empty_like(q)
    if g.get("dk") is None:
        g["dk"] = torch.empty_like(k)
    if g.get("dv") is None:
        g["dv"] = torch.empty_like(v)
    if L and g.get("dkd") is None:
        g["dkd"] = torch.empty_like(kd)
    if L and g.get("dvd") is None:
        g["dvd"] = torch.empty_like(vd)
    if not L:
        g["dkd"] = g["dvd"] = None
    bf, qs, kv, ds = torch.bfloat16, (B, Hq, T, d), (B, Hkv, T, d), (B, Hkv, T, L, d)
    spec = dict(q=(q, qs, bf), k=(k, kv, bf), v=(v, kv, bf), out=(out, qs, bf),
                lse=(lse, (B, Hq, T), torch.float32), dout=(dout, qs, bf),
                dq=(g["dq"], qs, bf), dk=(g["dk"], kv, bf), dv=(g["dv"], kv, bf))
    if L:
        spec.update(kd=(kd, ds, bf), vd=(vd, ds, bf), dkd=(g["dkd"], ds, bf),
                    dvd=(g["dvd"], ds, bf))
    _validate(q.device, spec, workspace)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(kd) if L else None, _ptr(vd) if L else None,
            _ptr(out), _ptr(lse), _ptr(dout), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
            _ptr(g["dkd"]), _ptr(g["dvd"]), _ptr(workspace), _nbytes(workspace),
            B, Hq, Hkv, T, L, d, float(scale), int(bool(causal)))
    if stages == 7:
        st = lib.moda_backward(*args, _stream_handle(q.device))
        _check(st, "moda_backward")
    else:
        st = lib.moda_backward_stages(*args, int(stages), _stream_handle(q.device))
        _check(st, "moda_backward_stages")
    return g


def check_device_errors(device=None):
    """Raise ModaError if a kernel on the current stream recorded a failure."""
    import torch
    st, flags = moda_check_device_errors(_stream_handle(device or torch.cuda.current_device()))
    _check(st, f"device error word 0x{flags:x}")


def depth_attention_forward(q, kd, vd, scale=None, out=None, lse=None):
    """Depth-only attention (Flash Depth Attention) forward on the current CUDA stream:
    each row attends to its own token's L >= 1 depth keys.  Returns (out bf16, lse fp32).

    q [B,Hq,T,d], kd/vd [B,Hkv,T,L,d]: contiguous bf16 CUDA tensors.
    """
    import torch
    _ndim("q", q, 4)
    _ndim("kd", kd, 5)
    B, Hq, T, d = q.shape
    Hkv, L = kd.shape[1], kd.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, T), device=q.device, dtype=torch.float32)
    bf, ds = torch.bfloat16, (B, Hkv, T, L, d)
    _validate(q.device, dict(q=(q, (B, Hq, T, d), bf), kd=(kd, ds, bf), vd=(vd, ds, bf),
                             out=(out, (B, Hq, T, d), bf),
                             lse=(lse, (B, Hq, T), torch.float32)))
    st = lib.moda_depth_attention_forward(_ptr(q), _ptr(kd), _ptr(vd), _ptr(out), _ptr(lse),
                                          B, Hq, Hkv, T, L, d, float(scale),
                                          _stream_handle(q.device))
    _check(st, "moda_depth_attention_forward")
    return out, lse


def depth_attention_backward(q, kd, vd, out, lse, dout, scale=None, workspace=None,
                             grads=None):
    """Depth-only attention backward on the current CUDA stream.  Returns dict(dq, dkd,
    dvd); ``workspace``/``grads`` as for backward()."""
    import torch
    _ndim("q", q, 4)
    _ndim("kd", kd, 5)
    B, Hq, T, d = q.shape
    Hkv, L = kd.shape[1], kd.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws = moda_backward_workspace_size(B, Hq, Hkv, T, L, d)
    if workspace is None:
        workspace = torch.empty(ws, device=q.device, dtype=torch.uint8)
    g = dict(grads or {})
    if g.get("dq") is None:
        g["dq"] = torch.empty_like(q)
    if g.get("dkd") is None:
        g["dkd"] = torch.empty_like(kd)
    if g.get("dvd") is None:
        g["dvd"] = torch.empty_like(vd)
    bf, qs, ds = torch.bfloat16, (B, Hq, T, d), (B, Hkv, T, L, d)
    _validate(q.device, dict(q=(q, qs, bf), kd=(kd, ds, bf), vd=(vd, ds, bf),
                             out=(out, qs, bf), lse=(lse, (B, Hq, T), torch.float32),
                             dout=(dout, qs, bf), dq=(g["dq"], qs, bf),
                             dkd=(g["dkd"], ds, bf), dvd=(g["dvd"], ds, bf)), workspace)
    st = lib.moda_depth_attention_backward(
        _ptr(q), _ptr(kd), _ptr(vd), _ptr(out), _ptr(lse), _ptr(dout), _ptr(g["dq"]),
        _ptr(g["dkd"]), _ptr(g["dvd"]), _ptr(workspace), _nbytes(workspace), B, Hq, Hkv, T,
        L, d, float(scale), _stream_handle(q.device))
    _check(st, "moda_depth_attention_backward")
    return g


def decode(q, k, v, kd=None, vd=None, scale=None, out=None, lse=None, workspace=None):
    """Single-token decode on the current CUDA stream: the newest token of each sequence
    (query q [B,Hq,d]) against its K/V cache k/v [B,Hkv,S,d] (the last entry its own) and
    its own depth entries kd/vd [B,Hkv,L,d] (or None for L = 0).  Returns (out [B,Hq,d]
    bf16, lse [B,Hq] fp32)."""
    import torch
    _ndim("q", q, 3)
    _ndim("k", k, 4)
    if kd is not None:
        _ndim("kd", kd, 4)
    B, Hq, d = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    L = 0 if kd is None else kd.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    ws = lib.moda_decode_workspace_size(B, Hq, Hkv, S, L, d)
    if workspace is None:
        workspace = torch.empty(max(ws, 256), device=q.device, dtype=torch.uint8)
    bf, kv = torch.bfloat16, (B, Hkv, S, d)
    spec = dict(q=(q, (B, Hq, d), bf), k=(k, kv, bf), v=(v, kv, bf), out=(out, (B, Hq, d), bf),
                lse=(lse, (B, Hq), torch.float32))
    if L:
        spec.update(kd=(kd, (B, Hkv, L, d), bf), vd=(vd, (B, Hkv, L, d), bf))
    _validate(q.device, spec, workspace)
    st = lib.moda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(kd) if L else None,
                         _ptr(vd) if L else None, _ptr(out), _ptr(lse), _ptr(workspace),
                         _nbytes(workspace), B, Hq, Hkv, S, L, d, float(scale),
                         _stream_handle(q.device))
    _check(st, "moda_decode")
    return out, lse


def depth_kv_write(x, w, kd, vd, slot):
    """Fused depth-stream write on the current CUDA stream: slot ``slot`` of kd / vd
    [B,Hkv,T,L,d] receives K|V = x w^T for x [B,T,hidden] and w [2*Hkv*d, hidden] (rows
    0..Hkv*d-1 project K, the rest V).  Other slots are untouched."""
    import torch
    _ndim("x", x, 3)
    _ndim("kd", kd, 5)
    B, T, hidden = x.shape
    _, Hkv, _, L, d = kd.shape
    bf, ds = torch.bfloat16, (B, Hkv, T, L, d)
    _validate(x.device, dict(x=(x, (B, T, hidden), bf), w=(w, (2 * Hkv * d, hidden), bf),
                             kd=(kd, ds, bf), vd=(vd, ds, bf)))
    st = lib.moda_depth_kv_write(_ptr(x), _ptr(w), _ptr(kd), _ptr(vd), B, T, hidden, Hkv, d,
                                 L, int(slot), _stream_handle(x.device))
    _check(st, "moda_depth_kv_write")
