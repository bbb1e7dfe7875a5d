"""fp64 CPU oracle for mixture-of-depths attention (MoDA) -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (``depth_aware_attention_b200``) never does:
it shares no code with it, and the oracle shares none with the CUDA library.

The arithmetic lives in ``moda_oracle.c`` (plain C, fp64, POSIX threads).  This module
only compiles it with gcc, loads it with ctypes and marshals numpy arrays.  Each entry
point follows the definition of the operator on the hyper.ai summary of arXiv
2603.15619, section "Mixture-of-Depths Attention (MoDA)": one softmax, jointly
normalised, over the query's causal sequence keys and its own token's depth keys.

``depth_forward`` / ``depth_backward`` run the pages' depth-only operator (Flash Depth
Attention: hyper.ai summary, section "Depth-stream mechanisms"): the same definition with
no sequence keys, each row attending to its own token's depth keys only.

Parity status: forward, backward, the backward with a given output, the row-weight view
and the depth-only forward/backward are pinned by the
``-m "not gpu"`` tests in ``tests/test_oracle_pins.py`` (library special cases, closed
forms, invariants, finite differences and hand-derived golden cases).
``tests/test_oracle_mutants.py`` plants single mistakes in copies of this package and
checks that those pins catch every one.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moda_oracle.c")
_LIB = os.path.join(_HERE, "libmoda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree with gcc; returns its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _configure(lib):
    """Declare the argument and return types of the oracle's entry points on ``lib``."""
    P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
    lib.moda_oracle_forward.argtypes = [P] * 7 + [I] * 8 + [D, I, I]
    lib.moda_oracle_backward.argtypes = [P] * 13 + [I] * 8 + [D, I, I]
    lib.moda_oracle_row_weights.argtypes = [P] * 3 + [I] * 9 + [D, I, P, P]
    lib.moda_oracle_backward_given_out.argtypes = [P] * 12 + [I] * 8 + [D, I, I]
    lib.moda_oracle_backward_given_out.restype = I
    lib.moda_oracle_depth_forward.argtypes = [P] * 5 + [I] * 8 + [D, I]
    lib.moda_oracle_depth_forward.restype = I
    lib.moda_oracle_depth_backward.argtypes = [P] * 10 + [I] * 8 + [D, I]
    lib.moda_oracle_depth_backward.restype = I
    for f in (lib.moda_oracle_forward, lib.moda_oracle_backward,
              lib.moda_oracle_row_weights):
        f.restype = I
    return lib


def _f64(x):
    """Contiguous float64 numpy copy of a numpy array or torch tensor (bf16 widens exactly)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return os.cpu_count() or 1


def forward(q, k, v, kd, vd, scale, causal=True, t0=0, nthreads=None):
    """Oracle forward over the query tokens [t0, t0+nt).

    Shapes: q [B,Hq,nt,d]; k,v [B,Hkv,T,d]; kd,vd [B,Hkv,nt,L,d] (L may be 0).
    Returns (out [B,Hq,nt,d], lse [B,Hq,nt]) as float64 numpy arrays.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, nt, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    if kd is None or kd.shape[3] == 0:
        L = 0
        kd = vd = np.zeros((1,), np.float64)
    else:
        kd, vd = _f64(kd), _f64(vd)
        L = kd.shape[3]
    out = np.empty((B, Hq, nt, d), np.float64)
    lse = np.empty((B, Hq, nt), np.float64)
    rc = _load().moda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd),
                                     _ptr(out), _ptr(lse), B, Hq, Hkv, T, L, d, t0, nt,
                                     float(scale), int(bool(causal)),
                                     nthreads or default_threads())
    if rc != 0:
        raise ValueError("moda_oracle_forward rejected the sizes")
    return out, lse


def backward(q, k, v, kd, vd, dout, scale, causal=True, t0=0, nthreads=None):
    """Oracle backward over the rows of the query tokens [t0, t0+nt).

    Returns dict(dq, dk, dv, dkd, dvd, out, lse) as float64 numpy arrays.  dq, dkd, dvd
    are exact for the window; dk, dv hold the window rows' contributions (exact for keys
    s >= t0 when causal and the window ends at T; exact everywhere for the full window).
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, nt, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    if kd is None or kd.shape[3] == 0:
        L = 0
        kd = vd = np.zeros((1,), np.float64)
    else:
        kd, vd = _f64(kd), _f64(vd)
        L = kd.shape[3]
    dq = np.empty((B, Hq, nt, d), np.float64)
    dk = np.empty((B, Hkv, T, d), np.float64)
    dv = np.empty((B, Hkv, T, d), np.float64)
    dkd = np.empty((B, Hkv, nt, L, d), np.float64)
    dvd = np.empty((B, Hkv, nt, L, d), np.float64)
    out = np.empty((B, Hq, nt, d), np.float64)
    lse = np.empty((B, Hq, nt), np.float64)
    rc = _load().moda_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd),
                                      _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dkd),
                                      _ptr(dvd), _ptr(out), _ptr(lse), B, Hq, Hkv, T, L, d,
                                      t0, nt, float(scale), int(bool(causal)),
                                      nthreads or default_threads())
    if rc != 0:
        raise ValueError("moda_oracle_backward rejected the sizes")
    return dict(dq=dq, dk=dk, dv=dv, dkd=dkd, dvd=dvd, out=out, lse=lse)


def backward_given_out(q, k, v, kd, vd, dout, out, scale, causal=True, t0=0, nthreads=None):
    """Oracle backward whose row terms D = <dO, out> use the given ``out`` (window-sized,
    e.g. the forward's bf16 output widened) instead of the oracle's exact output.

    Everything else is exactly moda's gradient: P comes from the exact logits and
    log-sum-exp.  This is the exact result a backward can reach when it is handed only
    the forward's rounded output.  Returns dict(dq, dk, dv, dkd, dvd), same windows as
    ``backward``.
    """
    q, k, v, dout, out = _f64(q), _f64(k), _f64(v), _f64(dout), _f64(out)
    B, Hq, nt, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    if kd is None or kd.shape[3] == 0:
        L = 0
        kd = vd = np.zeros((1,), np.float64)
    else:
        kd, vd = _f64(kd), _f64(vd)
        L = kd.shape[3]
    dq = np.empty((B, Hq, nt, d), np.float64)
    dk = np.empty((B, Hkv, T, d), np.float64)
    dv = np.empty((B, Hkv, T, d), np.float64)
    dkd = np.empty((B, Hkv, nt, L, d), np.float64)
    dvd = np.empty((B, Hkv, nt, L, d), np.float64)
    rc = _load().moda_oracle_backward_given_out(
        _ptr(q), _ptr(k), _ptr(v), _ptr(kd), _ptr(vd), _ptr(dout), _ptr(out), _ptr(dq),
        _ptr(dk), _ptr(dv), _ptr(dkd), _ptr(dvd), B, Hq, Hkv, T, L, d, t0, nt, float(scale),
        int(bool(causal)), nthreads or default_threads())
    if rc != 0:
        raise ValueError("moda_oracle_backward_given_out rejected the arguments")
    return dict(dq=dq, dk=dk, dv=dv, dkd=dkd, dvd=dvd)


def row_weights(q, k, kd, b, h, t, scale, causal=True):
    """Normalised joint-softmax weights of row (b,h,t): (w_seq [n_visible], w_depth [L])."""
    q, k = _f64(q), _f64(k)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if kd is None or kd.shape[3] == 0:
        L, kd = 0, np.zeros((1,), np.float64)
    else:
        kd = _f64(kd)
        L = kd.shape[3]
    n = t + 1 if causal else T
    ws = np.empty((n,), np.float64)
    wd = np.empty((max(L, 1),), np.float64)
    rc = _load().moda_oracle_row_weights(_ptr(q), _ptr(k), _ptr(kd), b, h, t, B, Hq, Hkv,
                                         T, L, d, float(scale), int(bool(causal)),
                                         _ptr(ws), _ptr(wd))
    if rc != 0:
        raise ValueError("moda_oracle_row_weights rejected the arguments")
    return ws, wd[:L]


def depth_forward(q, kd, vd, scale, t0=0, nthreads=None):
    """Depth-only attention forward over the query tokens [t0, t0+nt).

    q [B,Hq,nt,d]; kd,vd [B,Hkv,nt,L,d] with L >= 1.  Returns (out [B,Hq,nt,d],
    lse [B,Hq,nt]) as float64 numpy arrays.  T is taken as t0 + nt (no sequence keys).
    """
    q, kd, vd = _f64(q), _f64(kd), _f64(vd)
    B, Hq, nt, d = q.shape
    Hkv, L = kd.shape[1], kd.shape[3]
    out = np.empty((B, Hq, nt, d), np.float64)
    lse = np.empty((B, Hq, nt), np.float64)
    rc = _load().moda_oracle_depth_forward(_ptr(q), _ptr(kd), _ptr(vd), _ptr(out), _ptr(lse),
                                           B, Hq, Hkv, t0 + nt, L, d, t0, nt, float(scale),
                                           nthreads or default_threads())
    if rc != 0:
        raise ValueError("moda_oracle_depth_forward rejected the sizes")
    return out, lse


def depth_backward(q, kd, vd, dout, scale, out=None, t0=0, nthreads=None):
    """Depth-only attention backward over the query tokens [t0, t0+nt).

    Returns dict(dq, dkd, dvd, out, lse) as float64 numpy arrays.  With ``out`` given
    (window-sized, e.g. a forward's bf16 output widened), the row terms D = <dO, out> use
    it, as backward_given_out does; otherwise they use the oracle's exact output.
    """
    q, kd, vd, dout = _f64(q), _f64(kd), _f64(vd), _f64(dout)
    given = _f64(out)
    B, Hq, nt, d = q.shape
    Hkv, L = kd.shape[1], kd.shape[3]
    dq = np.empty((B, Hq, nt, d), np.float64)
    dkd = np.empty((B, Hkv, nt, L, d), np.float64)
    dvd = np.empty((B, Hkv, nt, L, d), np.float64)
    o = np.empty((B, Hq, nt, d), np.float64)
    lse = np.empty((B, Hq, nt), np.float64)
    rc = _load().moda_oracle_depth_backward(
        _ptr(q), _ptr(kd), _ptr(vd), _ptr(dout), _ptr(given), _ptr(dq), _ptr(dkd), _ptr(dvd),
        _ptr(o), _ptr(lse), B, Hq, Hkv, t0 + nt, L, d, t0, nt, float(scale),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("moda_oracle_depth_backward rejected the sizes")
    return dict(dq=dq, dkd=dkd, dvd=dvd, out=o, lse=lse)


def depth_kv_projection(x, w, Hkv, d):
    """The layer's depth-stream key/value pair that the fused write stores into slot l:
    K = x W_k^T and V = x W_v^T for every token, per KV head (hyper.ai summary,
    section "Hardware-efficient implementation": each layer appends its K/V to the depth
    stream that later layers read; the depth cache layout is [B, Hkv, T, L, d]).

    x [B,T,hidden]; w [2*Hkv*d, hidden] (rows 0..Hkv*d-1 project K, the rest V, the
    nn.Linear weight convention).  Returns (k_slot, v_slot), each [B,Hkv,T,d] float64: the
    values slot l of kd / vd must hold.  One fp64 matrix product, then a reshape.
    """
    x, w = _f64(x), _f64(w)
    B, T, _ = x.shape
    y = x.reshape(B * T, -1) @ w.T                       # [B*T, 2*Hkv*d]
    y = y.reshape(B, T, 2, Hkv, d).transpose(2, 0, 3, 1, 4)  # [2, B, Hkv, T, d]
    return np.ascontiguousarray(y[0]), np.ascontiguousarray(y[1])
