"""GPU depth-only attention (Flash Depth Attention: moda_depth_attention_forward/backward
through the C ABI) vs the fp64 oracle's depth-only mode, element by element.

Small problems are compared in full over group sizes that do and do not divide 128 (the
dense tensor-core depth path and the CUDA-core fold path), both head sizes, ragged token
counts, L = 1 and long depth caches.  The deep-stack head layout at 4K tokens is compared
on token windows (depth-only rows are independent per token, so a window is exact).  The
gradients are compared with the oracle's exact gradient of the definition.  The mean-abs
bound is applied beyond each element's bf16 rounding (the outputs average only L values,
so they are O(1)); the plain mean-abs of every case is logged beside it.
"""
import math

import pytest
import torch

import depth_aware_attention_b200 as moda
import workloads
import oracle
from parity_util import compare_forward, compare_grad, gpu_inputs, window_starts

pytestmark = pytest.mark.gpu

CASES = [
    ("g4-d128", dict(B=2, T=300, Hq=8, Hkv=2, d=128, L=5)),
    ("g1-d64", dict(B=1, T=200, Hq=2, Hkv=2, d=64, L=3)),
    ("g3-d128-fold", dict(B=1, T=130, Hq=6, Hkv=2, d=128, L=7)),
    ("g8-d128", dict(B=1, T=257, Hq=16, Hkv=2, d=128, L=9)),
    ("g16-d64", dict(B=1, T=100, Hq=16, Hkv=1, d=64, L=2)),
    ("L1", dict(B=1, T=77, Hq=4, Hkv=2, d=128, L=1)),
    ("g32-d128", dict(B=1, T=90, Hq=64, Hkv=2, d=128, L=6)),
    ("g64-d64", dict(B=1, T=70, Hq=64, Hkv=1, d=64, L=4)),
    ("longL", dict(B=1, T=64, Hq=4, Hkv=1, d=128, L=130)),
    # the gradient pass over staged (P, <dO, vd>) pairs at its shared-memory limit (tokens
    # per CTA x L x 4 heads x 8 bytes = 32 KB) and just past it (the recomputing pass)
    ("stage-limit-d128", dict(B=1, T=40, Hq=8, Hkv=2, d=128, L=128)),
    ("stage-limit-d64", dict(B=1, T=50, Hq=4, Hkv=1, d=64, L=64)),
    ("stage-over-d64", dict(B=1, T=50, Hq=4, Hkv=1, d=64, L=65)),
]


def _sel(x, t0, nt):
    sl = slice(t0, t0 + nt)
    return {n: x[n][:, :, sl].cpu() for n in ("q", "kd", "vd", "dout") if x.get(n) is not None}


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_depth_attention_small_full(name, cfg):
    x = gpu_inputs(cfg, seed_base=300 + [c[0] for c in CASES].index(name), with_dout=True)
    scale = 1.0 / math.sqrt(cfg["d"])
    out, lse = moda.depth_attention_forward(x["q"], x["kd"], x["vd"], scale)
    g = moda.depth_attention_backward(x["q"], x["kd"], x["vd"], out, lse, x["dout"], scale)
    moda.check_device_errors()
    w = _sel(x, 0, cfg["T"])
    ref_out, ref_lse = oracle.depth_forward(w["q"], w["kd"], w["vd"], scale)
    compare_forward(out, lse, ref_out, ref_lse, f"fda {name}", mean_beyond_rounding=True)
    # the exact gradient of the definition (the oracle's own out and row terms)
    ref = oracle.depth_backward(w["q"], w["kd"], w["vd"], w["dout"], scale)
    for n in ("dq", "dkd", "dvd"):
        compare_grad(g[n], ref[n], f"fda {name}:{n}", mean_beyond_rounding=True)


def test_depth_attention_is_deterministic():
    cfg = dict(B=1, T=515, Hq=8, Hkv=2, d=128, L=6)
    x = gpu_inputs(cfg, seed_base=320, with_dout=True)
    a, la = moda.depth_attention_forward(x["q"], x["kd"], x["vd"])
    b, lb = moda.depth_attention_forward(x["q"], x["kd"], x["vd"])
    ga = moda.depth_attention_backward(x["q"], x["kd"], x["vd"], a, la, x["dout"])
    gb = moda.depth_attention_backward(x["q"], x["kd"], x["vd"], a, la, x["dout"])
    moda.check_device_errors()
    assert torch.equal(a, b) and torch.equal(la, lb)
    for n in ("dq", "dkd", "dvd"):
        assert torch.equal(ga[n], gb[n]), n


def test_depth_attention_deep_windows():
    cfg = workloads.CONFIGS["deep-4k"]
    x = gpu_inputs(cfg, workloads.SEED_BASE["deep-4k"], with_dout=True)
    scale = workloads.default_scale(cfg["d"])
    out, lse = moda.depth_attention_forward(x["q"], x["kd"], x["vd"], scale)
    g = moda.depth_attention_backward(x["q"], x["kd"], x["vd"], out, lse, x["dout"], scale)
    moda.check_device_errors()
    T, nt = cfg["T"], 16
    for t0 in window_starts(T, nt, 6, seed=workloads.SEED_BASE["deep-4k"]):
        w = _sel(x, t0, nt)
        sl = slice(t0, t0 + nt)
        ref_out, ref_lse = oracle.depth_forward(w["q"], w["kd"], w["vd"], scale, t0=t0)
        compare_forward(out[:, :, sl], lse[:, :, sl], ref_out, ref_lse, f"deep-4k fda @{t0}",
                        mean_beyond_rounding=True)
        ref = oracle.depth_backward(w["q"], w["kd"], w["vd"], w["dout"], scale, t0=t0)
        compare_grad(g["dq"][:, :, sl], ref["dq"], f"deep-4k fda dq @{t0}",
                     mean_beyond_rounding=True)
        compare_grad(g["dkd"][:, :, sl], ref["dkd"], f"deep-4k fda dkd @{t0}",
                     mean_beyond_rounding=True)
        compare_grad(g["dvd"][:, :, sl], ref["dvd"], f"deep-4k fda dvd @{t0}",
                     mean_beyond_rounding=True)
    del x, out, lse, g
    torch.cuda.empty_cache()
