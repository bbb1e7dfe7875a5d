"""GPU backward (moda_backward through the C ABI) vs the fp64 CPU oracle, element by element.

The GPU backward takes the GPU forward's out (bf16) and lse (fp32); the oracle differentiates
its own fp64 forward.  Tolerances are those of parity_util: max-abs 1e-2 beyond the bf16 output's own rounding,
mean-abs 1e-3, relative RMS 1e-2.

Small problems are compared in full (all of dq, dk, dv, dkd, dvd) against the oracle's
exact gradient.  The 16K-token forward+backward workload, in the launch configuration the
benchmark times, is compared with the exact gradient on token windows: for a window
[t0, t0+nt) the oracle's dq, dkd and dvd are exact, and for the window that ends at T its
dk and dv are exact for every key s >= t0 (only tokens t >= s see key s under the causal
mask).
"""
import math

import numpy as np
import pytest
import torch

import depth_aware_attention_b200 as moda
import oracle
import workloads
from parity_util import (bf16_half_ulp, compare_grad, error_stats, gpu_inputs, log_stats,
                         window, window_starts)

pytestmark = pytest.mark.gpu

SMALL = [
    ("tiny", workloads.CONFIGS["tiny"], True),
    ("ragged-g4-d128", dict(B=2, T=300, Hq=8, Hkv=2, d=128, L=5), True),
    ("g1-d64", dict(B=1, T=200, Hq=2, Hkv=2, d=64, L=3), True),
    ("g3-d128", dict(B=1, T=130, Hq=6, Hkv=2, d=128, L=7), True),
    ("g8-d128", dict(B=1, T=257, Hq=16, Hkv=2, d=128, L=9), True),
    # (with L = 2 the first rows see three keys, and the bf16 rounding of out alone moves
    # dk by up to 6e-3 through D = <dO, out>: at T = 100 the GPU met the exact gradient
    # only to 1.01e-2 beyond the rounding, at T = 64 to a mean-abs of 1.12e-3; with L = 8
    # that shift stays under 2e-3)
    ("g16-d64", dict(B=1, T=200, Hq=16, Hkv=1, d=64, L=8), True),
    ("L0-d128", dict(B=1, T=333, Hq=8, Hkv=2, d=128, L=0), True),
    # groups above 16: the depth part runs per 16-head chunk with fp32 dkd/dvd sums.  The
    # shapes keep the outputs' own bf16 rounding well inside the mean-abs bound: entries of
    # dk and dv grow with the G*T rows a key collects (rounding alone: mean 6-8e-4 here)
    ("g32-d128", dict(B=1, T=384, Hq=32, Hkv=1, d=128, L=16), True),
    ("g64-d64", dict(B=1, T=512, Hq=64, Hkv=1, d=64, L=16), True),
    # four 16-head chunks writing the d = 128 sequence kernel's row-term records.  Shorter
    # sequences give larger weights and gradient entries: the bf16 rounding of the exact
    # dk alone averages 1.25e-3 at T = 130, 1.02e-3 at T = 260 and 7.5e-4 at T = 512 (L = 16)
    ("g64-d128", dict(B=1, T=512, Hq=64, Hkv=1, d=128, L=16), True),
    ("T1", dict(B=2, T=1, Hq=4, Hkv=2, d=128, L=6), True),
    ("longL-d128", dict(B=1, T=64, Hq=4, Hkv=1, d=128, L=130), True),
    ("noncausal-g4", dict(B=1, T=190, Hq=4, Hkv=1, d=128, L=4), False),
    ("multi-block-d64", dict(B=1, T=700, Hq=4, Hkv=2, d=64, L=11), True),
]

NAMES = ("dq", "dk", "dv", "dkd", "dvd")


def run_gpu(x, scale, causal, keep_out=False):
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal)
    g = moda.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"], scale,
                      causal)
    moda.check_device_errors()
    if keep_out:
        g["out"] = out
    return g


@pytest.mark.parametrize("name,cfg,causal", SMALL, ids=[s[0] for s in SMALL])
def test_backward_small_full(name, cfg, causal):
    """All five gradients in full against the oracle's exact gradient of the definition
    (its own fp64 forward, its own row terms D = <dO, out>).  The oracle's backward given
    the GPU forward's bf16 out, the most a backward handed only that out can reach, is
    logged beside it as a diagnostic of how much of the error the rounded out explains."""
    x = gpu_inputs(cfg, seed_base=200 + SMALL.index((name, cfg, causal)), with_dout=True)
    scale = 1.0 / math.sqrt(cfg["d"])
    g = run_gpu(x, scale, causal, keep_out=True)
    w = window(x, 0, cfg["T"])
    ref = oracle.backward(w["q"], w["k"], w["v"], w["kd"], w["vd"], w["dout"], scale, causal)
    given = oracle.backward_given_out(w["q"], w["k"], w["v"], w["kd"], w["vd"], w["dout"],
                                      g["out"].cpu(), scale, causal)
    for n in NAMES:
        if cfg["L"] == 0 and n in ("dkd", "dvd"):
            assert g[n] is None
            continue
        a = g[n].double().cpu().numpy()
        log_stats(f"{name}:{n} vs backward given the bf16 out", kind="diagnostic",
                  **error_stats(np.abs(a - given[n]), given[n]))
        compare_grad(g[n], ref[n], f"{name}:{n}")


def test_backward_is_deterministic_in_dkd_dvd_and_leaves_inputs_intact():
    cfg = dict(B=1, T=515, Hq=8, Hkv=2, d=128, L=6)
    x = gpu_inputs(cfg, seed_base=250, with_dout=True)
    before = {k: v.clone() for k, v in x.items() if v is not None}
    a = run_gpu(x, 1 / math.sqrt(128), True)
    b = run_gpu(x, 1 / math.sqrt(128), True)
    # dkd and dvd have one writer per element.  dq sums fp32 atomics, and dk, dv sum the
    # two half tiles' products in whichever order their issuers reach the tensor pipe:
    # those may differ between runs by the fp32 summation order, at most one bf16 step
    # after rounding.
    for n in ("dkd", "dvd"):
        assert torch.equal(a[n], b[n]), n
    for n in ("dk", "dv"):
        d = (a[n].float() - b[n].float()).abs()
        assert (d <= a[n].float().abs() * 2.0 ** -7 + 1e-6).all().item(), n
    assert (a["dq"].float() - b["dq"].float()).abs().max().item() < 1e-3
    for k, v in before.items():
        assert torch.equal(v, x[k]), k


def test_backward_stages_in_order_equal_one_backward_call():
    """moda_backward_stages 1, 2, 4 on one stream give moda_backward's results."""
    cfg = dict(B=1, T=400, Hq=8, Hkv=2, d=128, L=5)
    x = gpu_inputs(cfg, seed_base=252, with_dout=True)
    scale = 1 / math.sqrt(128)
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True)
    ref = moda.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"], scale)
    ws = torch.empty(moda.moda_backward_workspace_size(1, 8, 2, 400, 5, 128), device="cuda",
                     dtype=torch.uint8)
    g = {n: torch.empty_like(ref[n]) for n in NAMES}
    for st in (1, 2, 4):
        moda.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"], scale,
                      workspace=ws, grads=g, stages=st)
    moda.check_device_errors()
    for n in ("dk", "dv", "dkd", "dvd"):
        assert torch.equal(g[n], ref[n]), n
    assert (g["dq"].float() - ref["dq"].float()).abs().max().item() < 1e-3


def test_L0_backward_matches_torch_autograd():
    """Special case: with no depth entries the gradients are those of causal attention."""
    cfg = dict(B=1, T=600, Hq=8, Hkv=2, d=128, L=0)
    x = gpu_inputs(cfg, seed_base=251, with_dout=True)
    g = run_gpu(x, 1 / math.sqrt(128), True)
    G = cfg["Hq"] // cfg["Hkv"]
    q = x["q"].float().requires_grad_()
    k = x["k"].float().requires_grad_()
    v = x["v"].float().requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1), is_causal=True)
    o.backward(x["dout"].float())
    for n, ref in (("dq", q.grad), ("dk", k.grad), ("dv", v.grad)):
        r = ref.double().cpu().numpy()
        err = np.abs(g[n].double().cpu().numpy() - r)
        assert (err - bf16_half_ulp(r)).max() < 1e-2 and err.mean() < 1e-3, n


def test_backward_fwd_bwd_16k_windows():
    """The 16K-token forward+backward workload, in the launch configuration the benchmark
    times, against the oracle's exact gradient.  For a window [t0, t0+nt) the oracle's dq,
    dkd and dvd are exact; for the window that ends at T its dk and dv are exact for every
    key s >= t0 (only tokens t >= s see key s under the causal mask).  Sampled: dk and dv
    of the last 1024 keys; dq, dkd and dvd of those 1024 tokens and of 16-token windows at
    t = 0 and at seeded random positions (every head: over 20000 rows)."""
    name = "fwd-bwd-16k"
    cfg = workloads.CONFIGS[name]
    x = gpu_inputs(cfg, workloads.SEED_BASE[name], with_dout=True)
    scale = workloads.default_scale(cfg["d"])
    g = run_gpu(x, scale, True)
    T, late = cfg["T"], 1024
    k = x["k"].cpu().to(torch.float64).numpy()
    v = x["v"].cpu().to(torch.float64).numpy()
    windows = [(T - late, late)] + [(t0, 16) for t0 in
                                    window_starts(T - late, 16, 14, seed=41)]
    rows = 0
    for t0, nt in windows:
        w = window(x, t0, nt)
        ref = oracle.backward(w["q"], k, v, w["kd"], w["vd"], w["dout"], scale, True, t0=t0)
        sl = slice(t0, t0 + nt)
        compare_grad(g["dq"][:, :, sl], ref["dq"], f"{name}@{t0}+{nt}:dq")
        compare_grad(g["dkd"][:, :, sl], ref["dkd"], f"{name}@{t0}+{nt}:dkd")
        compare_grad(g["dvd"][:, :, sl], ref["dvd"], f"{name}@{t0}+{nt}:dvd")
        if t0 + nt == T:
            compare_grad(g["dk"][:, :, sl], ref["dk"][:, :, sl], f"{name}@{t0}+{nt}:dk")
            compare_grad(g["dv"][:, :, sl], ref["dv"][:, :, sl], f"{name}@{t0}+{nt}:dv")
        rows += cfg["B"] * cfg["Hq"] * nt
    assert rows >= 4096 + cfg["Hq"] * late
    del x, g
    torch.cuda.empty_cache()


def test_backward_dk_dv_sum_identities_at_16k():
    """Properties that hold at any size, checked on every key of the 16K workload:
    sum over keys of dv (sequence + depth) equals sum over rows of dout (the weights of a
    row sum to one), and sum over keys of dk + dkd is zero (a row's dS sums to zero),
    per KV head and column."""
    name = "fwd-bwd-16k"
    cfg = workloads.CONFIGS[name]
    x = gpu_inputs(cfg, workloads.SEED_BASE[name], with_dout=True)
    scale = workloads.default_scale(cfg["d"])
    g = run_gpu(x, scale, True)
    G = cfg["Hq"] // cfg["Hkv"]
    B, Hkv, d = cfg["B"], cfg["Hkv"], cfg["d"]
    dout_sum = x["dout"].double().view(B, Hkv, G, cfg["T"], d).sum(dim=(2, 3))
    dv_sum = g["dv"].double().sum(2) + g["dvd"].double().sum(dim=(2, 3))
    dk_sum = g["dk"].double().sum(2) + g["dkd"].double().sum(dim=(2, 3))
    scale_dv = dout_sum.abs().max().item()
    assert (dv_sum - dout_sum).abs().max().item() < 2e-3 * scale_dv + 0.5
    assert dk_sum.abs().max().item() < 0.5
    del x, g
    torch.cuda.empty_cache()
