"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the
fp64 oracle on the same bf16 bits (whole problem or token windows), compare with the
stated tolerances.

Tolerances (bf16 outputs, fp32 accumulation on the GPU): max-abs error <= 1e-2 and
mean-abs error <= 1e-3 against the fp64 oracle's unrounded result; lse within 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

OUT_MAX, OUT_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3


def gpu_inputs(cfg, seed_base, with_dout=False, device="cuda"):
    """Seeded inputs on the GPU.  Small problems draw on the CPU and copy up (so the CPU
    oracle can use the same draws cheaply); large ones draw directly on the device."""
    n = cfg["B"] * cfg["Hkv"] * cfg["T"] * max(cfg["L"], 1) * cfg["d"]
    if n <= (1 << 24):
        x = workloads.make_inputs(cfg, seed_base, "cpu", with_dout)
        return {k: (None if t is None else t.to(device)) for k, t in x.items()}
    return workloads.make_inputs(cfg, seed_base, device, with_dout)


def window(x, t0, nt):
    """CPU copies of what the oracle needs for query tokens [t0, t0+nt)."""
    sl = slice(t0, t0 + nt)
    w = dict(q=x["q"][:, :, sl].cpu(), k=x["k"].cpu(), v=x["v"].cpu())
    w["kd"] = None if x.get("kd") is None else x["kd"][:, :, sl].cpu()
    w["vd"] = None if x.get("vd") is None else x["vd"][:, :, sl].cpu()
    if x.get("dout") is not None:
        w["dout"] = x["dout"][:, :, sl].cpu()
    return w


def oracle_forward_window(x, t0, nt, scale, causal):
    w = window(x, t0, nt)
    return oracle.forward(w["q"], w["k"], w["v"], w["kd"], w["vd"], scale, causal, t0=t0)


def compare_forward(out, lse, ref_out, ref_lse, what=""):
    o = out.detach().to("cpu", torch.float64).numpy()
    ls = lse.detach().to("cpu", torch.float64).numpy()
    err = np.abs(o - ref_out)
    lerr = np.abs(ls - ref_lse)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err.max() <= OUT_MAX, f"{what}: out max-abs {err.max():.3e}"
    assert err.mean() <= OUT_MEAN, f"{what}: out mean-abs {err.mean():.3e}"
    assert lerr.max() <= LSE_MAX, f"{what}: lse max-abs {lerr.max():.3e}"
    return float(err.max()), float(err.mean()), float(lerr.max())


def compare_grad(g, ref, what, max_tol=OUT_MAX, mean_tol=OUT_MEAN):
    a = g.detach().to("cpu", torch.float64).numpy()
    err = np.abs(a - ref)
    assert np.isfinite(a).all(), f"{what}: non-finite"
    assert err.max() <= max_tol, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= mean_tol, f"{what}: mean-abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())
