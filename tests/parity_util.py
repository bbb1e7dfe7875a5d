"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the
fp64 oracle on the same bf16 bits (whole problem or token windows), compare with the
stated tolerances.

Tolerances (bf16 outputs, fp32 accumulation on the GPU), against the fp64 oracle's unrounded
result: max-abs error <= 1e-2 and mean-abs error <= 1e-3; lse within 1e-3.

The max-abs bound is applied beyond the output format's own rounding: element x may differ
from the exact value by 1e-2 plus half a bf16 ULP of x.  No bf16 number lies within 1e-2 of
some reals above 4 (bf16's spacing there is 1/32), so an exact kernel would otherwise fail
on large gradient entries.  For |x| < 2 the extra term is at most 2^-8.  Gradients are also
held to a relative RMS error of 1e-2 (bf16 operands carry 2^-9 relative rounding).

Depth-only attention's outputs average only the L values of one token's depth keys, so
they are O(1) and their bf16 rounding alone averages about |x| * 2^-10 (1e-3 at |x| ~ 1);
for it the mean-abs bound too is applied beyond the output rounding
(``mean_beyond_rounding``): the mean of max(0, err - half ULP).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

OUT_MAX, OUT_MEAN, LSE_MAX = 1e-2, 1e-3, 1e-3
GRAD_REL_RMS = 1e-2


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 8.0)


def excess(err, ref):
    """Error beyond the bf16 output rounding allowance (<= OUT_MAX passes)."""
    return err - bf16_half_ulp(ref)


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


def compare_forward(out, lse, ref_out, ref_lse, what="", mean_beyond_rounding=False):
    o = out.detach().to("cpu", torch.float64).numpy()
    ls = lse.detach().to("cpu", torch.float64).numpy()
    err = np.abs(o - ref_out)
    lerr = np.abs(ls - ref_lse)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    ex = excess(err, ref_out)
    assert ex.max() <= OUT_MAX, f"{what}: out max-abs {err.max():.3e} (beyond rounding {ex.max():.3e})"
    mean = np.maximum(ex, 0.0).mean() if mean_beyond_rounding else err.mean()
    assert mean <= OUT_MEAN, f"{what}: out mean-abs {mean:.3e}"
    assert lerr.max() <= LSE_MAX, f"{what}: lse max-abs {lerr.max():.3e}"
    return float(err.max()), float(err.mean()), float(lerr.max())


def compare_grad(g, ref, what, max_tol=OUT_MAX, mean_tol=OUT_MEAN, mean_beyond_rounding=False):
    a = g.detach().to("cpu", torch.float64).numpy()
    err = np.abs(a - ref)
    assert np.isfinite(a).all(), f"{what}: non-finite"
    ex = excess(err, ref)
    assert ex.max() <= max_tol, f"{what}: max-abs {err.max():.3e} (beyond rounding {ex.max():.3e})"
    mean = np.maximum(ex, 0.0).mean() if mean_beyond_rounding else err.mean()
    assert mean <= mean_tol, f"{what}: mean-abs {mean:.3e}"
    rms = float(np.sqrt((ref ** 2).mean()))
    if rms > 0:
        rel = float(np.sqrt((err ** 2).mean())) / rms
        assert rel <= GRAD_REL_RMS, f"{what}: relative RMS error {rel:.3e}"
    return float(err.max()), float(err.mean())
