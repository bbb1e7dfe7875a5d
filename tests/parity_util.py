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

import json
import os

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


def log_stats(what, **fields):
    """Appends one JSON line of measured errors to the file named by MODA_PARITY_STATS
    (when set), so that a run can record every case's figures, passing or not."""
    path = os.environ.get("MODA_PARITY_STATS")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(case=what, **fields)) + "\n")


def error_stats(err, ref):
    """max-abs, plain mean-abs, max beyond rounding and mean beyond rounding."""
    ex = excess(err, ref)
    return dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                max_beyond_rounding=float(ex.max()),
                mean_beyond_rounding=float(np.maximum(ex, 0.0).mean()))


def compare_forward(out, lse, ref_out, ref_lse, what="", mean_beyond_rounding=False):
    o = out.detach().to("cpu", torch.float64).numpy()
    ls = lse.detach().to("cpu", torch.float64).numpy()
    err = np.abs(o - ref_out)
    lerr = np.abs(ls - ref_lse)
    st = error_stats(err, ref_out)
    log_stats(what, kind="out", rows=int(np.prod(ref_lse.shape)), lse_max_abs=float(lerr.max()),
              **st)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert st["max_beyond_rounding"] <= OUT_MAX, (
        f"{what}: out max-abs {st['max_abs']:.3e} (beyond rounding "
        f"{st['max_beyond_rounding']:.3e})")
    mean = st["mean_beyond_rounding"] if mean_beyond_rounding else st["mean_abs"]
    assert mean <= OUT_MEAN, f"{what}: out mean-abs {mean:.3e} (plain {st['mean_abs']:.3e})"
    assert lerr.max() <= LSE_MAX, f"{what}: lse max-abs {lerr.max():.3e}"
    return st["max_abs"], st["mean_abs"], float(lerr.max())


def compare_grad(g, ref, what, max_tol=OUT_MAX, mean_tol=OUT_MEAN, mean_beyond_rounding=False):
    a = g.detach().to("cpu", torch.float64).numpy()
    err = np.abs(a - ref)
    st = error_stats(err, ref)
    rms = float(np.sqrt((ref ** 2).mean()))
    rel = float(np.sqrt((err ** 2).mean())) / rms if rms > 0 else 0.0
    log_stats(what, kind="grad", elements=int(ref.size), rel_rms=rel, **st)
    assert np.isfinite(a).all(), f"{what}: non-finite"
    assert st["max_beyond_rounding"] <= max_tol, (
        f"{what}: max-abs {st['max_abs']:.3e} (beyond rounding "
        f"{st['max_beyond_rounding']:.3e})")
    mean = st["mean_beyond_rounding"] if mean_beyond_rounding else st["mean_abs"]
    assert mean <= mean_tol, f"{what}: mean-abs {mean:.3e} (plain {st['mean_abs']:.3e})"
    assert rel <= GRAD_REL_RMS, f"{what}: relative RMS error {rel:.3e}"
    return st["max_abs"], st["mean_abs"]


def window_starts(T, nt, n_random, seed):
    """Starts of token windows of nt tokens: the first (t = 0), the last (t = T-1) and
    n_random more drawn uniformly from a seeded generator."""
    rng = np.random.RandomState(seed)
    starts = [0, T - nt] + [int(s) for s in rng.randint(0, T - nt + 1, size=n_random)]
    return sorted(set(starts))


def oracle_forward_windows(x, starts, nt, scale, causal):
    """Oracle forward on several token windows of one problem.  k and v are widened to
    fp64 once and shared by every window.  Yields (t0, ref_out, ref_lse)."""
    k = x["k"].cpu().to(torch.float64).numpy()
    v = x["v"].cpu().to(torch.float64).numpy()
    for t0 in starts:
        sl = slice(t0, t0 + nt)
        kd = None if x.get("kd") is None else x["kd"][:, :, sl].cpu()
        vd = None if x.get("vd") is None else x["vd"][:, :, sl].cpu()
        ref_out, ref_lse = oracle.forward(x["q"][:, :, sl].cpu(), k, v, kd, vd, scale,
                                          causal, t0=t0)
        yield t0, ref_out, ref_lse
