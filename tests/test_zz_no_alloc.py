"""moda_backward_noalloc: the backward for callers that cannot allocate device memory.

Those callers (device memory owned by another allocator or a fixed memory plan, or a plain
C binding with no device allocation API) cannot hand moda_backward a workspace, so the
library serves them from a 64 MiB static device array instead.  This test calls the new
entry point through the C ABI, twice in a row, and checks both results against
moda_backward run with a caller workspace, within the tolerance of the other GPU tests
(max-abs 1e-2, mean-abs 1e-3).  The second call sees the array as the first one left it.

The file is named to be collected last, so that a run stopping at its first failure has
already run every other test.  The test also passes alone in a fresh process.
"""
import ctypes
import math

import pytest
import torch

import depth_aware_attention_b200 as moda
from parity_util import gpu_inputs

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dkd", "dvd")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_backward_matches_workspace_backward_on_two_calls(cuda_device):
    cfg = dict(B=1, T=1000, Hq=8, Hkv=2, d=128, L=6)
    x = gpu_inputs(cfg, seed_base=300, with_dout=True)
    scale = 1.0 / math.sqrt(cfg["d"])
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True)
    ref = moda.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"], scale,
                        True)
    moda.check_device_errors()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        g = {n: torch.full_like(ref[n], float("nan")) for n in NAMES}
        st = moda.moda_backward_noalloc(
            _p(x["q"]), _p(x["k"]), _p(x["v"]), _p(x["kd"]), _p(x["vd"]), _p(out), _p(lse),
            _p(x["dout"]), _p(g["dq"]), _p(g["dk"]), _p(g["dv"]), _p(g["dkd"]), _p(g["dvd"]),
            cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["T"], cfg["L"], cfg["d"], scale, 1, stream)
        assert st == moda.MODA_OK, moda.moda_status_string(st)
        moda.check_device_errors()
        for n in NAMES:
            err = (g[n].float() - ref[n].float()).abs()
            assert torch.isfinite(g[n].float()).all(), f"call {call}: {n} not written"
            assert err.max().item() <= 1e-2, f"call {call}: {n} max-abs {err.max().item():.3e}"
            assert err.mean().item() <= 1e-3, f"call {call}: {n} mean-abs {err.mean().item():.3e}"
