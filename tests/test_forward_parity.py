"""GPU forward (moda_forward through the C ABI) vs the fp64 CPU oracle, element by element.

Small problems are compared in full: they span several query tiles and key blocks, ragged
tails, every supported group shape (including a group size that does not divide 128),
both head sizes, causal and full sequence masks, L = 0, T = 1 and long depth caches.  The
benchmark-size workloads are compared on token windows (start, middle and end of the
sequence) in the same launch configuration the benchmark times.
"""
import math

import pytest
import torch

import depth_aware_attention_b200 as moda
import workloads
from parity_util import (compare_forward, gpu_inputs, oracle_forward_window,
                         oracle_forward_windows, window_starts)
import oracle

pytestmark = pytest.mark.gpu

SMALL = [
    ("tiny", workloads.CONFIGS["tiny"], True),
    ("ragged-g4-d128", dict(B=2, T=300, Hq=8, Hkv=2, d=128, L=5), True),
    ("g1-d64", dict(B=1, T=200, Hq=2, Hkv=2, d=64, L=3), True),
    ("g3-d128", dict(B=1, T=130, Hq=6, Hkv=2, d=128, L=7), True),
    ("g8-d128", dict(B=1, T=257, Hq=16, Hkv=2, d=128, L=9), True),
    ("g16-d64", dict(B=1, T=100, Hq=16, Hkv=1, d=64, L=2), True),
    ("g32-d128", dict(B=1, T=150, Hq=32, Hkv=1, d=128, L=5), True),
    ("g64-d64", dict(B=1, T=90, Hq=64, Hkv=1, d=64, L=3), True),
    ("L0-d128", dict(B=1, T=333, Hq=8, Hkv=2, d=128, L=0), True),
    ("T1", dict(B=2, T=1, Hq=4, Hkv=2, d=128, L=6), True),
    ("longL-d128", dict(B=1, T=64, Hq=4, Hkv=1, d=128, L=130), True),
    ("noncausal-g4", dict(B=1, T=190, Hq=4, Hkv=1, d=128, L=4), False),
    ("noncausal-L0-d64", dict(B=1, T=129, Hq=2, Hkv=1, d=64, L=0), False),
    ("multi-tile-d64", dict(B=1, T=700, Hq=4, Hkv=2, d=64, L=11), True),
]


@pytest.mark.parametrize("name,cfg,causal", SMALL, ids=[s[0] for s in SMALL])
def test_forward_small_full(name, cfg, causal):
    x = gpu_inputs(cfg, seed_base=100 + SMALL.index((name, cfg, causal)))
    scale = 1.0 / math.sqrt(cfg["d"])
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal)
    moda.check_device_errors()
    ref_out, ref_lse = oracle_forward_window(x, 0, cfg["T"], scale, causal)
    compare_forward(out, lse, ref_out, ref_lse, name)


@pytest.mark.parametrize("path", [1, 2], ids=["fold", "dense"])
@pytest.mark.parametrize("name,cfg,causal", SMALL, ids=[s[0] for s in SMALL])
def test_forward_small_full_each_depth_path(name, cfg, causal, path):
    """Both depth paths (CUDA-core fold, dense tensor-core depth blocks) on every case;
    the dense path refuses groups that do not divide 128 or exceed 32 (a row sees only its
    warp's 32 columns of a depth block)."""
    x = gpu_inputs(cfg, seed_base=100 + SMALL.index((name, cfg, causal)))
    scale = 1.0 / math.sqrt(cfg["d"])
    G = cfg["Hq"] // cfg["Hkv"]
    if path == 2 and (128 % G != 0 or G > 32):
        with pytest.raises(moda.ModaError) as e:
            moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal,
                         depth_path=path)
        assert e.value.status == moda.MODA_ERR_UNSUPPORTED
        return
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal,
                            depth_path=path)
    moda.check_device_errors()
    ref_out, ref_lse = oracle_forward_window(x, 0, cfg["T"], scale, causal)
    compare_forward(out, lse, ref_out, ref_lse, f"{name} path {path}")


@pytest.mark.parametrize("path", [1, 2], ids=["fold", "dense"])
def test_forward_deep_windows_each_depth_path(path):
    """The deep-stack head layout (L = 128) at 4K tokens through each depth path, on
    16-token windows at the start, the end and seeded random positions (every head: at
    least 4096 rows); each path is also deterministic."""
    cfg = workloads.CONFIGS["deep-4k"]
    x = gpu_inputs(cfg, workloads.SEED_BASE["deep-4k"])
    scale = workloads.default_scale(cfg["d"])
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True,
                            depth_path=path)
    out2, lse2 = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True,
                              depth_path=path)
    moda.check_device_errors()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    T, nt = cfg["T"], 16
    starts = window_starts(T, nt, 6, seed=workloads.SEED_BASE["deep-4k"])
    for t0, ref_out, ref_lse in oracle_forward_windows(x, starts, nt, scale, True):
        sl = slice(t0, t0 + nt)
        compare_forward(out[:, :, sl], lse[:, :, sl], ref_out, ref_lse,
                        f"deep-4k path {path} @{t0}")
    del x, out, lse, out2, lse2
    torch.cuda.empty_cache()


def test_forward_is_deterministic_and_leaves_inputs_intact():
    cfg = dict(B=1, T=515, Hq=8, Hkv=2, d=128, L=6)
    x = gpu_inputs(cfg, seed_base=150)
    before = {k: v.clone() for k, v in x.items() if v is not None}
    a, la = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"])
    b, lb = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"])
    moda.check_device_errors()
    assert torch.equal(a, b) and torch.equal(la, lb)
    for k, v in before.items():
        assert torch.equal(v, x[k]), k


def test_forward_writes_only_its_outputs():
    """Canary fill around out/lse: the kernel must not write outside its rows."""
    cfg = dict(B=1, T=77, Hq=4, Hkv=2, d=64, L=3)
    x = gpu_inputs(cfg, seed_base=151)
    n_out = cfg["B"] * cfg["Hq"] * cfg["T"] * cfg["d"]
    n_lse = cfg["B"] * cfg["Hq"] * cfg["T"]
    big = torch.full((n_out + 4096,), -7.0, device="cuda", dtype=torch.bfloat16)
    out = big[2048:2048 + n_out].view(cfg["B"], cfg["Hq"], cfg["T"], cfg["d"])
    bigl = torch.full((n_lse + 256,), -7.0, device="cuda", dtype=torch.float32)
    lse = bigl[128:128 + n_lse].view(cfg["B"], cfg["Hq"], cfg["T"])
    moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], out=out, lse=lse)
    moda.check_device_errors()
    assert torch.all(big[:2048] == -7.0) and torch.all(big[2048 + n_out:] == -7.0)
    assert torch.all(bigl[:128] == -7.0) and torch.all(bigl[128 + n_lse:] == -7.0)
    ref_out, ref_lse = oracle_forward_window(x, 0, cfg["T"], 1 / 8, True)
    compare_forward(out, lse, ref_out, ref_lse, "canary")


def test_L0_matches_torch_causal_attention():
    """Special case: with no depth entries the kernel is causal GQA attention."""
    cfg = dict(B=2, T=1000, Hq=8, Hkv=2, d=128, L=0)
    x = gpu_inputs(cfg, seed_base=152)
    out, _ = moda.forward(x["q"], x["k"], x["v"], None, None)
    moda.check_device_errors()
    G = cfg["Hq"] // cfg["Hkv"]
    ref = torch.nn.functional.scaled_dot_product_attention(
        x["q"].float(), x["k"].float().repeat_interleave(G, 1),
        x["v"].float().repeat_interleave(G, 1), is_causal=True)
    assert (out.float() - ref).abs().max().item() < 1e-2


BIG = ["layer-4k", "long-64k", "long-64k-L0", "deep-stack", "fwd-bwd-16k"]


SAMPLE_ROWS = 4096


@pytest.mark.parametrize("name", BIG)
def test_forward_benchmark_workloads_windows(name):
    """A stratified sample of at least 4096 rows of each benchmark workload, in the launch
    configuration the benchmark times: every head of every batch entry on 8-token windows
    at t = 0, at t = T-1 and at seeded random positions.  Rows are independent, so each
    sampled row is compared with its exact oracle value."""
    cfg = workloads.CONFIGS[name]
    x = gpu_inputs(cfg, workloads.SEED_BASE[name])
    scale = workloads.default_scale(cfg["d"])
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True)
    moda.check_device_errors()
    T, nt = cfg["T"], 8
    per_window = cfg["B"] * cfg["Hq"] * nt
    n_windows = max(8, -(-SAMPLE_ROWS // per_window))
    starts = window_starts(T, nt, n_windows - 2, seed=workloads.SEED_BASE[name])
    assert len(starts) * per_window >= SAMPLE_ROWS and starts[0] == 0 and starts[-1] == T - nt
    for t0, ref_out, ref_lse in oracle_forward_windows(x, starts, nt, scale, True):
        sl = slice(t0, t0 + nt)
        compare_forward(out[:, :, sl], lse[:, :, sl], ref_out, ref_lse, f"{name}@{t0}")
    del x, out, lse
    torch.cuda.empty_cache()


def test_layer4k_full_oracle():
    cfg = workloads.CONFIGS["layer-4k"]
    x = gpu_inputs(cfg, workloads.SEED_BASE["layer-4k"])
    scale = workloads.default_scale(cfg["d"])
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True)
    moda.check_device_errors()
    ref_out, ref_lse = oracle_forward_window(x, 0, cfg["T"], scale, True)
    compare_forward(out, lse, ref_out, ref_lse, "layer-4k full")
