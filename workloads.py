"""Seeded synthetic workloads for MoDA -- shared by the tests, the benchmark and the smoke check.

This module holds shapes and random inputs only: none of the operator's arithmetic.  Both
sides of every parity check (the CUDA library and the fp64 CPU oracle) receive the exact
bf16 bits produced here.

Workloads are shaped like the pages' setting -- a 1.5B-parameter GQA decoder at 4K to 64K
tokens (hyper.ai summary of arXiv 2603.15619, sections "Main contributions" and
"Experiments") -- with head counts, head size and depth-cache length L chosen as stated
per entry, because the pages give none of them.  Every tensor is i.i.d. N(0, 1) rounded
to bf16; no dataset or trained weight is involved.
"""
from __future__ import annotations

import math

import torch

# name -> shape.  L is the number of depth K/V entries each token holds.
CONFIGS = {
    "tiny": dict(B=1, T=128, Hq=4, Hkv=2, d=64, L=4),
    "layer-4k": dict(B=1, T=4096, Hq=16, Hkv=4, d=128, L=24),
    "long-64k": dict(B=1, T=65536, Hq=16, Hkv=4, d=128, L=32),
    "long-64k-L0": dict(B=1, T=65536, Hq=16, Hkv=4, d=128, L=0),
    "deep-stack": dict(B=4, T=8192, Hq=32, Hkv=8, d=128, L=128),
    "fwd-bwd-16k": dict(B=1, T=16384, Hq=16, Hkv=4, d=128, L=48),
    # deep-stack head layout at 4K tokens: small enough (2.2 GB of depth cache) for an
    # ncu capture of the depth-dominated regime
    "deep-4k": dict(B=1, T=4096, Hq=32, Hkv=8, d=128, L=128),
    # the 16K fwd+bwd shape at head dimension 64, for the d = 64 kernels' ncu captures
    "fwd-bwd-16k-d64": dict(B=1, T=16384, Hq=16, Hkv=4, d=64, L=48),
}

# seed base per workload (inputs use base*1000 + index, index 0..5 = q,k,v,kd,vd,dout)
SEED_BASE = {"tiny": 0, "layer-4k": 1, "long-64k": 2, "long-64k-L0": 2, "deep-stack": 3,
             "fwd-bwd-16k": 4, "deep-4k": 5, "fwd-bwd-16k-d64": 6}

NAMES = ("q", "k", "v", "kd", "vd", "dout")


def shapes(B, T, Hq, Hkv, d, L):
    """Tensor shapes of one problem (row-major, contiguous)."""
    return dict(q=(B, Hq, T, d), k=(B, Hkv, T, d), v=(B, Hkv, T, d),
                kd=(B, Hkv, T, L, d), vd=(B, Hkv, T, L, d), dout=(B, Hq, T, d))


def make_inputs(cfg: dict, seed_base: int, device="cpu", with_dout=False):
    """i.i.d. N(0,1) bf16 tensors q,k,v,kd,vd (and dout) for shape dict ``cfg``.

    Each tensor draws from its own torch generator on ``device`` seeded with
    ``seed_base*1000 + index``.  CPU and CUDA generators give different bits; a check
    draws once, on one device, and copies the bits to the other side.
    """
    shp = shapes(**{k: cfg[k] for k in ("B", "T", "Hq", "Hkv", "d", "L")})
    dev = torch.device(device)
    out = {}
    names = NAMES if with_dout else NAMES[:5]
    for idx, name in enumerate(NAMES):
        if name not in names:
            continue
        if name in ("kd", "vd") and cfg["L"] == 0:
            out[name] = None
            continue
        g = torch.Generator(device=dev)
        g.manual_seed(seed_base * 1000 + idx)
        out[name] = torch.randn(shp[name], generator=g, device=dev, dtype=torch.bfloat16)
    return out


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def forward_flops(B, T, Hq, d, L, causal=True, **_):
    """Algorithmic forward FLOPs 4*B*Hq*d*(T^2/2 + T*L) (causal) / 4*B*Hq*d*(T^2 + T*L)."""
    seq = T * T / 2.0 if causal else float(T) * T
    return 4.0 * B * Hq * d * (seq + T * L)


def depth_bytes(B, T, Hkv, d, L, **_):
    """Bytes of the bf16 depth cache kd + vd, each read once."""
    return 2 * 2 * B * Hkv * T * L * d
