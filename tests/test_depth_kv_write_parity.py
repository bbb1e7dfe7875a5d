"""GPU fused depth-stream write (moda_depth_kv_write through the C ABI) vs the oracle's
fp64 projection: slot l of kd / vd must hold K|V = x W^T rounded to bf16, every other
slot must keep its previous bits.  Cases cover both head sizes, ragged token counts (the
last 128-token tile partly outside), a hidden size that is not a multiple of the 64-wide
K-slices, the first and the last slot, and the 1.5B-layer shape (hidden 2048, 4 KV heads
of 128).  Weights are drawn with standard deviation hidden^-1/2, as a trained projection's
scale, so the outputs are O(1) and the bf16 tolerances of the attention tests apply.
"""
import math

import pytest
import torch

import depth_aware_attention_b200 as moda
import oracle
from parity_util import compare_grad

pytestmark = pytest.mark.gpu

CASES = [
    ("d128", dict(B=2, T=300, hidden=256, Hkv=2, d=128, L=5, slot=0)),
    ("d64-last-slot", dict(B=1, T=200, hidden=128, Hkv=2, d=64, L=3, slot=2)),
    ("ragged-hidden", dict(B=1, T=129, hidden=200, Hkv=1, d=128, L=4, slot=1)),
    ("layer-1.5b", dict(B=1, T=4096, hidden=2048, Hkv=4, d=128, L=24, slot=7)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_depth_kv_write_matches_oracle(name, cfg):
    B, T, hidden, Hkv, d, L, slot = (cfg[n] for n in ("B", "T", "hidden", "Hkv", "d", "L",
                                                       "slot"))
    g = torch.Generator().manual_seed(700 + [c[0] for c in CASES].index(name))
    x = torch.randn(B, T, hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn(2 * Hkv * d, hidden, generator=g) / math.sqrt(hidden)).to(torch.bfloat16)
    kd0 = torch.randn(B, Hkv, T, L, d, generator=g).to(torch.bfloat16)
    vd0 = torch.randn(B, Hkv, T, L, d, generator=g).to(torch.bfloat16)
    kd, vd = kd0.cuda(), vd0.cuda()
    moda.depth_kv_write(x.cuda(), w.cuda(), kd, vd, slot)
    moda.check_device_errors()
    ref_k, ref_v = oracle.depth_kv_projection(x, w, Hkv, d)
    kd, vd = kd.cpu(), vd.cpu()
    compare_grad(kd[:, :, :, slot], ref_k, f"{name}:k", mean_beyond_rounding=True)
    compare_grad(vd[:, :, :, slot], ref_v, f"{name}:v", mean_beyond_rounding=True)
    others = [s for s in range(L) if s != slot]
    assert torch.equal(kd[:, :, :, others], kd0[:, :, :, others])
    assert torch.equal(vd[:, :, :, others], vd0[:, :, :, others])


def test_depth_kv_write_is_deterministic_and_feeds_the_forward():
    """Two writes give the same bits; slots written one layer at a time are what the
    forward reads as the depth cache."""
    B, T, hidden, Hkv, Hq, d, L = 1, 257, 256, 2, 8, 128, 3
    g = torch.Generator().manual_seed(790)
    xs = [torch.randn(B, T, hidden, generator=g).to(torch.bfloat16).cuda() for _ in range(L)]
    w = (torch.randn(2 * Hkv * d, hidden, generator=g) / 16).to(torch.bfloat16).cuda()
    kd = torch.zeros(B, Hkv, T, L, d, dtype=torch.bfloat16, device="cuda")
    vd = torch.zeros_like(kd)
    for l in range(L):
        moda.depth_kv_write(xs[l], w, kd, vd, l)
    kd2, vd2 = torch.zeros_like(kd), torch.zeros_like(vd)
    for l in range(L):
        moda.depth_kv_write(xs[l], w, kd2, vd2, l)
    moda.check_device_errors()
    assert torch.equal(kd, kd2) and torch.equal(vd, vd2)
    q = torch.randn(B, Hq, T, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16).cuda()
    out, lse = moda.forward(q, k, v, kd, vd)
    moda.check_device_errors()
    ref_out, ref_lse = oracle.forward(q.cpu(), k.cpu(), v.cpu(), kd.cpu(), vd.cpu(),
                                      1 / math.sqrt(d))
    assert (out.cpu().double().numpy() - ref_out).__abs__().max() < 2e-2
