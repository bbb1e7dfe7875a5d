"""GPU single-token decode (moda_decode through the C ABI) vs the fp64 oracle.

Decode is the forward's row for the newest token of each sequence: the oracle's forward
on the one-token window t0 = S-1 of a problem with T = S computes exactly it.  Cases
cover every group-size class (1, 3, 4, 8, 16), both head sizes, caches from 1 key (the
token alone) through ragged lengths to 64K keys, L = 0, 1, 5 and 130 depth entries, and
the split of the sequence over many CTAs.  The decode result is also checked against the
forward kernel's last row on the same data.
"""
import math

import pytest
import torch

import depth_aware_attention_b200 as moda
import oracle
from parity_util import compare_forward

pytestmark = pytest.mark.gpu

CASES = [
    ("g4-d128", dict(B=2, S=300, Hq=8, Hkv=2, d=128, L=5)),
    ("g1-d64", dict(B=1, S=200, Hq=2, Hkv=2, d=64, L=3)),
    ("g3-d128", dict(B=1, S=130, Hq=6, Hkv=2, d=128, L=7)),
    ("g8-d128-L0", dict(B=1, S=257, Hq=16, Hkv=2, d=128, L=0)),
    ("g16-d64", dict(B=1, S=100, Hq=16, Hkv=1, d=64, L=2)),
    ("g32-d128", dict(B=2, S=300, Hq=32, Hkv=1, d=128, L=5)),    # two 16-head chunks
    ("g64-d64", dict(B=1, S=150, Hq=128, Hkv=2, d=64, L=3)),     # four 16-head chunks
    ("S1", dict(B=3, S=1, Hq=4, Hkv=2, d=128, L=6)),
    ("longL", dict(B=1, S=64, Hq=4, Hkv=1, d=128, L=130)),
    ("many-splits", dict(B=1, S=20000, Hq=8, Hkv=2, d=128, L=24)),
    ("64k", dict(B=1, S=65536, Hq=16, Hkv=4, d=128, L=32)),
]


def _inputs(cfg, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, dtype=torch.float32).to(torch.bfloat16)
    B, S, Hq, Hkv, d, L = (cfg[n] for n in ("B", "S", "Hq", "Hkv", "d", "L"))
    x = dict(q=mk(B, Hq, d), k=mk(B, Hkv, S, d), v=mk(B, Hkv, S, d))
    x["kd"] = mk(B, Hkv, L, d) if L else None
    x["vd"] = mk(B, Hkv, L, d) if L else None
    return x


def _oracle(x, cfg, scale):
    S, L = cfg["S"], cfg["L"]
    q = x["q"][:, :, None, :]
    kd = None if not L else x["kd"][:, :, None]
    vd = None if not L else x["vd"][:, :, None]
    out, lse = oracle.forward(q, x["k"], x["v"], kd, vd, scale, True, t0=S - 1)
    return out[:, :, 0], lse[:, :, 0]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(name, cfg):
    x = _inputs(cfg, 500 + [c[0] for c in CASES].index(name))
    xg = {k: (None if t is None else t.cuda()) for k, t in x.items()}
    scale = 1.0 / math.sqrt(cfg["d"])
    out, lse = moda.decode(xg["q"], xg["k"], xg["v"], xg["kd"], xg["vd"], scale)
    moda.check_device_errors()
    ref_out, ref_lse = _oracle(x, cfg, scale)
    compare_forward(out, lse, ref_out, ref_lse, name)


def test_decode_is_deterministic_and_matches_forward_last_row():
    cfg = dict(B=2, S=700, Hq=8, Hkv=2, d=128, L=9)
    B, S, Hq, Hkv, d, L = (cfg[n] for n in ("B", "S", "Hq", "Hkv", "d", "L"))
    g = torch.Generator().manual_seed(599)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16).cuda()
    q, k, v = mk(B, Hq, S, d), mk(B, Hkv, S, d), mk(B, Hkv, S, d)
    kd, vd = mk(B, Hkv, S, L, d), mk(B, Hkv, S, L, d)
    fo, fl = moda.forward(q, k, v, kd, vd)
    a, la = moda.decode(q[:, :, -1].contiguous(), k, v, kd[:, :, -1].contiguous(),
                        vd[:, :, -1].contiguous())
    b, lb = moda.decode(q[:, :, -1].contiguous(), k, v, kd[:, :, -1].contiguous(),
                        vd[:, :, -1].contiguous())
    moda.check_device_errors()
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert (a.float() - fo[:, :, -1].float()).abs().max().item() <= 1.6e-2
    assert (la - fl[:, :, -1]).abs().max().item() <= 1e-3
