"""Pins of the fp64 CPU oracle to things other than itself (CPU only).

The operator (hyper.ai summary of arXiv 2603.15619, section "Mixture-of-Depths Attention
(MoDA)") is exact attention over an enlarged key set: the causal sequence keys plus the
query token's own L depth keys, all in one jointly normalised softmax.  So:

* it equals torch's scaled-dot-product attention over the concatenation [k ; kd] with a
  boolean visibility mask (library special case, forward and autograd backward);
* with L = 0 it is causal GQA attention (SDPA ``is_causal``);
* with T = 1 it is ordinary attention over the L + 1 keys;
* it is invariant to permuting depth entries, its weights sum to one, identical keys
  give the mean of the visible values with a closed-form log-sum-exp, and a depth key
  whose logit leads by 30 returns its value;
* its backward matches central finite differences of its own forward and obeys the
  key-shift / value-sum identities; hand-derived cases in tests/golden/ fix a few
  values outright.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def rand_problem(B, T, Hq, Hkv, d, L, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g, dtype=dtype)
    return dict(q=mk(B, Hq, T, d), k=mk(B, Hkv, T, d), v=mk(B, Hkv, T, d),
                kd=mk(B, Hkv, T, L, d), vd=mk(B, Hkv, T, L, d), dout=mk(B, Hq, T, d))


def sdpa_reference(q, k, v, kd, vd, scale, causal):
    """MoDA via torch SDPA over the concatenated keys [k ; kd flattened] with a mask.

    Row t may see sequence key s (s <= t if causal) and depth keys t*L .. t*L+L-1.
    Returns (out, lse) in fp64; lse by torch.logsumexp of the masked scores.
    """
    B, Hq, T, d = q.shape
    Hkv, L = k.shape[1], kd.shape[3]
    G = Hq // Hkv
    kcat = torch.cat([k, kd.reshape(B, Hkv, T * L, d)], dim=2).repeat_interleave(G, dim=1)
    vcat = torch.cat([v, vd.reshape(B, Hkv, T * L, d)], dim=2).repeat_interleave(G, dim=1)
    seq_mask = torch.ones(T, T, dtype=torch.bool)
    if causal:
        seq_mask = torch.tril(seq_mask)
    dep_mask = torch.zeros(T, T * L, dtype=torch.bool)
    for t in range(T):
        dep_mask[t, t * L:(t + 1) * L] = True
    mask = torch.cat([seq_mask, dep_mask], dim=1)
    out = F.scaled_dot_product_attention(q, kcat, vcat, attn_mask=mask, scale=scale)
    scores = torch.einsum("bhtc,bhsc->bhts", q, kcat) * scale
    lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
    return out, lse


SHAPES = [
    dict(B=1, T=9, Hq=4, Hkv=2, d=8, L=3),
    dict(B=2, T=7, Hq=3, Hkv=1, d=5, L=1),
    dict(B=1, T=16, Hq=2, Hkv=2, d=16, L=5),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_forward_equals_masked_sdpa(shape, causal):
    x = rand_problem(**shape, seed=11)
    scale = 0.7 / math.sqrt(shape["d"])
    out, lse = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal)
    ref_out, ref_lse = sdpa_reference(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal)
    np.testing.assert_allclose(out, ref_out.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_equals_sdpa_autograd(causal):
    shape = dict(B=1, T=8, Hq=4, Hkv=2, d=8, L=3)
    x = rand_problem(**shape, seed=12)
    scale = 1.0 / math.sqrt(shape["d"])
    g = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale, causal)
    leaves = {n: x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "kd", "vd")}
    ref_out, _ = sdpa_reference(leaves["q"], leaves["k"], leaves["v"], leaves["kd"],
                                leaves["vd"], scale, causal)
    ref_out.backward(x["dout"])
    for n in ("q", "k", "v", "kd", "vd"):
        np.testing.assert_allclose(g["d" + n], leaves[n].grad.numpy(), rtol=0, atol=1e-12,
                                   err_msg=n)


def test_L0_is_causal_gqa_attention():
    B, T, Hq, Hkv, d = 2, 33, 6, 2, 16
    x = rand_problem(B, T, Hq, Hkv, d, 1, seed=13)
    scale = 1.0 / math.sqrt(d)
    empty = torch.zeros(B, Hkv, T, 0, d, dtype=torch.float64)
    out, lse = oracle.forward(x["q"], x["k"], x["v"], empty, empty, scale, True)
    G = Hq // Hkv
    kk, vv = x["k"].repeat_interleave(G, 1), x["v"].repeat_interleave(G, 1)
    ref = F.scaled_dot_product_attention(x["q"], kk, vv, is_causal=True, scale=scale)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    # gradients with L=0 equal SDPA autograd
    dq_etc = oracle.backward(x["q"], x["k"], x["v"], empty, empty, x["dout"], scale, True)
    lq = x["q"].clone().requires_grad_(True)
    lk = x["k"].clone().requires_grad_(True)
    lv = x["v"].clone().requires_grad_(True)
    F.scaled_dot_product_attention(lq, lk.repeat_interleave(G, 1), lv.repeat_interleave(G, 1),
                                   is_causal=True, scale=scale).backward(x["dout"])
    np.testing.assert_allclose(dq_etc["dq"], lq.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dq_etc["dk"], lk.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dq_etc["dv"], lv.grad.numpy(), atol=1e-12, rtol=0)


def test_T1_is_attention_over_depth_plus_self():
    B, Hq, Hkv, d, L = 1, 4, 2, 8, 6
    x = rand_problem(B, 1, Hq, Hkv, d, L, seed=14)
    scale = 0.3
    out, lse = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True)
    G = Hq // Hkv
    keys = torch.cat([x["k"], x["kd"][:, :, 0]], dim=2).repeat_interleave(G, 1)  # [B,Hq,1+L,d]
    vals = torch.cat([x["v"], x["vd"][:, :, 0]], dim=2).repeat_interleave(G, 1)
    ref = F.scaled_dot_product_attention(x["q"], keys, vals, scale=scale)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("bhtc,bhsc->bhts", x["q"], keys) * scale
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_depth_permutation_invariance():
    shape = dict(B=1, T=10, Hq=4, Hkv=2, d=8, L=5)
    x = rand_problem(**shape, seed=15)
    perm = torch.tensor([3, 0, 4, 1, 2])
    scale = 0.4
    base = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale)
    pk, pv = x["kd"][:, :, :, perm], x["vd"][:, :, :, perm]
    permd = oracle.backward(x["q"], x["k"], x["v"], pk, pv, x["dout"], scale)
    for n in ("out", "lse", "dq", "dk", "dv"):
        np.testing.assert_allclose(permd[n], base[n], rtol=0, atol=1e-13, err_msg=n)
    np.testing.assert_allclose(permd["dkd"], base["dkd"][:, :, :, perm.numpy()], atol=1e-13)
    np.testing.assert_allclose(permd["dvd"], base["dvd"][:, :, :, perm.numpy()], atol=1e-13)


@pytest.mark.parametrize("causal", [True, False])
def test_row_weights_sum_to_one_and_match_softmax(causal):
    shape = dict(B=2, T=12, Hq=4, Hkv=2, d=8, L=3)
    x = rand_problem(**shape, seed=16)
    scale = 0.5
    for (b, h, t) in [(0, 0, 0), (1, 3, 11), (0, 2, 5)]:
        ws, wd = oracle.row_weights(x["q"], x["k"], x["kd"], b, h, t, scale, causal)
        assert abs(ws.sum() + wd.sum() - 1.0) < 1e-12
        g = h // 2
        n = t + 1 if causal else 12
        keys = torch.cat([x["k"][b, g, :n], x["kd"][b, g, t]], dim=0)
        p = torch.softmax(keys @ x["q"][b, h, t] * scale, dim=0).numpy()
        np.testing.assert_allclose(np.concatenate([ws, wd]), p, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [True, False])
def test_identical_keys_give_mean_of_values(causal):
    B, T, Hq, Hkv, d, L = 1, 9, 4, 2, 8, 3
    x = rand_problem(B, T, Hq, Hkv, d, L, seed=17)
    kappa = torch.randn(d, dtype=torch.float64, generator=torch.Generator().manual_seed(5))
    k = kappa.expand(B, Hkv, T, d).contiguous()
    kd = kappa.expand(B, Hkv, T, L, d).contiguous()
    scale = 0.9
    out, lse = oracle.forward(x["q"], k, x["v"], kd, x["vd"], scale, causal)
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        for t in range(T):
            n = t + 1 if causal else T
            mean = (x["v"][0, g, :n].sum(0) + x["vd"][0, g, t].sum(0)) / (n + L)
            np.testing.assert_allclose(out[0, h, t], mean.numpy(), rtol=0, atol=1e-12)
            want_lse = scale * float(x["q"][0, h, t] @ kappa) + math.log(n + L)
            assert abs(lse[0, h, t] - want_lse) < 1e-12


def test_plus30_depth_boost_returns_its_value():
    B, T, Hq, Hkv, d, L = 1, 12, 2, 1, 8, 4
    x = rand_problem(B, T, Hq, Hkv, d, L, seed=18)
    scale = 1.0 / math.sqrt(d)
    kd = x["kd"].clone()
    t, j, h = 7, 2, 1
    qv = x["q"][0, h, t]
    n = t + 1
    logits = torch.cat([x["k"][0, 0, :n], x["kd"][0, 0, t]]) @ qv * scale
    others = torch.cat([logits[:n], logits[n:][torch.arange(L) != j]])
    # choose kd[t,j] along q so that its logit leads every other one by 30
    target = float(others.max()) + 30.0
    kd[0, 0, t, j] = qv * (target / (scale * float(qv @ qv)))
    out, _ = oracle.forward(x["q"], x["k"], x["v"], kd, x["vd"], scale, True)
    bound = (n + L) * math.exp(-30.0) * float(torch.cat([x["v"][0, 0, :n].abs().flatten(),
                                                          x["vd"][0, 0, t].abs().flatten()]).max()) * 2
    np.testing.assert_allclose(out[0, h, t], x["vd"][0, 0, t, j].numpy(), rtol=0, atol=bound)


def test_backward_matches_finite_differences():
    shape = dict(B=1, T=5, Hq=2, Hkv=1, d=4, L=2)
    x = rand_problem(**shape, seed=19)
    scale = 0.6
    g = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale)
    dO = x["dout"].numpy()
    eps = 1e-6
    rng = np.random.default_rng(3)
    for n in ("q", "k", "v", "kd", "vd"):
        for _ in range(3):
            direction = torch.from_numpy(rng.standard_normal(tuple(x[n].shape)))
            plus = dict(x); minus = dict(x)
            plus[n] = x[n] + eps * direction
            minus[n] = x[n] - eps * direction
            fp, _ = oracle.forward(plus["q"], plus["k"], plus["v"], plus["kd"], plus["vd"], scale)
            fm, _ = oracle.forward(minus["q"], minus["k"], minus["v"], minus["kd"], minus["vd"], scale)
            numeric = float(((fp - fm) * dO).sum() / (2 * eps))
            analytic = float((g["d" + n] * direction.numpy()).sum())
            assert abs(numeric - analytic) < 1e-7 * max(1.0, abs(analytic)), (n, numeric, analytic)


def test_gradient_identities():
    """Per (b, g): sum of all key gradients is 0 (softmax is shift invariant in the keys);
    sum of all value gradients equals the sum of dO over the group's rows (weights sum to 1)."""
    shape = dict(B=2, T=11, Hq=6, Hkv=2, d=8, L=4)
    x = rand_problem(**shape, seed=20)
    g = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], 0.35)
    key_sum = g["dk"].sum(2) + g["dkd"].sum((2, 3))
    np.testing.assert_allclose(key_sum, 0.0, atol=1e-12)
    val_sum = g["dv"].sum(2) + g["dvd"].sum((2, 3))
    dO = x["dout"].numpy().reshape(2, 2, 3, 11, 8).sum((2, 3))
    np.testing.assert_allclose(val_sum, dO, atol=1e-12)


def test_windows_agree_with_full_problem():
    shape = dict(B=1, T=20, Hq=4, Hkv=2, d=8, L=3)
    x = rand_problem(**shape, seed=21)
    scale = 0.4
    full = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale)
    t0 = 13
    sl = slice(t0, None)
    out, lse = oracle.forward(x["q"][:, :, sl], x["k"], x["v"], x["kd"][:, :, sl],
                              x["vd"][:, :, sl], scale, t0=t0)
    np.testing.assert_allclose(out, full["out"][:, :, sl], atol=1e-14, rtol=0)
    np.testing.assert_allclose(lse, full["lse"][:, :, sl], atol=1e-14, rtol=0)
    win = oracle.backward(x["q"][:, :, sl], x["k"], x["v"], x["kd"][:, :, sl], x["vd"][:, :, sl],
                          x["dout"][:, :, sl], scale, t0=t0)
    for n in ("dq", "dkd", "dvd"):
        np.testing.assert_allclose(win[n], full[n][:, :, sl], atol=1e-13, rtol=0, err_msg=n)
    for n in ("dk", "dv"):
        np.testing.assert_allclose(win[n][:, :, sl], full[n][:, :, sl], atol=1e-13, rtol=0)


def _parse(v):
    if isinstance(v, list):
        return [_parse(e) for e in v]
    if isinstance(v, str):
        coef, _, rest = v.partition("ln")
        c = -1.0 if coef == "-" else (float(coef) if coef else 1.0)
        return c * math.log(float(rest))
    return float(v)


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["cases"], ids=lambda c: c["name"])
def test_golden_forward(case):
    arr = {n: np.array(_parse(case[n]), dtype=np.float64) for n in ("q", "k", "v", "kd", "vd")}
    out, lse = oracle.forward(arr["q"], arr["k"], arr["v"], arr["kd"], arr["vd"],
                              case["scale"], bool(case["causal"]))
    np.testing.assert_allclose(out, np.array(_parse(case["out"])), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, np.array(_parse(case["lse"])), atol=1e-12, rtol=0)


@pytest.mark.parametrize("case", _golden()["backward_cases"], ids=lambda c: c["name"])
def test_golden_backward(case):
    arr = {n: np.array(_parse(case[n]), dtype=np.float64)
           for n in ("q", "k", "v", "kd", "vd", "dout")}
    g = oracle.backward(arr["q"], arr["k"], arr["v"], arr["kd"], arr["vd"], arr["dout"],
                        case["scale"], bool(case["causal"]))
    for n in ("dq", "dk", "dv", "dkd", "dvd"):
        np.testing.assert_allclose(g[n], np.array(_parse(case[n])), atol=1e-12, rtol=0,
                                   err_msg=n)


def test_seeded_inputs_are_reproducible_bf16():
    cfg = workloads.CONFIGS["tiny"]
    a = workloads.make_inputs(cfg, 0, with_dout=True)
    b = workloads.make_inputs(cfg, 0, with_dout=True)
    for n in workloads.NAMES:
        assert a[n].dtype == torch.bfloat16
        assert torch.equal(a[n], b[n])
    assert a["kd"].shape == (1, 2, 128, 4, 64)
    # N(0,1): sample mean/std sanity on the largest tensor
    assert abs(float(a["kd"].float().mean())) < 0.05
    assert abs(float(a["kd"].float().std()) - 1.0) < 0.05


# ---------------------------------------------------------------- backward with a given out
def test_backward_given_own_out_equals_backward():
    x = rand_problem(B=1, T=11, Hq=4, Hkv=2, d=8, L=3, seed=41)
    scale = 0.35
    ref = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale, True)
    got = oracle.backward_given_out(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"],
                                    ref["out"], scale, True)
    for n in ("dq", "dk", "dv", "dkd", "dvd"):
        np.testing.assert_allclose(got[n], ref[n], rtol=0, atol=1e-13)


def test_backward_given_out_shifts_only_the_row_terms():
    """With out' = out + delta, D' = <dO, out'> replaces D.  The value gradients dv, dvd do
    not involve D; and since a row's dS then sums to D - D' instead of zero, the sum over
    all keys (sequence and depth) of dk + dkd equals scale * sum_r (D_r - D'_r) q_r per KV
    group -- zero for the exact out."""
    B, T, Hq, Hkv, d, L = 1, 9, 4, 2, 6, 2
    x = rand_problem(B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, L=L, seed=42)
    scale = 0.4
    ref = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale, True)
    g = torch.Generator().manual_seed(43)
    delta = 1e-3 * torch.randn(B, Hq, T, d, generator=g, dtype=torch.float64).numpy()
    got = oracle.backward_given_out(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"],
                                    ref["out"] + delta, scale, True)
    np.testing.assert_allclose(got["dv"], ref["dv"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(got["dvd"], ref["dvd"], rtol=0, atol=1e-13)
    dO, q = x["dout"].numpy(), x["q"].numpy()
    dD = -(dO * delta).sum(-1)                                   # D - D'  [B,Hq,T]
    G = Hq // Hkv
    expect = scale * np.einsum("bht,bhtc->bhc", dD, q).reshape(B, Hkv, G, d).sum(2)
    total = got["dk"].sum(2) + got["dkd"].sum(axis=(2, 3))
    np.testing.assert_allclose(total, expect, rtol=1e-9, atol=1e-13)
    assert np.abs(ref["dk"].sum(2) + ref["dkd"].sum(axis=(2, 3))).max() < 1e-12


# ---------------------------------------------------------------- depth-only attention
def sdpa_depth_reference(q, kd, vd, scale):
    """Depth-only attention via torch SDPA: row t sees exactly its own token's L depth
    keys (a block-diagonal mask over the flattened [T*L] depth keys).  fp64."""
    B, Hq, T, d = q.shape
    Hkv, L = kd.shape[1], kd.shape[3]
    G = Hq // Hkv
    kf = kd.reshape(B, Hkv, T * L, d).repeat_interleave(G, dim=1)
    vf = vd.reshape(B, Hkv, T * L, d).repeat_interleave(G, dim=1)
    mask = torch.zeros(T, T * L, dtype=torch.bool)
    for t in range(T):
        mask[t, t * L:(t + 1) * L] = True
    out = F.scaled_dot_product_attention(q, kf, vf, attn_mask=mask, scale=scale)
    scores = torch.einsum("bhtc,bhsc->bhts", q, kf) * scale
    lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
    return out, lse


@pytest.mark.parametrize("shape", SHAPES)
def test_depth_forward_equals_masked_sdpa(shape):
    x = rand_problem(**shape, seed=41)
    scale = 0.37
    out, lse = oracle.depth_forward(x["q"], x["kd"], x["vd"], scale)
    ref_out, ref_lse = sdpa_depth_reference(x["q"], x["kd"], x["vd"], scale)
    assert np.abs(out - ref_out.numpy()).max() < 1e-12
    assert np.abs(lse - ref_lse.numpy()).max() < 1e-12


def test_depth_backward_equals_sdpa_autograd():
    x = rand_problem(B=1, T=6, Hq=4, Hkv=2, d=8, L=3, seed=43)
    scale = 0.45
    g = oracle.depth_backward(x["q"], x["kd"], x["vd"], x["dout"], scale)
    leaves = {n: x[n].clone().requires_grad_(True) for n in ("q", "kd", "vd")}
    ref_out, _ = sdpa_depth_reference(leaves["q"], leaves["kd"], leaves["vd"], scale)
    (ref_out * x["dout"]).sum().backward()
    for n in ("q", "kd", "vd"):
        assert np.abs(g["d" + n] - leaves[n].grad.numpy()).max() < 1e-12, n


def test_depth_single_entry_closed_form():
    """L = 1: the one depth key takes all the weight, so out is its value, lse its logit,
    and only dvd is non-zero (the sum of the group's dO)."""
    x = rand_problem(B=2, T=4, Hq=6, Hkv=2, d=8, L=1, seed=45)
    scale = 0.5
    g = oracle.depth_backward(x["q"], x["kd"], x["vd"], x["dout"], scale)
    G = 3
    vd = x["vd"][:, :, :, 0].numpy().repeat(G, axis=1)
    kd = x["kd"][:, :, :, 0].numpy().repeat(G, axis=1)
    assert np.abs(g["out"] - vd).max() < 1e-14
    assert np.abs(g["lse"] - scale * (x["q"].numpy() * kd).sum(-1)).max() < 1e-13
    assert np.abs(g["dq"]).max() < 1e-14 and np.abs(g["dkd"]).max() < 1e-14
    dsum = x["dout"].numpy().reshape(2, 2, G, 4, 8).sum(2)
    assert np.abs(g["dvd"][:, :, :, 0] - dsum).max() < 1e-13


def test_depth_only_is_moda_at_one_token():
    """A one-token MoDA problem (its sequence key is its own k) equals depth-only attention
    over the depth keys with k prepended: the two oracle modes agree on the definition."""
    x = rand_problem(B=1, T=1, Hq=4, Hkv=2, d=8, L=3, seed=47)
    scale = 0.3
    out, lse = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    kd = torch.cat([x["k"][:, :, :, None], x["kd"]], dim=3)
    vd = torch.cat([x["v"][:, :, :, None], x["vd"]], dim=3)
    out2, lse2 = oracle.depth_forward(x["q"], kd, vd, scale)
    assert np.abs(out - out2).max() < 1e-14 and np.abs(lse - lse2).max() < 1e-14


def test_depth_backward_matches_finite_differences():
    x = rand_problem(B=1, T=3, Hq=2, Hkv=1, d=4, L=4, seed=49)
    scale = 0.7
    g = oracle.depth_backward(x["q"], x["kd"], x["vd"], x["dout"], scale)
    dO = x["dout"].numpy()
    eps = 1e-6
    rng = np.random.default_rng(5)
    for n in ("q", "kd", "vd"):
        for _ in range(3):
            direction = torch.from_numpy(rng.standard_normal(tuple(x[n].shape)))
            plus = dict(x); minus = dict(x)
            plus[n] = x[n] + eps * direction
            minus[n] = x[n] - eps * direction
            fp, _ = oracle.depth_forward(plus["q"], plus["kd"], plus["vd"], scale)
            fm, _ = oracle.depth_forward(minus["q"], minus["kd"], minus["vd"], scale)
            numeric = float(((fp - fm) * dO).sum() / (2 * eps))
            analytic = float((g["d" + n] * direction.numpy()).sum())
            assert abs(numeric - analytic) < 1e-7 * max(1.0, abs(analytic)), (n, numeric, analytic)


def test_depth_backward_given_own_out_equals_exact():
    x = rand_problem(B=1, T=5, Hq=4, Hkv=1, d=8, L=6, seed=51)
    g = oracle.depth_backward(x["q"], x["kd"], x["vd"], x["dout"], 0.4)
    h = oracle.depth_backward(x["q"], x["kd"], x["vd"], x["dout"], 0.4, out=g["out"])
    for n in ("dq", "dkd", "dvd"):
        assert np.abs(g[n] - h[n]).max() < 1e-14, n


# ---------------------------------------------------------------- depth-stream write
def test_depth_kv_projection_selects_columns_with_one_hot_weights():
    """A weight row that is one-hot at column c copies x[..., c]: checks the K/V split
    and the (head, column) placement of every output element."""
    B, T, hidden, Hkv, d = 2, 3, 16, 2, 4
    x = torch.randn(B, T, hidden, dtype=torch.float64)
    rng = np.random.default_rng(7)
    src = rng.integers(0, hidden, size=2 * Hkv * d)
    w = np.zeros((2 * Hkv * d, hidden))
    w[np.arange(2 * Hkv * d), src] = 1.0
    k, v = oracle.depth_kv_projection(x, w, Hkv, d)
    xn = x.numpy()
    for part, arr in ((0, k), (1, v)):
        for g in range(Hkv):
            for c in range(d):
                col = src[part * Hkv * d + g * d + c]
                assert np.array_equal(arr[:, g, :, c], xn[:, :, col])


def test_depth_kv_projection_is_linear_in_weights():
    B, T, hidden, Hkv, d = 1, 5, 8, 1, 4
    x = torch.randn(B, T, hidden, dtype=torch.float64)
    w1 = np.random.default_rng(1).standard_normal((2 * Hkv * d, hidden))
    w2 = np.random.default_rng(2).standard_normal((2 * Hkv * d, hidden))
    a1, b1 = oracle.depth_kv_projection(x, w1, Hkv, d)
    a2, b2 = oracle.depth_kv_projection(x, w2, Hkv, d)
    a3, b3 = oracle.depth_kv_projection(x, 2.0 * w1 - w2, Hkv, d)
    assert np.abs(a3 - (2 * a1 - a2)).max() < 1e-12 and np.abs(b3 - (2 * b1 - b2)).max() < 1e-12
