"""Property-based pins of the fp64 oracle: on randomly drawn small shapes (every group
size, L = 0 included, odd head sizes, one-token sequences, causal or not, any token
window), the oracle equals torch's scaled-dot-product attention over the concatenated
sequence and own-token depth keys with a visibility mask, and its backward equals that
reference's autograd gradients (CPU only).

The operator is exact attention over the enlarged key set (hyper.ai summary of arXiv
2603.15619, section "Mixture-of-Depths Attention (MoDA)": one softmax over the causal
sequence keys and the query token's own depth keys), so a library attention with the
matching mask is an independent statement of it.
"""
import math

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle
from test_oracle_pins import rand_problem, sdpa_reference


@st.composite
def problems(draw):
    Hkv = draw(st.integers(1, 3))
    G = draw(st.integers(1, 4))
    T = draw(st.integers(1, 12))
    shape = dict(B=draw(st.integers(1, 2)), T=T, Hq=Hkv * G, Hkv=Hkv,
                 d=draw(st.integers(1, 16)), L=draw(st.integers(0, 5)))
    t0 = draw(st.integers(0, T - 1))
    nt = draw(st.integers(1, T - t0))
    return shape, draw(st.booleans()), t0, nt, draw(st.integers(0, 2**31 - 1))


@settings(max_examples=60, deadline=None, derandomize=True)
@given(problems())
def test_forward_window_equals_masked_sdpa(p):
    shape, causal, t0, nt, seed = p
    x = rand_problem(**shape, seed=seed)
    scale = 1.0 / math.sqrt(shape["d"])
    ref_out, ref_lse = sdpa_reference(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, causal)
    w = slice(t0, t0 + nt)
    out, lse = oracle.forward(x["q"][:, :, w], x["k"], x["v"], x["kd"][:, :, w],
                              x["vd"][:, :, w], scale, causal, t0=t0)
    np.testing.assert_allclose(out, ref_out[:, :, w].numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse[:, :, w].numpy(), rtol=0, atol=1e-12)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(problems())
def test_backward_equals_sdpa_autograd(p):
    shape, causal, _, _, seed = p
    x = rand_problem(**shape, seed=seed)
    scale = 1.0 / math.sqrt(shape["d"])
    g = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale, causal)
    leaves = {n: x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "kd", "vd")}
    ref_out, _ = sdpa_reference(leaves["q"], leaves["k"], leaves["v"], leaves["kd"],
                                leaves["vd"], scale, causal)
    ref_out.backward(x["dout"])
    names = ("q", "k", "v") + (("kd", "vd") if shape["L"] else ())
    for n in names:
        np.testing.assert_allclose(g["d" + n], leaves[n].grad.numpy(), rtol=0, atol=1e-11,
                                   err_msg=n)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(problems())
def test_depth_only_equals_masked_sdpa_over_own_entries(p):
    shape, _, t0, nt, seed = p
    if shape["L"] == 0:
        shape = dict(shape, L=1)
    x = rand_problem(**shape, seed=seed)
    B, Hq, Hkv, d, L = (shape[n] for n in ("B", "Hq", "Hkv", "d", "L"))
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d)
    w = slice(t0, t0 + nt)
    out, lse = oracle.depth_forward(x["q"][:, :, w], x["kd"][:, :, w], x["vd"][:, :, w],
                                    scale, t0=t0)
    # per token, attention over that token's L entries only: a batch of L-key problems
    q = x["q"][:, :, w].reshape(B, Hkv, G, nt, d).permute(0, 1, 3, 2, 4)   # [B,Hkv,nt,G,d]
    kd = x["kd"][:, :, w]                                                   # [B,Hkv,nt,L,d]
    vd = x["vd"][:, :, w]
    ref = torch.nn.functional.scaled_dot_product_attention(q, kd, vd, scale=scale)
    ref = ref.permute(0, 1, 3, 2, 4).reshape(B, Hq, nt, d)
    ref_lse = torch.logsumexp(torch.einsum("bgtjc,bgtlc->bgtjl", q, kd) * scale, dim=-1)
    ref_lse = ref_lse.permute(0, 1, 3, 2).reshape(B, Hq, nt)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)
