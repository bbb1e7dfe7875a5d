"""The forward kernel's FMA-pipe exponential (used for a quarter of the exponentials of
unmasked sequence blocks) against exact 2^x and its stated error bound.

The softmax of the fused kernel (hyper.ai summary of arXiv 2603.15619, section
"Hardware-efficient implementation") needs p = 2^(s*scale*log2(e) - m); the kernel computes
some of these with a Cody-Waite reduction and a cubic instead of the exponent unit.  Its
relative error must stay far inside the bf16 rounding of P (2^-9): the bound checked here is
8e-5 on [-125, 8] (the arguments the online softmax can produce, the upper end being the
lazy-rescale threshold), and arguments below -125 must give the value at -125.
"""
import ctypes

import numpy as np
import pytest

import depth_aware_attention_b200 as moda


def test_exp2_fma_rejects_bad_arguments_before_any_cuda_call():
    fake = ctypes.c_void_p(1 << 32)
    assert moda.moda_test_exp2_fma(fake, fake, -1) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_test_exp2_fma(fake, fake, (1 << 30) + 1) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_test_exp2_fma(None, fake, 4) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_test_exp2_fma(fake, None, 4) == moda.MODA_ERR_INVALID_ARGUMENT
    odd = ctypes.c_void_p((1 << 32) + 2)
    assert moda.moda_test_exp2_fma(odd, fake, 4) == moda.MODA_ERR_INVALID_ARGUMENT


@pytest.mark.gpu
def test_exp2_fma_relative_error_bound():
    import torch
    dev = torch.device("cuda", 0)
    grid = np.linspace(-125.0, 8.0, 2_000_001)
    # the reduction's edges: integers, half-integers and their float neighbours
    k = np.arange(-125, 9, dtype=np.float64)
    edges = np.concatenate([k, k + 0.5, k - 0.5])
    edges = np.concatenate([edges, np.nextafter(edges.astype(np.float32), np.float32(np.inf)),
                            np.nextafter(edges.astype(np.float32), np.float32(-np.inf))])
    xs = np.concatenate([grid, edges]).astype(np.float32)
    xs = xs[(xs >= -125.0) & (xs <= 8.0)]
    x = torch.from_numpy(xs).to(dev)
    y = moda.test_exp2_fma(x)
    torch.cuda.synchronize(dev)
    ref = np.exp2(xs.astype(np.float64))
    rel = np.abs(y.cpu().numpy().astype(np.float64) / ref - 1.0)
    assert np.all(np.isfinite(rel))
    assert rel.max() <= 8e-5, (rel.max(), xs[rel.argmax()])
    # an odd count takes the kernel's single-element tail
    y3 = moda.test_exp2_fma(x[:3].contiguous())
    assert torch.equal(y3, y[:3])


@pytest.mark.gpu
def test_exp2_fma_clamps_below_minus_125():
    import torch
    dev = torch.device("cuda", 0)
    xs = torch.tensor([-125.0, -125.25, -126.0, -149.0, -1000.0, -3.0e38, float("-inf")],
                      dtype=torch.float32, device=dev)
    y = moda.test_exp2_fma(xs).cpu().double().numpy()
    at = y[0]
    assert abs(at / 2.0 ** -125 - 1.0) <= 8e-5
    assert np.all(y[1:] == at)
