"""The torch-level wrappers check tensor metadata before any pointer reaches the library.

The C ABI sees only pointers and sizes, and the wrappers take the sizes from q, k and kd.
A tensor smaller than those sizes say, a strided view or another dtype would make a kernel
read or write outside a buffer, so each of these must raise before the call.  CPU tensors
with consistent metadata get as far as the device check; no test here reaches a kernel.
"""
import pytest
import torch

import depth_aware_attention_b200 as moda

BF = torch.bfloat16
B, Hq, Hkv, T, L, d = 1, 4, 2, 16, 3, 64


def _t(*shape, dtype=BF, device="cpu"):
    return torch.zeros(*shape, dtype=dtype, device=device)


def _fwd_inputs():
    return dict(q=_t(B, Hq, T, d), k=_t(B, Hkv, T, d), v=_t(B, Hkv, T, d),
                kd=_t(B, Hkv, T, L, d), vd=_t(B, Hkv, T, L, d))


def test_forward_consistent_cpu_tensors_stop_at_the_device_check():
    x = _fwd_inputs()
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"])
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.forward(x["q"], x["k"], x["v"], None, None)


@pytest.mark.parametrize("name,bad,err,match", [
    ("k", _t(B, Hkv, T - 1, d), ValueError, "k has shape"),
    ("v", _t(B, Hkv + 1, T, d), ValueError, "v has shape"),
    ("vd", _t(B, Hkv, T, L - 1, d), ValueError, "vd has shape"),
    ("vd", None, ValueError, "vd is required"),
    ("q", _t(B, Hq, T, d, dtype=torch.float32), TypeError, "q has dtype"),
    ("kd", _t(B, Hkv, T, d, L).transpose(3, 4), ValueError, "kd must be contiguous"),
    ("v", _t(B, Hkv, T, d, device="meta"), ValueError, "v is on meta"),
    ("q", _t(B, Hq, T), ValueError, "q must be a 4-D tensor"),
])
def test_forward_rejects_bad_tensors(name, bad, err, match):
    x = _fwd_inputs()
    x[name] = bad
    with pytest.raises(err, match=match):
        moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"])


def test_forward_rejects_bad_outputs():
    x = _fwd_inputs()
    with pytest.raises(ValueError, match="out has shape"):
        moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], out=_t(B, Hq, T - 1, d))
    with pytest.raises(TypeError, match="lse has dtype"):
        moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], lse=_t(B, Hq, T))
    with pytest.raises(ValueError, match="out must be contiguous"):
        moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"],
                     out=_t(B, Hq, d, T).transpose(2, 3))


def test_backward_checks_gradients_and_workspace():
    x = _fwd_inputs()
    out, lse, dout = _t(B, Hq, T, d), _t(B, Hq, T, dtype=torch.float32), _t(B, Hq, T, d)
    args = (x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, dout)
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.backward(*args)
    with pytest.raises(ValueError, match="dk has shape"):
        moda.backward(*args, grads=dict(dk=_t(B, Hkv, T + 1, d)))
    with pytest.raises(TypeError, match="dvd has dtype"):
        moda.backward(*args, grads=dict(dvd=_t(B, Hkv, T, L, d, dtype=torch.float16)))
    with pytest.raises(ValueError, match="dout has shape"):
        moda.backward(*args[:7], _t(B, Hq, T, d + 1))
    with pytest.raises(ValueError, match="workspace must be a contiguous tensor"):
        moda.backward(*args, workspace=_t(64, dtype=torch.uint8, device="meta"))


def test_depth_attention_checks_its_tensors():
    x = _fwd_inputs()
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.depth_attention_forward(x["q"], x["kd"], x["vd"])
    with pytest.raises(ValueError, match="vd has shape"):
        moda.depth_attention_forward(x["q"], x["kd"], _t(B, Hkv, T, L + 1, d))
    out, lse, dout = _t(B, Hq, T, d), _t(B, Hq, T, dtype=torch.float32), _t(B, Hq, T, d)
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.depth_attention_backward(x["q"], x["kd"], x["vd"], out, lse, dout)
    with pytest.raises(TypeError, match="lse has dtype"):
        moda.depth_attention_backward(x["q"], x["kd"], x["vd"], out, lse.double(), dout)


def test_decode_checks_its_tensors():
    S = 40
    q, k, v = _t(B, Hq, d), _t(B, Hkv, S, d), _t(B, Hkv, S, d)
    kd, vd = _t(B, Hkv, L, d), _t(B, Hkv, L, d)
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.decode(q, k, v, kd, vd)
    with pytest.raises(ValueError, match="v has shape"):
        moda.decode(q, k, _t(B, Hkv, S - 1, d), kd, vd)
    with pytest.raises(ValueError, match="q must be a 3-D tensor"):
        moda.decode(_t(B, Hq, 1, d), k, v, kd, vd)
    with pytest.raises(ValueError, match="lse has shape"):
        moda.decode(q, k, v, kd, vd, lse=_t(B, Hq, 1, dtype=torch.float32))


def test_depth_kv_write_checks_its_tensors():
    hidden = 96
    x, w = _t(B, T, hidden), _t(2 * Hkv * d, hidden)
    kd, vd = _t(B, Hkv, T, L, d), _t(B, Hkv, T, L, d)
    with pytest.raises(ValueError, match="runs on CUDA tensors"):
        moda.depth_kv_write(x, w, kd, vd, 0)
    with pytest.raises(ValueError, match="w has shape"):
        moda.depth_kv_write(x, _t(Hkv * d, hidden), kd, vd, 0)
    with pytest.raises(ValueError, match="vd has shape"):
        moda.depth_kv_write(x, w, kd, _t(B, Hkv, T, L + 1, d), 0)
    with pytest.raises(TypeError, match="x has dtype"):
        moda.depth_kv_write(x.float(), w, kd, vd, 0)
