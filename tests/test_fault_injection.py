"""Host-side fault injection (MODA_FAULT_INJECT), on CPU: every compute entry point of the
C ABI returns the injected status without launching anything.

MODA_FAULT_INJECT=validate fails each call before its argument checks with
MODA_ERR_INVALID_ARGUMENT; =launch lets the argument checks run and then fails with
MODA_ERR_CUDA in place of the device query and the launch.  The calls below pass fake
device addresses with otherwise valid arguments, so they run only where no GPU is present:
if the injection failed there, nothing could be launched either.
"""
import ctypes

import pytest
import torch

import depth_aware_attention_b200 as moda

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake device addresses: CPU-only test")

A = 1 << 20  # fake, 16-byte aligned addresses 1 MiB apart (never dereferenced)


def _p(i):
    return ctypes.c_void_p(A * i)


def calls():
    """One call of every compute entry point with valid sizes and non-overlapping fake
    buffers (tiny problem: B=1, Hq=4, Hkv=2, T=16, L=2, d=64)."""
    B, Hq, Hkv, T, L, d, sc = 1, 4, 2, 16, 2, 64, 0.125
    f = moda.lib
    return {
        "moda_forward": lambda: f.moda_forward(_p(1), _p(2), _p(3), _p(4), _p(5), _p(6), _p(7),
                                               B, Hq, Hkv, T, L, d, sc, 1, None),
        "moda_forward_depth_path": lambda: f.moda_forward_depth_path(
            _p(1), _p(2), _p(3), _p(4), _p(5), _p(6), _p(7), B, Hq, Hkv, T, L, d, sc, 1, 1,
            None),
        "moda_depth_attention_forward": lambda: f.moda_depth_attention_forward(
            _p(1), _p(4), _p(5), _p(6), _p(7), B, Hq, Hkv, T, L, d, sc, None),
        "moda_depth_attention_backward": lambda: f.moda_depth_attention_backward(
            _p(1), _p(4), _p(5), _p(6), _p(7), _p(8), _p(9), _p(12), _p(13), _p(64),
            1 << 20, B, Hq, Hkv, T, L, d, sc, None),
        "moda_decode": lambda: f.moda_decode(_p(1), _p(2), _p(3), _p(4), _p(5), _p(6), _p(7),
                                             _p(64), 1 << 20, B, Hq, Hkv, T, L, d, sc, None),
        "moda_depth_kv_write": lambda: f.moda_depth_kv_write(_p(1), _p(2), _p(4), _p(5), B, T,
                                                             64, Hkv, d, L, 0, None),
        "moda_backward": lambda: f.moda_backward(
            *[_p(i) for i in range(1, 14)], _p(64), 1 << 20, B, Hq, Hkv, T, L, d, sc, 1, None),
        "moda_backward_stages": lambda: f.moda_backward_stages(
            *[_p(i) for i in range(1, 14)], _p(64), 1 << 20, B, Hq, Hkv, T, L, d, sc, 1, 7,
            None),
        "moda_backward_noalloc": lambda: f.moda_backward_noalloc(
            *[_p(i) for i in range(1, 14)], B, Hq, Hkv, T, L, d, sc, 1, None),
    }


@pytest.mark.parametrize("name", sorted(calls()))
def test_validate_injection_fails_before_the_argument_checks(name, monkeypatch):
    monkeypatch.setenv("MODA_FAULT_INJECT", "validate")
    assert calls()[name]() == moda.MODA_ERR_INVALID_ARGUMENT
    assert b"MODA_FAULT_INJECT=validate" in moda.lib.moda_last_error_message()


@pytest.mark.parametrize("name", sorted(calls()))
def test_launch_injection_fails_after_the_argument_checks(name, monkeypatch):
    monkeypatch.setenv("MODA_FAULT_INJECT", "launch")
    assert calls()[name]() == moda.MODA_ERR_CUDA
    assert b"MODA_FAULT_INJECT=launch" in moda.lib.moda_last_error_message()


def test_launch_injection_leaves_argument_errors_first(monkeypatch):
    monkeypatch.setenv("MODA_FAULT_INJECT", "launch")
    st = moda.lib.moda_forward(None, _p(2), _p(3), _p(4), _p(5), _p(6), _p(7),
                               1, 4, 2, 16, 2, 64, 0.125, 1, None)
    assert st == moda.MODA_ERR_INVALID_ARGUMENT
    assert b"injected" not in moda.lib.moda_last_error_message()


@pytest.mark.parametrize("value", ["", "other"])
def test_other_values_inject_nothing(value, monkeypatch):
    monkeypatch.setenv("MODA_FAULT_INJECT", value)
    st = moda.lib.moda_forward(None, _p(2), _p(3), _p(4), _p(5), _p(6), _p(7),
                               1, 4, 2, 16, 2, 64, 0.125, 1, None)
    assert st == moda.MODA_ERR_INVALID_ARGUMENT
    assert b"injected" not in moda.lib.moda_last_error_message()
