"""The C-ABI library loads, exports every entry point include/moda.h declares, and
rejects bad arguments before touching the GPU (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

import depth_aware_attention_b200 as moda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moda.h")

# A fake, 16-byte aligned "device pointer" that is never dereferenced.  Every call in this
# file must fail an argument check: on a machine with a GPU, a call whose arguments are all
# valid would launch a kernel on these addresses.
A = 1 << 20


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moda_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert set(names) == set(moda.EXPORTED)
    lib = ctypes.CDLL(moda.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_library_is_sm100a_only_and_self_contained():
    # no link-time dependency on the CUDA driver or a shared CUDA runtime
    deps = os.popen(f"ldd {moda.LIB_PATH}").read()
    assert "libcuda.so" not in deps
    assert "libcudart" not in deps


def test_status_strings():
    for s in range(6):
        assert moda.moda_status_string(s)
    assert moda.moda_status_string(99) == "unknown status"


def fwd(**kw):
    args = dict(q=A, k=A * 2, v=A * 3, kd=A * 4, vd=A * 5, out=A * 64, lse=A * 128, B=1,
                Hq=4, Hkv=2, T=16, L=2, d=64, scale=0.125, causal=1, stream=None)
    args.update(kw)
    return moda.moda_forward(**args)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(T=0), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(L=-1), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(Hq=3, Hkv=2), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(d=96), moda.MODA_ERR_UNSUPPORTED),
    (dict(Hq=256, Hkv=2), moda.MODA_ERR_UNSUPPORTED),
    (dict(Hq=130, Hkv=1), moda.MODA_ERR_UNSUPPORTED),  # G = 130: beyond groups of 64
    (dict(q=None), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(kd=None), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(q=A + 8), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(lse=A * 3 + 4), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(out=A * 2), moda.MODA_ERR_INVALID_ARGUMENT),  # out aliases k
    (dict(scale=float("nan")), moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(scale=float("inf")), moda.MODA_ERR_INVALID_ARGUMENT),
    # beyond the kernels' index ranges
    (dict(B=40000), moda.MODA_ERR_UNSUPPORTED),                 # B*Hkv > 65535
    (dict(T=(1 << 30) + 16), moda.MODA_ERR_UNSUPPORTED),        # T > 2^30
    (dict(L=70000), moda.MODA_ERR_UNSUPPORTED),                 # L > 65535
    (dict(B=600, Hq=64, Hkv=64, T=1 << 16), moda.MODA_ERR_UNSUPPORTED),  # rows > 2^31
    (dict(lse=A * 64 + 64), moda.MODA_ERR_INVALID_ARGUMENT),    # lse overlaps out
])
def test_forward_rejects_bad_arguments_before_launch(kw, status):
    assert fwd(**kw) == status


@pytest.mark.parametrize("kw,path,status", [
    (dict(), 3, moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(), -1, moda.MODA_ERR_INVALID_ARGUMENT),
    (dict(Hq=6, Hkv=2), 2, moda.MODA_ERR_UNSUPPORTED),  # group of 3 does not divide 128
    (dict(Hq=128, Hkv=2), 2, moda.MODA_ERR_UNSUPPORTED),  # group of 64: beyond a warp's columns
    (dict(q=None), 2, moda.MODA_ERR_INVALID_ARGUMENT),
])
def test_forward_depth_path_rejects_bad_arguments(kw, path, status):
    args = dict(q=A, k=A * 2, v=A * 3, kd=A * 4, vd=A * 5, out=A * 64, lse=A * 128, B=1,
                Hq=4, Hkv=2, T=16, L=2, d=64, scale=0.125, causal=1, depth_path=path,
                stream=None)
    args.update(kw)
    assert moda.moda_forward_depth_path(**args) == status


def test_depth_attention_rejects_bad_arguments():
    f = dict(q=A, kd=A * 4, vd=A * 5, out=A * 64, lse=A * 128, B=1, Hq=4, Hkv=2, T=16, L=2,
             d=64, scale=0.125, stream=None)
    assert moda.moda_depth_attention_forward(**dict(f, L=0)) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_depth_attention_forward(**dict(f, kd=None)) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_depth_attention_forward(**dict(f, d=96)) == moda.MODA_ERR_UNSUPPORTED
    b = dict(q=A, kd=A * 4, vd=A * 5, out=A * 6, lse=A * 7, dout=A * 8, dq=A * 9, dkd=A * 12,
             dvd=A * 13, workspace=A * 64, workspace_bytes=1 << 20, B=1, Hq=4, Hkv=2, T=16,
             L=2, d=64, scale=0.125, stream=None)
    assert moda.moda_depth_attention_backward(**dict(b, L=0)) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_depth_attention_backward(**dict(b, dq=None)) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_depth_attention_backward(**dict(b, workspace_bytes=16)) == \
        moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_depth_attention_backward(**dict(b, dkd=A * 4)) == \
        moda.MODA_ERR_INVALID_ARGUMENT  # dkd aliases kd


def test_decode_rejects_bad_arguments():
    base = dict(q=A, k=A * 2, v=A * 3, kd=A * 4, vd=A * 5, out=A * 64, lse=A * 128,
                workspace=A * 256, workspace_bytes=1 << 24, B=1, Hq=4, Hkv=2, S=16, L=2, d=64,
                scale=0.125, stream=None)
    st = lambda **kw: moda.moda_decode(**dict(base, **kw))
    assert st(S=0) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(kd=None) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(workspace_bytes=16) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(workspace=A * 256 + 16) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(out=A * 2) == moda.MODA_ERR_INVALID_ARGUMENT  # out aliases k
    assert st(Hq=130, Hkv=1) == moda.MODA_ERR_UNSUPPORTED
    assert st(d=96) == moda.MODA_ERR_UNSUPPORTED
    assert moda.moda_decode_workspace_size(1, 16, 4, 65536, 32, 128) > 0
    assert moda.moda_decode_workspace_size(1, 130, 1, 100, 1, 128) == 0


def test_depth_kv_write_rejects_bad_arguments():
    base = dict(x=A, w=A * 2, kd=A * 64, vd=A * 128, B=1, T=16, hidden=64, Hkv=2, d=64, L=3,
                slot=1, stream=None)
    st = lambda **kw: moda.moda_depth_kv_write(**dict(base, **kw))
    assert st(slot=3) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(slot=-1) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(L=0) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(x=None) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(kd=A * 64 + 8) == moda.MODA_ERR_INVALID_ARGUMENT
    assert st(vd=A * 64 + 16) == moda.MODA_ERR_INVALID_ARGUMENT  # vd overlaps kd
    assert st(kd=A) == moda.MODA_ERR_INVALID_ARGUMENT            # kd overlaps x
    assert st(vd=A * 2) == moda.MODA_ERR_INVALID_ARGUMENT        # vd overlaps w
    assert st(d=96) == moda.MODA_ERR_UNSUPPORTED
    assert st(Hkv=1) == moda.MODA_ERR_UNSUPPORTED      # Hkv*d = 64
    assert st(hidden=60) == moda.MODA_ERR_UNSUPPORTED  # rows not 16-byte multiples
    assert st(B=1 << 16, T=1 << 15) == moda.MODA_ERR_UNSUPPORTED  # B*T = 2^31 tokens


def test_forward_L0_allows_null_depth():
    # With L = 0, NULL kd/vd pass the pointer checks: the call is refused only by the
    # later scale check.  A call with every argument valid would launch the kernel on
    # these fake pointers wherever a GPU is present, so no test here makes one.
    assert fwd(kd=None, vd=None) == moda.MODA_ERR_INVALID_ARGUMENT
    assert "kd and vd" in moda.moda_last_error_message()
    assert fwd(L=0, kd=None, vd=None, scale=float("nan")) == moda.MODA_ERR_INVALID_ARGUMENT
    assert "scale" in moda.moda_last_error_message()


def test_backward_workspace_size():
    B, Hq, Hkv, T, L, d = 1, 16, 4, 16384, 48, 128
    ws = moda.moda_backward_workspace_size(B, Hq, Hkv, T, L, d)
    assert ws >= B * Hq * T * d * 4 + B * Hq * T * 4
    assert moda.moda_backward_workspace_size(0, Hq, Hkv, T, L, d) == 0


def test_backward_rejects_small_workspace_and_aliasing():
    args = dict(q=A, k=A * 2, v=A * 3, kd=A * 4, vd=A * 5, out=A * 6, lse=A * 7, dout=A * 8,
                dq=A * 9, dk=A * 10, dv=A * 11, dkd=A * 12, vd_=None)
    args.pop("vd_")
    base = dict(dvd=A * 13, workspace=A * 64, workspace_bytes=1 << 20, B=1, Hq=4, Hkv=2,
                T=16, L=2, d=64, scale=0.125, causal=1, stream=None)
    st = moda.moda_backward(**args, **dict(base, workspace_bytes=16))
    assert st == moda.MODA_ERR_INVALID_ARGUMENT
    st = moda.moda_backward(**dict(args, dq=A * 2), **base)  # dq aliases k
    assert st == moda.MODA_ERR_INVALID_ARGUMENT
    st = moda.moda_backward(**args, **dict(base, workspace=A * 64 + 16))  # not 256-aligned
    assert st == moda.MODA_ERR_INVALID_ARGUMENT
    st = moda.moda_backward(**args, **dict(base, Hq=256, Hkv=2))  # group of 128 heads
    assert st == moda.MODA_ERR_UNSUPPORTED


@pytest.mark.parametrize("stages", [0, 8, 15])
def test_backward_stages_rejects_bad_masks(stages):
    args = [A * (i + 1) for i in range(13)] + [A * 64, 1 << 20, 1, 4, 2, 16, 2, 64, 0.125, 1,
                                               stages, None]
    assert moda.moda_backward_stages(*args) == moda.MODA_ERR_INVALID_ARGUMENT


def test_binding_has_no_fallback():
    src = open(os.path.join(ROOT, "depth_aware_attention_b200", "__init__.py")).read()
    assert "oracle" not in src.lower().replace("no cpu", "")


NOALLOC_LIMIT = 64 << 20  # bytes of the no-allocation backward's static scratch


def _noalloc(ptrs, B, Hq, Hkv, T, L, d, scale=0.088):
    return moda.moda_backward_noalloc(*[None if p is None else ctypes.c_void_p(p) for p in ptrs],
                                      B, Hq, Hkv, T, L, d, scale, 1, None)


def test_noalloc_rejects_sizes_beyond_its_scratch_before_touching_the_gpu():
    # 13 buffers 4 GiB apart, so that no size check sees an overlap.  The sizes must need
    # more workspace than the static scratch holds: the call is then refused by that check
    # and nothing is launched on the fake addresses.
    sizes = (1, 16, 4, 16384, 4, 128)
    assert moda.moda_backward_workspace_size(*sizes) > NOALLOC_LIMIT, \
        "these sizes must exceed the no-allocation scratch, or the call would launch"
    ptrs = [(i + 1) << 32 for i in range(13)]
    assert _noalloc(ptrs, *sizes) == moda.MODA_ERR_UNSUPPORTED
    assert "static scratch" in moda.moda_last_error_message()


def test_noalloc_rejects_bad_pointers_before_touching_the_gpu():
    sizes = (1, 4, 2, 64, 2, 64)
    ptrs = [A * (i + 1) for i in range(13)]
    assert _noalloc([None] + ptrs[1:], *sizes) == moda.MODA_ERR_INVALID_ARGUMENT
    assert _noalloc([A * 1 + 8] + ptrs[1:], *sizes) == moda.MODA_ERR_INVALID_ARGUMENT
    assert _noalloc(ptrs[:8] + [A * 2] + ptrs[9:], *sizes) == moda.MODA_ERR_INVALID_ARGUMENT
    assert _noalloc(ptrs, *sizes, scale=float("inf")) == moda.MODA_ERR_INVALID_ARGUMENT


def test_test_fault_knob_rejects_bad_values_before_touching_the_gpu():
    assert moda.moda_test_set_device_fault(2, 0) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_test_set_device_fault(-1, 0) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_test_set_device_fault(0, 5) == moda.MODA_ERR_INVALID_ARGUMENT
    assert moda.moda_test_set_device_fault(0, 20_000_000_000) == moda.MODA_ERR_INVALID_ARGUMENT
