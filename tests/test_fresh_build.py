"""__graft_entry__.build() works on a checkout that holds no built library (CPU only).

The sources are copied without any .so into a temporary directory, and build() runs
there in a fresh interpreter: nvcc cross-compiles the sm_100a library, gcc the oracle,
and the binding then imports.  (The binding refuses to import without its library, so a
build step that imported the package first could never bootstrap.)
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_build_from_sources_alone(tmp_path):
    dst = tmp_path / "repo"
    ignore = shutil.ignore_patterns("*.so", "*.so.tmp*", "__pycache__")
    for d in ("depth_aware_attention_b200", "include", "oracle"):
        shutil.copytree(os.path.join(ROOT, d), dst / d, ignore=ignore)
    for f in ("__graft_entry__.py", "workloads.py"):
        shutil.copy(os.path.join(ROOT, f), dst / f)
    assert not list(dst.rglob("*.so"))
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    r = subprocess.run([sys.executable, "-c", "import __graft_entry__ as g; g.build()"],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    assert (dst / "depth_aware_attention_b200" / "libmoda_b200.so").exists()
    assert (dst / "oracle" / "libmoda_oracle.so").exists()
