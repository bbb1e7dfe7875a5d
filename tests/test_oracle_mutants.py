"""The oracle's pins catch plausible mistakes: each mutant below plants one in a copy of
the oracle (a dropped term, a wrong sign, a wrong index or scale, a transposed operand),
and the pin suite tests/test_oracle_pins.py must fail on it.

Each mutant is a copy of the ``oracle`` package with one exact text substitution, built
with its own gcc call and imported ahead of the real package in a subprocess that runs
the pins.  The unmutated copy must pass the same run first, so that a broken harness
cannot pass for a killed mutant.  Only CPU code is touched.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

C, PY = "moda_oracle.c", "__init__.py"

# (name, file, original text, planted mistake); each original occurs once in its file.
MUTANTS = [
    ("causal mask drops the diagonal", C,
     "return causal ? t + 1 : T;", "return causal ? t : T;"),
    ("sequence keys of the wrong KV group", C,
     "G = J->Hq / J->Hkv, g = h / G;\n    const int t = J->t0 + w;",
     "G = J->Hq / J->Hkv, g = h % J->Hkv;\n    const int t = J->t0 + w;"),
    ("depth logits not scaled", C,
     "scratch[ns + j] = J->scale * dot(qr, kdt", "scratch[ns + j] = dot(qr, kdt"),
    ("depth entries of the wrong token", C,
     "J->kd + dtok(J, b, g, w) * L * d : NULL;\n    const double *vdt = L ? J->vd + dtok(J, b, g, w)",
     "J->kd + dtok(J, b, g, 0) * L * d : NULL;\n    const double *vdt = L ? J->vd + dtok(J, b, g, 0)"),
    ("depth values dropped from the output", C,
     "const double *vr = vdt + (int64_t)j * d;\n        Z += p;\n"
     "        for (int c = 0; c < d; ++c) out_row[c] += p * vr[c];",
     "const double *vr = vdt + (int64_t)j * d;\n        Z += p;\n        (void)vr;"),
    ("depth keys dropped from the normaliser", C,
     "const double *vr = vdt + (int64_t)j * d;\n        Z += p;",
     "const double *vr = vdt + (int64_t)j * d;"),
    ("log-sum-exp without the max", C,
     "*lse_row = m + log(Z);", "*lse_row = log(Z);"),
    ("depth dS with the wrong sign", C,
     "const double dP = dot(dor, vdt + (int64_t)j * d, d);\n"
     "            const double dS = P * (dP - D);",
     "const double dP = dot(dor, vdt + (int64_t)j * d, d);\n"
     "            const double dS = P * (D - dP);"),
    ("sequence dk without the scale", C,
     "double *dkr = dkb + (int64_t)s * d, *dvr = dvb + (int64_t)s * d;\n"
     "            for (int c = 0; c < d; ++c) {\n"
     "                dqr[c] += J->scale * dS * kr[c];\n"
     "                dkr[c] += J->scale * dS * qr[c];",
     "double *dkr = dkb + (int64_t)s * d, *dvr = dvb + (int64_t)s * d;\n"
     "            for (int c = 0; c < d; ++c) {\n"
     "                dqr[c] += J->scale * dS * kr[c];\n"
     "                dkr[c] += dS * qr[c];"),
    ("dvd from q instead of dO", C,
     "*dvr = dvdt + (int64_t)j * d;\n"
     "            for (int c = 0; c < d; ++c) {\n"
     "                dqr[c] += J->scale * dS * kr[c];\n"
     "                dkr[c] += J->scale * dS * qr[c];\n"
     "                dvr[c] += P * dor[c];",
     "*dvr = dvdt + (int64_t)j * d;\n"
     "            for (int c = 0; c < d; ++c) {\n"
     "                dqr[c] += J->scale * dS * kr[c];\n"
     "                dkr[c] += J->scale * dS * qr[c];\n"
     "                dvr[c] += P * qr[c];"),
    ("dq misses the depth keys", C,
     "*dvr = dvdt + (int64_t)j * d;\n"
     "            for (int c = 0; c < d; ++c) {\n"
     "                dqr[c] += J->scale * dS * kr[c];",
     "*dvr = dvdt + (int64_t)j * d;\n"
     "            for (int c = 0; c < d; ++c) {\n"
     "            (void)kr;"),
    ("only one thread's key-gradient buffer summed", C,
     "for (int i = 0; i < nthreads; ++i)\n                    for (int64_t e = 0; e < n; ++e) {",
     "for (int i = 0; i < 1; ++i)\n                    for (int64_t e = 0; e < n; ++e) {"),
    ("row term D dropped", C,
     "const double D = dot(dor, J->out_given ? J->out_given + r * d : o_row, d);",
     "const double D = 0.0 * dot(dor, J->out_given ? J->out_given + r * d : o_row, d);"),
    ("K and V halves of the projection swapped", PY,
     "return np.ascontiguousarray(y[0]), np.ascontiguousarray(y[1])",
     "return np.ascontiguousarray(y[1]), np.ascontiguousarray(y[0])"),
    ("projection heads and halves transposed", PY,
     "y = y.reshape(B, T, 2, Hkv, d).transpose(2, 0, 3, 1, 4)",
     "y = y.reshape(B, T, Hkv, 2, d).transpose(3, 0, 2, 1, 4)"),
    ("forward window offset ignored", PY,
     "_ptr(out), _ptr(lse), B, Hq, Hkv, T, L, d, t0, nt,",
     "_ptr(out), _ptr(lse), B, Hq, Hkv, T, L, d, 0, nt,"),
]

RUNNER = """
import sys
sys.path.insert(0, sys.argv[1])
sys.path.insert(1, sys.argv[2])
import oracle
assert oracle.__file__.startswith(sys.argv[1]), oracle.__file__
import pytest
sys.exit(pytest.main([sys.argv[3], "-x", "-q", "-p", "no:cacheprovider"]))
"""


def _run_copy(tmp, name, mutation):
    """Copy the oracle package under tmp/<name>/, apply the mutation, run the pins.
    Returns (exit code, output tail)."""
    base = os.path.join(tmp, name)
    pkg = os.path.join(base, "oracle")
    os.makedirs(pkg)
    for f in (C, PY):
        shutil.copy(os.path.join(ROOT, "oracle", f), os.path.join(pkg, f))
    if mutation is not None:
        f, old, new = mutation
        path = os.path.join(pkg, f)
        src = open(path).read()
        assert src.count(old) == 1, f"{name}: the original text occurs {src.count(old)} times"
        open(path, "w").write(src.replace(old, new))
    r = subprocess.run([sys.executable, "-c", RUNNER, base, ROOT, PINS], cwd=base,
                       capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout + r.stderr)[-1500:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    tmp = str(tmp_path)
    rc, out = _run_copy(tmp, "unmutated", None)
    assert rc == 0, "the unmutated copy must pass the pins:\n" + out
    jobs = {}
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for i, (name, f, old, new) in enumerate(MUTANTS):
            jobs[name] = ex.submit(_run_copy, tmp, f"m{i}", (f, old, new))
    survived = []
    for name, job in jobs.items():
        rc, out = job.result()
        # pytest exits 1 when a test failed; anything else (0: all pins passed, a crash,
        # a collection error) is not a pin catching the mistake
        if rc != 1:
            survived.append(f"{name} (exit {rc}):\n{out}")
    assert not survived, "mutants the pins did not catch:\n" + "\n".join(survived)
