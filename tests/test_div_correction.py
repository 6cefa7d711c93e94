"""The packed quantizer routes take fl32(v / s) as y0 = fl32(v rs) plus one
fma correction (Markstein's theorem) instead of a division; this checks the
identity on the host in binary32 arithmetic (C, fmaf): every binary16 input
significand against a strided sweep of the scale significands, and random
binary32 significands.  SSMQ_FULL_DIVCHECK=1 sweeps every scale significand
(2^34 pairs per mode, about a minute on 8 cores)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("divcheck") / "div_correction_check")
    src = os.path.join(HERE, "div_correction_check.c")
    base = [cc, "-O2", "-ffp-contract=off", src, "-o", exe, "-lm"]
    try:
        subprocess.run(base[:1] + ["-fopenmp"] + base[1:], check=True, capture_output=True)
    except subprocess.CalledProcessError:
        subprocess.run(base, check=True, capture_output=True)
    return exe


@pytest.mark.parametrize("mode", [0, 1])
def test_division_correction_is_correctly_rounded(checker, mode):
    stride = 1 if os.environ.get("SSMQ_FULL_DIVCHECK") == "1" else 97
    r = subprocess.run([checker, str(mode), str(stride)], capture_output=True, text=True,
                       timeout=1800)
    pairs, mism = (int(t) for t in r.stdout.split()[1::2])
    assert pairs >= 2048 * ((1 << 23) // stride)
    assert mism == 0 and r.returncode == 0, r.stdout
