"""The float64 exp used by the draft-logit row sums, checked on the host against math.exp (an
independent libm) within 2 ulp over the argument range the kernel sees, including the cutoff."""
import math
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc) and shutil.which("nvcc") is None:
        pytest.skip("nvcc not available")
    out = tmp_path_factory.mktemp("exp64") / "exp64_check"
    subprocess.run([nvcc, "-O2", "-x", "cu", os.path.join(HERE, "exp64_check.cu"), "-o", str(out)], check=True)
    return str(out)


def run(exe, xs):
    res = subprocess.run([exe], input="\n".join(repr(float(x)) for x in xs), capture_output=True, text=True,
                         check=True)
    return np.array([float(v) for v in res.stdout.split()])


def test_within_two_ulp(exe):
    rng = np.random.default_rng(0)
    xs = np.concatenate([-rng.exponential(5.0, 4000), -rng.uniform(0, 708, 4000), -rng.uniform(0, 1e-3, 500),
                         [0.0, -0.0, -1e-300, -0.34657359027997264, -0.3465735902799727, -707.9, -1.0, -2.0]])
    got = run(exe, xs)
    want = np.array([math.exp(x) for x in xs])
    ulp = np.abs(got - want) / np.spacing(want)
    assert ulp.max() <= 2.0, (ulp.max(), xs[ulp.argmax()])


def test_cutoff_and_specials(exe):
    got = run(exe, [-708.5, -1e6, float("-inf"), 0.0])
    assert got[0] == 0.0 and got[1] == 0.0 and got[2] == 0.0 and got[3] == 1.0
