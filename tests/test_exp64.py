"""The float64 exp used by the draft-logit row sums, checked on the host against math.exp (an
independent libm) over the argument range the kernel sees, including the cutoff, and its table of
2^(j/128) against exact decimal arithmetic.  The bound is 1e-14 relative: the row sums only need to keep
the tree's float64 keys within far less than the 1e-9 decision margins the build tests guard.  At and below
the cutoff (-709, where 2^k reaches 2^-1023) the result is a subnormal below 2.3e-308 rather than 0: next to the
row maximum's exact 1 such a term changes no double-precision sum."""
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


def run(exe, xs, args=()):
    res = subprocess.run([exe, *args], input="\n".join(repr(float(x)) for x in xs), capture_output=True,
                         text=True, check=True)
    return np.array([float(v) for v in res.stdout.split()])


def test_within_1e14_relative(exe):
    rng = np.random.default_rng(0)
    xs = np.concatenate([-rng.exponential(5.0, 4000), -rng.uniform(0, 708, 4000), -rng.uniform(0, 1e-3, 500),
                         [0.0, -0.0, -1e-300, -0.34657359027997264, -0.3465735902799727, -707.9, -1.0, -2.0]])
    got = run(exe, xs)
    want = np.array([math.exp(x) for x in xs])
    rel = np.abs(got - want) / want
    assert rel.max() <= 1e-14, (rel.max(), xs[rel.argmax()])


def test_cutoff_and_specials(exe):
    got = run(exe, [-709.5, -1e6, float("-inf"), float("nan"), 0.0, -708.0])
    assert all(0.0 <= g < 2.3e-308 for g in got[:4]), got[:4]
    assert got[4] == 1.0
    assert abs(got[5] - math.exp(-708.0)) <= 1e-14 * math.exp(-708.0)
    # next to a row maximum's 1, a term at the cutoff leaves the sum unchanged
    assert 1.0 + got[0] == 1.0


def test_table_is_correctly_rounded(exe):
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    res = subprocess.run([exe, "table"], capture_output=True, text=True, check=True)
    tab = [float.fromhex(v) for v in res.stdout.split()]
    assert len(tab) == 128
    for j, d in enumerate(tab):
        exact = Decimal(2) ** (Decimal(j) / Decimal(128))
        err = abs(Decimal(d) - exact)
        # no neighbouring double is closer
        assert err <= abs(Decimal(math.nextafter(d, 0.0)) - exact), j
        assert err <= abs(Decimal(math.nextafter(d, 4.0)) - exact), j
