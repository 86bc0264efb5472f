import os
import sys
from fractions import Fraction

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def _ensure_built():
    """Build libbitlinear.so and the oracle if they are missing or stale."""
    from ternary_weight_bitlinear_b200 import build as lib_build
    from oracle import build as oracle_build
    lib_build.build()
    oracle_build.build()


def pytest_configure(config):
    _ensure_built()
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size oracle work)")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def load_golden(name):
    """Parse a tests/golden/*.txt fixture: 'key v1 v2 ...' lines, '#' comments."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def parse_float(s):
    return float.fromhex(s) if "0x" in s else float(s)


def rn32_of_fraction(fr):
    """Correctly rounded binary32 value of an exact rational (ties to even).

    Independent of the oracle: picks, among the binary32 neighbours of the
    rational, the nearest one by exact Fraction comparison.
    """
    fr = Fraction(fr)
    if fr == 0:
        return np.float32(0.0)
    guess = np.float32(float(fr))
    cands = {guess, np.nextafter(guess, np.float32(np.inf)),
             np.nextafter(guess, np.float32(-np.inf))}
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - fr)
        if best is None or d < best[0] or (d == best[0] and
                                           (np.float32(c).view(np.uint32) & 1) == 0):
            best = (d, c)
    return np.float32(best[1])


@pytest.fixture(scope="session")
def O():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture
def guard():
    """Guarded device buffers (see gpu_util.Guard); checked after the test."""
    from gpu_util import Guard
    g = Guard()
    yield g
    g.check()
