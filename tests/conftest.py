import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def read_golden(name):
    """Parse a `key = value` fixture under tests/golden (comments start with #)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line or "=" not in line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            out[key] = val
    return out


def parse_numbers(val):
    """'0x4F 0x98' / '1.75 -1' / '0x88 x62' -> list of numbers."""
    toks = val.split()
    res = []
    i = 0
    while i < len(toks):
        t = toks[i]
        if t.startswith("x") and res:
            res.extend([res[-1]] * (int(t[1:]) - 1))
        elif t.lower().startswith(("0x", "-0x")):
            res.append(int(t, 16))
        else:
            res.append(float(t) if any(c in t for c in ".eE") else int(t))
        i += 1
    return res


@pytest.fixture
def golden():
    return read_golden
