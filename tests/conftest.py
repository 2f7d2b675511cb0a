import os
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


GOLDEN = Path(__file__).resolve().parent / "golden"


def read_golden(name):
    """Parse a `key = value` fixture; repeated `value k = v` lines become a dict."""
    kv, values = {}, {}
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = [s.strip() for s in line.split("=", 1)]
        if key.startswith("value "):
            values[int(key.split()[1])] = float(val)
        else:
            kv[key] = val
    kv["values"] = values
    return kv
