import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    from oracle.oracle import Oracle
    return Oracle()


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def golden_two_tiles_weights(d):
    rows, cols = d["rows"], d["cols"]
    w = np.zeros((rows, cols), np.uint16)
    w[0, :] = int(d["fill"][0], 16)
    w[1, :] = int(d["fill"][1], 16)
    w[1, 1::2] = int(d["row1_odd"], 16)
    for r, c, v in d["overrides"]:
        w[r, c] = int(v, 16)
    return w


def golden_expected_bytes(d):
    out = np.zeros(d["total_bytes"], np.uint8)
    for item in d["nonzero_bytes"]:
        off, hexs = item[0], item[1]
        reps = item[2] if len(item) > 2 else 1
        chunk = bytes.fromhex(hexs) * reps
        out[off:off + len(chunk)] = np.frombuffer(chunk, np.uint8)
    return out


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True
