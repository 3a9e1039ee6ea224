"""Shared test setup: the `gpu` marker, import paths, golden-file parsing."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a); calls the CUDA path")


@pytest.fixture(scope="session")
def cuda_device():
    """The first CUDA device, with the library built; skips where there is no GPU."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4a4_mxfp4_post_b200 import build

    build.build()
    torch.cuda.init()
    return torch.device("cuda:0")


def parse_blocks(path):
    """Cases of a hand_blocks-style golden file: name, factors, x, scale, codes."""
    cases = []
    cur = None
    with open(path) as fh:
        for raw in fh:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            val = val.strip()
            if key == "case":
                cur = {"name": val}
                cases.append(cur)
            elif key == "factors":
                cur["factors"] = np.array([float(t) for t in val.split()], np.float32).reshape(1, 5, 2, 2)
            elif key == "x":
                cur["x"] = np.array([float(t) for t in val.split()], np.float32).reshape(1, 32)
            elif key == "scale":
                cur["scale"] = int(val, 16)
            elif key == "codes":
                cur["codes"] = np.array([int(t, 16) for t in val.split()], np.uint8)
            else:
                raise ValueError(f"bad golden line: {raw!r}")
    for c in cases:
        assert c["factors"].size == 20 and c["x"].size == 32 and c["codes"].size == 16, c["name"]
    return cases
