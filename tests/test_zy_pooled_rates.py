"""The exempt-code rate, pooled over every KroQuant-type parity case of the session.

The criterion bounds near-boundary code flips as a rate over all compared
codes (at most 1e-6 of them), so it is checked once over the sum of every case
that tests/parity_check.py counted in this process: the quantizers of every
workload at full size, the sampled full-size sweep launches, the LU form, the
fused normalisation, the tensor-core variant and the scale-factor-layout
writer.  This file is collected after the parity test files so that the pool
is complete when it runs.
"""
import json
import os

import pytest

import parity_check as pc

pytestmark = pytest.mark.gpu


def test_pooled_exempt_rate(cuda_device):
    v = pc.pooled_verdict()
    if v["cases"] == 0:
        pytest.skip("no KroQuant parity case ran in this session")
    print("\npooled KroQuant parity:", json.dumps(v))
    out = os.environ.get("KQ_PARITY_REPORT", "")
    if out:
        with open(out, "a") as fh:
            fh.write(json.dumps({"case": "pooled", **v}) + "\n")
    assert v["ok"], v
