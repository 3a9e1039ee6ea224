"""CUDA path vs CPU oracle, element by element, on every workload.

The CUDA calls go through the C ABI (ctypes binding); the oracle is the plain
C implementation under oracle/.  Both are fed the same seeded inputs from
w4a4_mxfp4_post_b200.synth.  Criteria: tests/parity_check.py.
"""
import json
import os

import numpy as np
import pytest

import oracle
import parity_check as pc
import w4a4_mxfp4_post_b200 as kq
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu

OUT = os.environ.get("KQ_PARITY_REPORT", "")


def report(name, res):
    if OUT:
        with open(OUT, "a") as fh:
            fh.write(json.dumps({"case": name, **res}) + "\n")


def dev_bf16(bits, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def dev_f32(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def run_gpu_kq(x_dev, F_dev, shared):
    if shared:
        c, s = kq.kq_quantize_shared(x_dev, F_dev)
    else:
        c, s = kq.kq_quantize(x_dev, F_dev)
    return c.cpu().numpy(), s.cpu().numpy()


def layer_inputs(M, d, model, shared, seed, rows=None):
    x = synth.activation(model, M, d, seed, rows=rows)
    F = synth.factors(d // 32, seed, shared=shared)
    return x, F


FULL_CASES = [(M, d, model, shared, seed) for name in ("tiny", "pixart", "sana", "flux")
              for (M, d, model, shared, seed) in synth.workload_layers(name)]


@pytest.mark.parametrize("M,d,model,shared,seed", FULL_CASES,
                         ids=[f"{c[2]}-{c[0]}x{c[1]}" for c in FULL_CASES])
def test_kq_sq_mx_full(cuda_device, M, d, model, shared, seed):
    x, F = layer_inputs(M, d, model, shared, seed)
    xd = dev_bf16(x, cuda_device)
    Fd = dev_f32(F, cuda_device)
    # KroQuant
    cg, sg = run_gpu_kq(xd, Fd, shared)
    cr, sr = oracle.kq_quantize(x, F, shared=shared)
    yr, ab = oracle.kq_transform(x, F, shared=shared, want_absbound=True)
    res = pc.check_kq(cg, sg, cr, sr, yr, ab)
    report(f"kq-{model}-{M}x{d}", res)
    assert res["ok"], res
    # fp32 transform
    yg = kq.kq_transform_f32(xd, Fd, shared=shared).cpu().numpy()
    tr = pc.check_transform(yg, yr, ab)
    report(f"transform-{model}-{M}x{d}", tr)
    assert tr["bad"] == 0, tr
    del yr, ab, yg
    # SmoothQuant and plain MX: bit-exact
    m = synth.sq_multipliers(x)
    c, s = kq.sq_quantize(xd, dev_f32(m, cuda_device))
    r = pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *oracle.sq_quantize(x, m))
    report(f"sq-{model}-{M}x{d}", r)
    assert r["ok"], r
    c, s = kq.mx_quantize(xd)
    r = pc.check_exact(c.cpu().numpy(), s.cpu().numpy(), *oracle.mx_quantize(x))
    report(f"mx-{model}-{M}x{d}", r)
    assert r["ok"], r
    assert kq.kq_wait_timeouts() == 0       # no bounded wait gave up on the normal path


SWEEP = [(M, d) for M in synth.WORKLOADS["sweep"]["Ms"] for d in synth.WORKLOADS["sweep"]["ds"]]


def sample_rows(M, rng):
    """Rows the oracle recomputes at full size: head, tail (ragged end) and random rows."""
    if M <= 4096:
        return np.arange(M)
    pick = np.concatenate([np.arange(64), np.arange(M - 64, M), rng.choice(M, 128, replace=False)])
    return np.unique(pick)


@pytest.mark.parametrize("M,d", SWEEP, ids=[f"{M}x{d}" for M, d in SWEEP])
def test_sweep_kq_sampled(cuda_device, M, d):
    """Full-size launches (the benchmark's configuration); the oracle checks sampled rows."""
    import torch

    seed = synth.WORKLOADS["sweep"]["seed"]
    x = synth.activation("pixart", M, d, seed)
    F = synth.factors(d // 32, seed)
    xd = dev_bf16(x, cuda_device)
    Fd = dev_f32(F, cuda_device)
    c, s = kq.kq_quantize(xd, Fd)
    rows = sample_rows(M, np.random.default_rng(M + d))
    idx = torch.from_numpy(rows).to(cuda_device)
    cg = c.index_select(0, idx).cpu().numpy()
    sg = s.index_select(0, idx).cpu().numpy()
    xs = x[rows]
    cr, sr = oracle.kq_quantize(xs, F)
    yr, ab = oracle.kq_transform(xs, F, want_absbound=True)
    res = pc.check_kq(cg, sg, cr, sr, yr, ab)
    res["rows_checked"] = int(rows.size)
    report(f"kq-sweep-{M}x{d}", res)
    assert res["ok"], res
    # the baselines at the same size, same rows
    m = synth.sq_multipliers(x)
    c2, s2 = kq.sq_quantize(xd, dev_f32(m, cuda_device))
    r = pc.check_exact(c2.index_select(0, idx).cpu().numpy(), s2.index_select(0, idx).cpu().numpy(),
                       *oracle.sq_quantize(xs, m))
    assert r["ok"], r
    c3, s3 = kq.mx_quantize(xd)
    r = pc.check_exact(c3.index_select(0, idx).cpu().numpy(), s3.index_select(0, idx).cpu().numpy(),
                       *oracle.mx_quantize(xs))
    assert r["ok"], r


def test_fold_weights_and_product_identity(cuda_device):
    import torch

    M, N, d = 64, 64, 128
    x = synth.activation("tiny", M, d, 0)
    W = synth.weights(N, d, 0)
    F = synth.factors(d // 32, 0)
    Wd, Fd = dev_f32(W, cuda_device), dev_f32(F, cuda_device)
    Wf = kq.kq_fold_weights(Wd, Fd).cpu().numpy()
    Wr, abw = oracle.fold_weights(W, F, want_absbound=True)
    err = np.abs(Wf.astype(np.float64) - Wr)
    assert np.all(err <= pc.REL * abw + 1e-37), float(np.max(err / abw))
    # X W^T == (X T^T)(W T^-1)^T in fp32 on the GPU (TF32 off)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        xd = dev_bf16(x, cuda_device)
        Y = kq.kq_transform_f32(xd, Fd)
        lhs = xd.float() @ Wd.T
        rhs = Y @ torch.from_numpy(Wf).to(cuda_device).T
        rel = float((lhs - rhs).abs().max() / lhs.abs().max())
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    report("fold-identity-64x128", {"max_rel": rel})
    assert rel <= 1e-4, rel
    # shared mode
    F1 = synth.factors(1, 0, shared=True)
    Wf1 = kq.kq_fold_weights(Wd, dev_f32(F1, cuda_device), shared=True).cpu().numpy()
    Wr1, abw1 = oracle.fold_weights(W, F1, shared=True, want_absbound=True)
    assert np.all(np.abs(Wf1.astype(np.float64) - Wr1) <= pc.REL * abw1 + 1e-37)
