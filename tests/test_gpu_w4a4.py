"""The W4A4 consumer against the oracle: scales in the tensor core's
scale-factor layout, the fp32-input MXFP4 quantizer, and the block-scaled
tcgen05 product D = A B^T over MXFP4 operands.

Criteria:
- layouts, codes and scale bytes are integer work: bit-exact (the whole
  scale-factor buffer is compared, pre-filled with 0xFF, so a stray write
  fails);
- the product: the tensor core multiplies exactly and accumulates in fp32 in
  some order, so |D_gpu - D| <= K * 2^-23 * sum_k |a_k b_k| (the bound of any
  fp32 summation of K terms, with a rounding unit of 2^-23 that also covers
  truncating adds); bf16 output adds its rounding to nearest, at most 2^-8
  (bf16's unit roundoff: 8 significant bits) of the fp32 value.
"""
import numpy as np
import pytest

import oracle
import parity_check as pc
import w4a4_mxfp4_post_b200 as kq
from w4a4_mxfp4_post_b200 import synth

pytestmark = pytest.mark.gpu


def dev(a, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def dev_bf16(bits, device):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def sf_buffer(rows, d, device):
    import torch

    return torch.full((kq.kq_sf_bytes(rows, d),), 0xFF, dtype=torch.uint8, device=device)


def gather_rowmajor(sf, rows, nb):
    """Row-major scales read back out of a scale-factor buffer (oracle layout)."""
    r = np.arange(rows)[:, None]
    j = np.arange(nb)[None, :]
    ka = (nb + 3) // 4
    off = ((r // 128) * ka + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)
    assert oracle.sf_offset(rows - 1, nb - 1, nb) == off[-1, -1]
    return sf[off]


def check_gemm(Dg, D, absd, K, bf16_out):
    """The per-element fp32-summation bound and, for fp32 output, the rms
    statistic (tests/parity_check.py)."""
    res = pc.check_gemm(Dg, D, absd, K, bf16_out)
    assert res["ok"], res
    return res["worst"]


# -- scale-factor-layout writers ------------------------------------------------------
SF_CASES = [(64, 128, "tiny", False, 0), (300, 1152, "pixart", False, 1), (200, 5600, "sana", True, 2),
            (129, 96, "tiny", False, 3)]


@pytest.mark.parametrize("M,d,model,shared,seed", SF_CASES, ids=[f"{c[0]}x{c[1]}" for c in SF_CASES])
def test_kq_quantize_sf_matches_oracle_and_row_major_kernel(cuda_device, M, d, model, shared, seed):
    x = synth.activation(model, M, d, seed)
    F = synth.factors(d // 32, seed, shared=shared)
    xd, Fd = dev_bf16(x, cuda_device), dev(F, cuda_device)
    codes = kq.kq_quantize_sf(xd, Fd, shared=shared, out_sf=sf_buffer(M, d, cuda_device))
    cg, sfg = codes[0].cpu().numpy(), codes[1].cpu().numpy()
    # the oracle: codes and scales within the quantizer's criteria
    cr, sr = oracle.kq_quantize(x, F, shared=shared)
    yr, ab = oracle.kq_transform(x, F, shared=shared, want_absbound=True)
    res = pc.check_kq(cg, gather_rowmajor(sfg, M, d // 32), cr, sr, yr, ab)
    assert res["ok"], res
    # the same arithmetic as kq_quantize: codes identical, scales relaid exactly
    c2, s2 = (kq.kq_quantize_shared if shared else kq.kq_quantize)(xd, Fd)
    np.testing.assert_array_equal(cg, c2.cpu().numpy())
    np.testing.assert_array_equal(sfg, oracle.scales_to_sf(s2.cpu().numpy()))


@pytest.mark.parametrize("M,d", [(1, 32), (130, 96), (257, 5600), (64, 1152)])
def test_mx_scales_to_sf_is_the_oracle_layout(cuda_device, M, d):
    _, sc = synth.mx_operand(M, d, 11)
    out = kq.mx_scales_to_sf(dev(sc, cuda_device), out_sf=sf_buffer(M, d, cuda_device)).cpu().numpy()
    np.testing.assert_array_equal(out, oracle.scales_to_sf(sc))


@pytest.mark.parametrize("M,d", [(64, 128), (257, 1152), (33, 96)])
def test_mx_quantize_f32_bit_exact(cuda_device, M, d):
    W = synth.weights(M, d, 4)
    W[0, :32] = 0.0                             # an all-zero block
    W[1, 5] = -0.0
    W[2, :32] *= 1e-40                          # subnormal block amax
    Wd = dev(W, cuda_device)
    cr, sr = oracle.mx_quantize_f32(W)
    c, s = kq.mx_quantize_f32(Wd)
    np.testing.assert_array_equal(c.cpu().numpy(), cr)
    np.testing.assert_array_equal(s.cpu().numpy(), sr)
    c2, sf = kq.mx_quantize_f32(Wd, sf_layout=True, out_scales=sf_buffer(M, d, cuda_device))
    np.testing.assert_array_equal(c2.cpu().numpy(), cr)
    np.testing.assert_array_equal(sf.cpu().numpy(), oracle.scales_to_sf(sr))


# -- the product ----------------------------------------------------------------------
GEMM_CASES = [(1, 8, 32), (128, 256, 64), (300, 520, 1152), (200, 264, 2240), (77, 136, 5600), (513, 1032, 256)]


@pytest.mark.parametrize("M,N,K", GEMM_CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}" for c in GEMM_CASES])
@pytest.mark.parametrize("f32", [True, False], ids=["f32", "bf16"])
def test_mxf4_gemm_random_operands(cuda_device, M, N, K, f32):
    import torch

    ca, sa = synth.mx_operand(M, K, 21)
    cb, sb = synth.mx_operand(N, K, 22)
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    out = kq.mxf4_gemm(dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device), dev(cb, cuda_device),
                       dev(oracle.scales_to_sf(sb), cuda_device),
                       out_dtype=torch.float32 if f32 else torch.bfloat16)
    check_gemm(out.float().cpu().numpy(), D, absd, K, not f32)
    assert kq.kq_wait_timeouts() == 0


# The SM-pair forms (cta_group::2): 256 x 256 and 256 x 192 tiles.  Cases add
# to the above: more tiles than SM pairs (every pair walks several tiles, both
# accumulators cycle), a 256-row tile whose second CTA is past M, 192-column
# tiles starting in the middle of a scale unit, K of one chunk and ragged K.
PAIR_FORMS = (7, 8)
PAIR_CASES = GEMM_CASES + [(2100, 3000, 192), (520, 1160, 640), (4096, 4608, 128)]


@pytest.mark.parametrize("variant", PAIR_FORMS)
@pytest.mark.parametrize("M,N,K", PAIR_CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}" for c in PAIR_CASES])
@pytest.mark.parametrize("f32", [True, False], ids=["f32", "bf16"])
def test_mxf4_gemm_sm_pair_forms(cuda_device, M, N, K, f32, variant):
    import torch

    ca, sa = synth.mx_operand(M, K, 23)
    cb, sb = synth.mx_operand(N, K, 24)
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    kq.kq_wait_timeouts(reset=True)
    out = kq.mxf4_gemm_variant(variant, dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device),
                               dev(cb, cuda_device), dev(oracle.scales_to_sf(sb), cuda_device),
                               out_dtype=torch.float32 if f32 else torch.bfloat16)
    assert kq.kq_wait_timeouts() == 0
    check_gemm(out.float().cpu().numpy(), D, absd, K, not f32)


@pytest.mark.parametrize("M,N,K", [(300, 520, 1152), (77, 136, 5600), (256, 264, 96)])
def test_mxf4_gemm_configurations_agree(cuda_device, M, N, K):
    """Every tile configuration gives the same bits (same K order), and the
    oracle's bound holds for each."""
    import torch

    ca, sa = synth.mx_operand(M, K, 51)
    cb, sb = synth.mx_operand(N, K, 52)
    args = [dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device), dev(cb, cuda_device),
            dev(oracle.scales_to_sf(sb), cuda_device)]
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    for dtype in (torch.float32, torch.bfloat16):
        ref = kq.mxf4_gemm_variant(1, *args, out_dtype=dtype)
        check_gemm(ref.float().cpu().numpy(), D, absd, K, dtype == torch.bfloat16)
        for v in (0, 2, 3, 4, 5, 6) + PAIR_FORMS:
            got = kq.mxf4_gemm_variant(v, *args, out_dtype=dtype)
            assert torch.equal(got, ref), (v, dtype)


def test_mxf4_gemm_repeated_calls_and_other_stream(cuda_device):
    import torch

    M, N, K = 260, 512, 1152
    ca, sa = synth.mx_operand(M, K, 31)
    cb, sb = synth.mx_operand(N, K, 32)
    args = [dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device), dev(cb, cuda_device),
            dev(oracle.scales_to_sf(sb), cuda_device)]
    first = kq.mxf4_gemm(*args, out_dtype=torch.float32)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        second = kq.mxf4_gemm(*args, out_dtype=torch.float32)
    s.synchronize()
    assert torch.equal(first, second)        # deterministic: same order of accumulation


def hadamard_factors(nb):
    s = np.float32(1.0 / np.sqrt(2.0))
    return np.tile(np.array([[s, s], [s, -s]], np.float32), (nb, 5, 1, 1))


def test_w4a4_chain_on_oracle_operands(cuda_device):
    """Activation quantized by KroQuant and weights folded and quantized (all by
    the oracle), multiplied on the tensor cores, against the oracle product.
    Then, on the oracle alone, that the chain computes X W^T: with Hadamard
    factors it is closer to X W^T than plain MXFP4 on both operands, and
    leaving the fold out makes it far worse."""
    import torch

    M, N, d, seed = 256, 384, 1152, 1
    x = synth.activation("pixart", M, d, seed)
    W = synth.weights(N, d, seed)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ W.astype(np.float64).T
    rel = {}
    for name, F in (("random", synth.factors(d // 32, seed)), ("hadamard", hadamard_factors(d // 32))):
        ca, sa = oracle.kq_quantize(x, F)
        cb, sb = oracle.mx_quantize_f32(oracle.fold_weights(W, F))
        D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
        out = kq.mxf4_gemm(dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device), dev(cb, cuda_device),
                           dev(oracle.scales_to_sf(sb), cuda_device), out_dtype=torch.float32).cpu().numpy()
        check_gemm(out, D, absd, d, False)
        rel[name] = np.linalg.norm(D - ref) / np.linalg.norm(ref)
        if name == "hadamard":
            cbu, sbu = oracle.mx_quantize_f32(W)            # the fold left out
            Du = oracle.mxf4_gemm(ca, sa, cbu, sbu)
            rel["unfolded"] = np.linalg.norm(Du - ref) / np.linalg.norm(ref)
    cam, sam = oracle.mx_quantize(x)
    cbm, sbm = oracle.mx_quantize_f32(W)
    rel["mx"] = np.linalg.norm(oracle.mxf4_gemm(cam, sam, cbm, sbm) - ref) / np.linalg.norm(ref)
    assert rel["hadamard"] < rel["mx"], rel
    assert rel["unfolded"] > 0.9 and rel["hadamard"] < 0.5 * rel["unfolded"], rel


@pytest.mark.parametrize("variant", (0,) + PAIR_FORMS)
@pytest.mark.parametrize("N,K", synth.GEMM_LAYERS["pixart_mlp"]["layers"])
def test_mxf4_gemm_full_size_sampled_rows(cuda_device, N, K, variant):
    """The benchmark's launch (8192 tokens, PixArt-Sigma MLP layer), checked on
    sampled rows: head, tail and random rows of every row tile class."""
    import torch

    M = synth.GEMM_LAYERS["pixart_mlp"]["M"]
    ca, sa = synth.mx_operand(M, K, 41)
    cb, sb = synth.mx_operand(N, K, 42)
    out = kq.mxf4_gemm_variant(variant, dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device),
                               dev(cb, cuda_device), dev(oracle.scales_to_sf(sb), cuda_device))
    rng = np.random.default_rng(N + K)
    rows = np.unique(np.concatenate([np.arange(8), np.arange(M - 8, M), rng.choice(M, 24, replace=False)]))
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, rows=rows, want_absbound=True)
    got = out.index_select(0, torch.from_numpy(rows).to(cuda_device)).float().cpu().numpy()
    check_gemm(got, D, absd, K, True)


@pytest.mark.parametrize("variant", (0, 7))
def test_mxf4_gemm_extreme_scale_exponents(cuda_device, variant):
    """Scale bytes at both ends of E8M0: A at 2^127 (0xFE) and 2^126, B at
    2^-127 (0x00) and 2^-126, so every product is of order one; the tensor
    core must apply both exponents exactly (oracle bound as above)."""
    import torch

    M, N, K = 130, 136, 320
    ca, _ = synth.mx_operand(M, K, 61)
    cb, _ = synth.mx_operand(N, K, 62)
    rng = np.random.default_rng(63)
    sa = rng.choice(np.array([0xFE, 0xFD], np.uint8), size=(M, K // 32))
    sb = rng.choice(np.array([0x00, 0x01], np.uint8), size=(N, K // 32))
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    out = kq.mxf4_gemm_variant(variant, dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device),
                               dev(cb, cuda_device), dev(oracle.scales_to_sf(sb), cuda_device), out_dtype=torch.float32)
    assert np.all(np.isfinite(D))
    check_gemm(out.cpu().numpy(), D, absd, K, False)


@pytest.mark.parametrize("variant", (0, 7))
def test_mxf4_gemm_nan_scale_reaches_only_its_row(cuda_device, variant):
    """A scale byte 0xFF (E8M0 NaN) in one row of A makes exactly that output
    row NaN (the header's stated behaviour); every other row is unaffected."""
    import torch

    M, N, K = 96, 64, 256
    ca, sa = synth.mx_operand(M, K, 71)
    cb, sb = synth.mx_operand(N, K, 72)
    sa = sa.copy()
    sa[5, 3] = 0xFF
    D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
    out = kq.mxf4_gemm_variant(variant, dev(ca, cuda_device), dev(oracle.scales_to_sf(sa), cuda_device),
                               dev(cb, cuda_device), dev(oracle.scales_to_sf(sb), cuda_device),
                               out_dtype=torch.float32).cpu().numpy()
    assert np.all(np.isnan(out[5])) and np.all(np.isnan(D[5]))
    keep = np.arange(M) != 5
    assert np.all(np.isfinite(out[keep]))
    check_gemm(out[keep], D[keep], absd[keep], K, False)


def test_back_to_back_launches_see_their_producers_writes(cuda_device):
    """Every launch allows programmatic dependent launch, and every kernel waits
    for its predecessor's writes before it touches memory.  Fold -> quantize the
    weights -> quantize the activation -> product, on one stream with no
    synchronisation, three times into the same code and scale buffers (which
    start out holding other bytes): each product must be the oracle's product of
    the codes its own quantizer wrote, so a kernel that read early, or a
    quantizer that overwrote codes the previous product still needed, fails."""
    import torch

    M, N, d = 520, 392, 1152
    F = synth.factors(d // 32, 8)
    Fd = dev(F, cuda_device)
    codes = torch.full((M, d // 2), 0x77, dtype=torch.uint8, device=cuda_device)
    sf = torch.full((kq.kq_sf_bytes(M, d),), 0x7F, dtype=torch.uint8, device=cuda_device)
    wcodes = torch.full((N, d // 2), 0x77, dtype=torch.uint8, device=cuda_device)
    wsf = torch.full((kq.kq_sf_bytes(N, d),), 0x7F, dtype=torch.uint8, device=cuda_device)
    xs = [synth.activation("pixart", M, d, seed) for seed in range(3)]
    Ws = [synth.weights(N, d, 10 + seed) for seed in range(3)]
    xds = [dev_bf16(x, cuda_device) for x in xs]
    Wds = [dev(W, cuda_device) for W in Ws]
    torch.cuda.synchronize()
    outs = []
    for xd, Wd in zip(xds, Wds):
        kq.mx_quantize_f32(kq.kq_fold_weights(Wd, Fd), sf_layout=True, out_codes=wcodes, out_scales=wsf)
        kq.kq_quantize_sf(xd, Fd, out_codes=codes, out_sf=sf)
        outs.append(kq.mxf4_gemm(codes, sf, wcodes, wsf, out_dtype=torch.float32))
    torch.cuda.synchronize()
    for xd, Wd, out in zip(xds, Wds, outs):
        # the same (deterministic) kernels once more, one at a time
        wc, ws = kq.mx_quantize_f32(kq.kq_fold_weights(Wd, Fd), sf_layout=True)
        c, s = kq.kq_quantize_sf(xd, Fd)
        torch.cuda.synchronize()
        ca, cb = c.cpu().numpy(), wc.cpu().numpy()
        sa = gather_rowmajor(s.cpu().numpy(), M, d // 32)
        sb = gather_rowmajor(ws.cpu().numpy(), N, d // 32)
        D, absd = oracle.mxf4_gemm(ca, sa, cb, sb, want_absbound=True)
        check_gemm(out.cpu().numpy(), D, absd, d, False)
    assert kq.kq_wait_timeouts() == 0
