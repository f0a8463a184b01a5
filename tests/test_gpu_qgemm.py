"""GPU parity: wush_qgemm (tcgen05 block-scaled FP4 GEMM) against the oracle.

Two kinds of check: the GEMM alone on seeded random codes and scales (inputs
that never pass through the CUDA path), and the whole layer end to end
(transform + quantise + GEMM) against the oracle's layer.  The bar is a
relative Frobenius error <= 1e-3 on fp32 output.
"""
import numpy as np
import pytest

import synth
from oracle import calibrate as C
from oracle import formats as F
from oracle import gemm as G
from oracle import quant as Q
from oracle import transforms as T
from tests import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _random_operand(seed, rows, k, fmt):
    """Seeded random codes + scales: (packed codes, scale buffer, dequantised fp64)."""
    u = synth.uniform(seed, rows * k + rows * k // 16).astype(np.float64)
    codes = (u[: rows * k] * 16).astype(np.uint8).reshape(rows, k)
    v = F.e2m1_value(codes)
    b = 32 if fmt == "mxfp4" else 16
    su = u[rows * k: rows * k + rows * (k // b)].reshape(rows, k // b)
    if fmt == "mxfp4":
        sb = (120 + (su * 14).astype(np.int64)).astype(np.uint8)          # 2^-7 .. 2^6
        sv = F.e8m0_value(sb)
    else:
        sb = (0x28 + (su * 0x30).astype(np.int64)).astype(np.uint8)       # UE4M3 0.03 .. 30
        sv = F.e4m3_value(sb)
    dq = v * np.repeat(sv, b, axis=1)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, P.swizzle_scales(sb), dq


def _rel_fro(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


SHAPES = [(128, 256, 256), (256, 512, 2048), (384, 384, 1280), (128, 128, 4096),
          (256, 256, 256), (512, 768, 1536), (1024, 1024, 4096)]


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("mnk", SHAPES)
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_gemm_random_codes(lib, fmt, mnk, variant):
    # variant 0: CTA-pair 256x256 tiles when M, N % 256 == 0; 1: single-CTA 128x256; 2: single-CTA 128x128
    m, n, k = mnk
    if variant == 1 and (m % 256 or n % 256):
        pytest.skip("same kernel as variant 0")
    if variant == 2 and n % 256:
        pytest.skip("same kernel as variant 0")
    lib.wush_debug_set_gemm_variant(variant)
    a_c, a_s, a_dq = _random_operand(101 + m + k, m, k, fmt)
    b_c, b_s, b_dq = _random_operand(202 + n + k, n, k, fmt)
    alpha = 0.37 if fmt == "nvfp4" else 1.0
    dev = "cuda"
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev)
    try:
        lib.wush_qgemm(torch.from_numpy(a_c).to(dev), torch.from_numpy(a_s).to(dev), torch.from_numpy(b_c).to(dev),
                       torch.from_numpy(b_s).to(dev), m, n, k, fmt, alpha, y)
        assert lib.wush_check_device_status() == 0
    finally:
        lib.wush_debug_set_gemm_variant(0)
    got = y.cpu().numpy().astype(np.float64)
    want = G.gemm_dequantized(a_dq, b_dq, alpha)
    assert np.isfinite(got).all()
    err = _rel_fro(got, want)
    assert err <= 1e-5, err          # exact products, fp32 accumulation
    assert err <= P.GEMM_REL_FRO


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_layer_end_to_end(lib, fmt):
    w = synth.WORKLOADS["up_proj" if fmt == "mxfp4" else "down_proj"]
    m, n, k = 256, 512, 2048
    b = Q.BLOCK[fmt]
    x = synth.activations(w, tokens=m)[:, :k]
    wt = synth.weights(w)[:n, :k]
    xc = synth.activations(w, tokens=1024, calib=True)[:, :k]
    tx, tw = C.calibrate(xc, wt, b, "wush")
    tx, tw = tx.astype(np.float32), tw.astype(np.float32)
    gx = gw = None
    alpha = 1.0
    if fmt == "nvfp4":
        gx = C.nvfp4_global_scale(T.apply_block_transform(xc, tx).astype(np.float32))
        gw = C.nvfp4_global_scale(T.apply_block_transform(wt, tw).astype(np.float32))
        alpha = float(np.float32(gx) * np.float32(gw))
    dev = "cuda"
    ac, as_ = lib.alloc_quant_outputs(m, k, fmt)
    bc, bs = lib.alloc_quant_outputs(n, k, fmt)
    xt = torch.from_numpy(x).to(torch.bfloat16).to(dev)
    wtt = torch.from_numpy(wt).to(torch.bfloat16).to(dev)
    lib.wush_transform_quant(xt, torch.from_numpy(tx).to(dev), "wush", fmt, ac, as_, gx or 0.0)
    lib.wush_transform_quant(wtt, torch.from_numpy(tw).to(dev), "wush", fmt, bc, bs, gw or 0.0)
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    lib.wush_qgemm(ac, as_, bc, bs, m, n, k, fmt, alpha, y)
    assert lib.wush_check_device_status() == 0
    qa = Q.transform_quantize(x, tx, fmt, gx)
    qb = Q.transform_quantize(wt, tw, fmt, gw)
    if fmt == "nvfp4":   # the GEMM applies the two per-tensor scales through alpha
        want = G.gemm_dequantized(qa["dq"] / np.float64(gx), qb["dq"] / np.float64(gw), alpha)
    else:
        want = G.gemm_dequantized(qa["dq"], qb["dq"])
    err = _rel_fro(y.cpu().numpy().astype(np.float64), want)
    assert err <= P.GEMM_REL_FRO, err
    # and the quantised layer approximates the exact product W^T X
    ref = x.astype(np.float64) @ wt.astype(np.float64).T
    assert _rel_fro(y.cpu().numpy().astype(np.float64), ref) < 0.3


def test_full_size_up_proj_sampled(lib):
    # the bench's launch configuration: M 4096, N 12288, K 4096, MXFP4; the oracle
    # checks a sample of 48 rows x 256 columns of y
    w = synth.WORKLOADS["up_proj"]
    x = synth.activations(w)
    wt = synth.weights(w)
    xc = synth.activations(w, tokens=1024, calib=True)
    tx, tw = C.calibrate(xc, wt[:2048], 32, "wush")
    tx, tw = tx.astype(np.float32), tw.astype(np.float32)
    dev = "cuda"
    m, n, k = w.tokens, w.d_out, w.d_in
    ac, as_ = lib.alloc_quant_outputs(m, k, "mxfp4")
    bc, bs = lib.alloc_quant_outputs(n, k, "mxfp4")
    lib.wush_transform_quant(torch.from_numpy(x).to(torch.bfloat16).to(dev), torch.from_numpy(tx).to(dev),
                             "wush", "mxfp4", ac, as_)
    lib.wush_transform_quant(torch.from_numpy(wt).to(torch.bfloat16).to(dev), torch.from_numpy(tw).to(dev),
                             "wush", "mxfp4", bc, bs)
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    lib.wush_qgemm(ac, as_, bc, bs, m, n, k, "mxfp4", 1.0, y)
    assert lib.wush_check_device_status() == 0
    rng = np.random.default_rng(9)
    rows = np.sort(rng.choice(m, 48, replace=False))
    cols = np.sort(rng.choice(n, 256, replace=False))
    qa = Q.transform_quantize(x[rows], tx, "mxfp4")
    qb = Q.transform_quantize(wt[cols], tw, "mxfp4")
    want = G.gemm_dequantized(qa["dq"], qb["dq"])
    got = y.cpu().numpy()[np.ix_(rows, cols)].astype(np.float64)
    assert _rel_fro(got, want) <= P.GEMM_REL_FRO


@pytest.mark.parametrize("fmt, mnk", [("nvfp4", (4096, 4096, 12288)), ("nvfp4", (4096, 4096, 1024)),
                                      ("mxfp4", (4096, 4096, 1024)), ("mxfp4", (4096, 12288, 4096))])
def test_gemm_random_codes_many_tiles_per_pair(lib, fmt, mnk):
    # 16 x 16 = 256 pair tiles of 256 x 256 for 74 CTA pairs: every pair runs three
    # or four tiles, handing its accumulator back between them; (4096, 4096, 12288) is
    # the NVFP4 down_proj launch and (4096, 12288, 4096) the MXFP4 up_proj launch (10
    # or 11 tiles per pair).  The oracle checks 64 sampled rows, all columns.
    m, n, k = mnk
    a_c, a_s, a_dq = _random_operand(301 + k, m, k, fmt)
    b_c, b_s, b_dq = _random_operand(402 + k, n, k, fmt)
    alpha = 0.37 if fmt == "nvfp4" else 1.0
    dev = "cuda"
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev)
    lib.wush_qgemm(torch.from_numpy(a_c).to(dev), torch.from_numpy(a_s).to(dev), torch.from_numpy(b_c).to(dev),
                   torch.from_numpy(b_s).to(dev), m, n, k, fmt, alpha, y)
    assert lib.wush_check_device_status() == 0
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    rows = np.sort(np.random.default_rng(17).choice(m, 64, replace=False))
    rows[0], rows[-1] = 0, m - 1
    err = _rel_fro(got[rows], G.gemm_dequantized(a_dq[rows], b_dq, alpha))
    assert err <= 1e-5, err


def test_full_size_down_proj_sampled(lib):
    # the NVFP4 down_proj launch: M 4096, N 4096, K 12288, WUSH b = 16 with static
    # per-tensor scales; the oracle checks 48 rows x 256 columns of y
    w = synth.WORKLOADS["down_proj"]
    x = synth.activations(w)
    wt = synth.weights(w)
    xc = synth.activations(w, tokens=1024, calib=True)
    tx, tw = C.calibrate(xc, wt[:2048], 16, "wush")
    tx, tw = tx.astype(np.float32), tw.astype(np.float32)
    gx = C.nvfp4_global_scale(T.apply_block_transform(xc, tx).astype(np.float32))
    gw = C.nvfp4_global_scale(T.apply_block_transform(wt, tw).astype(np.float32))
    alpha = lib.wush_nvfp4_alpha(float(gx), float(gw))
    dev = "cuda"
    m, n, k = w.tokens, w.d_out, w.d_in
    ac, as_ = lib.alloc_quant_outputs(m, k, "nvfp4")
    bc, bs = lib.alloc_quant_outputs(n, k, "nvfp4")
    lib.wush_transform_quant(torch.from_numpy(x).to(torch.bfloat16).to(dev), torch.from_numpy(tx).to(dev),
                             "wush", "nvfp4", ac, as_, float(gx))
    lib.wush_transform_quant(torch.from_numpy(wt).to(torch.bfloat16).to(dev), torch.from_numpy(tw).to(dev),
                             "wush", "nvfp4", bc, bs, float(gw))
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    lib.wush_qgemm(ac, as_, bc, bs, m, n, k, "nvfp4", alpha, y)
    assert lib.wush_check_device_status() == 0
    rng = np.random.default_rng(19)
    rows = np.sort(rng.choice(m, 48, replace=False))
    cols = np.sort(rng.choice(n, 256, replace=False))
    qa = Q.transform_quantize(x[rows], tx, "nvfp4", gx)
    qb = Q.transform_quantize(wt[cols], tw, "nvfp4", gw)
    want = G.gemm_dequantized(qa["dq"] / np.float64(gx), qb["dq"] / np.float64(gw), alpha)
    got = y.cpu().numpy()[np.ix_(rows, cols)].astype(np.float64)
    assert _rel_fro(got, want) <= P.GEMM_REL_FRO


@pytest.mark.parametrize("m", [128, 256])     # single-CTA kernel, CTA-pair kernel
def test_bounded_wait_gives_up_and_context_survives(lib, m):
    n, k = 256, 512
    a_c, a_s, a_dq = _random_operand(7, m, k, "mxfp4")
    b_c, b_s, b_dq = _random_operand(8, n, k, "mxfp4")
    dev = "cuda"
    args = [torch.from_numpy(v).to(dev) for v in (a_c, a_s, b_c, b_s)]
    y = torch.zeros((m, n), dtype=torch.float32, device=dev)
    lib.wush_debug_set_wait_limit(64)     # the MMA role waits on a barrier nothing arrives on
    try:
        lib.wush_qgemm(*args, m, n, k, "mxfp4", 1.0, y)
        assert lib.wush_check_device_status() == -5
    finally:
        lib.wush_debug_set_wait_limit(0)
    lib.wush_qgemm(*args, m, n, k, "mxfp4", 1.0, y)
    assert lib.wush_check_device_status() == 0
    assert _rel_fro(y.cpu().numpy().astype(np.float64), G.gemm_dequantized(a_dq, b_dq)) < 1e-5


def test_gemm_rejects_bad_shapes(lib):
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    y = torch.zeros(1 << 14, dtype=torch.float32, device="cuda")
    for mnk in ((100, 256, 256), (128, 200, 256), (128, 256, 128), (0, 256, 256)):
        with pytest.raises(lib.WushError):
            lib.wush_qgemm(z, z, z, z, *mnk, "mxfp4", 1.0, y)
    with pytest.raises(lib.WushError):
        lib.wush_qgemm(z, z, z, z, 128, 256, 256, "int4", 1.0, y)
