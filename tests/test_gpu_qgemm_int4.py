"""GPU parity: wush_qgemm_int4 against the oracle's fp64 GEMM on dequantised INT4.

The kernel rounds each dequantised element to fp16 (relative error <= 2^-11), so
its relative Frobenius error against the exact product stays well inside the
1e-3 bar; the test checks both bars.
"""
import numpy as np
import pytest

import synth
from oracle import calibrate as C
from oracle import gemm as G
from oracle import quant as Q
from tests import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _random_int4(seed, rows, k):
    u = synth.uniform(seed, rows * k + rows * (k // 32))
    q = np.floor(u[: rows * k] * 15).astype(np.int64).reshape(rows, k) - 7          # -7 .. 7
    s = (2.0 ** (u[rows * k:] * 10 - 8)).reshape(rows, k // 32).astype(np.float16)  # 2^-8 .. 2^2
    dq = q * np.repeat(s.astype(np.float64), 32, axis=1)
    nib = (q & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return packed, s, dq


def _rel(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


@pytest.mark.parametrize("mnk", [(128, 256, 64), (256, 512, 640), (384, 768, 2048), (128, 256, 5120)])
def test_int4_gemm_random(lib, mnk):
    m, n, k = mnk
    a_c, a_s, a_dq = _random_int4(11 + m, m, k)
    b_c, b_s, b_dq = _random_int4(22 + n, n, k)
    dev = "cuda"
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev)
    lib.wush_qgemm_int4(torch.from_numpy(a_c).to(dev), torch.from_numpy(a_s).to(dev), torch.from_numpy(b_c).to(dev),
                        torch.from_numpy(b_s).to(dev), m, n, k, y)
    assert lib.wush_check_device_status() == 0
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    err = _rel(got, G.gemm_dequantized(a_dq, b_dq))
    assert err <= 5e-4, err
    assert err <= P.GEMM_REL_FRO


def test_int4_layer_end_to_end_sampled(lib):
    # the int4 workload at 2048 tokens (full K and N), oracle on 40 rows x 256 columns
    w = synth.WORKLOADS["int4"]
    m, n, k = 2048, w.d_out, w.d_in
    x = synth.activations(w, tokens=m)
    wt = synth.weights(w)
    xc = synth.activations(w, tokens=1024, calib=True)
    tx, tw = C.calibrate(xc, wt[:2048], 32, "wush")
    tx, tw = tx.astype(np.float32), tw.astype(np.float32)
    dev = "cuda"
    ac, as_ = lib.alloc_quant_outputs(m, k, "int4")
    bc, bs = lib.alloc_quant_outputs(n, k, "int4")
    lib.wush_transform_quant(torch.from_numpy(x).to(torch.bfloat16).to(dev), torch.from_numpy(tx).to(dev),
                             "wush", "int4", ac, as_)
    lib.wush_transform_quant(torch.from_numpy(wt).to(torch.bfloat16).to(dev), torch.from_numpy(tw).to(dev),
                             "wush", "int4", bc, bs)
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    lib.wush_qgemm_int4(ac, as_, bc, bs, m, n, k, y)
    assert lib.wush_check_device_status() == 0
    rng = np.random.default_rng(4)
    rows = np.sort(rng.choice(m, 40, replace=False))
    cols = np.sort(rng.choice(n, 256, replace=False))
    want = G.gemm_dequantized(Q.transform_quantize(x[rows], tx, "int4")["dq"],
                              Q.transform_quantize(wt[cols], tw, "int4")["dq"])
    got = y.cpu().numpy()[np.ix_(rows, cols)].astype(np.float64)
    assert _rel(got, want) <= P.GEMM_REL_FRO


def test_int4_rejects_bad_shapes(lib):
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    y = torch.zeros(1 << 14, dtype=torch.float32, device="cuda")
    for mnk in ((100, 256, 64), (128, 200, 64), (128, 256, 48)):
        with pytest.raises(lib.WushError):
            lib.wush_qgemm_int4(z, z, z, z, *mnk, y)


def _run_ws(lib, a_c, a_s, b_c, b_s, m, n, k, y):
    ws = torch.empty(lib.wush_qgemm_int4_workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    lib.wush_qgemm_int4_ws(a_c, a_s, b_c, b_s, m, n, k, ws, y)


@pytest.mark.parametrize("mnk", [(256, 256, 64), (256, 512, 640), (512, 768, 2048), (256, 256, 5120)])
def test_int4_gemm_two_pass_random(lib, mnk):
    m, n, k = mnk
    a_c, a_s, a_dq = _random_int4(31 + m, m, k)
    b_c, b_s, b_dq = _random_int4(42 + n, n, k)
    dev = "cuda"
    args = [torch.from_numpy(v).to(dev) for v in (a_c, a_s, b_c, b_s)]
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev)
    _run_ws(lib, *args, m, n, k, y)
    assert lib.wush_check_device_status() == 0
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    err = _rel(got, G.gemm_dequantized(a_dq, b_dq))
    assert err <= 5e-4, err
    # the fused form rounds the same fp16 operands: the two agree to fp32 accumulation order
    y2 = torch.empty_like(y)
    lib.wush_qgemm_int4(*args, m, n, k, y2)
    diff = _rel(got, y2.cpu().numpy().astype(np.float64))
    assert diff <= 1e-5, diff


def test_int4_two_pass_random_full_size_sampled(lib):
    # the int4 workload's launch (8192 x 17408 x 5120) on seeded random codes: the pair
    # GEMM walks its tiles in groups of row blocks sized to L2, so every group, every
    # tile of a column and the last, partial group are reached; the oracle checks 64
    # sampled rows (the first and the last included) against all 17408 columns
    m, n, k = 8192, 17408, 5120
    a_c, a_s, a_dq = _random_int4(51, m, k)
    b_c, b_s, b_dq = _random_int4(52, n, k)
    dev = "cuda"
    args = [torch.from_numpy(v).to(dev) for v in (a_c, a_s, b_c, b_s)]
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=dev)
    _run_ws(lib, *args, m, n, k, y)
    assert lib.wush_check_device_status() == 0
    rows = np.sort(np.random.default_rng(53).choice(m, 64, replace=False))
    rows[0], rows[-1] = 0, m - 1
    got = y[torch.from_numpy(rows).to(dev)].cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    err = _rel(got, G.gemm_dequantized(a_dq[rows], b_dq))
    assert err <= 5e-4, err


@pytest.mark.parametrize("m", [2048, 8192])
def test_int4_two_pass_end_to_end_sampled(lib, m):
    # the int4 workload at 2048 and 8192 tokens (the bench's launches) through the
    # two-pass form, oracle on 40 x 256
    w = synth.WORKLOADS["int4"]
    n, k = w.d_out, w.d_in
    x = synth.activations(w, tokens=m)
    wt = synth.weights(w)
    xc = synth.activations(w, tokens=1024, calib=True)
    tx, tw = C.calibrate(xc, wt[:2048], 32, "wush")
    tx, tw = tx.astype(np.float32), tw.astype(np.float32)
    dev = "cuda"
    ac, as_ = lib.alloc_quant_outputs(m, k, "int4")
    bc, bs = lib.alloc_quant_outputs(n, k, "int4")
    lib.wush_transform_quant(torch.from_numpy(x).to(torch.bfloat16).to(dev), torch.from_numpy(tx).to(dev),
                             "wush", "int4", ac, as_)
    lib.wush_transform_quant(torch.from_numpy(wt).to(torch.bfloat16).to(dev), torch.from_numpy(tw).to(dev),
                             "wush", "int4", bc, bs)
    y = torch.empty((m, n), dtype=torch.float32, device=dev)
    _run_ws(lib, ac, as_, bc, bs, m, n, k, y)
    assert lib.wush_check_device_status() == 0
    rng = np.random.default_rng(6)
    rows = np.sort(rng.choice(m, 40, replace=False))
    cols = np.sort(rng.choice(n, 256, replace=False))
    want = G.gemm_dequantized(Q.transform_quantize(x[rows], tx, "int4")["dq"],
                              Q.transform_quantize(wt[cols], tw, "int4")["dq"])
    got = y.cpu().numpy()[np.ix_(rows, cols)].astype(np.float64)
    assert _rel(got, want) <= P.GEMM_REL_FRO


def test_int4_two_pass_rejects_bad_arguments(lib):
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    y = torch.zeros(1 << 14, dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    for mnk in ((128, 256, 64), (256, 384, 64), (256, 256, 48)):
        with pytest.raises(lib.WushError):
            lib.wush_qgemm_int4_ws(z, z, z, z, *mnk, ws, y)
    small = torch.zeros(lib.wush_qgemm_int4_workspace_bytes(256, 256, 64) - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.WushError, match="BUFFER_TOO_SMALL|too small"):
        lib.wush_qgemm_int4_ws(z, z, z, z, 256, 256, 64, small, y)
