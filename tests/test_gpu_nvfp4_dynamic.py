"""GPU parity: the per-batch (dynamic) NVFP4 per-tensor scale.

Chain: wush_transform_amax (device amax of T x) -> wush_transform_quant_nvfp4_dynamic
(scale fp32(amax / 2688) derived on the device) -> wush_qgemm_nvfp4_dynamic
(alpha = scale_x * scale_w formed on the device).  The device amax comes from
fp32 transform arithmetic, so it may sit an ulp away from the oracle's; the
tests therefore (1) bound the device scale against the oracle's rule, (2) check
codes and scales against the oracle quantiser given the device's own scale, and
(3) require the dynamic path to equal the static path fed the same scale, bit
for bit, in the quantiser and the GEMM.
"""
import numpy as np
import pytest

import synth
from oracle import calibrate as C
from oracle import formats as F
from oracle import gemm as G
from oracle import transforms as T
from tests import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _ulps(a, b):
    a, b = np.float32(a), np.float32(b)
    return abs(int(a.view(np.int32)) - int(b.view(np.int32)))


def _setup(tokens=300, x_dtype="bf16"):
    w = synth.WORKLOADS["down_proj"]
    x = synth.activations(w, tokens=tokens)
    xc, wt = synth.activations(w, tokens=1024, calib=True), synth.weights(w)[:2048]
    tx, _ = C.calibrate(xc, wt, 16, "wush")
    t = tx.astype(np.float32)
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    if x_dtype == "bf16":
        xt = xt.to(torch.bfloat16)
    return x, t, xt.cuda(), torch.from_numpy(t).cuda()


def _dynamic(lib, xt, tt, kind="wush"):
    rows, d_in = xt.shape
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    gs = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    lib.wush_transform_amax(xt, tt, kind, 16, amax)
    codes, scales = lib.alloc_quant_outputs(rows, d_in, "nvfp4")
    lib.wush_transform_quant_nvfp4_dynamic(xt, tt, kind, amax, codes, scales, gs)
    torch.cuda.synchronize()
    assert lib.wush_check_device_status() == 0
    return amax, gs, codes, scales


@pytest.mark.parametrize("x_dtype", ["bf16", "fp32"])
def test_dynamic_scale_matches_rule_and_oracle_codes(lib, x_dtype):
    # bf16 runs the tensor-core kernel, fp32 the one-row-per-thread kernel
    x, t, xt, tt = _setup(x_dtype=x_dtype)
    rows, d_in = x.shape
    amax, gs, codes, scales = _dynamic(lib, xt, tt)
    gs_dev = np.float32(gs.item())
    want = C.nvfp4_dynamic_global_scale(T.apply_block_transform(x, t).astype(np.float32))
    assert _ulps(gs_dev, want) <= 2, (gs_dev, want)
    assert gs_dev == C.nvfp4_dynamic_global_scale(np.array([amax.item()], np.float32))
    P.compare_transform_quant(x, t, "nvfp4", float(gs_dev), P.unpack_nibbles(codes.cpu().numpy(), rows, d_in),
                              P.decode_scales(scales.cpu().numpy(), rows, d_in, "nvfp4"))


def test_dynamic_equals_static_with_same_scale_and_gemm(lib):
    x, t, xt, tt = _setup(tokens=256)
    rows, d_in = x.shape
    _, gs, codes_d, scales_d = _dynamic(lib, xt, tt)
    codes_s, scales_s = lib.alloc_quant_outputs(rows, d_in, "nvfp4")
    lib.wush_transform_quant(xt, tt, "wush", "nvfp4", codes_s, scales_s, float(gs.item()))
    torch.cuda.synchronize()
    assert torch.equal(codes_d, codes_s) and torch.equal(scales_d, scales_s)

    # weights: 256 rows of the down_proj W, static scale
    w = synth.WORKLOADS["down_proj"]
    xc, wt = synth.activations(w, tokens=1024, calib=True), synth.weights(w)[:256]
    _, tw = C.calibrate(xc, synth.weights(w)[:2048], 16, "wush")
    tw = tw.astype(np.float32)
    gw = float(C.nvfp4_global_scale(T.apply_block_transform(wt, tw).astype(np.float32)))
    wd = torch.from_numpy(np.ascontiguousarray(wt, np.float32)).to(torch.bfloat16).cuda()
    bc, bs = lib.alloc_quant_outputs(256, d_in, "nvfp4")
    lib.wush_transform_quant(wd, torch.from_numpy(tw).cuda(), "wush", "nvfp4", bc, bs, gw)
    y_dyn = torch.full((rows, 256), float("nan"), dtype=torch.float32, device="cuda")
    y_sta = torch.full((rows, 256), float("nan"), dtype=torch.float32, device="cuda")
    lib.wush_qgemm_nvfp4_dynamic(codes_d, scales_d, bc, bs, rows, 256, d_in, gs, gw, y_dyn)
    alpha = float(np.float32(gs.item()) * np.float32(gw))
    lib.wush_qgemm(codes_s, scales_s, bc, bs, rows, 256, d_in, "nvfp4", alpha, y_sta)
    torch.cuda.synchronize()
    assert lib.wush_check_device_status() == 0
    assert torch.equal(y_dyn, y_sta)
    # and against the oracle's product of the device's own operands, dequantised
    # (E2M1 value x UE4M3 block scale; the per-tensor scales enter through alpha)
    def dq(codes, scales, n):
        c = P.unpack_nibbles(codes.cpu().numpy(), n, d_in)
        sb = P.decode_scales(scales.cpu().numpy(), n, d_in, "nvfp4")
        return F.e2m1_value(c) * np.repeat(F.e4m3_value(sb), 16, axis=1)
    want = np.float64(np.float32(alpha)) * G.gemm_dequantized(dq(codes_d, scales_d, rows), dq(bc, bs, 256))
    got = y_dyn.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-5


def test_all_zero_tensor_gets_unit_scale_and_zero_codes(lib):
    rows, d_in = 128, 256
    xt = torch.zeros((rows, d_in), dtype=torch.bfloat16, device="cuda")
    _, gs, codes, scales = _dynamic(lib, xt, None, kind="hadamard")
    assert gs.item() == 1.0
    assert not codes.any() and not scales.any()


def test_dynamic_rejects_missing_amax(lib):
    xt = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    codes, scales = lib.alloc_quant_outputs(128, 256, "nvfp4")
    with pytest.raises(lib.WushError):
        lib.wush_transform_quant_nvfp4_dynamic(xt, None, "identity", None, codes, scales)
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    y = torch.zeros(128 * 128, dtype=torch.float32, device="cuda")
    with pytest.raises(lib.WushError):
        lib.wush_qgemm_nvfp4_dynamic(z, z, z, z, 128, 128, 256, None, 1.0, y)


@pytest.mark.parametrize("m, n", [(256, 256), (128, 256), (128, 384)])   # pair, 128 x 256, 128 x 128 tiles
def test_dynamic_alpha_in_every_gemm_kernel(lib, m, n):
    # random NVFP4 operands; the device factor must give the same y as host alpha,
    # bit for bit, in each of the GEMM's kernel forms
    k = 512
    rng = np.random.default_rng(m + n)
    a_codes = torch.from_numpy(rng.integers(0, 256, m * k // 2, dtype=np.uint8)).cuda()
    b_codes = torch.from_numpy(rng.integers(0, 256, n * k // 2, dtype=np.uint8)).cuda()
    def scales(rows):
        sb = (0x28 + rng.integers(0, 0x30, (rows, k // 16))).astype(np.uint8)   # UE4M3 0.03 .. 30
        return torch.from_numpy(P.swizzle_scales(sb)).cuda()
    a_s, b_s = scales(m), scales(n)
    gx = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    gw = 0.0377
    y_dyn = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    y_sta = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    lib.wush_qgemm_nvfp4_dynamic(a_codes, a_s, b_codes, b_s, m, n, k, gx, gw, y_dyn)
    lib.wush_qgemm(a_codes, a_s, b_codes, b_s, m, n, k, "nvfp4", float(np.float32(0.0123) * np.float32(gw)), y_sta)
    torch.cuda.synchronize()
    assert lib.wush_check_device_status() == 0
    assert torch.isfinite(y_dyn).all() and torch.equal(y_dyn, y_sta)
