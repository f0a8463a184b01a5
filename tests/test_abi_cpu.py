"""C-ABI library checks that need no GPU: exports, host calibration and ITQ3
quantisation against the oracle, buffer sizes and argument validation."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from oracle import calibrate as C
from oracle import itq3 as I

aq = pytest.importorskip("activation_quantization_b200")
HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "wush.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(aq.LIB_PATH)
    names = _declared()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(aq._SIGNATURES), "binding lacks a signature"


@pytest.mark.parametrize("kind", ["identity", "hadamard", "wus", "wush", "wush_diag"])
def test_calibrate_matches_oracle(kind):
    w = synth.WORKLOADS["tiny"]
    xc, wt = synth.activations(w, calib=True), synth.weights(w)
    for b in (16, 32):
        tx, tw = aq.wush_calibrate(xc, wt, b, kind)
        ox, ow = C.calibrate(xc, wt, b, kind)
        for got, want in ((tx, ox), (tw, ow)):
            scale = np.abs(want).max(axis=(1, 2), keepdims=True)
            assert np.max(np.abs(got - want) / scale) < 1e-6


def test_calibrate_from_moments_matches_calibrate():
    w = synth.WORKLOADS["tiny"]
    xc, wt = synth.activations(w, calib=True), synth.weights(w)
    tx, tw = aq.wush_calibrate(xc, wt, 32, "wush")
    mx, mw = C.block_moments(xc, 32), C.block_moments(wt, 32)
    tx2, tw2 = aq.wush_calibrate_from_moments(mx, mw, "wush")
    assert np.allclose(tx, tx2, rtol=1e-5, atol=1e-6 * np.abs(tx).max())


def test_not_spd_status():
    sx = np.broadcast_to(np.eye(4), (2, 4, 4)).copy()
    with pytest.raises(aq.WushError) as e:
        aq.wush_calibrate_from_moments(sx, -sx, "wush")
    assert e.value.status == -3


def _unpack_itq3(packed, d_out, d_in):
    bits = np.unpackbits(packed.reshape(-1, 96), axis=1, bitorder="little").reshape(-1, 256, 3)
    c = bits[:, :, 0] | (bits[:, :, 1] << 1) | (bits[:, :, 2] << 2)
    return c.reshape(d_out, d_in).astype(np.uint8)


@pytest.mark.parametrize("shape", [(8, 256), (64, 1024)])
def test_itq3_quantize_matches_oracle_bit_exact(shape):
    w = synth.itq3_weights(*shape)
    w[0, :256] = 0.0                                   # an all-zero block: s = 0, codes 0
    codes, scales = aq.itq3_quantize_weights(w.astype(np.float16))
    oc, os_ = I.quantize(w.astype(np.float16).astype(np.float64))
    assert np.array_equal(scales.view(np.uint16), os_.view(np.uint16))
    assert np.array_equal(_unpack_itq3(codes, *shape), oc)


def test_buffer_sizes():
    assert aq.wush_codes_bytes(4096, 4096, "mxfp4") == 8388608
    assert aq.wush_scales_bytes(4096, 4096, "mxfp4") == 524288
    assert aq.wush_scales_bytes(4096, 12288, "nvfp4") == 3145728
    assert aq.wush_scales_bytes(8192, 5120, "int4") == 2621440
    assert aq.wush_scales_bytes(130, 96, "mxfp4") == 2 * 1 * 512      # 2 row atoms x 1 col atom
    assert aq.wush_block_size("nvfp4") == 16 and aq.wush_block_size(7) == 0


def test_argument_validation_before_launch():
    lib = aq._lib
    # d_in not a multiple of the block, unknown format/kind, NULL pointers: no launch happens
    assert lib.wush_transform_quant(16, 0, 4, 48, None, 0, 0, 0.0, 16, 16, None, None) == -1
    assert lib.wush_transform_quant(16, 0, 4, 64, None, 0, 9, 0.0, 16, 16, None, None) == -2
    assert lib.wush_transform_quant(16, 0, 4, 64, None, 7, 0, 0.0, 16, 16, None, None) == -2
    assert lib.wush_transform_quant(None, 0, 4, 64, None, 0, 0, 0.0, 16, 16, None, None) == -1
    assert lib.wush_transform_quant(16, 0, 4, 64, None, 3, 0, 0.0, 16, 16, None, None) == -1  # WUSH needs t
    assert lib.wush_transform_quant(17, 0, 4, 64, None, 0, 0, 0.0, 16, 16, None, None) == -1  # misaligned
    assert lib.wush_transform_quant(16, 0, 4, 64, None, 0, 1, 0.0, 16, 16, None, None) == -1  # NVFP4 s_g
    assert lib.wush_transform_quant(16, 0, 0, 64, None, 0, 0, 0.0, 16, 16, None, None) == 0   # empty
    assert lib.wush_calibrate(None, 0, None, 0, 64, 24, 3, 16, 16) == -1                      # block
    assert lib.itq3_quantize_weights(16, 4, 100, 16, 16) == -1
    assert lib.wush_status_string(-5) == b"a bounded device wait gave up"


@pytest.mark.parametrize("kind", ["wus", "wush", "wush_diag"])
def test_calibrate_shared_matches_oracle(kind):
    w = synth.WORKLOADS["tiny"]
    xc, wt = synth.activations(w, calib=True), synth.weights(w)
    for b in (16, 32):
        for groups in (1, 2, 3, 256 // b):
            tx, tw, idx = aq.wush_calibrate_shared(xc, wt, b, kind, groups)
            ox, ow, oidx = C.shared_transforms(C.block_moments(xc, b), C.block_moments(wt, b), kind, groups)
            assert np.array_equal(idx, oidx)
            for got, want in ((tx, ox), (tw, ow)):
                scale = np.abs(want).max(axis=(1, 2), keepdims=True)
                assert np.max(np.abs(got - want) / scale) < 1e-6
    with pytest.raises(aq.WushError):
        aq.wush_calibrate_shared(xc, wt, 32, kind, 0)
    with pytest.raises(aq.WushError):
        aq.wush_calibrate_shared(xc, wt, 32, kind, 9)      # more groups than blocks


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_host_calls_reject_non_finite_inputs(bad):
    # one planted NaN or infinity anywhere in an input gives WUSH_ERR_INVALID_ARG
    w = synth.WORKLOADS["tiny"]
    xc, wt = synth.activations(w, calib=True), synth.weights(w)

    def planted(a):
        a = np.array(a, copy=True)
        a.flat[a.size // 3] = bad
        return a

    def status(fn, *args):
        with pytest.raises(aq.WushError) as e:
            fn(*args)
        return e.value.status

    for kind in ("wus", "wush", "wush_diag"):
        assert status(aq.wush_calibrate, planted(xc), wt, 32, kind) == -1
        assert status(aq.wush_calibrate, xc, planted(wt), 32, kind) == -1
        assert status(aq.wush_calibrate_shared, planted(xc), wt, 32, kind, 2) == -1
        sx, sw = C.block_moments(xc, 32), C.block_moments(wt, 32)
        assert status(aq.wush_calibrate_from_moments, planted(sx), sw, kind) == -1
        assert status(aq.wush_calibrate_shared_from_moments, sx, planted(sw), kind, 2) == -1
    # identity and Hadamard read no data, so there is nothing to check
    aq.wush_calibrate(planted(xc), wt, 32, "hadamard")
    w3 = synth.itq3_weights(4, 512).astype(np.float16)
    assert status(aq.itq3_quantize_weights, planted(w3)) == -1
    aq.itq3_quantize_weights(w3)                      # the clean copy is accepted


@pytest.mark.parametrize("b", [2, 4, 8, 64, 128, 256])
@pytest.mark.parametrize("kind", ["hadamard", "wus", "wush", "wush_diag"])
def test_calibrate_every_block_size_matches_oracle(kind, b):
    # the host calibration accepts any power-of-two block up to 256; the device
    # kernels use 16 and 32, checked above, and here the rest of the range
    w = synth.WORKLOADS["tiny"]
    xc, wt = synth.activations(w, calib=True), synth.weights(w)
    tx, tw = aq.wush_calibrate(xc, wt, b, kind)
    ox, ow = C.calibrate(xc, wt, b, kind)
    for got, want in ((tx, ox), (tw, ow)):
        scale = np.abs(want).max(axis=(1, 2), keepdims=True)
        assert np.max(np.abs(got - want) / scale) < 1e-6
    if kind != "hadamard":
        # the defining property T_W^T T_X = I, in fp32 storage
        eye = np.einsum("jki,jkl->jil", tw.astype(np.float64), tx.astype(np.float64))
        assert np.max(np.abs(eye - np.eye(b))) < 1e-4


def test_nvfp4_static_scale_and_alpha_match_the_oracle_rule():
    # s_g = amax / 2688 rounded once to fp32 (the oracle's static rule, which
    # rounds the fp64 quotient; with 53 >= 2*24 + 2 bits that double rounding is
    # the correctly rounded fp32 quotient); alpha = fp32(s_gx * s_gw)
    from oracle import calibrate as C
    rng = np.random.default_rng(21)
    amaxes = np.concatenate([np.float32(10.0) ** rng.uniform(-20, 20, 2000),
                             np.float32([1.0, 2688.0, 448.0 * 6, 1e-3, 3.4e38])]).astype(np.float32)
    for a in amaxes:
        want = C.nvfp4_global_scale(np.array([[a]], np.float32))
        assert np.float32(aq.wush_nvfp4_global_scale(float(a))) == want, a
    assert aq.wush_nvfp4_global_scale(0.0) == 1.0
    assert np.float32(aq.wush_nvfp4_global_scale(0.0)) == C.nvfp4_dynamic_global_scale(np.zeros((1, 16), np.float32))
    for _ in range(500):
        gx, gw = np.float32(10.0 ** rng.uniform(-8, 2, 2))
        assert np.float32(aq.wush_nvfp4_alpha(float(gx), float(gw))) == np.float32(np.float64(gx) * np.float64(gw))
    for bad in (-1.0, float("nan"), float("inf")):
        with pytest.raises(aq.WushError):
            aq.wush_nvfp4_global_scale(bad)
    for bad in ((0.0, 1.0), (1.0, -2.0), (float("nan"), 1.0), (1.0, float("inf"))):
        with pytest.raises(aq.WushError):
            aq.wush_nvfp4_alpha(*bad)
