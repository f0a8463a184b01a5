"""GPU parity: the tensor-core form of the ITQ3 activation-side GEMV (mode 1).

Mode 1 runs on the tensor cores when tokens >= 3 and d_out % 128 == 0 (one or two
tokens take the CUDA-core kernel, which is faster there): the 3-bit levels are exact
fp16 MMA operands and each 256-block of rotated x is scaled by a power of two and
split into fp16 hi + lo parts.  Cases cover one to eight CTAs per cluster (the
host picks the cluster width from d_out), one and two MMA widths (up to 8 tokens
and 9 to 16), ragged token counts, x values from fp16 subnormals to near the fp16
maximum, zero blocks and zero tokens, bit-for-bit repeatability, agreement with
the CUDA-core kernel, the allocation-free entry point, and a tiny wait limit.
"""
import functools

import numpy as np
import pytest

import synth
from oracle import itq3 as I
from tests.test_gpu_itq3 import pack_codes

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = 1e-5          # relative Frobenius bound of the ITQ3 GEMV, per token here


@functools.lru_cache(maxsize=None)
def _layer(d_out, d_in):
    """Device codes and scales plus the oracle's fp64 w_hat for a synthetic layer."""
    c, s = I.quantize(synth.itq3_weights(d_out, d_in))
    w_hat = I.dequantize(c, s)
    return torch.from_numpy(pack_codes(c)).cuda(), torch.from_numpy(s).cuda(), w_hat


def _gemv(lib, layer, x, d_out, variant=0, noalloc=False):
    codes, scales, _ = layer
    tokens, d_in = x.shape
    xd = torch.from_numpy(np.asarray(x, dtype=np.float16)).cuda()
    y = torch.full((tokens, d_out), float("nan"), dtype=torch.float32, device="cuda")
    lib.wush_debug_set_itq3_variant(variant)
    try:
        if noalloc:
            lib.itq3_dequant_gemv_noalloc(codes, scales, xd, d_out, y)
        else:
            ws = torch.full((tokens, d_in), float("nan"), dtype=torch.float32, device="cuda")
            lib.itq3_dequant_gemv(codes, scales, xd, d_out, 1, y, ws)
        torch.cuda.synchronize()
    finally:
        lib.wush_debug_set_itq3_variant(0)
    assert lib.wush_check_device_status() == 0
    return y.cpu().numpy().astype(np.float64)


def _per_token_err(got, want):
    errs = []
    for t in range(want.shape[0]):
        n = np.linalg.norm(want[t])
        errs.append(np.linalg.norm(got[t] - want[t]) / n if n > 0 else np.abs(got[t]).max())
    return max(errs)


@pytest.mark.parametrize("shape", [(128, 256), (384, 768), (256, 4096), (4096, 4096), (1024, 16384)])
@pytest.mark.parametrize("tokens", [1, 3, 8, 9, 16])
def test_tc_gemv_matches_oracle(lib, shape, tokens):
    d_out, d_in = shape
    layer = _layer(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in)
    want = np.asarray(x, dtype=np.float64) @ layer[2].T
    got = _gemv(lib, layer, x, d_out)
    assert np.isfinite(got).all()
    assert _per_token_err(got, want) <= TOL


@pytest.mark.parametrize("tokens", [5, 16])
def test_tc_gemv_value_ranges(lib, tokens):
    # tokens of very different magnitude, a zero token and zero blocks: each
    # (token, block) slice gets its own power-of-two scale, so every token meets
    # the bound on its own
    d_out, d_in = 512, 2048
    layer = _layer(d_out, d_in)
    x = np.asarray(synth.itq3_activations(tokens, d_in), dtype=np.float64)
    mags = [1.0, 2.0 ** -20, 0.0, 4000.0, 2.0 ** -10]
    for t in range(tokens):
        x[t] *= mags[t % len(mags)]
    x[0, 256:512] = 0.0                           # one zero block in a live token
    x[tokens - 1, :256] = 0.0
    x = x.astype(np.float16).astype(np.float64)  # the fp16 values the GEMV sees
    want = x @ layer[2].T
    got = _gemv(lib, layer, x, d_out)
    assert np.isfinite(got).all()
    assert _per_token_err(got, want) <= TOL
    assert not got[2].any()                       # the zero token gives exact zeros


@pytest.mark.parametrize("tokens", [3, 9])
def test_tc_gemv_agrees_with_cuda_core_kernel_and_repeats(lib, tokens):
    d_out, d_in = 4096, 4096
    layer = _layer(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in)
    tc1 = _gemv(lib, layer, x, d_out, variant=0)
    tc2 = _gemv(lib, layer, x, d_out, variant=0)
    cc = _gemv(lib, layer, x, d_out, variant=1)
    assert np.array_equal(tc1, tc2)               # cluster partials are added in rank order
    assert np.linalg.norm(tc1 - cc) / np.linalg.norm(cc) <= 2 * TOL


def test_tc_gemv_noalloc_matches_workspace_form(lib):
    d_out, d_in, tokens = 4096, 4096, 16
    layer = _layer(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in)
    assert np.array_equal(_gemv(lib, layer, x, d_out, noalloc=True), _gemv(lib, layer, x, d_out))


def test_tc_gemv_falls_back_for_rows_not_multiple_of_128(lib):
    # d_out % 128 != 0 takes the CUDA-core kernel; the result still meets the bound
    d_out, d_in, tokens = 200, 512, 3
    layer = _layer(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in)
    want = np.asarray(x, dtype=np.float64) @ layer[2].T
    assert _per_token_err(_gemv(lib, layer, x, d_out), want) <= TOL


def test_tc_gemv_tiny_wait_limit_never_hangs_and_context_survives(lib):
    # The accumulator waits end within a try_wait's hardware suspend window here,
    # so even a one-poll limit may not make them give up; either way the call
    # ends, reports honestly, and the next call is exact.
    d_out, d_in, tokens = 256, 1024, 4
    codes, scales, w_hat = _layer(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in)
    want = np.asarray(x, dtype=np.float64) @ w_hat.T
    xd = torch.from_numpy(x.astype(np.float16)).cuda()
    ws = torch.empty((tokens, d_in), dtype=torch.float32, device="cuda")
    y = torch.zeros((tokens, d_out), dtype=torch.float32, device="cuda")
    lib.wush_debug_set_wait_limit(1)
    try:
        lib.itq3_dequant_gemv(codes, scales, xd, d_out, 1, y, ws)
        status = lib.wush_check_device_status()
    finally:
        lib.wush_debug_set_wait_limit(0)
    assert status in (0, -5)
    if status == 0:
        assert _per_token_err(y.cpu().numpy().astype(np.float64), want) <= TOL
    lib.itq3_dequant_gemv(codes, scales, xd, d_out, 1, y, ws)
    assert lib.wush_check_device_status() == 0
    assert _per_token_err(y.cpu().numpy().astype(np.float64), want) <= TOL
