"""GPU parity: itq3_dequant_gemv (both modes) against the oracle's fp64 GEMV."""
import numpy as np
import pytest

import synth
from oracle import itq3 as I

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def pack_codes(c):
    """Test-side packer restating the header's layout: 3-bit codes, element e of a
    256-block at bits 3e .. 3e + 2 of the block's 96 little-endian bytes."""
    d_out, d_in = c.shape
    cb = c.reshape(d_out * d_in // 256, 256).astype(np.uint8)
    bits = ((cb[:, :, None] >> np.arange(3, dtype=np.uint8)) & 1).reshape(-1, 768)   # bit 3e + p
    return np.packbits(bits, axis=1, bitorder="little").reshape(-1)


@pytest.mark.parametrize("shape", [(256, 1024), (4096, 4096)])
@pytest.mark.parametrize("tokens", [1, 2, 3, 4, 16])
@pytest.mark.parametrize("mode", [0, 1])
def test_itq3_gemv(lib, shape, tokens, mode):
    d_out, d_in = shape
    w = synth.itq3_weights(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in)
    c, s = I.quantize(w)
    want = I.gemv(c, s, x)
    dev = "cuda"
    y = torch.full((tokens, d_out), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.empty((tokens, d_in), dtype=torch.float32, device=dev) if mode == 1 else None
    lib.itq3_dequant_gemv(torch.from_numpy(pack_codes(c)).to(dev), torch.from_numpy(s).to(dev),
                          torch.from_numpy(x.astype(np.float16)).to(dev), d_out, mode, y, ws)
    got = y.cpu().numpy().astype(np.float64)
    err = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert err <= 1e-5, err


def test_itq3_library_quantiser_feeds_gemv(lib):
    w = synth.itq3_weights(512, 2048)
    codes, scales = lib.itq3_quantize_weights(w.astype(np.float16))
    x = synth.itq3_activations(4, 2048)
    c, s = I.quantize(w)
    want = I.gemv(c, s, x)
    y = torch.empty((4, 512), dtype=torch.float32, device="cuda")
    lib.itq3_dequant_gemv(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                          torch.from_numpy(x.astype(np.float16)).cuda(), 512, 0, y)
    err = np.linalg.norm(y.cpu().numpy() - want) / np.linalg.norm(want)
    assert err <= 1e-5


@pytest.mark.parametrize("tokens, d_in", [(1, 40960), (2, 20480), (2, 24576), (1, 43008), (1, 256), (3, 4096),
                                          (8, 4096), (5, 1024)])
@pytest.mark.parametrize("variant", [0, 2, 3])
def test_itq3_mode1_rotation_inside_or_outside_the_gemv(lib, tokens, d_in, variant):
    # the single-kernel form rotates x inside the GEMV while the tokens' rotated x
    # fits shared memory (tokens * d_in <= 40960): by default for one and two
    # tokens, for up to eight as variant 3.  Otherwise, and for every call as variant
    # 2, the call rotates into the workspace first and then runs the GEMV (the
    # tensor-core kernel from 3 tokens when d_out % 128 == 0).  Against the oracle.
    d_out = 64
    w = synth.itq3_weights(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in).astype(np.float16)
    c, s = I.quantize(w)
    want = I.gemv(c, s, x.astype(np.float64))
    y = torch.full((tokens, d_out), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty((tokens, d_in), dtype=torch.float32, device="cuda")
    lib.wush_debug_set_itq3_variant(variant)
    try:
        lib.itq3_dequant_gemv(torch.from_numpy(pack_codes(c)).cuda(), torch.from_numpy(s).cuda(),
                              torch.from_numpy(x).cuda(), d_out, 1, y, ws)
        assert lib.wush_check_device_status() == 0
    finally:
        lib.wush_debug_set_itq3_variant(0)
    got = y.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-5


@pytest.mark.parametrize("d_out", [8, 40, 72, 1000])
@pytest.mark.parametrize("tokens, d_in", [(1, 256), (1, 2048), (2, 2048)])
def test_itq3_one_launch_ragged_rows(lib, d_out, tokens, d_in):
    # the one-launch form gives each CTA 32 rows: row counts that leave the last CTA
    # partly empty (and a single CTA of 8 rows) against the oracle
    w = synth.itq3_weights(d_out, d_in)
    x = synth.itq3_activations(tokens, d_in).astype(np.float16)
    c, s = I.quantize(w)
    want = I.gemv(c, s, x.astype(np.float64))
    y = torch.full((tokens, d_out), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty((tokens, d_in), dtype=torch.float32, device="cuda")
    lib.itq3_dequant_gemv(torch.from_numpy(pack_codes(c)).cuda(), torch.from_numpy(s).cuda(),
                          torch.from_numpy(x).cuda(), d_out, 1, y, ws)
    assert lib.wush_check_device_status() == 0
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 1e-5
