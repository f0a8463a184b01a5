"""The allocation-free ITQ3 GEMV entry point, called through the C ABI.

It must give the same output as the workspace form (itq3_dequant_gemv mode 1)
on consecutive calls that reuse the library's fixed scratch array.  This file
is collected last so that a run stopping at the first failure has run every
other test already.
"""
import ctypes

import numpy as np
import pytest

import synth
from oracle import itq3 as I
from tests.test_gpu_itq3 import pack_codes

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL_TOL = 1e-5          # the ITQ3 GEMV tolerance used by the other GPU tests


def _call_noalloc(lib, codes, scales, x, d_out, y):
    fn = lib._lib.itq3_dequant_gemv_noalloc
    tokens, d_in = x.shape
    return fn(ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
              ctypes.c_void_p(x.data_ptr()), tokens, d_out, d_in, ctypes.c_void_p(y.data_ptr()),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_form_on_consecutive_calls(lib):
    d_out, d_in = 1024, 4096
    w = synth.itq3_weights(d_out, d_in)
    c, s = I.quantize(w)
    codes = torch.from_numpy(pack_codes(c)).cuda()
    scales = torch.from_numpy(s).cuda()
    for tokens in (16, 3):                       # two calls in a row, different sizes and inputs
        x = torch.from_numpy(synth.itq3_activations(tokens, d_in).astype(np.float16)).cuda()
        if tokens == 3:
            x = -x * 0.5
        y_ref = torch.empty((tokens, d_out), dtype=torch.float32, device="cuda")
        ws = torch.empty((tokens, d_in), dtype=torch.float32, device="cuda")
        lib.itq3_dequant_gemv(codes, scales, x, d_out, 1, y_ref, ws)
        y = torch.full((tokens, d_out), float("nan"), dtype=torch.float32, device="cuda")
        assert _call_noalloc(lib, codes, scales, x, d_out, y) == 0
        torch.cuda.synchronize()
        got, want = y.cpu().numpy().astype(np.float64), y_ref.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert np.linalg.norm(got - want) / np.linalg.norm(want) <= REL_TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    y = torch.empty(16, dtype=torch.float32, device="cuda")
    z = torch.zeros(256, dtype=torch.uint8, device="cuda")
    # 16 tokens x 32768 inputs needs 524,288 floats of scratch: more than the 262,144 it has
    fn = lib._lib.itq3_dequant_gemv_noalloc
    st = fn(ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(z.data_ptr()),
            16, 8, 32768, ctypes.c_void_p(y.data_ptr()), None)
    assert st == -6
