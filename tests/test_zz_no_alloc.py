"""The allocation-free ITQ3 GEMV entry point, called through the C ABI.

Callers that cannot allocate device memory where the GEMV runs (an engine that
owns all device memory in its own pool, a real-time loop) use this form; it keeps
the rotated activations in one fixed array inside the library.  Its output must
match the oracle's fp64 GEMV and the workspace form (itq3_dequant_gemv mode 1),
also on consecutive calls that reuse the fixed array with different sizes and
inputs.  This file is collected last so that a run stopping at the first failure
has run every other test already.
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
SCRATCH_FLOATS = 262144  # the fixed array's capacity, tokens * d_in


def _call_noalloc(lib, codes, scales, x, d_out, y):
    fn = lib._lib.itq3_dequant_gemv_noalloc
    tokens, d_in = x.shape
    return fn(ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
              ctypes.c_void_p(x.data_ptr()), tokens, d_out, d_in, ctypes.c_void_p(y.data_ptr()),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _rel(got, want):
    return np.linalg.norm(got - want) / np.linalg.norm(want)


# tokens 1-2 with tokens * d_in <= 40960 run the single-kernel form, which does not
# touch the array; 2 x 32768 rotates into the array and runs the CUDA-core GEMV, 3
# and 16 the tensor-core one; the last case fills the array exactly (16 x 16384)
@pytest.mark.parametrize("tokens, d_out, d_in", [(1, 1024, 4096), (2, 1024, 4096), (2, 64, 32768), (3, 1024, 4096),
                                                 (16, 1024, 4096), (16, 256, 16384)])
def test_noalloc_matches_oracle_and_workspace_form_on_consecutive_calls(lib, tokens, d_out, d_in):
    assert tokens * d_in <= SCRATCH_FLOATS
    w = synth.itq3_weights(d_out, d_in)
    c, s = I.quantize(w)
    codes = torch.from_numpy(pack_codes(c)).cuda()
    scales = torch.from_numpy(s).cuda()
    x0 = synth.itq3_activations(tokens, d_in).astype(np.float16)
    # two calls in a row on the shared array: the second with other inputs (and a
    # smaller size for the multi-token cases), so stale contents would show
    calls = [x0, (-0.5 * x0[: max(1, tokens // 2)]).astype(np.float16)]
    for x16 in calls:
        t = x16.shape[0]
        want = I.gemv(c, s, x16.astype(np.float64))
        x = torch.from_numpy(x16).cuda()
        y = torch.full((t, d_out), float("nan"), dtype=torch.float32, device="cuda")
        assert _call_noalloc(lib, codes, scales, x, d_out, y) == 0
        y_ws = torch.empty((t, d_out), dtype=torch.float32, device="cuda")
        ws = torch.empty((t, d_in), dtype=torch.float32, device="cuda")
        lib.itq3_dequant_gemv(codes, scales, x, d_out, 1, y_ws, ws)
        torch.cuda.synchronize()
        assert lib.wush_check_device_status() == 0
        got = y.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert _rel(got, want) <= REL_TOL
        assert _rel(got, y_ws.cpu().numpy().astype(np.float64)) <= REL_TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    y = torch.empty(16, dtype=torch.float32, device="cuda")
    z = torch.zeros(256, dtype=torch.uint8, device="cuda")
    # 16 tokens x 32768 inputs needs 524,288 floats of scratch: more than the 262,144 it has
    fn = lib._lib.itq3_dequant_gemv_noalloc
    st = fn(ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(z.data_ptr()),
            16, 8, 32768, ctypes.c_void_p(y.data_ptr()), None)
    assert st == -6
    # one float over the capacity is refused too
    st = fn(ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(z.data_ptr()),
            1, 8, SCRATCH_FLOATS + 256, ctypes.c_void_p(y.data_ptr()), None)
    assert st == -6
