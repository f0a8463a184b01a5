"""The Python binding's own argument checks, on CPU tensors (no GPU needed).

The C entry points take bare pointers, so the binding checks element types and
buffer sizes before it hands a pointer over: a buffer one byte short gives
WushError with WUSH_ERR_BUFFER_TOO_SMALL and names the tensor, a wrong element
type gives ValueError, and a call whose buffers are exactly large enough gets
past the checks and stops only at the CUDA-tensor requirement."""
import pytest

aq = pytest.importorskip("activation_quantization_b200")
torch = pytest.importorskip("torch")

TOO_SMALL = -6


def u8(n):
    return torch.zeros(max(n, 0), dtype=torch.uint8)


def f32(n):
    return torch.zeros(max(n, 0), dtype=torch.float32)


def _passes_checks(fn, *args, **kw):
    with pytest.raises(ValueError, match="expected a CUDA tensor"):
        fn(*args, **kw)


def _too_small(name, fn, *args, **kw):
    with pytest.raises(aq.WushError, match=name) as e:
        fn(*args, **kw)
    assert e.value.status == TOO_SMALL


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_transform_quant_buffers(fmt):
    rows, d_in = 130, 256
    b = aq.wush_block_size(fmt)
    x = torch.zeros((rows, d_in), dtype=torch.bfloat16)
    nc, ns = aq.wush_codes_bytes(rows, d_in, fmt), aq.wush_scales_bytes(rows, d_in, fmt)
    t = f32(d_in * b)
    _passes_checks(aq.wush_transform_quant, x, t, "wush", fmt, u8(nc), u8(ns), 0.01, f32(rows * d_in))
    _too_small("codes", aq.wush_transform_quant, x, t, "wush", fmt, u8(nc - 1), u8(ns), 0.01)
    _too_small("scales", aq.wush_transform_quant, x, t, "wush", fmt, u8(nc), u8(ns - 1), 0.01)
    _too_small("'t'|t holds", aq.wush_transform_quant, x, f32(d_in * b - 1), "wush", fmt, u8(nc), u8(ns), 0.01)
    _too_small("y_debug", aq.wush_transform_quant, x, t, "wush", fmt, u8(nc), u8(ns), 0.01, f32(rows * d_in - 1))
    with pytest.raises(ValueError, match="t must be"):
        aq.wush_transform_quant(x, t.double(), "wush", fmt, u8(nc), u8(ns), 0.01)
    # identity and Hadamard read no T
    _passes_checks(aq.wush_transform_quant, x, None, "hadamard", fmt, u8(nc), u8(ns), 0.01)


def test_indexed_and_dynamic_buffers():
    rows, d_in, b = 128, 512, 32
    x = torch.zeros((rows, d_in), dtype=torch.bfloat16)
    nc, ns = aq.wush_codes_bytes(rows, d_in, "mxfp4"), aq.wush_scales_bytes(rows, d_in, "mxfp4")
    t = torch.zeros((3, b, b), dtype=torch.float32)
    idx = torch.zeros(d_in // b, dtype=torch.int32)
    _passes_checks(aq.wush_transform_quant_indexed, x, t, idx, "wush", "mxfp4", u8(nc), u8(ns))
    _too_small("t_index", aq.wush_transform_quant_indexed, x, t, idx[:-1], "wush", "mxfp4", u8(nc), u8(ns))
    with pytest.raises(ValueError, match="t_index must be"):
        aq.wush_transform_quant_indexed(x, t, idx.long(), "wush", "mxfp4", u8(nc), u8(ns))
    # T whose blocks are smaller than b: n_t blocks of b x b would overrun it
    _too_small("holds", aq.wush_transform_quant_indexed, x, torch.zeros((3, 16, 16)), idx, "wush", "mxfp4",
               u8(nc), u8(ns))
    nc, ns = aq.wush_codes_bytes(rows, d_in, "nvfp4"), aq.wush_scales_bytes(rows, d_in, "nvfp4")
    t16 = f32(d_in * 16)
    _passes_checks(aq.wush_transform_quant_nvfp4_dynamic, x, t16, "wush", f32(1), u8(nc), u8(ns), f32(1))
    _too_small("amax", aq.wush_transform_quant_nvfp4_dynamic, x, t16, "wush", f32(0), u8(nc), u8(ns))
    _too_small("global_scale_out", aq.wush_transform_quant_nvfp4_dynamic, x, t16, "wush", f32(1), u8(nc), u8(ns),
               f32(0))
    _passes_checks(aq.wush_transform_amax, x, t16, "wush", 16, f32(1))
    _too_small("amax_out", aq.wush_transform_amax, x, t16, "wush", 16, f32(0))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_gemm_buffers(fmt):
    m, n, k = 256, 384, 512
    ac, bc = u8(m * k // 2), u8(n * k // 2)
    as_, bs = u8(aq.wush_scales_bytes(m, k, fmt)), u8(aq.wush_scales_bytes(n, k, fmt))
    y = f32(m * n)
    _passes_checks(aq.wush_qgemm, ac, as_, bc, bs, m, n, k, fmt, 1.0, y)
    _too_small("a_codes", aq.wush_qgemm, ac[:-1], as_, bc, bs, m, n, k, fmt, 1.0, y)
    _too_small("b_codes", aq.wush_qgemm, ac, as_, bc[:-1], bs, m, n, k, fmt, 1.0, y)
    _too_small("a_scales", aq.wush_qgemm, ac, as_[:-1], bc, bs, m, n, k, fmt, 1.0, y)
    _too_small("b_scales", aq.wush_qgemm, ac, as_, bc, bs[:-1], m, n, k, fmt, 1.0, y)
    _too_small("'y'|y holds", aq.wush_qgemm, ac, as_, bc, bs, m, n, k, fmt, 1.0, y[:-1])
    with pytest.raises(ValueError, match="y must be"):
        aq.wush_qgemm(ac, as_, bc, bs, m, n, k, fmt, 1.0, torch.zeros(m * n, dtype=torch.bfloat16))
    if fmt == "nvfp4":
        _passes_checks(aq.wush_qgemm_nvfp4_dynamic, ac, as_, bc, bs, m, n, k, f32(1), 1.0, y)
        _too_small("a_global_scale", aq.wush_qgemm_nvfp4_dynamic, ac, as_, bc, bs, m, n, k, f32(0), 1.0, y)


def test_int4_gemm_buffers():
    m, n, k = 256, 256, 64
    ac, bc = u8(m * k // 2), u8(n * k // 2)
    as_, bs = u8(m * (k // 32) * 2), u8(n * (k // 32) * 2)
    y = f32(m * n)
    _passes_checks(aq.wush_qgemm_int4, ac, as_, bc, bs, m, n, k, y)
    _too_small("b_scales", aq.wush_qgemm_int4, ac, as_, bc, bs[:-1], m, n, k, y)
    ws = u8(aq.wush_qgemm_int4_workspace_bytes(m, n, k))
    _passes_checks(aq.wush_qgemm_int4_ws, ac, as_, bc, bs, m, n, k, ws, y)
    _too_small("a_codes", aq.wush_qgemm_int4_ws, ac[:-1], as_, bc, bs, m, n, k, ws, y)


def test_itq3_buffers():
    d_out, d_in, tokens = 256, 512, 4
    codes, scales = u8(d_out * d_in * 3 // 8), torch.zeros((d_out, d_in // 256), dtype=torch.float16)
    x = torch.zeros((tokens, d_in), dtype=torch.float16)
    y, ws = f32(tokens * d_out), f32(tokens * d_in)
    for mode in (0, 1):
        _passes_checks(aq.itq3_dequant_gemv, codes, scales, x, d_out, mode, y, ws)
    _passes_checks(aq.itq3_dequant_gemv_noalloc, codes, scales, x, d_out, y)
    _too_small("codes", aq.itq3_dequant_gemv, codes[:-1], scales, x, d_out, 0, y)
    _too_small("scales", aq.itq3_dequant_gemv, codes, scales[:-1], x, d_out, 0, y)
    _too_small("'y'|y holds", aq.itq3_dequant_gemv_noalloc, codes, scales, x, d_out, y[:-1])
    _too_small("workspace", aq.itq3_dequant_gemv, codes, scales, x, d_out, 1, y, ws[:-1])
    _passes_checks(aq.itq3_dequant_gemv, codes, scales, x, d_out, 0, y, ws[:-1])   # mode 0 uses none
    with pytest.raises(ValueError, match="x must be"):
        aq.itq3_dequant_gemv(codes, scales, x.float(), d_out, 0, y)
