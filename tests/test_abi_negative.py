"""Host-side argument validation of every device entry point, without a GPU.

Each call below breaks one documented requirement (shape, alignment, NULL,
unsupported format, kind or mode, buffer size) and must return its status
before anything touches the device, so the calls run here with made-up,
never-dereferenced pointer values."""
import pytest

aq = pytest.importorskip("activation_quantization_b200")
lib = aq._lib

OK, INVALID, UNSUPPORTED, TOO_SMALL = 0, -1, -2, -6
P, P2, ODD, HALF = 4096, 8192, 4097, 4098     # aligned, aligned, odd, 2-byte aligned only
MX, NV, I4 = 0, 1, 2
BF16, F32 = 0, 1
IDENT, HAD, WUS, WUSH, DIAG = 0, 1, 2, 3, 4


def test_transform_quant_indexed():
    f = lib.wush_transform_quant_indexed
    args = dict(x=P, dt=BF16, rows=128, d_in=256, t=P, idx=P2, n_t=2, kind=WUSH, fmt=MX, gs=0.0,
                codes=P, scales=P2, y=None, s=None)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["x"], a["dt"], a["rows"], a["d_in"], a["t"], a["idx"], a["n_t"], a["kind"], a["fmt"], a["gs"],
                 a["codes"], a["scales"], a["y"], a["s"])

    assert call(kind=IDENT) == INVALID and call(kind=HAD) == INVALID     # only dense transforms are shared
    assert call(fmt=9) == UNSUPPORTED
    assert call(kind=7) == UNSUPPORTED                                    # kinds past WUSH_DIAG
    assert call(idx=None) == INVALID and call(idx=HALF) == INVALID and call(n_t=0) == INVALID
    assert call(t=None) == INVALID and call(t=ODD) == INVALID
    assert call(d_in=48) == INVALID                                       # not a multiple of b = 32
    assert call(dt=3) == UNSUPPORTED
    assert call(codes=ODD) == INVALID and call(scales=None) == INVALID and call(y=ODD) == INVALID
    assert call(fmt=NV, gs=0.0) == INVALID and call(fmt=NV, gs=float("nan")) == INVALID
    assert call(rows=0) == OK                                            # nothing to do, nothing launched
    assert call(rows=-1) == INVALID


def test_transform_quant_nvfp4_dynamic_and_amax():
    f = lib.wush_transform_quant_nvfp4_dynamic
    base = [P, BF16, 128, 256, P, WUSH, P2, None, P, P2, None, None]

    def call(i, v):
        a = list(base)
        a[i] = v
        return f(*a)

    assert call(6, None) == INVALID and call(6, HALF) == INVALID          # amax
    assert call(7, ODD) == INVALID                                        # global_scale_out alignment
    assert call(3, 40) == INVALID                                         # d_in % 16
    assert call(1, 7) == UNSUPPORTED
    assert call(4, None) == INVALID                                       # WUSH needs T
    assert call(8, ODD) == INVALID and call(9, None) == INVALID
    assert call(2, 0) == OK
    g = lib.wush_transform_amax
    assert g(P, BF16, 128, 256, P, WUSH, 8, P2, None) == UNSUPPORTED     # block 8
    assert g(P, BF16, 128, 256, P, WUSH, 32, None, None) == INVALID
    assert g(P, BF16, 128, 256, P, WUSH, 32, HALF, None) == INVALID
    assert g(P, BF16, 128, 256, None, DIAG, 16, P2, None) == INVALID
    assert g(P, BF16, 128, 48, None, IDENT, 32, P2, None) == INVALID      # d_in % block


def test_fp4_gemm():
    f = lib.wush_qgemm
    base = [P, P2, P, P2, 256, 256, 512, MX, 1.0, P, None]

    def call(i, v):
        a = list(base)
        a[i] = v
        return f(*a)

    assert call(7, I4) == UNSUPPORTED and call(7, 5) == UNSUPPORTED
    for i, v in ((4, 100), (5, 200), (6, 128), (4, 0), (6, -256)):        # M, N % 128; K % 256; > 0
        assert call(i, v) == INVALID, (i, v)
    assert call(4, 1 << 31) == UNSUPPORTED
    for i in (0, 1, 2, 3, 9):
        assert call(i, None) == INVALID and call(i, ODD) == INVALID, i
    g = lib.wush_qgemm_nvfp4_dynamic
    assert g(P, P2, P, P2, 256, 256, 512, None, 1.0, P, None) == INVALID
    assert g(P, P2, P, P2, 256, 256, 512, HALF, 1.0, P, None) == INVALID
    assert g(P, P2, P, P2, 100, 256, 512, P, 1.0, P, None) == INVALID


def test_int4_gemm():
    f = lib.wush_qgemm_int4
    assert f(P, P2, P, P2, 128, 128, 64, P, None) == INVALID              # N % 256
    assert f(P, P2, P, P2, 128, 256, 48, P, None) == INVALID              # K % 64
    assert f(P, HALF, P, P2, 128, 256, 64, P, None) == INVALID            # fp16 scales need 4-byte alignment
    assert f(P, P2, P, P2, 128, 256, 64, None, None) == INVALID
    assert f(P, P2, P, P2, 1 << 31, 256, 64, P, None) == UNSUPPORTED
    g = lib.wush_qgemm_int4_ws
    need = aq.wush_qgemm_int4_workspace_bytes(256, 256, 64)
    assert need == (256 + 256) * 64 * 2
    assert aq.wush_qgemm_int4_workspace_bytes(0, 256, 64) == 0
    assert g(P, P2, P, P2, 128, 256, 64, P, need, P, None) == INVALID    # M % 256 in the two-pass form
    assert g(P, P2, P, P2, 256, 256, 64, None, need, P, None) == INVALID
    assert g(P, P2, P, P2, 256, 256, 64, ODD, need, P, None) == INVALID
    assert g(P, ODD, P, P2, 256, 256, 64, P, need, P, None) == INVALID
    assert g(P, P2, P, P2, 256, 256, 64, P, need - 1, P, None) == TOO_SMALL


def test_itq3_gemv():
    f = lib.itq3_dequant_gemv
    base = [P, P2, P, 4, 256, 512, 0, None, P, None]

    def call(i, v):
        a = list(base)
        a[i] = v
        return f(*a)

    for i, v in ((3, 0), (3, 17), (4, 12), (4, 0), (5, 100), (5, 0)):    # tokens 1..16, d_out % 8, d_in % 256
        assert call(i, v) == INVALID, (i, v)
    assert call(6, 2) == UNSUPPORTED
    assert call(6, 1) == INVALID                                          # mode 1 needs a workspace
    for i in (0, 1, 2):
        assert call(i, None) == INVALID and call(i, ODD) == INVALID, i
    assert call(8, None) == INVALID
    g = lib.itq3_dequant_gemv_noalloc
    assert g(P, P2, P, 16, 256, 32768, P, None) == TOO_SMALL              # 524,288 floats of scratch
    assert g(P, P2, P, 4, 12, 512, P, None) == INVALID
    assert g(P, P2, None, 4, 256, 512, P, None) == INVALID


def test_debug_hooks_reject_out_of_range_values():
    assert lib.wush_debug_set_gemm_variant(3) == INVALID and lib.wush_debug_set_gemm_variant(-1) == INVALID
    assert lib.wush_debug_set_itq3_variant(4) == INVALID
    assert lib.wush_debug_set_wait_limit(-5) == INVALID
    assert lib.wush_status_string(-7) == b"file could not be opened, read or written"
    assert lib.wush_status_string(-99) == b"unknown status"
