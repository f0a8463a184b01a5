"""Python binding of libwush.so: the B200 WUSH transform-then-quantize linear layer.

Argument marshalling only: every step of the path runs in the library (host
calibration in C++, everything else in sm_100a CUDA kernels).  Functions carry
the C names declared in include/wush.h; device buffers are torch CUDA tensors
(PyTorch provides memory and streams, nothing else), host buffers are numpy
arrays.  A missing library raises ImportError: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwush.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m activation_quantization_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

FORMATS = {"mxfp4": 0, "nvfp4": 1, "int4": 2}
TRANSFORMS = {"identity": 0, "hadamard": 1, "wus": 2, "wush": 3, "wush_diag": 4}
IN_BF16, IN_FP32 = 0, 1

_i64, _i32, _f32, _vp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

_SIGNATURES = {
    "wush_status_string": (ctypes.c_char_p, [_i32]),
    "wush_block_size": (_i32, [_i32]),
    "wush_calibrate": (_i32, [_vp, _i64, _vp, _i64, _i64, _i32, _i32, _vp, _vp]),
    "wush_calibrate_from_moments": (_i32, [_vp, _vp, _i64, _i32, _i32, _vp, _vp]),
    "wush_calibrate_shared": (_i32, [_vp, _i64, _vp, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp]),
    "wush_calibrate_shared_from_moments": (_i32, [_vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp, _vp]),
    "wush_save_transforms": (_i32, [ctypes.c_char_p, _i32, _i32, _i32, _i64, _vp, _vp, _vp, _i64]),
    "wush_transforms_file_info": (_i32, [ctypes.c_char_p, _vp, _vp, _vp, _vp, _vp, _vp]),
    "wush_load_transforms": (_i32, [ctypes.c_char_p, _vp, _vp, _i64, _vp, _i64]),
    "wush_nvfp4_global_scale": (_i32, [_f32, _vp]),
    "wush_nvfp4_alpha": (_i32, [_f32, _f32, _vp]),
    "wush_codes_bytes": (_sz, [_i64, _i64, _i32]),
    "wush_scales_bytes": (_sz, [_i64, _i64, _i32]),
    "wush_transform_quant": (_i32, [_vp, _i32, _i64, _i64, _vp, _i32, _i32, _f32, _vp, _vp, _vp, _vp]),
    "wush_transform_amax": (_i32, [_vp, _i32, _i64, _i64, _vp, _i32, _i32, _vp, _vp]),
    "wush_transform_quant_indexed": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _i32, _i32, _i32, _f32, _vp, _vp, _vp,
                                             _vp]),
    "wush_transform_quant_nvfp4_dynamic": (_i32, [_vp, _i32, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp]),
    "wush_qgemm": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _f32, _vp, _vp]),
    "wush_qgemm_nvfp4_dynamic": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _f32, _vp, _vp]),
    "wush_qgemm_int4": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "wush_qgemm_int4_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "wush_qgemm_int4_ws": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp, _vp]),
    "itq3_quantize_weights": (_i32, [_vp, _i64, _i64, _vp, _vp]),
    "itq3_dequant_gemv": (_i32, [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp, _vp]),
    "itq3_dequant_gemv_noalloc": (_i32, [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "wush_check_device_status": (_i32, [_vp]),
    "wush_debug_set_wait_limit": (_i32, [_i64]),
    "wush_debug_set_gemm_variant": (_i32, [_i32]),
    "wush_debug_set_itq3_variant": (_i32, [_i32]),
}

EXPORTED = []
for _name, (_res, _args) in _SIGNATURES.items():
    _fn = getattr(_lib, _name, None)
    if _fn is None:
        continue
    _fn.restype = _res
    _fn.argtypes = _args
    EXPORTED.append(_name)


WUSH_ERR_BUFFER_TOO_SMALL = -6


class WushError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str | None = None):
        self.status = status
        msg = f"{fn}: {_lib.wush_status_string(status).decode()} ({status})"
        super().__init__(msg + (f": {detail}" if detail else ""))


def _check(fn: str, status: int):
    if status != 0:
        raise WushError(fn, status)


def _enum(table, v):
    return table[v] if isinstance(v, str) else int(v)


def _ptr(t):
    """Device pointer of a torch tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _need(fn: str, name: str, t, nbytes: int, dtypes=None):
    """The C calls take bare pointers, so the binding checks what it can see: the
    element type (ValueError) and that ``t`` holds at least ``nbytes`` bytes
    (WushError with WUSH_ERR_BUFFER_TOO_SMALL).  None passes through to the
    library's own checks."""
    if t is None:
        return
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{fn}: {name} must be {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise WushError(fn, WUSH_ERR_BUFFER_TOO_SMALL, f"{name} holds {have} bytes, needs {nbytes}")


def _quant_outputs_ok(fn, rows, d_in, fmt, kind, t, codes, scales, y_debug, n_t=None):
    import torch
    f = _enum(FORMATS, fmt)
    b = _lib.wush_block_size(f)
    if b > 0 and _enum(TRANSFORMS, kind) >= TRANSFORMS["wus"]:
        count = n_t if n_t is not None else d_in // b
        _need(fn, "t", t, count * b * b * 4, (torch.float32,))
    _need(fn, "codes", codes, wush_codes_bytes(rows, d_in, f))
    _need(fn, "scales", scales, wush_scales_bytes(rows, d_in, f))
    _need(fn, "y_debug", y_debug, rows * d_in * 4, (torch.float32,))


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _host(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


# --------------------------------------------------------------------------- host

def wush_block_size(fmt) -> int:
    return _lib.wush_block_size(_enum(FORMATS, fmt))


def wush_calibrate(x_calib: np.ndarray, w: np.ndarray, block: int, kind):
    """(t_x, t_w) fp32 [d_in/block, block, block] from calibration tokens [n, d_in] and W^T [d_out, d_in]."""
    x, xp = _host(x_calib, np.float32)
    wt, wp = _host(w, np.float32)
    d_in = x.shape[1]
    if wt.shape[1] != d_in:
        raise ValueError("d_in mismatch")
    tx = np.empty((d_in // block, block, block), np.float32)
    tw = np.empty_like(tx)
    _check("wush_calibrate", _lib.wush_calibrate(xp, x.shape[0], wp, wt.shape[0], d_in, block,
                                                 _enum(TRANSFORMS, kind), tx.ctypes.data, tw.ctypes.data))
    return tx, tw


def wush_calibrate_shared(x_calib: np.ndarray, w: np.ndarray, block: int, kind, groups: int):
    """(t_x, t_w) fp32 [groups, block, block] and the block -> group index int32 [d_in/block]."""
    x, xp = _host(x_calib, np.float32)
    wt, wp = _host(w, np.float32)
    d_in = x.shape[1]
    if wt.shape[1] != d_in:
        raise ValueError("d_in mismatch")
    tx = np.empty((groups, block, block), np.float32)
    tw = np.empty_like(tx)
    index = np.empty(d_in // block, np.int32)
    _check("wush_calibrate_shared",
           _lib.wush_calibrate_shared(xp, x.shape[0], wp, wt.shape[0], d_in, block, _enum(TRANSFORMS, kind),
                                      int(groups), tx.ctypes.data, tw.ctypes.data, index.ctypes.data))
    return tx, tw, index


SIGMA_NORMS = {"unknown": 0, "mean": 1}


def wush_save_transforms(path, t_x: np.ndarray, t_w: np.ndarray, kind, index: np.ndarray | None = None,
                         sigma_norm="mean"):
    """Write fp32 T_X, T_W [n_t, b, b] (and the block -> transform index, if given) to ``path``.

    ``sigma_norm`` "mean" is the normalisation of wush_calibrate*; "unknown" marks other transforms."""
    tx, txp = _host(t_x, np.float32)
    tw, twp = _host(t_w, np.float32)
    if tx.ndim != 3 or tx.shape != tw.shape or tx.shape[1] != tx.shape[2]:
        raise ValueError("t_x and t_w must both be [n_t, b, b]")
    ip, n_blocks = None, 0
    if index is not None:
        idx, ip = _host(index, np.int32)
        n_blocks = idx.size
    _check("wush_save_transforms",
           _lib.wush_save_transforms(os.fsencode(path), tx.shape[1], _enum(TRANSFORMS, kind),
                                     _enum(SIGMA_NORMS, sigma_norm), tx.shape[0], txp, twp, ip, n_blocks))


def wush_transforms_file_info(path) -> dict:
    """Header of a transforms file: block, kind, sigma_norm, n_t, n_blocks, has_index."""
    b, k, sn, hi = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    nt, nb = ctypes.c_int64(), ctypes.c_int64()
    _check("wush_transforms_file_info",
           _lib.wush_transforms_file_info(os.fsencode(path), ctypes.byref(b), ctypes.byref(k), ctypes.byref(sn),
                                          ctypes.byref(nt), ctypes.byref(nb), ctypes.byref(hi)))
    return {"block": b.value, "kind": k.value, "sigma_norm": sn.value, "n_t": nt.value, "n_blocks": nb.value,
            "has_index": bool(hi.value)}


def wush_load_transforms(path):
    """(t_x, t_w, index or None, kind) from a file written by wush_save_transforms."""
    info = wush_transforms_file_info(path)
    b, nt = info["block"], info["n_t"]
    tx = np.empty((nt, b, b), np.float32)
    tw = np.empty_like(tx)
    index = np.empty(info["n_blocks"], np.int32) if info["has_index"] else None
    _check("wush_load_transforms",
           _lib.wush_load_transforms(os.fsencode(path), tx.ctypes.data, tw.ctypes.data, tx.size,
                                     None if index is None else index.ctypes.data,
                                     0 if index is None else index.size))
    return tx, tw, index, info["kind"]


def wush_calibrate_shared_from_moments(sigma_x: np.ndarray, sigma_w: np.ndarray, kind, groups: int):
    sx, sxp = _host(sigma_x, np.float64)
    sw, swp = _host(sigma_w, np.float64)
    nb, b, _ = sx.shape
    tx = np.empty((groups, b, b), np.float32)
    tw = np.empty_like(tx)
    index = np.empty(nb, np.int32)
    _check("wush_calibrate_shared_from_moments",
           _lib.wush_calibrate_shared_from_moments(sxp, swp, nb * b, b, _enum(TRANSFORMS, kind), int(groups),
                                                   tx.ctypes.data, tw.ctypes.data, index.ctypes.data))
    return tx, tw, index


def wush_calibrate_from_moments(sigma_x: np.ndarray, sigma_w: np.ndarray, kind):
    sx, sxp = _host(sigma_x, np.float64)
    sw, swp = _host(sigma_w, np.float64)
    nb, b, _ = sx.shape
    tx = np.empty((nb, b, b), np.float32)
    tw = np.empty_like(tx)
    _check("wush_calibrate_from_moments",
           _lib.wush_calibrate_from_moments(sxp, swp, nb * b, b, _enum(TRANSFORMS, kind),
                                            tx.ctypes.data, tw.ctypes.data))
    return tx, tw


def itq3_quantize_weights(w_fp16: np.ndarray):
    """(packed codes uint8 [d_out * d_in * 3 / 8], scales fp16 [d_out, d_in/256]) from fp16 W [d_out, d_in]."""
    w, wp = _host(w_fp16, np.float16)
    d_out, d_in = w.shape
    codes = np.empty(d_out * d_in * 3 // 8, np.uint8)
    scales = np.empty((d_out, d_in // 256), np.float16)
    _check("itq3_quantize_weights",
           _lib.itq3_quantize_weights(wp, d_out, d_in, codes.ctypes.data, scales.ctypes.data))
    return codes, scales


# --------------------------------------------------------------------------- device

def wush_nvfp4_global_scale(amax: float) -> float:
    """Static NVFP4 per-tensor scale s_g = fp32(amax / 2688) (1 for an all-zero tensor)."""
    out = ctypes.c_float()
    _check("wush_nvfp4_global_scale", _lib.wush_nvfp4_global_scale(float(amax), ctypes.byref(out)))
    return out.value


def wush_nvfp4_alpha(s_gx: float, s_gw: float) -> float:
    """The NVFP4 GEMM's alpha = fp32(s_gx * s_gw)."""
    out = ctypes.c_float()
    _check("wush_nvfp4_alpha", _lib.wush_nvfp4_alpha(float(s_gx), float(s_gw), ctypes.byref(out)))
    return out.value


def wush_codes_bytes(rows: int, d_in: int, fmt) -> int:
    return _lib.wush_codes_bytes(rows, d_in, _enum(FORMATS, fmt))


def wush_scales_bytes(rows: int, d_in: int, fmt) -> int:
    return _lib.wush_scales_bytes(rows, d_in, _enum(FORMATS, fmt))


def alloc_quant_outputs(rows: int, d_in: int, fmt, device="cuda"):
    """Empty (codes, scales) uint8 CUDA tensors sized for wush_transform_quant."""
    import torch
    codes = torch.empty(wush_codes_bytes(rows, d_in, fmt), dtype=torch.uint8, device=device)
    scales = torch.empty(max(wush_scales_bytes(rows, d_in, fmt), 16), dtype=torch.uint8, device=device)
    return codes, scales


def wush_transform_quant(x, t, kind, fmt, codes, scales, global_scale: float = 0.0, y_debug=None,
                         stream=None):
    """x: CUDA [rows, d_in] bf16 or fp32; t: CUDA fp32 [d_in/b, b, b] or None."""
    import torch
    x_dtype = IN_FP32 if x.dtype == torch.float32 else IN_BF16
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("x must be bf16 or fp32")
    rows, d_in = x.shape
    _quant_outputs_ok("wush_transform_quant", rows, d_in, fmt, kind, t, codes, scales, y_debug)
    _check("wush_transform_quant",
           _lib.wush_transform_quant(_ptr(x), x_dtype, rows, d_in, _ptr(t), _enum(TRANSFORMS, kind),
                                     _enum(FORMATS, fmt), float(global_scale), _ptr(codes), _ptr(scales),
                                     _ptr(y_debug), _stream(stream)))


def wush_transform_quant_indexed(x, t, t_index, kind, fmt, codes, scales, global_scale: float = 0.0, y_debug=None,
                                 stream=None):
    """wush_transform_quant with shared transforms: t CUDA fp32 [n_t, b, b], t_index CUDA int32 [d_in/b]."""
    import torch
    x_dtype = IN_FP32 if x.dtype == torch.float32 else IN_BF16
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("x must be bf16 or fp32")
    rows, d_in = x.shape
    b = _lib.wush_block_size(_enum(FORMATS, fmt))
    _quant_outputs_ok("wush_transform_quant_indexed", rows, d_in, fmt, kind, t, codes, scales, y_debug,
                      n_t=int(t.shape[0]))
    _need("wush_transform_quant_indexed", "t_index", t_index, max(d_in // max(b, 1), 0) * 4, (torch.int32,))
    _check("wush_transform_quant_indexed",
           _lib.wush_transform_quant_indexed(_ptr(x), x_dtype, rows, d_in, _ptr(t), _ptr(t_index), int(t.shape[0]),
                                             _enum(TRANSFORMS, kind), _enum(FORMATS, fmt), float(global_scale),
                                             _ptr(codes), _ptr(scales), _ptr(y_debug), _stream(stream)))


def wush_transform_amax(x, t, kind, block: int, amax_out, stream=None):
    import torch
    x_dtype = IN_FP32 if x.dtype == torch.float32 else IN_BF16
    rows, d_in = x.shape
    if _enum(TRANSFORMS, kind) >= TRANSFORMS["wus"] and block > 0:
        _need("wush_transform_amax", "t", t, (d_in // block) * block * block * 4, (torch.float32,))
    _need("wush_transform_amax", "amax_out", amax_out, 4, (torch.float32,))
    _check("wush_transform_amax",
           _lib.wush_transform_amax(_ptr(x), x_dtype, rows, d_in, _ptr(t), _enum(TRANSFORMS, kind), block,
                                    _ptr(amax_out), _stream(stream)))


def wush_transform_quant_nvfp4_dynamic(x, t, kind, amax, codes, scales, global_scale_out=None, y_debug=None,
                                       stream=None):
    """NVFP4 transform + quantisation whose per-tensor scale is derived on the device from
    ``amax`` (a CUDA fp32 scalar, e.g. from wush_transform_amax); the scale is written to
    ``global_scale_out`` (CUDA fp32 scalar) if given."""
    import torch
    x_dtype = IN_FP32 if x.dtype == torch.float32 else IN_BF16
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("x must be bf16 or fp32")
    rows, d_in = x.shape
    fn = "wush_transform_quant_nvfp4_dynamic"
    _quant_outputs_ok(fn, rows, d_in, "nvfp4", kind, t, codes, scales, y_debug)
    _need(fn, "amax", amax, 4, (torch.float32,))
    _need(fn, "global_scale_out", global_scale_out, 4, (torch.float32,))
    _check("wush_transform_quant_nvfp4_dynamic",
           _lib.wush_transform_quant_nvfp4_dynamic(_ptr(x), x_dtype, rows, d_in, _ptr(t), _enum(TRANSFORMS, kind),
                                                   _ptr(amax), _ptr(global_scale_out), _ptr(codes), _ptr(scales),
                                                   _ptr(y_debug), _stream(stream)))


def wush_qgemm_nvfp4_dynamic(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int, a_global_scale,
                             b_global_scale: float, y, stream=None):
    """NVFP4 GEMM with alpha = *a_global_scale (CUDA fp32 scalar) * b_global_scale, formed on the device."""
    import torch
    _gemm_operands_ok("wush_qgemm_nvfp4_dynamic", a_codes, a_scales, b_codes, b_scales, M, N, K, "nvfp4", y)
    _need("wush_qgemm_nvfp4_dynamic", "a_global_scale", a_global_scale, 4, (torch.float32,))
    _check("wush_qgemm_nvfp4_dynamic",
           _lib.wush_qgemm_nvfp4_dynamic(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K,
                                         _ptr(a_global_scale), float(b_global_scale), _ptr(y), _stream(stream)))


def _gemm_operands_ok(fn, a_codes, a_scales, b_codes, b_scales, M, N, K, fmt, y):
    import torch
    if M <= 0 or N <= 0 or K <= 0:
        return                                      # the library rejects the shape
    f = _enum(FORMATS, fmt)
    _need(fn, "a_codes", a_codes, M * K // 2)
    _need(fn, "b_codes", b_codes, N * K // 2)
    _need(fn, "a_scales", a_scales, wush_scales_bytes(M, K, f))
    _need(fn, "b_scales", b_scales, wush_scales_bytes(N, K, f))
    _need(fn, "y", y, M * N * 4, (torch.float32,))


def wush_qgemm(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int, fmt, alpha: float, y,
               stream=None):
    _gemm_operands_ok("wush_qgemm", a_codes, a_scales, b_codes, b_scales, M, N, K, fmt, y)
    _check("wush_qgemm",
           _lib.wush_qgemm(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K,
                           _enum(FORMATS, fmt), float(alpha), _ptr(y), _stream(stream)))


def wush_qgemm_int4(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int, y, stream=None):
    _gemm_operands_ok("wush_qgemm_int4", a_codes, a_scales, b_codes, b_scales, M, N, K, "int4", y)
    _check("wush_qgemm_int4",
           _lib.wush_qgemm_int4(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K, _ptr(y),
                                _stream(stream)))


def wush_qgemm_int4_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(_lib.wush_qgemm_int4_workspace_bytes(M, N, K))


def wush_qgemm_int4_ws(a_codes, a_scales, b_codes, b_scales, M: int, N: int, K: int, workspace, y, stream=None):
    """workspace: CUDA tensor of at least wush_qgemm_int4_workspace_bytes(M, N, K) bytes."""
    _gemm_operands_ok("wush_qgemm_int4_ws", a_codes, a_scales, b_codes, b_scales, M, N, K, "int4", y)
    nbytes = workspace.numel() * workspace.element_size()
    _check("wush_qgemm_int4_ws",
           _lib.wush_qgemm_int4_ws(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), M, N, K,
                                   _ptr(workspace), nbytes, _ptr(y), _stream(stream)))

def _itq3_operands_ok(fn, codes, scales, x, d_out, y, workspace=None):
    import torch
    tokens, d_in = x.shape
    _need(fn, "x", x, 0, (torch.float16,))
    if d_out <= 0 or d_in <= 0:
        return                                      # the library rejects the shape
    _need(fn, "codes", codes, d_out * d_in * 3 // 8)
    _need(fn, "scales", scales, d_out * (d_in // 256) * 2)
    _need(fn, "y", y, tokens * d_out * 4, (torch.float32,))
    _need(fn, "workspace", workspace, tokens * d_in * 4, (torch.float32,))


def itq3_dequant_gemv(codes, scales, x, d_out: int, mode: int, y, workspace=None, stream=None):
    tokens, d_in = x.shape
    _itq3_operands_ok("itq3_dequant_gemv", codes, scales, x, d_out, y, workspace if int(mode) == 1 else None)
    _check("itq3_dequant_gemv",
           _lib.itq3_dequant_gemv(_ptr(codes), _ptr(scales), _ptr(x), tokens, d_out, d_in, int(mode),
                                  _ptr(workspace), _ptr(y), _stream(stream)))


def itq3_dequant_gemv_noalloc(codes, scales, x, d_out: int, y, stream=None):
    """Mode-1 ITQ3 GEMV with the library's fixed scratch instead of a workspace."""
    tokens, d_in = x.shape
    _itq3_operands_ok("itq3_dequant_gemv_noalloc", codes, scales, x, d_out, y)
    _check("itq3_dequant_gemv_noalloc",
           _lib.itq3_dequant_gemv_noalloc(_ptr(codes), _ptr(scales), _ptr(x), tokens, d_out, d_in, _ptr(y),
                                          _stream(stream)))


def wush_check_device_status(stream=None) -> int:
    return _lib.wush_check_device_status(_stream(stream))


def wush_debug_set_gemm_variant(variant: int):
    _check("wush_debug_set_gemm_variant", _lib.wush_debug_set_gemm_variant(int(variant)))


def wush_debug_set_itq3_variant(variant: int):
    _check("wush_debug_set_itq3_variant", _lib.wush_debug_set_itq3_variant(int(variant)))


def wush_debug_set_wait_limit(max_polls: int):
    _check("wush_debug_set_wait_limit", _lib.wush_debug_set_wait_limit(int(max_polls)))
