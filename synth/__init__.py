"""Seeded synthetic inputs for the WUSH transform-then-quantize linear layer.

This module produces data only. It holds none of the method's arithmetic (no
transform, no rounding onto a quantisation grid, no GEMM), so both the CPU
oracle's tests and the CUDA path's tests and bench can draw the same inputs from
it without sharing any of the computation under test.

Generator
---------
Every stream is a counter-based splitmix64 sequence: element ``i`` of the stream
with seed ``s`` is ``mix64(s + (i + 1) * 0x9E3779B97F4A7C15)`` where ``mix64`` is
the splitmix64 finaliser (xor-shift 30, multiply 0xBF58476D1CE4E5B9, xor-shift
27, multiply 0x94D049BB133111EB, xor-shift 31).  A 64-bit draw becomes a uniform
in (0, 1) as ``((z >> 11) + 0.5) * 2**-53``.

Distributions (all in fp64):
  * Gaussian: Box-Muller on consecutive uniform pairs (cos and sin branches).
  * Student-t(nu): z / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared normals.
  * Laplace(0, 1): inverse CDF, -sign(u - 1/2) * ln(1 - 2|u - 1/2|).

Stream seeds follow ``0x5EED0000 + 16 * cfg + stream`` with stream 0 = the
evaluation activations, 1 = calibration activations, 2 = weights, 3 = the
outlier-channel choice, 4 = ITQ3 activations.

Workloads (the pages measure WUSH on Qwen3 layers and ITQ3_S on an LLM forward;
neither model is available, so these seeded stand-ins keep the shapes and the
outlier structure the pages describe -- a few input channels with much larger
magnitude than the rest):

  tiny          X fp32 [128 tok, 256], N(0,1), 4 channels x20; 512 calib tokens;
                W fp32 [256 out, 256 in] N(0, 0.02^2); MXFP4, block 32.
  up_proj       X bf16 [4096 tok, 4096] Student-t(3), 41 channels x50;
                8192 calib tokens; W bf16 [12288, 4096] N(0, 0.02^2); MXFP4.
  down_proj     X bf16 [4096 tok, 12288] Laplace(0,1), 61 channels x30;
                8192 calib tokens; W bf16 [4096, 12288] N(0, 0.02^2); NVFP4.
  int4          X bf16 [8192 tok (and 2048), 5120] Laplace, 51 channels x50;
                8192 calib tokens; W bf16 [17408, 5120] N(0, 0.02^2); INT4 g32.
  itq3          W fp16 [4096, 4096] Student-t(4) x 0.02; x fp16 [t, 4096] N(0,1),
                t in {1, 4, 16}.
"""
from __future__ import annotations

import dataclasses

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_X, STREAM_CALIB, STREAM_W, STREAM_OUTLIER, STREAM_ITQ3_X = 0, 1, 2, 3, 4


def seed_for(cfg: int, stream: int) -> int:
    return 0x5EED0000 + 16 * cfg + stream


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def raw64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """n consecutive 64-bit draws of the counter-based stream ``seed``."""
    with np.errstate(over="ignore"):
        ctr = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        return _mix64(np.uint64(seed) + ctr * _GAMMA)


def uniform(seed: int, n: int, offset: int = 0) -> np.ndarray:
    z = raw64(seed, n, offset)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """n standard normals (Box-Muller, fp64): normals offset .. offset+n-1 (offset even)."""
    if offset % 2:
        raise ValueError("normal stream offset must be even")
    m = (n + 1) // 2
    u = uniform(seed, 2 * m, offset)
    r = np.sqrt(-2.0 * np.log(u[0::2]))
    th = 2.0 * np.pi * u[1::2]
    out = np.empty(2 * m)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    return out[:n]


def student_t(seed: int, n: int, nu: int) -> np.ndarray:
    g = normal(seed, n * (nu + 1)).reshape(n, nu + 1)
    chi2 = np.sum(g[:, 1:] ** 2, axis=1)
    return g[:, 0] / np.sqrt(chi2 / nu)


def laplace(seed: int, n: int) -> np.ndarray:
    u = uniform(seed, n) - 0.5
    return -np.sign(u) * np.log1p(-2.0 * np.abs(u))


def outlier_channels(seed: int, d_in: int, count: int) -> np.ndarray:
    """A seeded set of ``count`` distinct channel indices in [0, d_in), sorted."""
    keys = uniform(seed, d_in)
    return np.sort(np.argsort(keys, kind="stable")[:count])


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round fp64 data to bf16 (fp64 -> fp32 -> bf16, each RNE); returned as fp32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def to_fp16_values(a: np.ndarray) -> np.ndarray:
    """Round fp64 data to fp16 (RNE); returned as fp32."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg: int              # index used in stream seeds
    tokens: int
    d_in: int
    d_out: int
    n_calib: int
    x_dist: str           # "normal" | "t3" | "laplace"
    n_outlier: int
    outlier_factor: float
    x_dtype: str          # "fp32" | "bf16"
    fmt: str              # "mxfp4" | "nvfp4" | "int4"
    block: int


WORKLOADS = {
    "tiny": Workload("tiny", 0, 128, 256, 256, 512, "normal", 4, 20.0, "fp32", "mxfp4", 32),
    "up_proj": Workload("up_proj", 1, 4096, 4096, 12288, 8192, "t3", 41, 50.0, "bf16", "mxfp4", 32),
    "down_proj": Workload("down_proj", 2, 4096, 12288, 4096, 8192, "laplace", 61, 30.0, "bf16", "nvfp4", 16),
    "int4": Workload("int4", 3, 8192, 5120, 17408, 8192, "laplace", 51, 50.0, "bf16", "int4", 32),
}


def _draw(dist: str, seed: int, n: int) -> np.ndarray:
    if dist == "normal":
        return normal(seed, n)
    if dist == "t3":
        return student_t(seed, n, 3)
    if dist == "laplace":
        return laplace(seed, n)
    raise ValueError(dist)


def activations(w: Workload, tokens: int | None = None, calib: bool = False,
                token_offset: int = 0) -> np.ndarray:
    """Activations X^T as [tokens, d_in] fp32 (bf16-valued for bf16 workloads).

    Rows ``token_offset .. token_offset + tokens`` of the workload's stream are
    returned, so a sample of rows equals the matching rows of the full matrix for
    the Gaussian and Laplace streams (the Student-t stream draws per element and
    is regenerated whole, then sliced).
    """
    t = (w.n_calib if calib else w.tokens) if tokens is None else tokens
    seed = seed_for(w.cfg, STREAM_CALIB if calib else STREAM_X)
    if w.x_dist == "t3":
        total = token_offset + t
        x = student_t(seed, total * w.d_in, 3).reshape(total, w.d_in)[token_offset:]
    elif w.x_dist == "normal":
        x = normal(seed, t * w.d_in, token_offset * w.d_in).reshape(t, w.d_in)
    else:
        u = uniform(seed, t * w.d_in, token_offset * w.d_in) - 0.5
        x = (-np.sign(u) * np.log1p(-2.0 * np.abs(u))).reshape(t, w.d_in)
    ch = outlier_channels(seed_for(w.cfg, STREAM_OUTLIER), w.d_in, w.n_outlier)
    x = x.copy()
    x[:, ch] *= w.outlier_factor
    if w.x_dtype == "bf16":
        return to_bf16_values(x)
    return x.astype(np.float32)


def weights(w: Workload) -> np.ndarray:
    """Weights W^T as [d_out, d_in] fp32 (bf16-valued for bf16 workloads), N(0, 0.02^2)."""
    g = normal(seed_for(w.cfg, STREAM_W), w.d_out * w.d_in).reshape(w.d_out, w.d_in) * 0.02
    if w.x_dtype == "bf16":
        return to_bf16_values(g)
    return g.astype(np.float32)


# ITQ3_S-style weight-only workload
ITQ3_CFG = 4
ITQ3_D_OUT = 4096
ITQ3_D_IN = 4096
ITQ3_TOKENS = (1, 4, 16)


def itq3_weights(d_out: int = ITQ3_D_OUT, d_in: int = ITQ3_D_IN) -> np.ndarray:
    """W as [d_out, d_in] fp16 values (returned as fp32): Student-t(4) x 0.02."""
    w = student_t(seed_for(ITQ3_CFG, STREAM_W), d_out * d_in, 4).reshape(d_out, d_in) * 0.02
    return to_fp16_values(w)


def itq3_activations(tokens: int, d_in: int = ITQ3_D_IN) -> np.ndarray:
    """x as [tokens, d_in] fp16 values (returned as fp32): N(0, 1)."""
    x = normal(seed_for(ITQ3_CFG, STREAM_ITQ3_X), tokens * d_in).reshape(tokens, d_in)
    return to_fp16_values(x)


def small_random(seed: int, shape, scale: float = 1.0) -> np.ndarray:
    """Generic seeded N(0, scale^2) fp64 array for small test cases."""
    n = int(np.prod(shape))
    return normal(seed, n).reshape(shape) * scale
