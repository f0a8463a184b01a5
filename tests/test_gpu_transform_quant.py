"""GPU parity: wush_transform_quant against the oracle, element by element.

Codes and scales are bit-exact except where the oracle's pre-rounding value sits
within 1e-6 (relative to the magnitude of the terms that form it) of a rounding
boundary; those are counted and bounded (tests/parity.py).  Transformed values
agree within 1e-5 of that magnitude.
"""
import functools

import numpy as np
import pytest

import synth
from oracle import calibrate as C
from oracle import transforms as T
from tests import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

FMT_WORKLOAD = {"mxfp4": "up_proj", "nvfp4": "down_proj", "int4": "int4"}


@functools.lru_cache(maxsize=None)
def _calib_inputs(name, n_calib):
    w = synth.WORKLOADS[name]
    return synth.activations(w, tokens=n_calib, calib=True), synth.weights(w)[:2048]


@functools.lru_cache(maxsize=None)
def _transform_cached(kind, fmt, name, n_calib):
    w = synth.WORKLOADS[name]
    b = P.Q.BLOCK[fmt]
    if kind in ("identity", "hadamard"):
        return (T.identity_blocks(w.d_in, b) if kind == "identity" else T.hadamard_blocks(w.d_in, b)).astype(np.float32)
    xc, wt = _calib_inputs(name, n_calib)
    tx, _ = C.calibrate(xc, wt, b, kind)
    return tx.astype(np.float32)


def _transform(kind, fmt, w, n_calib=1024):
    return _transform_cached(kind, fmt, w.name, n_calib)


def _global_scale(x, t, fmt):
    if fmt != "nvfp4":
        return 0.0
    return float(C.nvfp4_global_scale(T.apply_block_transform(x, t).astype(np.float32)))


def _as_input(x, bf16):
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, np.float32))


def run_gpu_t(lib, xt_cpu, t, kind, fmt, gs):
    rows, d_in = xt_cpu.shape
    xt = xt_cpu.cuda()
    tt = None if kind in ("identity", "hadamard") else torch.from_numpy(t).cuda()
    codes, scales = lib.alloc_quant_outputs(rows, d_in, fmt)
    y = torch.empty((rows, d_in), dtype=torch.float32, device="cuda")
    lib.wush_transform_quant(xt, tt, kind, fmt, codes, scales, gs, y)
    torch.cuda.synchronize()
    return (P.unpack_nibbles(codes.cpu().numpy(), rows, d_in),
            P.decode_scales(scales.cpu().numpy(), rows, d_in, fmt), y.cpu().numpy())


@pytest.mark.parametrize("kind", ["identity", "hadamard", "wus", "wush", "wush_diag"])
def test_tiny_fp32_mxfp4(lib, kind):
    w = synth.WORKLOADS["tiny"]
    x = synth.activations(w)
    t = _transform(kind, "mxfp4", w, n_calib=512)
    c, s, y = run_gpu_t(lib, _as_input(x, False), t, kind, "mxfp4", 0.0)
    out = P.compare_transform_quant(x, t, "mxfp4", None, c, s, y)
    assert out["elements"] == x.size


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
@pytest.mark.parametrize("kind", ["identity", "hadamard", "wus", "wush", "wush_diag"])
def test_ragged_rows_bf16(lib, fmt, kind):
    # 300 rows: two full 128-row tiles and a ragged tail; the full d_in of the workload
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    x = synth.activations(w, tokens=300)
    t = _transform(kind, fmt, w)
    gs = _global_scale(x, t, fmt)
    c, s, y = run_gpu_t(lib, _as_input(x, True), t, kind, fmt, gs)
    P.compare_transform_quant(x, t, fmt, gs, c, s, y)


def _run_raw(lib, x, t, kind, fmt, gs):
    """bf16 x through wush_transform_quant: (codes, raw scale buffer, y) on the host;
    the scale buffer is poisoned first, so every byte left in it was written."""
    rows, d_in = x.shape
    xt = _as_input(x, True).cuda()
    tt = None if kind in ("identity", "hadamard") else torch.from_numpy(np.ascontiguousarray(t)).cuda()
    codes, scales = lib.alloc_quant_outputs(rows, d_in, fmt)
    scales.fill_(0x5A)
    y = torch.empty((rows, d_in), dtype=torch.float32, device="cuda")
    lib.wush_transform_quant(xt, tt, kind, fmt, codes, scales, gs, y)
    torch.cuda.synchronize()
    assert lib.wush_check_device_status() == 0
    return P.unpack_nibbles(codes.cpu().numpy(), rows, d_in), scales.cpu().numpy(), y.cpu().numpy()


@pytest.mark.parametrize("fmt, d_in", [("mxfp4", 160), ("nvfp4", 176), ("nvfp4", 48), ("int4", 224)])
@pytest.mark.parametrize("kind", ["identity", "hadamard", "wush"])
def test_ragged_columns_bf16(lib, fmt, d_in, kind):
    # d_in not a multiple of the 128-column tile (d_in = 48 is even narrower than
    # one TMA box): the tensor-core kernel's last tile column reaches past the end of
    # X, which the TMA fills with zeros.  Blocks are independent, so every real block
    # must come out bit for bit as in the same rows zero-padded to whole tiles (a
    # path the other tests check against the oracle); blocks beyond d_in must write
    # no codes, and the scale atoms' padding must be written as zero.  Identity and
    # Hadamard, exact on both sides, are also checked against the oracle directly.
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    b = P.Q.BLOCK[fmt]
    x = np.ascontiguousarray(synth.activations(w, tokens=200)[:, :d_in])
    rows, nb = x.shape[0], d_in // b
    d_pad = (d_in + 127) // 128 * 128
    if kind == "identity":
        t, t_pad = T.identity_blocks(d_in, b), T.identity_blocks(d_pad, b)
    elif kind == "hadamard":
        t, t_pad = T.hadamard_blocks(d_in, b), T.hadamard_blocks(d_pad, b)
    else:
        xc, wt = _calib_inputs(w.name, 1024)
        t = C.calibrate(xc[:, :d_in], wt[:, :d_in], b, kind)[0]
        t_pad = np.concatenate([t, T.identity_blocks(d_pad - d_in, b)])
    t, t_pad = t.astype(np.float32), t_pad.astype(np.float32)
    gs = _global_scale(x, t, fmt)
    c, raw, y = _run_raw(lib, x, t, kind, fmt, gs)
    x_pad = np.zeros((rows, d_pad), np.float32)
    x_pad[:, :d_in] = x
    c_pad, raw_pad, y_pad = _run_raw(lib, x_pad, t_pad, kind, fmt, gs)
    assert np.array_equal(c, c_pad[:, :d_in])
    assert np.array_equal(P.decode_scales(raw, rows, d_in, fmt), P.decode_scales(raw_pad, rows, d_pad, fmt)[:, :nb])
    assert np.array_equal(y, y_pad[:, :d_in])
    if fmt != "int4":
        full = P.unswizzle_scales(raw, (rows + 127) // 128 * 128, (nb + 3) // 4 * 4)
        assert not full[rows:, :].any() and not full[:, nb:].any()
    if kind != "wush":
        P.compare_transform_quant(x, t, fmt, gs if fmt == "nvfp4" else None, c,
                                  P.decode_scales(raw, rows, d_in, fmt), y)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_partial_scale_atom_and_special_values(lib, fmt):
    # d_in = 3 blocks (a partial 4-column scale atom), 5 rows; zero blocks, tiny and
    # huge values, negative values that round to -0, exact grid values
    b = P.Q.BLOCK[fmt]
    d_in = 3 * b
    x = synth.small_random(11, (5, d_in)).astype(np.float32)
    x[0, :b] = 0.0
    x[1, :b] = -1e-30
    x[1, 3] = 1.0
    x[2, b:2 * b] *= 1e4 if fmt == "int4" else 1e20
    x[3, :] = np.array([0.0, 0.5, 1, 1.5, 2, 3, 4, 6] * (d_in // 8), np.float32)
    x[4, 2 * b:] = -x[4, 2 * b:] * 1e-12
    t = T.identity_blocks(d_in, b).astype(np.float32)
    gs = 1e-3 if fmt == "nvfp4" else 0.0
    c, s, y = run_gpu_t(lib, _as_input(x, False), t, "identity", fmt, gs)
    P.compare_transform_quant(x, t, fmt, gs if fmt == "nvfp4" else None, c, s, y)
    if fmt == "mxfp4":
        assert s[0, 0] == 0 and np.all(c[0, :b] == 0)


def test_dense_path_matches_hadamard_path(lib):
    # the WUS code path fed H/sqrt(b) must agree with the butterfly path
    w = synth.WORKLOADS["up_proj"]
    x = synth.activations(w, tokens=256)
    t = T.hadamard_blocks(w.d_in, 32).astype(np.float32)
    c1, s1, y1 = run_gpu_t(lib, _as_input(x, True), t, "wus", "mxfp4", 0.0)
    P.compare_transform_quant(x, t, "mxfp4", None, c1, s1, y1)
    c2, s2, y2 = run_gpu_t(lib, _as_input(x, True), t, "hadamard", "mxfp4", 0.0)
    mag = P.magnitude(x, t)
    assert np.all(np.abs(y1 - y2) <= 2e-6 * mag)


def test_empty_rows_is_noop(lib):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros(16, dtype=torch.uint8, device="cuda")
    lib.wush_transform_quant(x, None, "identity", "mxfp4", codes, codes)
    torch.cuda.synchronize()
    assert int(codes.sum()) == 0


@pytest.mark.parametrize("kind", ["identity", "hadamard", "wush"])
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_amax_matches_oracle(lib, kind, fmt):
    # bf16 x runs the tensor-core kernel's amax mode, fp32 x the one-row-per-thread
    # kernel; 300 rows leave a ragged row tile, whose padding rows must not count
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    x = synth.activations(w, tokens=300)
    t = _transform(kind, fmt, w)
    tt = None if kind in ("identity", "hadamard") else torch.from_numpy(t).cuda()
    want = np.max(np.abs(T.apply_block_transform(x, t)))
    for bf16 in (True, False):
        out = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        lib.wush_transform_amax(_as_input(x, bf16).cuda(), tt, kind, P.Q.BLOCK[fmt], out)
        torch.cuda.synchronize()
        assert abs(float(out.item()) - want) <= 1e-5 * want, (bf16, float(out.item()), want)


@pytest.mark.parametrize("fmt, d_in", [("nvfp4", 176), ("mxfp4", 160), ("nvfp4", 48)])
@pytest.mark.parametrize("kind", ["hadamard", "wush"])
def test_amax_ragged_columns(lib, fmt, d_in, kind):
    # the amax mode over a last tile column that reaches past the end of X (TMA zero
    # fill), for both kernels
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    b = P.Q.BLOCK[fmt]
    x = np.ascontiguousarray(synth.activations(w, tokens=200)[:, :d_in])
    if kind == "hadamard":
        t = T.hadamard_blocks(d_in, b).astype(np.float32)
    else:
        xc, wt = _calib_inputs(w.name, 1024)
        t = C.calibrate(xc[:, :d_in], wt[:, :d_in], b, kind)[0].astype(np.float32)
    tt = None if kind == "hadamard" else torch.from_numpy(t).cuda()
    want = np.max(np.abs(T.apply_block_transform(x, t)))
    for bf16 in (True, False):
        out = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        lib.wush_transform_amax(_as_input(x, bf16).cuda(), tt, kind, b, out)
        torch.cuda.synchronize()
        assert lib.wush_check_device_status() == 0
        assert abs(float(out.item()) - want) <= 1e-5 * want, (bf16, float(out.item()), want)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_full_size_sampled_rows(lib, fmt):
    # the bench's launch configuration (full workload, WUSH), oracle on sampled rows
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    x = synth.activations(w)
    t = _transform("wush", fmt, w)
    gs = _global_scale(x[:512], t, fmt) * 1.5
    c, s, y = run_gpu_t(lib, _as_input(x, True), t, "wush", fmt, gs)
    rng = np.random.default_rng(5)
    sel = np.unique(np.concatenate([rng.integers(0, w.tokens, 96), [0, w.tokens - 1]]))
    P.compare_transform_quant(x, t, fmt, gs if fmt == "nvfp4" else None, c, s, y, rows_sel=sel)
    # properties over every block: MXFP4 scale rule amax / 2^e in [4, 8)
    if fmt == "mxfp4":
        yb = np.abs(y.reshape(w.tokens, -1, 32)).max(axis=2)
        e = s.astype(np.int64) - 127
        r = yb / np.ldexp(1.0, e)
        assert np.all((r >= 4) & (r < 8) | (yb == 0))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
@pytest.mark.parametrize("kind", ["identity", "hadamard", "wush"])
def test_full_size_ring_repeatable(lib, kind, fmt):
    # At the full sizes each CTA walks a long run of shared-memory stages and TMEM
    # slots (about 20 tiles per CTA at the NVFP4 size); identity and Hadamard read X
    # straight from the ring, WUSH from the tensor cores.  Three launches in a row
    # must agree bit for bit, and sampled rows must match the oracle.
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    x = synth.activations(w)
    t = _transform(kind, fmt, w)
    gs = _global_scale(x[:512], t, fmt) * 1.5
    xt = _as_input(x, True).cuda()
    tt = None if kind in ("identity", "hadamard") else torch.from_numpy(t).cuda()
    outs = []
    for _ in range(3):
        codes, scales = lib.alloc_quant_outputs(w.tokens, w.d_in, fmt)
        lib.wush_transform_quant(xt, tt, kind, fmt, codes, scales, gs)
        outs.append((codes, scales))
    torch.cuda.synchronize()
    assert lib.wush_check_device_status() == 0
    for codes, scales in outs[1:]:
        assert torch.equal(codes, outs[0][0]) and torch.equal(scales, outs[0][1])
    c = P.unpack_nibbles(outs[0][0].cpu().numpy(), w.tokens, w.d_in)
    s = P.decode_scales(outs[0][1].cpu().numpy(), w.tokens, w.d_in, fmt)
    rng = np.random.default_rng(11)
    sel = np.unique(np.concatenate([rng.integers(0, w.tokens, 48), [0, w.tokens - 1]]))
    P.compare_transform_quant(x, t, fmt, gs if fmt == "nvfp4" else None, c, s, None, rows_sel=sel)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
@pytest.mark.parametrize("bf16", [True, False])
def test_indexed_transforms_equal_expanded(lib, fmt, bf16):
    # shared transforms (4 groups of similar blocks) through the index map give the
    # same codes and scales as the same transforms expanded to one per block; two
    # planted out-of-range entries are clamped to the first and last transform
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    b = P.Q.BLOCK[fmt]
    x = synth.activations(w, tokens=300)
    xc, wt = _calib_inputs(w.name, 1024)
    tx, _, idx = C.shared_transforms(C.block_moments(xc, b), C.block_moments(wt, b), "wush", 4)
    ts = tx.astype(np.float32)
    idx = idx.astype(np.int32)
    idx[0], idx[-1] = -3, 99
    t_full = ts[np.clip(idx, 0, len(ts) - 1)]
    gs = _global_scale(x, t_full, fmt)
    xt = _as_input(x, bf16).cuda()
    rows, d_in = x.shape
    c1, s1 = lib.alloc_quant_outputs(rows, d_in, fmt)
    c2, s2 = lib.alloc_quant_outputs(rows, d_in, fmt)
    lib.wush_transform_quant_indexed(xt, torch.from_numpy(ts).cuda(), torch.from_numpy(idx).cuda(), "wush", fmt,
                                     c1, s1, gs)
    lib.wush_transform_quant(xt, torch.from_numpy(t_full).cuda(), "wush", fmt, c2, s2, gs)
    torch.cuda.synchronize()
    assert lib.wush_check_device_status() == 0
    assert torch.equal(c1, c2) and torch.equal(s1, s2)
    P.compare_transform_quant(x, t_full, fmt, gs if fmt == "nvfp4" else None,
                              P.unpack_nibbles(c1.cpu().numpy(), rows, d_in), P.decode_scales(s1.cpu().numpy(), rows, d_in, fmt))


def test_indexed_transform_rejects_non_dense_kinds(lib):
    xt = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    t = torch.zeros((1, 32, 32), dtype=torch.float32, device="cuda")
    idx = torch.zeros(8, dtype=torch.int32, device="cuda")
    codes, scales = lib.alloc_quant_outputs(128, 256, "mxfp4")
    for kind in ("identity", "hadamard"):
        with pytest.raises(lib.WushError):
            lib.wush_transform_quant_indexed(xt, t, idx, kind, "mxfp4", codes, scales)


def _near_tie_rows(fmt, rng, rows=64):
    """fp32 rows whose quotients sit on, and one fp32 ulp either side of, element
    and scale rounding boundaries (the cases where a reciprocal-multiply order would
    round differently from the exact quotient); with the identity transform both
    sides see the same fp32 values, so every code and scale must match exactly."""
    from oracle import formats as F
    b = P.Q.BLOCK[fmt]
    out = np.zeros((rows, 4 * b), np.float32)
    gs = np.float32(0.0123)
    for r in range(rows):
        for j in range(4):
            if fmt == "nvfp4":
                sbv = float(rng.choice(F.E4M3_GRID[40:110]))
                d = sbv * float(gs)
                mids = (F.E2M1_GRID[:-1] + F.E2M1_GRID[1:]) / 2
                blk = [np.float32(6.0 * d)]
            else:
                s = float(np.float16(rng.uniform(1e-3, 50)))
                d = s
                mids = np.arange(7) + 0.5
                blk = [np.float32(7.0 * d)]
            while len(blk) < b:
                v = np.float32(float(rng.choice(mids)) * d * (1 if rng.random() < 0.5 else -1))
                k = rng.integers(0, 3)
                v = v if k == 0 else np.nextafter(v, np.float32(np.inf if k == 1 else -np.inf))
                blk.append(v)
            out[r, j * b:(j + 1) * b] = blk
    return out, float(gs)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_exact_decisions_next_to_ties_fp32(lib, fmt):
    # one-row-per-thread kernel (fp32 input), identity transform: bit-exact against
    # the oracle's exact-quotient rule with no boundary window
    rng = np.random.default_rng(31)
    x, gs = _near_tie_rows(fmt, rng)
    t = T.identity_blocks(x.shape[1], P.Q.BLOCK[fmt]).astype(np.float32)
    c, s, y = run_gpu_t(lib, _as_input(x, False), t, "identity", fmt, gs if fmt == "nvfp4" else 0.0)
    P.compare_transform_quant(x, t, fmt, gs if fmt == "nvfp4" else None, c, s, y, strict=True)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
@pytest.mark.parametrize("kind", ["identity", "hadamard"])
def test_exact_decisions_structured_bf16(lib, fmt, kind):
    # tensor-core kernel, bf16 input with 8-bit significands and a per-tensor scale
    # derived from a bf16 amax (amax / 2688 = amax / (2^7 * 21)): many quotients fall
    # on or within an fp32 ulp of a boundary.  The identity transform is exact in
    # fp32 on both sides, so its codes and scales must match the oracle exactly;
    # Hadamard's fp32 butterflies may round, so it gets the boundary window.
    w = synth.WORKLOADS[FMT_WORKLOAD[fmt]]
    x = synth.activations(w, tokens=256)[:, :1024]
    t = (T.identity_blocks if kind == "identity" else T.hadamard_blocks)(1024, P.Q.BLOCK[fmt]).astype(np.float32)
    gs = _global_scale(x, t, fmt)
    c, s, y = run_gpu_t(lib, _as_input(x, True), t, kind, fmt, gs)
    P.compare_transform_quant(x, t, fmt, gs if fmt == "nvfp4" else None, c, s, y, strict=kind == "identity")
