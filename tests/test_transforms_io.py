"""Checkpointing calibrated transforms through the C ABI (host only, no GPU).

The file layout is pinned by parsing it here with ``struct`` and numpy, written
from the layout the header documents, independently of the library's reader;
round trips must be bit exact; every malformed file must give its documented
status and never a crash.
"""
import ctypes
import os
import struct

import numpy as np
import pytest

import synth

aq = pytest.importorskip("activation_quantization_b200")
_lib = ctypes.CDLL(aq.LIB_PATH)

OK, INVALID, TOO_SMALL, IO = 0, -1, -6, -7
HDR = struct.Struct("<8sIIIIIIqq")


@pytest.fixture(scope="module")
def calibrated():
    w = synth.WORKLOADS["tiny"]
    xc, wt = synth.activations(w, calib=True), synth.weights(w)
    tx, tw = aq.wush_calibrate(xc, wt, 16, "wush")
    sx, sw, idx = aq.wush_calibrate_shared(xc, wt, 16, "wush", 2)
    return (tx, tw), (sx, sw, idx)


def _parse(path):
    raw = open(path, "rb").read()
    magic, ver, b, kind, dtype, norm, has_index, n_t, n_blocks = HDR.unpack_from(raw, 0)
    assert HDR.size == 48
    off, m = HDR.size, n_t * b * b
    tx = np.frombuffer(raw, "<f4", m, off).reshape(n_t, b, b)
    tw = np.frombuffer(raw, "<f4", m, off + 4 * m).reshape(n_t, b, b)
    off += 8 * m
    idx = None
    if has_index:
        idx = np.frombuffer(raw, "<i4", n_blocks, off)
        off += 4 * n_blocks
    assert off == len(raw)
    return dict(magic=magic, version=ver, block=b, kind=kind, dtype=dtype, sigma_norm=norm, n_t=n_t,
                n_blocks=n_blocks), tx, tw, idx


def test_per_block_round_trip_and_layout(tmp_path, calibrated):
    (tx, tw), _ = calibrated
    p = tmp_path / "t.wush"
    aq.wush_save_transforms(p, tx, tw, "wush")
    hdr, fx, fw, fi = _parse(p)
    assert hdr == dict(magic=b"WUSHTRF1", version=1, block=16, kind=aq.TRANSFORMS["wush"], dtype=0,
                       sigma_norm=1, n_t=tx.shape[0], n_blocks=tx.shape[0])
    assert fi is None and np.array_equal(fx, tx) and np.array_equal(fw, tw)
    lx, lw, li, kind = aq.wush_load_transforms(p)
    assert li is None and kind == aq.TRANSFORMS["wush"]
    assert lx.tobytes() == tx.tobytes() and lw.tobytes() == tw.tobytes()


def test_shared_round_trip_keeps_index(tmp_path, calibrated):
    _, (sx, sw, idx) = calibrated
    p = tmp_path / "s.wush"
    aq.wush_save_transforms(p, sx, sw, "wush", idx)
    info = aq.wush_transforms_file_info(p)
    assert info == {"block": 16, "kind": aq.TRANSFORMS["wush"], "sigma_norm": 1, "n_t": 2, "n_blocks": idx.size,
                    "has_index": True}
    hdr, fx, fw, fi = _parse(p)
    assert np.array_equal(fi, idx)
    lx, lw, li, _ = aq.wush_load_transforms(p)
    assert lx.tobytes() == sx.tobytes() and lw.tobytes() == sw.tobytes() and np.array_equal(li, idx)


def test_special_values_survive(tmp_path):
    # every fp32 bit pattern goes through unchanged (no conversion on the way)
    t = np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, 3.4e38, np.nan, 1.0], np.float32).reshape(1, 2, 4)
    t = np.concatenate([t, t[:, :, ::-1]], axis=2).reshape(1, 4, 4)
    p = tmp_path / "v.wush"
    aq.wush_save_transforms(p, t, -t, "identity", sigma_norm="unknown")
    assert aq.wush_transforms_file_info(p)["sigma_norm"] == 0
    lx, lw, _, _ = aq.wush_load_transforms(p)
    assert lx.tobytes() == t.tobytes() and lw.tobytes() == (-t).tobytes()


def _write(path, raw):
    with open(path, "wb") as f:
        f.write(raw)


def _raw_load(path, cap, icap=64):
    tx = np.zeros(max(cap, 1), np.float32)
    tw = np.zeros_like(tx)
    ix = np.zeros(max(icap, 1), np.int32)
    return _lib.wush_load_transforms(os.fsencode(str(path)), ctypes.c_void_p(tx.ctypes.data),
                                     ctypes.c_void_p(tw.ctypes.data), ctypes.c_int64(cap),
                                     ctypes.c_void_p(ix.ctypes.data), ctypes.c_int64(icap))


def _status(fn, *args):
    with pytest.raises(aq.WushError) as e:
        fn(*args)
    return e.value.status


def test_malformed_files_are_rejected(tmp_path, calibrated):
    _, (sx, sw, idx) = calibrated
    good = tmp_path / "g.wush"
    aq.wush_save_transforms(good, sx, sw, "wush", idx)
    raw = good.read_bytes()
    cap = sx.size
    cases = {
        "magic": (b"WUSHTRF2" + raw[8:], INVALID),
        "version": (raw[:8] + struct.pack("<I", 2) + raw[12:], INVALID),
        "block_not_pow2": (raw[:12] + struct.pack("<I", 24) + raw[16:], INVALID),
        "kind": (raw[:16] + struct.pack("<I", 9) + raw[20:], INVALID),
        "dtype": (raw[:20] + struct.pack("<I", 1) + raw[24:], INVALID),
        "sigma_norm": (raw[:24] + struct.pack("<I", 2) + raw[28:], INVALID),
        "has_index_2": (raw[:28] + struct.pack("<I", 2) + raw[32:], INVALID),
        "n_t_zero": (raw[:32] + struct.pack("<q", 0) + raw[40:], INVALID),
        "header_short": (raw[:47], IO),
        "body_short": (raw[:-5], INVALID),
        "extra_bytes": (raw + b"\0", INVALID),
        "index_out_of_range": (raw[:-4] + struct.pack("<i", 2), INVALID),
        "index_negative": (raw[:-4] + struct.pack("<i", -1), INVALID),
        # an index that does not cover the blocks: has_index = 0 but n_t != n_blocks
        "no_index_count_mismatch": (raw[:28] + struct.pack("<I", 0) + raw[32:], INVALID),
    }
    for name, (blob, want) in cases.items():
        p = tmp_path / f"{name}.wush"
        _write(p, blob)
        assert _raw_load(p, cap) == want, name
    assert _raw_load(good, cap) == OK
    assert _raw_load(good, cap - 1) == TOO_SMALL
    assert _raw_load(good, cap, icap=idx.size - 1) == TOO_SMALL
    assert _raw_load(tmp_path / "missing.wush", cap) == IO
    assert _status(aq.wush_transforms_file_info, tmp_path / "missing.wush") == IO
    _write(tmp_path / "m.wush", b"WUSHTRF2" + raw[8:])
    assert _status(aq.wush_transforms_file_info, tmp_path / "m.wush") == INVALID


def test_save_rejects_bad_arguments_before_writing(tmp_path, calibrated):
    (tx, tw), (sx, sw, idx) = calibrated
    p = tmp_path / "x.wush"
    bad = idx.copy()
    bad[0] = sx.shape[0]
    assert _status(aq.wush_save_transforms, p, sx, sw, "wush", bad) == INVALID
    assert _status(aq.wush_save_transforms, p, sx[:, :3, :3], sw[:, :3, :3], "wush") == INVALID
    assert _status(aq.wush_save_transforms, p, tx, tw, 7) == INVALID
    assert _status(aq.wush_save_transforms, p, tx, tw, "wush", None, 5) == INVALID
    assert not p.exists()
    assert _status(aq.wush_save_transforms, tmp_path / "no_dir" / "x.wush", tx, tw, "wush") == IO
    with pytest.raises(ValueError):
        aq.wush_save_transforms(p, tx, tw[:1], "wush")


def test_header_that_overstates_the_body_is_rejected_before_allocation(tmp_path, calibrated):
    # a header claiming 2^31 transforms over a short body: info refuses it, so the
    # binding never sizes a buffer from it
    (tx, tw), _ = calibrated
    good = tmp_path / "g.wush"
    aq.wush_save_transforms(good, tx, tw, "wush")
    raw = good.read_bytes()
    p = tmp_path / "huge.wush"
    _write(p, raw[:32] + struct.pack("<qq", 1 << 31, 1 << 31) + raw[48:])
    assert _status(aq.wush_transforms_file_info, p) == INVALID
    assert _status(aq.wush_load_transforms, p) == INVALID
    _write(p, raw + b"\0\0\0\0")
    assert _status(aq.wush_transforms_file_info, p) == INVALID
