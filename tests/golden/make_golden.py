"""Write the stored expected values under tests/golden/ from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
Only ``oracle`` and the seeded generators in ``synth`` are used.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import synth  # noqa: E402
from oracle import calibrate, loss, transforms  # noqa: E402


def tiny_layer_losses():
    w = synth.WORKLOADS["tiny"]
    x = synth.activations(w)
    xc = synth.activations(w, calib=True)
    wt = synth.weights(w)
    out = {}
    for fmt, b in (("mxfp4", 32), ("nvfp4", 16), ("int4", 32)):
        for kind in ("identity", "hadamard", "wus", "wush", "wush_diag"):
            tx, tw = calibrate.calibrate(xc, wt, b, kind)
            tx32, tw32 = tx.astype(np.float32), tw.astype(np.float32)
            gs = None
            if fmt == "nvfp4":
                gs = calibrate.nvfp4_global_scale(
                    transforms.apply_block_transform(xc, tx32).astype(np.float32))
            out[f"{fmt}/{kind}"] = loss.layer_loss(x, wt, tx32, tw32, fmt, gs)
    # WUSH shared among groups of similar blocks (MXFP4, 8 blocks of 32)
    mx, mw = calibrate.block_moments(xc, 32), calibrate.block_moments(wt, 32)
    for groups in (1, 2, 4):
        sx, sw, idx = calibrate.shared_transforms(mx, mw, "wush", groups)
        out[f"mxfp4/wush_shared{groups}"] = loss.layer_loss(x, wt, sx[idx].astype(np.float32),
                                                            sw[idx].astype(np.float32), "mxfp4")
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_layer_losses.json"), "w") as f:
        json.dump({"source": "oracle only (tests/golden/make_golden.py); seeded tiny layer "
                             "X [128, 256] N(0,1) with 4 channels x20, W [256, 256] N(0, 0.02^2), "
                             "512 calibration tokens",
                   "losses": tiny_layer_losses()}, f, indent=1, sort_keys=True)
