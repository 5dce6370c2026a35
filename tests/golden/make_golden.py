"""Writes tests/golden/tiny_w4a4.json from the CPU oracle alone (no CUDA path).

The pages print no worked numeric example for the layer, so this fixture is a
regression pin of the oracle itself on the tiny W4A4 configuration (X [64,256]
N(0,1) with 1% outlier channels x20, W [256,256] N(0,0.02), seed 0): digests of
the codes, scales, exact int32 accumulators and bf16 outputs, plus a few values
written out.  Run:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import rbd_oracle as O  # noqa: E402
from rotated_bit_dit_b200 import inputs as I  # noqa: E402


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def compute():
    t = I.make_layer_inputs(I.CONFIGS["tiny_w4a4"], seed=0)
    ref = O.linear_reference(t["x"], t["w"], 4, 256, 0)
    acc = O.gemm_acc(ref["codes"], O.unpack_int4(ref["wq"]))
    return {
        "config": "tiny_w4a4 seed 0: X [64,256], W [256,256], INT4, group-256 rotation, per-row scales",
        "x_sha256": digest(t["x"]),
        "codes_sha256": digest(ref["codes"].astype(np.int8)),
        "act_scales_sha256": digest(ref["sx"].astype(np.float32)),
        "weights_packed_sha256": digest(ref["wq"].astype(np.uint8)),
        "acc_sha256": digest(acc.astype(np.int64)),
        "out_bf16_sha256": digest(ref["ref_bf16"].astype(np.uint16)),
        "codes_row0_first16": [int(v) for v in ref["codes"][0, :16]],
        "act_scale_row0_hex": float(ref["sx"][0]).hex(),
        "acc_00": int(acc[0, 0]),
        "out_bf16_row0_first8": [int(v) for v in ref["ref_bf16"][0, :8]],
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_w4a4.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=1)
        f.write("\n")
    print("wrote", out)
