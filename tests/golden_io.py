"""Reader for the hand-worked fixtures under tests/golden/."""

import glob
import os

import numpy as np

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

_INT_LISTS = {"x_shape", "w_shape", "y_shape", "strides", "dilations", "pads",
              "output_padding", "output_shape", "kernel_shape"}
_FLOAT_LISTS = {"x", "w", "bias", "y"}


def load(path):
    rec = {"layout": "nchw", "auto_pad": "NOTSET", "group": 1}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = [t.strip() for t in line.split(":", 1)]
            if key in _INT_LISTS:
                rec[key] = [int(v) for v in val.split()]
            elif key in _FLOAT_LISTS:
                rec[key] = [float(v) for v in val.split()]
            elif key == "group":
                rec[key] = int(val)
            else:
                rec[key] = val
    rec["x"] = np.array(rec["x"], dtype=np.float64).reshape(rec["x_shape"])
    rec["w"] = np.array(rec["w"], dtype=np.float64).reshape(rec["w_shape"])
    rec["y"] = np.array(rec["y"], dtype=np.float64).reshape(rec["y_shape"])
    if "bias" in rec:
        rec["bias"] = np.array(rec["bias"], dtype=np.float64)
    else:
        rec["bias"] = None
    return rec


def all_fixtures():
    return sorted(glob.glob(os.path.join(GOLDEN_DIR, "*.txt")))
