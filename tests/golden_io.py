"""Loading of the stored expected values under tests/golden/."""
import json
import os

import numpy as np
import ml_dtypes

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_bits(v):
    if isinstance(v, str):
        if v.startswith("0x"):
            return int(v, 16)
        v = float(v)
    return int(np.array([v], np.float32).astype(ml_dtypes.bfloat16)
               .view(np.uint16)[0])


def hand_groups():
    """[(name, x bf16[32], scale byte, codes[32])] from hand_groups.json."""
    out = []
    for g in load("hand_groups.json")["groups"]:
        bits = np.zeros(32, np.uint16)
        for pos, v in g["values"].items():
            bits[int(pos)] = _bf16_bits(v)
        codes = np.zeros(32, np.uint8)
        for pos, c in g["codes"].items():
            codes[int(pos)] = c
        out.append((g["name"], bits.view(ml_dtypes.bfloat16), g["scale_byte"],
                    codes))
    return out


def unpack_nibbles(codes):
    """[..., n] packed bytes -> [..., 2n] codes, even index in the low nibble."""
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = codes & 0x0F
    out[..., 1::2] = codes >> 4
    return out
