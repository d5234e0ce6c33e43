"""Readers for the hand-derived fixtures under tests/golden (test code only)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def nvfp4_hand_blocks():
    """The row of tests/golden/nvfp4_hand_blocks.txt.

    Returns (W [1, 96] float64, tensor scale, block scale codes [6] uint8,
    element codes [96] uint8 (4-bit), W / value(scale) per element [96])."""
    W = np.zeros((1, 96))
    sb = np.zeros(6, dtype=np.uint8)
    q = np.zeros(96, dtype=np.uint8)
    ratio = np.zeros(96)
    st = None
    with open(os.path.join(GOLDEN, "nvfp4_hand_blocks.txt")) as f:
        for line in f:
            t = line.split()
            if not t:
                continue
            if t[0] == "#" and len(t) >= 3 and t[1] == "tensor_scale":
                st = float(t[2])
            elif t[0] == "block":
                sb[int(t[1])] = int(t[4], 16)
            elif t[0] == "elem":
                col = int(t[1])
                W[0, col] = float(t[2])
                ratio[col] = float(t[3])
                q[col] = int(t[4], 16)
    assert st is not None
    return W, st, sb, q, ratio
