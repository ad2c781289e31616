"""Oracle calls for process pools started with spawn (imports no torch)."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def e4m3_codes(rng):
    """The oracle's E4M3 codes of the fp32 bit patterns [a, b)."""
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import oracle
    a, b = rng
    return oracle.f32_to_e4m3(np.arange(a, b, dtype=np.uint32).view(np.float32))
