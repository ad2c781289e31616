"""Writes the stored expected values under tests/golden/ from the CPU oracle.

Calls only oracle/ and the seeded input generators of workloads/.  The pages
print no worked example for this path, so no fixture holds their numbers;
these freeze the oracle's results on two small cases, so that a change to
the oracle's arithmetic shows up as a failing test (and has to name the
passage that justifies it), and so that the GPU tests can compare the CUDA
path with values written before it ran.

    python tests/golden/make_golden.py
"""

import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import CONFIGS, make_workload  # noqa: E402

TILE = 16
ALIGN = 4

# A hand-written routing with duplicates (token 1 sends two slots to expert
# 2), ids outside [0, E) (-1, 5, 9) and an expert nobody picks (4).
EDGE_IDS = [[2, 0, 1], [2, 2, 3], [-1, 1, 0], [3, 5, 2], [0, 1, 9], [1, 0, 3], [2, 3, 0]]
EDGE_E = 5


def digest(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def bits(t):
    import torch
    t = t.contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def case_inputs(name):
    """ids, weights, x (bf16), y (bf16) of a golden case, drawn on the CPU."""
    import torch
    if name == "tiny_t32_h4096_e256_k8":
        w = CONFIGS[name]
        ids, wt, x, y = make_workload(w, device="cpu")
        return ids, wt, x, y, w.E
    ids = np.array(EDGE_IDS, np.int32)
    T, k = ids.shape
    g = torch.Generator().manual_seed(7)
    x = torch.randn(T, 256, generator=g).to(torch.bfloat16)
    y = torch.randn(T * k, 256, generator=g).to(torch.bfloat16)
    wt = torch.rand(T, k, generator=g).numpy().astype(np.float32)
    return ids, wt, x, y, EDGE_E


def expected(name):
    ids, wt, x, y, E = case_inputs(name)
    T, k = ids.shape
    H = x.shape[1]
    m = oracle.prepare(ids, E, ALIGN)
    rows = int(m["bso"][-1])
    out = {"T": T, "k": k, "E": E, "H": H, "blockscale_align": ALIGN, "tile": TILE}
    for key in ("counts", "offsets", "bso", "input_perm", "output_perm"):
        out[key] = m[key].tolist()
    out["dispatch_bf16_sha256"] = digest(oracle.dispatch(bits(x), k, m["input_perm"],
                                                         out=np.zeros((T * k, H), np.uint16)))
    q, sc = oracle.dispatch_fp8(bits(x), "bf16", ids, m, np.zeros((T * k, H), np.uint8),
                                np.zeros((rows, H // 128), np.float32))
    out["fp8_q_sha256"], out["fp8_scales_sha256"] = digest(q), digest(sc)
    q, sc = oracle.dispatch_nvfp4(bits(x), "bf16", ids, m, np.zeros((T * k, H // 2), np.uint8),
                                  np.zeros((rows, H // 16), np.uint8))
    out["nvfp4_q_sha256"], out["nvfp4_scales_sha256"] = digest(q), digest(sc)
    out["combine_bf16_sha256"] = digest(oracle.combine(bits(y), "bf16", m["output_perm"], wt, "bf16"))
    out["combine_fp32_sha256"] = digest(oracle.combine(bits(y), "bf16", m["output_perm"], wt, "fp32"))
    max_tiles = -(-(T * k) // TILE) + min(E, T * k)
    lay = oracle.tile_layout(ids, m, E, TILE, max_tiles)
    out["max_tiles"] = max_tiles
    for key, v in lay.items():
        out["tile_" + key] = np.asarray(v).tolist()
    return out


CASES = ["tiny_t32_h4096_e256_k8", "edge_t7_k3_e5"]


def path(name):
    return os.path.join(HERE, f"oracle_{name}.json")


if __name__ == "__main__":
    for name in CASES:
        with open(path(name), "w") as f:
            json.dump(expected(name), f, indent=0, sort_keys=True)
            f.write("\n")
        print("wrote", path(name))
