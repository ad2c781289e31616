"""Exhaustive check of the fp32 -> FP8 E4M3 conversion the quantised
dispatch uses (moe::cvt_e4m3x2: cvt.rn.satfinite.e4m3x2.f32, round to
nearest even, saturating) against the oracle's encoder, written from the
format definition: every non-negative finite fp32 bit pattern and +inf
(2^31 - 2^23 + 1 values; the codes above 448 all saturate), and, on the
GPU, that -v always encodes as the code of v with the sign bit set.

The dispatch tests reach the converter only through quotients x / s of
bf16 values; this covers every fp32 it could be handed.  The oracle runs
in a pool of processes started with spawn, chunk by chunk.
"""

import ctypes
import multiprocessing as mp
import os
import subprocess

import numpy as np
import pytest
import torch

from tests._oracle_workers import e4m3_codes

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = [pytest.mark.gpu, pytest.mark.slow]

LAST = 0x7F800000          # +inf: the last pattern checked
CHUNK = 1 << 27            # patterns per GPU call
PIECE = 1 << 23            # patterns per oracle task


def _build():
    src = os.path.join(ROOT, "tests", "cuda", "cvt_sweep.cu")
    out = os.path.join(ROOT, "_build", "libcvt_sweep.so")
    os.makedirs(os.path.dirname(out), exist_ok=True)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-Xcompiler", "-fPIC", "-shared", "-I",
                    os.path.join(ROOT, "combine_permute_b200", "csrc"), "-o", out, src], check=True)
    lib = ctypes.CDLL(out)
    lib.sweep_codes.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p]
    lib.sweep_sign.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p]
    return lib


def test_e4m3_converter_matches_oracle_on_every_fp32():
    ctx = mp.get_context("spawn")
    with ctx.Pool(max(1, min(32, os.cpu_count() or 1))) as pool:
        lib = _build()
        dev = torch.device("cuda:0")
        codes = torch.empty(CHUNK, dtype=torch.uint8, device=dev)
        bad = torch.zeros(1, dtype=torch.int64, device=dev)
        mismatches, checked = 0, 0
        for first in range(0, LAST + 1, CHUNK):
            n = min(CHUNK, LAST + 1 - first)
            assert lib.sweep_codes(first, n, codes.data_ptr()) == 0
            assert lib.sweep_sign(first, n, bad.data_ptr()) == 0
            got = codes[:n].cpu().numpy()
            pieces = [(first + o, first + min(n, o + PIECE)) for o in range(0, n, PIECE)]
            want = np.concatenate(pool.map(e4m3_codes, pieces))
            diff = np.nonzero(got != want)[0]
            if len(diff) and mismatches == 0:
                i = int(diff[0])
                print(f"first mismatch: pattern {first + i:#010x} gpu {got[i]:#04x} oracle {want[i]:#04x}")
            mismatches += len(diff)
            checked += n
        torch.cuda.synchronize(dev)
    assert checked == LAST + 1
    assert mismatches == 0
    assert int(bad.item()) == 0
