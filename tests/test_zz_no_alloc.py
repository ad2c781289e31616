"""moe_prepare_no_alloc: the prepare entry point for callers that cannot
allocate device memory (work recorded into a CUDA graph, serving loops where
a cudaMalloc would synchronise the device, processes whose GPU memory is all
handed to a pool allocator).  Its scratch is a fixed device array inside the
library; these tests call it through the C ABI and compare it with
moe_prepare given a workspace of its own.

This file runs last in a full test run (pytest collects it last), so that a
failure here never hides the other tests; it also passes on its own in a
fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from combine_permute_b200 import _lib
from workloads import CONFIGS, make_workload

MOE_OK, MOE_ERR_UNSUPPORTED = 0, 2
SCRATCH_BYTES = 4 << 20


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() else None


def _outputs(S, E, dev):
    i32 = dict(dtype=torch.int32, device=dev)
    return dict(counts=torch.full((E,), -9, **i32), offsets=torch.full((E + 1,), -9, **i32),
                bso=torch.full((E + 1,), -9, **i32), inp=torch.full((S,), -9, **i32),
                outp=torch.full((S,), -9, **i32), diag=torch.full((2,), -9, **i32))


def _no_alloc(lib, ids, T, k, E, A, o, stream):
    return lib.moe_prepare_no_alloc(_p(ids), T, k, E, _p(o["counts"]), _p(o["offsets"]),
                                    _p(o["bso"]), A, _p(o["inp"]), _p(o["outp"]), _p(o["diag"]),
                                    ctypes.c_void_p(stream))


def _with_workspace(lib, ids, T, k, E, A, o, stream, dev):
    need = lib.moe_prepare_workspace_bytes(T, k, E)
    ws = torch.zeros(max(need, 1), dtype=torch.uint8, device=dev)
    return lib.moe_prepare(_p(ids), T, k, E, _p(o["counts"]), _p(o["offsets"]), _p(o["bso"]), A,
                           _p(o["inp"]), _p(o["outp"]), _p(o["diag"]), _p(ws), need,
                           ctypes.c_void_p(stream))


def test_rejects_problems_larger_than_its_scratch():
    lib = _lib.load()
    T, k, E = 300000, 8, 1024            # needs about 9.4 MB of scratch
    assert lib.moe_prepare_workspace_bytes(T, k, E) > SCRATCH_BYTES
    st = lib.moe_prepare_no_alloc(ctypes.c_void_p(0x1000), T, k, E, ctypes.c_void_p(0x1000),
                                  ctypes.c_void_p(0x1000), None, 1, ctypes.c_void_p(0x1000),
                                  ctypes.c_void_p(0x1000), None, None)
    assert st == MOE_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_no_alloc_matches_moe_prepare_on_consecutive_calls():
    """Two calls in a row (a large problem, then a smaller one with other
    routing, so that the second must not see the first's scratch), each
    bit-exact against moe_prepare with its own zeroed workspace."""
    lib = _lib.load()
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev).cuda_stream
    cases = [CONFIGS["zipf_fp16_t131072_h2048_e64_k6"],                  # 786432 slots, tiled
             CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(20000),       # 160000 slots, tiled
             CONFIGS["tiny_t32_h4096_e256_k8"]]                          # one block, no scratch
    for w in cases:
        ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
        ids_np[::97, 0] = -1                                             # some invalid ids
        ids = torch.from_numpy(ids_np).to(dev)
        A = 128
        got, ref = _outputs(w.S, w.E, dev), _outputs(w.S, w.E, dev)
        assert _no_alloc(lib, ids, w.T, w.k, w.E, A, got, stream) == MOE_OK
        assert _with_workspace(lib, ids, w.T, w.k, w.E, A, ref, stream, dev) == MOE_OK
        torch.cuda.synchronize(dev)
        for key in ("counts", "offsets", "bso", "inp", "outp", "diag"):
            assert torch.equal(got[key], ref[key]), (w.name, key)
        assert int(got["diag"][0]) == int((ids_np < 0).sum()) and int(got["diag"][1]) == 0
        # the stable order itself: dispatched rows sorted by expert, then slot
        flat = ids_np.ravel()
        perm = got["inp"].cpu().numpy()[: int(got["offsets"][-1])]
        keys = flat[perm].astype(np.int64) * (1 << 32) + perm
        assert (np.diff(keys) > 0).all()
