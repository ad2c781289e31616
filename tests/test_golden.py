"""The stored expected values of tests/golden/, written by
tests/golden/make_golden.py from the oracle and the seeded generators alone:
the oracle still produces them (CPU), and the CUDA path, called through the
C ABI, reproduces them bit for bit (GPU)."""

import json
import os
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))
import make_golden  # noqa: E402

LISTS = ("counts", "offsets", "bso", "input_perm", "output_perm")


def stored(name):
    with open(make_golden.path(name)) as f:
        return json.load(f)


@pytest.mark.parametrize("name", make_golden.CASES)
def test_oracle_reproduces_stored_values(name):
    assert make_golden.expected(name) == stored(name)


@pytest.mark.gpu
@pytest.mark.parametrize("name", make_golden.CASES)
def test_cuda_path_reproduces_stored_values(name):
    import combine_permute_b200 as moe
    g = stored(name)
    dev = torch.device("cuda:0")
    ids_np, wt, x, y, E = make_golden.case_inputs(name)
    T, k = ids_np.shape
    H = x.shape[1]
    A = g["blockscale_align"]
    ids, x, y = torch.from_numpy(ids_np).to(dev), x.to(dev), y.to(dev)
    wt = torch.from_numpy(wt).to(dev)
    meta = moe.moe_prepare(ids, E, blockscale_align=A)
    got = dict(counts=meta.expert_counts, offsets=meta.expert_offsets,
               bso=meta.blockscale_offsets, input_perm=meta.input_permutation,
               output_perm=meta.output_permutation)
    for key in LISTS:
        assert got[key].cpu().numpy().tolist() == g[key], key
    S, rows = T * k, g["bso"][-1]
    out = moe.moe_dispatch_rows(x, k, meta.input_permutation, meta.output_permutation,
                                out=torch.zeros(S, H, dtype=x.dtype, device=dev))
    assert make_golden.digest(make_golden.bits(out.cpu())) == g["dispatch_bf16_sha256"]
    q, sc = moe.moe_dispatch_rows_fp8(
        x, k, meta.output_permutation, meta.expert_offsets, meta.blockscale_offsets,
        out_q=torch.zeros(S, H, dtype=torch.uint8, device=dev),
        out_scales=torch.zeros(rows, H // 128, dtype=torch.float32, device=dev))
    assert make_golden.digest(q.cpu().numpy()) == g["fp8_q_sha256"]
    assert make_golden.digest(sc.cpu().numpy()) == g["fp8_scales_sha256"]
    q, sc = moe.moe_dispatch_rows_nvfp4(
        x, k, meta.output_permutation, meta.expert_offsets, meta.blockscale_offsets,
        out_q=torch.zeros(S, H // 2, dtype=torch.uint8, device=dev),
        out_scales=torch.zeros(rows, H // 16, dtype=torch.uint8, device=dev))
    assert make_golden.digest(q.cpu().numpy()) == g["nvfp4_q_sha256"]
    assert make_golden.digest(sc.cpu().numpy()) == g["nvfp4_scales_sha256"]
    for odt, key in ((torch.bfloat16, "combine_bf16_sha256"), (torch.float32, "combine_fp32_sha256")):
        o = moe.moe_combine(y, meta.output_permutation, wt, out_dtype=odt)
        assert make_golden.digest(make_golden.bits(o.cpu())) == g[key], key
    lay = moe.moe_tile_layout(meta, k, g["tile"], g["max_tiles"])
    torch.cuda.synchronize()
    assert lay.padded_offsets.cpu().numpy().tolist() == g["tile_padded_offsets"]
    assert lay.tile_idx_to_group_idx.cpu().numpy().tolist() == g["tile_tile_group"]
    assert lay.tile_idx_to_mn_limit.cpu().numpy().tolist() == g["tile_tile_mn_limit"]
    assert lay.expanded_idx_to_permuted_idx.cpu().numpy().tolist() == g["tile_exp2perm"]
    assert lay.permuted_idx_to_expanded_idx.cpu().numpy().tolist() == g["tile_perm2exp"]
    assert int(lay.num_non_exiting_tiles.item()) == g["tile_num_tiles"]
    assert int(lay.total_num_padded_tokens.item()) == g["tile_total_padded"]
