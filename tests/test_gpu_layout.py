"""Parity of the grouped-GEMM metadata kernels (problem sizes and the
tile-padded layout, the step after prepare) with the oracle, bit-exact."""

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
import oracle
from workloads import CONFIGS, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _layout_case(ids_np, E, tile, max_tiles=None):
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, E)
    got = moe.moe_tile_layout(meta, ids_np.shape[1], tile, max_tiles)
    torch.cuda.synchronize()
    T, k = ids_np.shape
    S = T * k
    mt = max_tiles if max_tiles is not None else max(1, -(-S // tile) + min(E, S))
    ref_meta = oracle.prepare(ids_np, E)
    ref = oracle.tile_layout(ids_np, ref_meta, E, tile, mt)
    return got, ref


@pytest.mark.parametrize("name", list(CONFIGS))
@pytest.mark.parametrize("tile", [128, 1, 37])
def test_tile_layout_workloads(name, tile):
    w = CONFIGS[name]
    if w.S > 200_000:
        w = w.scaled(200_000 // w.k)
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids_np = ids_np.copy()
    ids_np[::41, -1] = -1  # some invalid ids
    got, ref = _layout_case(ids_np, w.E, tile)
    np.testing.assert_array_equal(got.padded_offsets.cpu().numpy(), ref["padded_offsets"])
    assert int(got.num_non_exiting_tiles) == ref["num_tiles"]
    assert int(got.total_num_padded_tokens) == ref["total_padded"]
    np.testing.assert_array_equal(got.tile_idx_to_group_idx.cpu().numpy(), ref["tile_group"])
    np.testing.assert_array_equal(got.tile_idx_to_mn_limit.cpu().numpy(), ref["tile_mn_limit"])
    np.testing.assert_array_equal(got.expanded_idx_to_permuted_idx.cpu().numpy(), ref["exp2perm"])
    np.testing.assert_array_equal(got.permuted_idx_to_expanded_idx.cpu().numpy(), ref["perm2exp"])


def test_tile_layout_capacity_overflow_is_reported():
    rng = np.random.default_rng(3)
    ids_np = rng.integers(0, 64, size=(500, 4)).astype(np.int32)
    got, ref = _layout_case(ids_np, 64, 128, max_tiles=10)  # 2000 slots over 64 experts need more
    assert ref is None
    assert int(got.num_non_exiting_tiles) == -1
    assert int(got.total_num_padded_tokens) > 10 * 128


def test_tile_layout_edge_cases():
    # a single expert, every id invalid, an empty batch
    for ids_np, E in [(np.zeros((300, 2), np.int32), 1), (np.full((50, 3), -1, np.int32), 8),
                      (np.zeros((0, 4), np.int32), 8)]:
        got, ref = _layout_case(ids_np, E, 16)
        np.testing.assert_array_equal(got.padded_offsets.cpu().numpy(), ref["padded_offsets"])
        np.testing.assert_array_equal(got.tile_idx_to_group_idx.cpu().numpy(), ref["tile_group"])
        np.testing.assert_array_equal(got.permuted_idx_to_expanded_idx.cpu().numpy(), ref["perm2exp"])


def test_problem_sizes_vs_oracle():
    w = CONFIGS["zipf_fp8_t16384_h4096_e288_k8"]
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), w.E)
    ps1, ps2 = moe.moe_problem_sizes(meta.expert_counts, 2 * 2048, w.H, w.H, 2048)
    torch.cuda.synchronize()
    r1, r2 = oracle.problem_sizes(oracle.prepare(ids_np, w.E)["counts"], 2 * 2048, w.H, w.H, 2048)
    np.testing.assert_array_equal(ps1.cpu().numpy(), r1)
    np.testing.assert_array_equal(ps2.cpu().numpy(), r2)
