"""Parity of the expert-window / int64-id prepare, of the steps after it
(fp8 dispatch, tile layout) and of the output memset with the oracle."""

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
import oracle
from workloads import CONFIGS, make_workload

from _helpers import TORCH_DT, bits

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _shifted(ids, base, E):
    s = ids.astype(np.int64) - base
    s[(s < 0) | (s >= E)] = -1
    return s.astype(np.int32)


def _check_local(ids_np, base, E, A=16):
    meta = moe.moe_prepare_local(torch.from_numpy(ids_np).to(DEV), base, E, blockscale_align=A)
    torch.cuda.synchronize()
    ref = oracle.prepare_local(ids_np.astype(np.int64), base, E, A)
    np.testing.assert_array_equal(meta.expert_counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(meta.expert_offsets.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(meta.blockscale_offsets.cpu().numpy(), ref["bso"])
    np.testing.assert_array_equal(meta.input_permutation.cpu().numpy(), ref["input_perm"])
    np.testing.assert_array_equal(meta.output_permutation.cpu().numpy(), ref["output_perm"])
    assert meta.diag.cpu().tolist() == [ref["n_invalid"], 0]
    return meta, ref


@pytest.mark.parametrize("id_dtype", [np.int32, np.int64])
@pytest.mark.parametrize("T,base,E", [(40, 64, 32), (3000, 0, 256), (3000, 96, 64),
                                      (40000, 128, 128), (262144, 16, 40), (660000, 16, 40)])
def test_prepare_local_vs_oracle(id_dtype, T, base, E):
    # top-8 slots: one block, 1 round, 5 rounds (input_permutation staged),
    # 28 rounds (one launch, slot by slot) and 5.28 M slots (two kernels)
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(T)
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids_np = ids_np.astype(id_dtype)
    _check_local(ids_np, base, E)


def test_prepare_local_int64_ids_beyond_int32():
    rng = np.random.default_rng(5)
    base = 3 * 2**32 + 17
    ids_np = (base - 8 + rng.integers(0, 48, size=(5000, 6))).astype(np.int64)
    _check_local(ids_np, base, 32)


def test_fp8_dispatch_and_tile_layout_on_an_expert_window():
    w = CONFIGS["zipf_fp8_t16384_h4096_e288_k8"].scaled(1500)
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    base, E, A = 100, 96, 128
    meta, ref = _check_local(ids_np, base, E, A)
    q, sc = moe.moe_dispatch_rows_fp8(x, w.k, meta.output_permutation, meta.expert_offsets,
                                      meta.blockscale_offsets, blockscale_align=A,
                                      out_q=torch.full((w.S, w.H), 0xAB, dtype=torch.uint8, device=DEV),
                                      out_scales=torch.full((w.S + E * (A - 1), w.H // 128), float("nan"),
                                                            device=DEV))
    lay = moe.moe_tile_layout(meta, w.k, 64)
    torch.cuda.synchronize()
    local = _shifted(ids_np, base, E)
    q_ref = np.full((w.S, w.H), 0xAB, np.uint8)
    sc_ref = np.full((w.S + E * (A - 1), w.H // 128), np.nan, np.float32)
    oracle.dispatch_fp8(bits(x), "bf16", local, ref, q_ref, sc_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), sc_ref.view(np.uint32))
    S = w.S
    lref = oracle.tile_layout(local, ref, E, 64, max(1, -(-S // 64) + min(E, S)))
    np.testing.assert_array_equal(lay.tile_idx_to_group_idx.cpu().numpy(), lref["tile_group"])
    np.testing.assert_array_equal(lay.expanded_idx_to_permuted_idx.cpu().numpy(), lref["exp2perm"])
    np.testing.assert_array_equal(lay.permuted_idx_to_expanded_idx.cpu().numpy(), lref["perm2exp"])


def test_nvfp4_dispatch_on_an_expert_window_int64_ids():
    """One rank's window of experts from int64 ids, then the NVFP4 dispatch
    of its rows (scale rows padded to 16 per expert)."""
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(900)
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    ids64 = ids_np.astype(np.int64) + (1 << 33)   # ids beyond the int32 range
    base, E, A = (1 << 33) + 64, 64, 16
    meta, ref = _check_local(ids64, base, E, A)
    rows = w.S + E * (A - 1)
    q, sc = moe.moe_dispatch_rows_nvfp4(
        x, w.k, meta.output_permutation, meta.expert_offsets, meta.blockscale_offsets,
        out_q=torch.full((w.S, w.H // 2), 0xAB, dtype=torch.uint8, device=DEV),
        out_scales=torch.full((rows, w.H // 16), 0xCD, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    local = _shifted(ids64, base, E)
    q_ref = np.full((w.S, w.H // 2), 0xAB, np.uint8)
    sc_ref = np.full((rows, w.H // 16), 0xCD, np.uint8)
    oracle.dispatch_nvfp4(bits(x), "bf16", local, ref, q_ref, sc_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sc.cpu().numpy(), sc_ref)


@pytest.mark.parametrize("dtype,H", [("bf16", 7168), ("fp32", 1000), ("fp16", 8)])
def test_output_memset_vs_oracle(dtype, H):
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(700)
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    meta = moe.moe_prepare_local(torch.from_numpy(ids_np).to(DEV), 200, 56)  # many tokens unrouted
    out = torch.randn(w.T, H, device=DEV).to(TORCH_DT[dtype])
    ref = bits(out).copy()
    moe.moe_output_memset(out, meta.output_permutation, w.k)
    torch.cuda.synchronize()
    oracle.output_memset(ref, meta.output_permutation.cpu().numpy(), w.k)
    np.testing.assert_array_equal(bits(out), ref)
    routed = (meta.output_permutation.cpu().numpy().reshape(w.T, w.k) >= 0).any(axis=1)
    assert routed.any() and (~routed).any()
