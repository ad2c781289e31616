"""Parity of the NVFP4 dispatch (E2M1 codes, one E4M3 scale per 16 elements)
with the CPU oracle, through the C ABI.

Bar: codes and scale bytes bit-exact (both sides take every rounding
decision in fp32 with the same operation order).  Bytes that no valid slot
maps to keep their fill value.
"""

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
import oracle
from workloads import CONFIGS, make_workload

from _helpers import TORCH_DT, bits

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _ids(rng, T, k, E, p_invalid=0.0):
    if k <= E:
        ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    else:
        ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if p_invalid:
        bad = rng.random((T, k)) < p_invalid
        ids[bad] = rng.choice(np.array([-1, E, E + 3], np.int32), size=bad.sum())
    return ids


def _run(ids_np, E, x, A):
    T, k = ids_np.shape
    H = x.shape[1]
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), E, blockscale_align=A)
    rows = T * k + E * (A - 1)
    q = torch.full((T * k, H // 2), 0xAB, dtype=torch.uint8, device=DEV)
    sc = torch.full((rows, H // 16), 0xCD, dtype=torch.uint8, device=DEV)
    moe.moe_dispatch_rows_nvfp4(x, k, meta.output_permutation, meta.expert_offsets,
                                meta.blockscale_offsets, out_q=q, out_scales=sc)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, E, A)
    q_ref = np.full((T * k, H // 2), 0xAB, np.uint8)
    sc_ref = np.full((rows, H // 16), 0xCD, np.uint8)
    xdt = "bf16" if x.dtype == torch.bfloat16 else "fp16"
    oracle.dispatch_nvfp4(bits(x), xdt, ids_np, ref_meta, q_ref, sc_ref)
    return q.cpu().numpy(), sc.cpu().numpy(), q_ref, sc_ref


@pytest.mark.parametrize("xdt", ["bf16", "fp16"])
@pytest.mark.parametrize("T,H,E,k,A", [(300, 4096, 288, 8, 128), (77, 48, 16, 3, 1),
                                       (40, 16, 5, 2, 32), (513, 7168, 64, 6, 4),
                                       (50, 4096, 64, 40, 4), (31, 2048, 40, 32, 1)])
def test_dispatch_nvfp4_vs_oracle(xdt, T, H, E, k, A):
    rng = np.random.default_rng(T + H)
    ids_np = _ids(rng, T, k, E, p_invalid=0.02)
    x = torch.randn(T, H, device=DEV)
    x[1, :16] = 0.0                        # an all-zero group: scale byte 0
    x[2, :16] *= 1e-4                      # scale in the e4m3 subnormal range
    x[3, :16] *= 1e-9                      # scale underflows to 0: codes 0
    if xdt == "bf16":
        x[4, :16] *= 1e5                   # amax / 6 above 448: scale saturates
    x = x.to(TORCH_DT[xdt])
    q, sc, q_ref, sc_ref = _run(ids_np, E, x, A)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sc, sc_ref)


@pytest.mark.parametrize("mant", range(8, 16))
@pytest.mark.parametrize("scale_exp", [0, -7, 5])
def test_dispatch_nvfp4_every_bf16_value(mant, scale_exp):
    """Every bf16 value of magnitude <= amax in groups whose amax is
    0.75 * mant * 2^scale_exp, so that amax / 6 is (mant / 8) * 2^scale_exp:
    each of the 8 scale mantissas (at 2^-7 the odd ones round to the E4M3
    subnormal grid), and on each every e2m1 rounding tie, the subnormal step, signed zeros and the
    saturation edge."""
    top = 0.75 * mant * 2.0 ** scale_exp
    allv = torch.arange(-(2 ** 15), 2 ** 15, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    v = allv[torch.isfinite(allv.float()) & (allv.float().abs() <= top)]
    per = 15
    ngrp = (v.numel() + per - 1) // per
    groups = torch.zeros(ngrp, 16, dtype=torch.bfloat16)
    groups[:, 0] = top
    flat = groups[:, 1:].reshape(-1)
    flat[: v.numel()] = v
    groups[:, 1:] = flat.view(ngrp, per)
    H = 16 * 64
    rows = (ngrp + 63) // 64
    x = torch.zeros(rows * 64, 16, dtype=torch.bfloat16)
    x[:ngrp] = groups
    x = x.view(rows, H).to(DEV)
    T = x.shape[0]
    ids_np = (np.arange(T, dtype=np.int32) % 3).reshape(T, 1)
    q, sc, q_ref, sc_ref = _run(ids_np, 3, x, 1)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sc, sc_ref)


def test_dispatch_nvfp4_every_fp16_value():
    """Every finite fp16 value, in groups with amax 6 * 1.375 (scale
    mantissa 11) and with amax 448 * 6 * 2 (the scale saturates at 448 and
    x / d reaches 12: the e2m1 saturation)."""
    allv = torch.arange(-(2 ** 15), 2 ** 15, dtype=torch.int32).to(torch.int16).view(torch.float16)
    for top in (6 * 1.375, 448 * 6 * 2):
        v = allv[torch.isfinite(allv.float()) & (allv.float().abs() <= top)]
        per = 15
        ngrp = (v.numel() + per - 1) // per
        groups = torch.zeros(ngrp, 16, dtype=torch.float16)
        groups[:, 0] = top
        flat = groups[:, 1:].reshape(-1)
        flat[: v.numel()] = v
        groups[:, 1:] = flat.view(ngrp, per)
        rows = (ngrp + 63) // 64
        x = torch.zeros(rows * 64, 16, dtype=torch.float16)
        x[:ngrp] = groups
        x = x.view(rows, 16 * 64).to(DEV)
        ids_np = (np.arange(rows, dtype=np.int32) % 2).reshape(rows, 1)
        q, sc, q_ref, sc_ref = _run(ids_np, 2, x, 1)
        np.testing.assert_array_equal(q, q_ref)
        np.testing.assert_array_equal(sc, sc_ref)


def test_dispatch_nvfp4_full_workload_sampled():
    """The fp8 block-scale routing workload at full size (16384 tokens,
    hidden 4096, 288 experts, top-8, scale rows padded to 128), dispatched
    to NVFP4; sampled tokens checked against the oracle run on them alone."""
    w = CONFIGS["zipf_fp8_t16384_h4096_e288_k8"]
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    A = w.block_align
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), w.E, blockscale_align=A)
    q, sc = moe.moe_dispatch_rows_nvfp4(x, w.k, meta.output_permutation, meta.expert_offsets,
                                        meta.blockscale_offsets, blockscale_align=A)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, w.E, A)
    rng = np.random.default_rng(3)
    toks = np.unique(rng.integers(0, w.T, 300))
    slots = (toks[:, None] * w.k + np.arange(w.k)).ravel()
    p = ref_meta["output_perm"][slots]
    e = ids_np.ravel()[slots]
    srow = ref_meta["bso"][e] + p - ref_meta["offsets"][e]
    # with zero offsets the oracle writes scale row r for sampled slot r
    sub_meta = dict(input_perm=np.arange(slots.size, dtype=np.int32),
                    offsets=np.zeros(w.E + 1, np.int32), bso=np.zeros(w.E + 1, np.int32))
    q_sub, sc_sub = oracle.dispatch_nvfp4(bits(x[torch.from_numpy(toks).to(DEV)]), "bf16",
                                          ids_np[toks], sub_meta,
                                          scales=np.zeros((slots.size, w.H // 16), np.uint8))
    np.testing.assert_array_equal(q[torch.from_numpy(p).long().to(DEV)].cpu().numpy(), q_sub)
    np.testing.assert_array_equal(sc[torch.from_numpy(srow).long().to(DEV)].cpu().numpy(), sc_sub)


@pytest.mark.parametrize("H", [4096, 7168])
def test_dispatch_nvfp4_unaligned_outputs(H):
    """Code rows and scale rows that start 8 bytes past a 16-byte boundary
    (the contract asks for 8-byte alignment only): same bytes as the oracle."""
    T, E, k, A = 150, 64, 6, 4
    rng = np.random.default_rng(H)
    ids_np = _ids(rng, T, k, E, p_invalid=0.02)
    x = torch.randn(T, H, device=DEV).to(torch.bfloat16)
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), E, blockscale_align=A)
    rows = T * k + E * (A - 1)
    qbuf = torch.full((T * k * (H // 2) + 8,), 0xAB, dtype=torch.uint8, device=DEV)
    sbuf = torch.full((rows * (H // 16) + 8,), 0xCD, dtype=torch.uint8, device=DEV)
    q = qbuf[8:].view(T * k, H // 2)
    sc = sbuf[8:].view(rows, H // 16)
    assert q.data_ptr() % 16 == 8
    moe.moe_dispatch_rows_nvfp4(x, k, meta.output_permutation, meta.expert_offsets,
                                meta.blockscale_offsets, out_q=q, out_scales=sc)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, E, A)
    q_ref = np.full((T * k, H // 2), 0xAB, np.uint8)
    sc_ref = np.full((rows, H // 16), 0xCD, np.uint8)
    oracle.dispatch_nvfp4(bits(x), "bf16", ids_np, ref_meta, q_ref, sc_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sc.cpu().numpy(), sc_ref)


def test_dispatch_nvfp4_validation():
    lib = moe._lib.load()
    x = torch.zeros(4, 24, dtype=torch.bfloat16, device=DEV)
    perm = torch.zeros(4, dtype=torch.int32, device=DEV)
    off = torch.zeros(2, dtype=torch.int32, device=DEV)
    q = torch.zeros(4, 12, dtype=torch.uint8, device=DEV)
    st = lib.moe_dispatch_rows_nvfp4(x.data_ptr(), moe._lib.MOE_BF16, 4, 24, 1, 1, perm.data_ptr(),
                                     off.data_ptr(), off.data_ptr(), q.data_ptr(), q.data_ptr(), None)
    assert st == moe._lib.MOE_ERR_INVALID_ARG           # H not a multiple of 16
    x32 = torch.zeros(4, 32, dtype=torch.float32, device=DEV)
    st = lib.moe_dispatch_rows_nvfp4(x32.data_ptr(), moe._lib.MOE_F32, 4, 32, 1, 1, perm.data_ptr(),
                                     off.data_ptr(), off.data_ptr(), q.data_ptr(), q.data_ptr(), None)
    assert st == moe._lib.MOE_ERR_UNSUPPORTED
    # no tokens: nothing to do, NULL buffers accepted
    st = lib.moe_dispatch_rows_nvfp4(None, moe._lib.MOE_BF16, 0, 32, 1, 1, None, None, None, None,
                                     None, None)
    assert st == moe._lib.MOE_OK
