"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Bar: routing metadata, dispatched rows and fp8 bytes/scales bit-exact;
combine within one bf16/fp16 ulp for half outputs and 1e-5 relative (to
sum_j |w_j y_j|) for fp32 outputs.  The kernels use the oracle's operation
order, so combine is also expected to be bit-exact and the tests check that
too.  Sizes span several tiles with a ragged tail; full-size workloads are
compared on sampled rows / tokens that the oracle computes one by one.
"""

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
import oracle
from workloads import CONFIGS, make_workload

from _helpers import TORCH_DT, assert_f32_within_rel, assert_half_within_one_ulp, bits, combine_magnitude

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _ids_random(rng, T, k, E, p_invalid=0.0, distinct=True):
    if distinct and k <= E:
        ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    else:
        ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if p_invalid:
        bad = rng.random((T, k)) < p_invalid
        ids[bad] = rng.choice(np.array([-1, E, E + 7, -(2 ** 31)], np.int32), size=bad.sum())
    return ids


def _check_prepare(ids_np, E, A=None, workspace=None):
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, E, blockscale_align=A, workspace=workspace)
    torch.cuda.synchronize()
    ref = oracle.prepare(ids_np, E, A or 1)
    np.testing.assert_array_equal(meta.expert_counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(meta.expert_offsets.cpu().numpy(), ref["offsets"])
    if A is not None:
        np.testing.assert_array_equal(meta.blockscale_offsets.cpu().numpy(), ref["bso"])
    np.testing.assert_array_equal(meta.input_permutation.cpu().numpy(), ref["input_perm"])
    np.testing.assert_array_equal(meta.output_permutation.cpu().numpy(), ref["output_perm"])
    diag = meta.diag.cpu().numpy()
    assert diag[0] == ref["n_invalid"] and diag[1] == 0
    return meta, ref


# ---------------------------------------------------------------------------
# prepare
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("trial", range(40))
def test_prepare_tiny_vs_oracle(trial):
    rng = np.random.default_rng(100 + trial)
    T, k, E = int(rng.integers(0, 9)), int(rng.integers(1, 5)), int(rng.integers(1, 7))
    ids = rng.integers(-1, E + 1, size=(T, k)).astype(np.int32)  # duplicates + invalid
    _check_prepare(ids, E, A=int(rng.integers(1, 5)))


@pytest.mark.parametrize("T,k,E", [
    (1, 8, 256), (63, 8, 256), (64, 8, 1024), (65, 8, 3),  # small path up to 512 slots, then
    (512, 8, 256),                                     # single block, full single tile
    (513, 8, 256), (1024, 8, 7), (3001, 6, 64),          # two or more tiles, ragged tails
    (4095, 1, 1), (20000, 8, 1024), (9216, 8, 256),
    (40000, 3, 5), (70000, 8, 288),
    (131072, 8, 1024), (140000, 8, 64), (262144, 6, 256),
])
def test_prepare_sizes_vs_oracle(T, k, E):
    rng = np.random.default_rng(T * 31 + k * 7 + E)
    ids = _ids_random(rng, T, k, E, p_invalid=0.03, distinct=False)
    _check_prepare(ids, E, A=128)
    _check_prepare(ids, E, A=None)


def test_prepare_large_batch():
    """100 M slots (2^24 tokens, top-6 of 4 experts; three quarters of the
    slots on one expert, about 5 % invalid ids): about 49 000 tiles through
    the two-kernel path, offsets near 10^8."""
    T, k, E = 1 << 24, 6, 4
    rng = np.random.default_rng(2024)
    ids = rng.integers(-1, E, size=(T, k), dtype=np.int32)
    ids[rng.random((T, k), dtype=np.float32) < 0.75] = 2
    _check_prepare(ids, E, A=128)


@pytest.mark.parametrize("T", [100, 5000])
def test_prepare_degenerate_routing(T):
    k, E = 8, 1024
    _check_prepare(np.full((T, k), E - 1, np.int32), E, A=128)   # one expert takes everything
    _check_prepare(np.full((T, k), -1, np.int32), E, A=7)         # every id invalid
    _check_prepare(np.zeros((T, k), np.int32), 1, A=1)            # a single expert


def test_prepare_empty():
    meta, _ = _check_prepare(np.zeros((0, 8), np.int32), 16, A=4)
    assert meta.expert_offsets.cpu().numpy().tolist() == [0] * 17


@pytest.mark.parametrize("name", list(CONFIGS))
def test_prepare_full_workloads(name):
    w = CONFIGS[name]
    ids, _, _, _ = make_workload(w, with_x=False, with_y=False)
    _check_prepare(ids, w.E, A=w.block_align if w.block_align > 1 else 128)


@pytest.mark.parametrize("T", [131072, 200000])
def test_prepare_deterministic_and_workspace_reusable(T):
    """Repeated calls give identical results, and one workspace serves calls
    of different sizes in any order (look-back words left by an earlier call
    never count for a later one)."""
    w = CONFIGS["zipf_fp16_t131072_h2048_e64_k6"].scaled(T)
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids = torch.from_numpy(ids_np).to(DEV)
    nbytes = moe.moe_prepare_workspace_bytes(w.T, w.k, w.E)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    runs = [moe.moe_prepare(ids, w.E, blockscale_align=16, workspace=ws) for _ in range(3)]
    small = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(3000)
    sids_np, _, _, _ = make_workload(small, with_x=False, with_y=False)
    smeta = moe.moe_prepare(torch.from_numpy(sids_np).to(DEV), small.E, workspace=ws)
    runs.append(moe.moe_prepare(ids, w.E, blockscale_align=16, workspace=ws))
    torch.cuda.synchronize()
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)
    ref = oracle.prepare(ids_np, w.E, 16)
    np.testing.assert_array_equal(runs[-1].output_permutation.cpu().numpy(), ref["output_perm"])
    sref = oracle.prepare(sids_np, small.E)
    np.testing.assert_array_equal(smeta.input_permutation.cpu().numpy(), sref["input_perm"])
    assert runs[-1].diag.cpu().tolist() == [0, 0]


def test_one_workspace_shared_by_both_tiled_paths():
    """One workspace, calls alternating between the one-launch path (grid
    barrier, histogram rows) and the two-kernel path (look-back words) with
    different sizes and expert counts: neither path may read the other's
    data (or an earlier call's) as its own."""
    rng = np.random.default_rng(4242)
    # one launch (input_permutation staged or not) and two kernels (more
    # than 511 experts), in turn
    shapes = [(15000, 8, 5), (20000, 8, 600), (40000, 3, 64), (30000, 6, 700),
              (60000, 8, 288), (20000, 8, 600), (320000, 8, 288), (30000, 6, 700),
              (300000, 6, 64), (9000, 8, 256)]
    need = max(moe.moe_prepare_workspace_bytes(T, k, E) for T, k, E in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for T, k, E in shapes:
        ids = _ids_random(rng, T, k, E, p_invalid=0.02, distinct=False)
        _check_prepare(ids, E, A=64, workspace=ws)


# ---------------------------------------------------------------------------
# dispatch (same dtype)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("form", ["scatter", "gather"])
@pytest.mark.parametrize("dtype,H", [("bf16", 7168), ("fp16", 2048), ("fp32", 1000), ("bf16", 8)])
def test_dispatch_vs_oracle(form, dtype, H):
    rng = np.random.default_rng(H)
    T, k, E = 301, 8, 64
    ids_np = _ids_random(rng, T, k, E, p_invalid=0.02)
    x = torch.randn(T, H, device=DEV).to(TORCH_DT[dtype])
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, E)
    out = torch.full((T * k, H), -3.0, device=DEV).to(TORCH_DT[dtype])   # sentinel rows
    if form == "scatter":
        moe.moe_dispatch_rows(x, k, None, meta.output_permutation, out=out)
    else:
        moe.moe_dispatch_rows(x, k, meta.input_permutation, None, out=out)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, E)
    ref = bits(torch.full((T * k, H), -3.0).to(TORCH_DT[dtype]))
    oracle.dispatch(bits(x), k, ref_meta["input_perm"], ref)
    np.testing.assert_array_equal(bits(out), ref)


@pytest.mark.parametrize("T,H", [(40, 300_000), (32, 600_000)])
def test_dispatch_rows_wider_than_the_stage_ring(T, H):
    """bf16 rows of 600 KB and 1.2 MB: the scatter dispatch cuts them into
    chunks of at most half its 64 KB ring of stages (the chunk rule alone
    would give one or no stage)."""
    rng = np.random.default_rng(T)
    k, E = 3, 16
    ids_np = _ids_random(rng, T, k, E, p_invalid=0.05)
    x = torch.randn(T, H, device=DEV).to(torch.bfloat16)
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), E)
    out = torch.full((T * k, H), -3.0, device=DEV).to(torch.bfloat16)
    moe.moe_dispatch_rows(x, k, None, meta.output_permutation, out=out)
    err = moe.moe_dispatch_error()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref_meta = oracle.prepare(ids_np, E)
    ref = bits(torch.full((T * k, H), -3.0).to(torch.bfloat16))
    oracle.dispatch(bits(x), k, ref_meta["input_perm"], ref)
    np.testing.assert_array_equal(bits(out), ref)


@pytest.mark.parametrize("name", ["uniform_t4096_h7168_e256_k8", "khot_t9216_h7168_e256_k8",
                                  "zipf_fp16_t131072_h2048_e64_k6"])
def test_dispatch_full_workloads_sampled(name):
    w = CONFIGS[name]
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, w.E)
    out = moe.moe_dispatch_rows(x, w.k, meta.input_permutation, meta.output_permutation)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, w.E)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.integers(0, w.S, 2000), [0, w.S - 1]]))
    ref = oracle.dispatch(bits(x), w.k, ref_meta["input_perm"][rows])
    np.testing.assert_array_equal(bits(out[torch.from_numpy(rows).to(DEV)]), ref)
    # any-size property: every dispatched row equals its token row (exact
    # integer fingerprint of the raw bits)
    fp_x = x.view(torch.int16).to(torch.int32).sum(dim=1)
    fp_out = out.view(torch.int16).to(torch.int32).sum(dim=1)
    counts = torch.bincount(meta.input_permutation.long() // w.k, minlength=w.T)
    assert bool((counts == w.k).all())
    assert torch.equal(fp_out, fp_x[meta.input_permutation.long() // w.k])


# ---------------------------------------------------------------------------
# fp8 dispatch
# ---------------------------------------------------------------------------

def _fp8_run(ids_np, E, x, A):
    T, k = ids_np.shape
    H = x.shape[1]
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, E, blockscale_align=A)
    q = torch.full((T * k, H), 0xAB, dtype=torch.uint8, device=DEV)
    rows = T * k + E * (A - 1)
    sc = torch.full((rows, H // 128), float("nan"), device=DEV)
    moe.moe_dispatch_rows_fp8(x, k, meta.output_permutation, meta.expert_offsets,
                              meta.blockscale_offsets, out_q=q, out_scales=sc)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, E, A)
    q_ref = np.full((T * k, H), 0xAB, np.uint8)
    sc_ref = np.full((rows, H // 128), np.nan, np.float32)
    xdt = "bf16" if x.dtype == torch.bfloat16 else "fp16"
    oracle.dispatch_fp8(bits(x), xdt, ids_np, ref_meta, q_ref, sc_ref)
    return q.cpu().numpy(), sc.cpu().numpy(), q_ref, sc_ref


@pytest.mark.parametrize("xdt", ["bf16", "fp16"])
@pytest.mark.parametrize("T,H,E,k,A", [(300, 4096, 288, 8, 128), (129, 7168, 64, 4, 8),
                                       (77, 384, 16, 3, 1), (40, 128, 5, 2, 32),
                                       (50, 4096, 64, 40, 4), (33, 7168, 48, 33, 2)])
def test_dispatch_fp8_vs_oracle(xdt, T, H, E, k, A):
    # H = 7168: two 16-element groups a thread; the others one; top-k up to 40
    rng = np.random.default_rng(T + H)
    ids_np = _ids_random(rng, T, k, E, p_invalid=0.02)
    x = torch.randn(T, H, device=DEV)
    x[1, :128] = 0.0                       # an all-zero block
    x[2, 128 % H:128 % H + 128] *= 1e-6    # tiny values: subnormal e4m3 codes
    x = x.to(TORCH_DT[xdt])
    q, sc, q_ref, sc_ref = _fp8_run(ids_np, E, x, A)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))  # NaN padding kept


def test_dispatch_fp8_every_bf16_value():
    """Every bf16 value of magnitude <= 448 quantised with s = 1 (blocks whose
    amax is 448) and with s = 2^-10: covers every e4m3 rounding tie."""
    allv = torch.arange(-(2 ** 15), 2 ** 15, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    v = allv[torch.isfinite(allv.float()) & (allv.float().abs() <= 448)]
    per = 127
    nblk = (v.numel() + per - 1) // per
    blocks = torch.zeros(nblk, 128, dtype=torch.bfloat16)
    blocks[:, 0] = 448.0
    flat = blocks[:, 1:].reshape(-1)
    flat[: v.numel()] = v
    blocks[:, 1:] = flat.view(nblk, per)
    H = 128 * 16
    rows = (nblk + 15) // 16
    x = torch.zeros(rows * 16, 128, dtype=torch.bfloat16)
    x[:nblk] = blocks
    x = x.view(rows, H)
    x = torch.cat([x, (x.float() * 2.0 ** -10).to(torch.bfloat16)]).to(DEV)
    T = x.shape[0]
    ids_np = (np.arange(T, dtype=np.int32) % 3).reshape(T, 1)
    q, sc, q_ref, sc_ref = _fp8_run(ids_np, 3, x, 1)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))


@pytest.mark.parametrize("amax", [417.5, 0.0999755859375, 3.0e15])
def test_dispatch_fp8_every_bf16_value_odd_scale(amax):
    """Every bf16 value of magnitude <= amax in 128-blocks whose amax is a
    value with a non-power-of-two scale amax / 448: x / s is then a general
    fp32 quotient, so this checks the correctly rounded division on every
    bf16 dividend against the oracle's."""
    allv = torch.arange(-(2 ** 15), 2 ** 15, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    v = allv[torch.isfinite(allv.float()) & (allv.float().abs() <= amax)]
    per = 127
    nblk = (v.numel() + per - 1) // per
    blocks = torch.zeros(nblk, 128, dtype=torch.bfloat16)
    blocks[:, 0] = amax
    flat = blocks[:, 1:].reshape(-1)
    flat[: v.numel()] = v
    blocks[:, 1:] = flat.view(nblk, per)
    rows = (nblk + 15) // 16
    x = torch.zeros(rows * 16, 128, dtype=torch.bfloat16)
    x[:nblk] = blocks
    x = x.view(rows, 128 * 16).to(DEV)
    T = x.shape[0]
    ids_np = (np.arange(T, dtype=np.int32) % 3).reshape(T, 1)
    q, sc, q_ref, sc_ref = _fp8_run(ids_np, 3, x, 1)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))


def test_dispatch_fp8_extreme_scales():
    """Blocks whose scale amax / 448 lies near and beyond 2^-60 and 2^60
    (the range where the quotient takes the one-reciprocal route), with
    random values and signed zeros inside them; all finite (2^110 * 448 is
    below the bf16 maximum), since the contract is for finite activations."""
    T, H = 64, 128 * 12
    g = torch.Generator().manual_seed(5)
    x = torch.randn(T, H, generator=g)
    exps = torch.tensor([-130, -80, -62, -61, -60, -59, -20, 0, 20, 59, 60, 61, 62, 70, 100, 110],
                        dtype=torch.float32)
    blk = x.view(T, 12, 128)
    e = exps[torch.randint(0, exps.numel(), (T, 12), generator=g)]
    blk *= (2.0 ** e)[:, :, None] * 448.0 / blk.abs().amax(dim=2, keepdim=True)
    x = blk.view(T, H)
    x[:, 5::17] = -0.0
    x = x.to(torch.bfloat16)
    ids_np = (np.arange(T, dtype=np.int32) % 4).reshape(T, 1)
    q, sc, q_ref, sc_ref = _fp8_run(ids_np, 4, x.to(DEV), 1)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(sc.view(np.uint32), sc_ref.view(np.uint32))


def test_dispatch_fp8_unaligned_scales():
    """Scale rows that start 4 bytes past a 16-byte boundary (the contract
    asks for 4-byte alignment only): same bytes as the oracle."""
    T, H, E, k, A = 150, 4096, 64, 6, 4
    rng = np.random.default_rng(11)
    ids_np = _ids_random(rng, T, k, E, p_invalid=0.02)
    x = torch.randn(T, H, device=DEV).to(torch.bfloat16)
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), E, blockscale_align=A)
    rows = T * k + E * (A - 1)
    q = torch.full((T * k, H), 0xAB, dtype=torch.uint8, device=DEV)
    sbuf = torch.full((rows * (H // 128) + 1,), float("nan"), device=DEV)
    sc = sbuf[1:].view(rows, H // 128)
    assert sc.data_ptr() % 16 == 4
    moe.moe_dispatch_rows_fp8(x, k, meta.output_permutation, meta.expert_offsets,
                              meta.blockscale_offsets, out_q=q, out_scales=sc)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, E, A)
    q_ref = np.full((T * k, H), 0xAB, np.uint8)
    sc_ref = np.full((rows, H // 128), np.nan, np.float32)
    oracle.dispatch_fp8(bits(x), "bf16", ids_np, ref_meta, q_ref, sc_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), sc_ref.view(np.uint32))


def test_dispatch_fp8_full_workload_sampled():
    w = CONFIGS["zipf_fp8_t16384_h4096_e288_k8"]
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    ids = torch.from_numpy(ids_np).to(DEV)
    A = w.block_align
    meta = moe.moe_prepare(ids, w.E, blockscale_align=A)
    q, sc = moe.moe_dispatch_rows_fp8(x, w.k, meta.output_permutation, meta.expert_offsets,
                                      meta.blockscale_offsets, blockscale_align=A)
    torch.cuda.synchronize()
    ref_meta = oracle.prepare(ids_np, w.E, A)
    rng = np.random.default_rng(1)
    toks = np.unique(rng.integers(0, w.T, 300))
    sub_ids = ids_np[toks]
    # oracle on the sampled tokens alone, placed at the rows / scale rows the
    # full problem gives them
    slots = (toks[:, None] * w.k + np.arange(w.k)).ravel()
    p = ref_meta["output_perm"][slots]
    e = ids_np.ravel()[slots]
    srow = ref_meta["bso"][e] + p - ref_meta["offsets"][e]
    sub_meta = dict(input_perm=np.arange(slots.size, dtype=np.int32),
                    offsets=np.zeros(w.E + 1, np.int32),
                    bso=np.zeros(w.E + 1, np.int32))
    # with zero offsets the oracle writes scale row p for row p: remap after
    q_sub, sc_sub = oracle.dispatch_fp8(bits(x[torch.from_numpy(toks).to(DEV)]), "bf16",
                                        sub_ids, sub_meta,
                                        scales=np.zeros((slots.size, w.H // 128), np.float32))
    np.testing.assert_array_equal(q[torch.from_numpy(p).long().to(DEV)].cpu().numpy(), q_sub)
    np.testing.assert_array_equal(sc[torch.from_numpy(srow).long().to(DEV)].cpu().numpy(), sc_sub)


# ---------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------

def _combine_check(y, out_perm_np, w_np, out_dtype, got):
    """Contract tolerance, then bit-exactness with the oracle."""
    ydt = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[y.dtype]
    ref = oracle.combine(bits(y), ydt, out_perm_np, w_np, out_dtype)
    g = bits(got)
    if out_dtype == "fp32":
        T, k = w_np.shape
        rows = y.double().cpu().numpy()[np.maximum(out_perm_np, 0)].reshape(T, k, -1)
        rows = rows * (out_perm_np.reshape(T, k, 1) >= 0)
        assert_f32_within_rel(g, ref, combine_magnitude(rows, w_np))
        np.testing.assert_array_equal(g.view(np.uint32), ref.view(np.uint32))
    else:
        assert_half_within_one_ulp(g, ref)
        np.testing.assert_array_equal(g, ref)


@pytest.mark.parametrize("ydt,odt", [("bf16", "bf16"), ("fp16", "fp16"), ("fp16", "fp32"),
                                     ("bf16", "fp32"), ("fp32", "fp32"), ("fp32", "bf16"),
                                     ("bf16", "fp16")])
@pytest.mark.parametrize("k", [1, 6, 8, 9, 16])
def test_combine_vs_oracle(ydt, odt, k):
    rng = np.random.default_rng(k)
    T, H = 211, 1024
    S = T * k
    y = torch.randn(S, H, device=DEV).to(TORCH_DT[ydt])
    out_perm = rng.permutation(S).astype(np.int32)
    out_perm[rng.random(S) < 0.03] = -1                 # slots with invalid ids
    w = rng.random((T, k)).astype(np.float32)
    w /= w.sum(axis=1, keepdims=True)
    got = moe.moe_combine(y, torch.from_numpy(out_perm).to(DEV), torch.from_numpy(w).to(DEV),
                          out_dtype=TORCH_DT[odt])
    torch.cuda.synchronize()
    _combine_check(y, out_perm, w, odt, got)


@pytest.mark.parametrize("name", ["uniform_t4096_h7168_e256_k8", "khot_t9216_h7168_e256_k8",
                                  "zipf_fp8_t16384_h4096_e288_k8", "zipf_fp16_t131072_h2048_e64_k6"])
def test_combine_full_workloads_sampled(name):
    w = CONFIGS[name]
    ids_np, wt_np, _, y = make_workload(w, device=DEV, with_x=False)
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, w.E)
    got = moe.moe_combine(y, meta.output_permutation, torch.from_numpy(wt_np).to(DEV),
                          out_dtype=TORCH_DT[w.out_dtype])
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    toks = np.unique(np.concatenate([rng.integers(0, w.T, 256), [0, w.T - 1]]))
    op = meta.output_permutation.cpu().numpy().reshape(w.T, w.k)[toks]
    y_sub = y[torch.from_numpy(op.ravel()).long().to(DEV)]
    local = np.arange(op.size, dtype=np.int32)
    _combine_check(y_sub, local, wt_np[toks], w.out_dtype, got[torch.from_numpy(toks).to(DEV)])


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_identity_expert_round_trip(dtype):
    """dispatch, then combine of the dispatched rows themselves with weights
    summing to 1, returns x bit-exactly."""
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(777)
    ids_np, wt_np, x, _ = make_workload(w, device=DEV, with_y=False)
    x = x.to(TORCH_DT[dtype])
    ids = torch.from_numpy(ids_np).to(DEV)
    meta = moe.moe_prepare(ids, w.E)
    xd = moe.moe_dispatch_rows(x, w.k, meta.input_permutation, meta.output_permutation)
    back = moe.moe_combine(xd, meta.output_permutation, torch.from_numpy(wt_np).to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(back, x)


# ---------------------------------------------------------------------------
# tiny fused path and the chained step
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("trial", range(12))
def test_prepare_dispatch_fused_vs_oracle(trial):
    rng = np.random.default_rng(500 + trial)
    if trial == 0:
        w = CONFIGS["tiny_t32_h4096_e256_k8"]
        ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
        E, k, A = w.E, w.k, 128
    else:
        T = int(rng.integers(0, 512))
        k = int(rng.integers(1, 9))
        E = int(rng.choice([1, 3, 64, 256, 1024]))
        A = int(rng.integers(1, 9))
        ids_np = _ids_random(rng, T, k, E, p_invalid=0.05, distinct=False)
        H = int(rng.choice([8, 64, 4096]))
        x = torch.randn(T, H, device=DEV).to(torch.bfloat16)
    T, H = x.shape
    ids = torch.from_numpy(ids_np).to(DEV)
    out = torch.full((T * k, H), 7.0, device=DEV).to(x.dtype)
    meta, out = moe.moe_prepare_dispatch(ids, E, x, blockscale_align=A, out=out)
    torch.cuda.synchronize()
    ref = oracle.prepare(ids_np, E, A)
    np.testing.assert_array_equal(meta.expert_counts.cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(meta.expert_offsets.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(meta.blockscale_offsets.cpu().numpy(), ref["bso"])
    np.testing.assert_array_equal(meta.input_permutation.cpu().numpy(), ref["input_perm"])
    np.testing.assert_array_equal(meta.output_permutation.cpu().numpy(), ref["output_perm"])
    assert meta.diag.cpu().numpy().tolist() == [ref["n_invalid"], 0]
    out_ref = bits(torch.full((T * k, H), 7.0).to(x.dtype))
    oracle.dispatch(bits(x), k, ref["input_perm"], out_ref)
    np.testing.assert_array_equal(bits(out), out_ref)


def test_chained_step_on_one_stream():
    """prepare -> dispatch -> combine enqueued back to back (programmatic
    dependent launch between them), checked at the end."""
    w = CONFIGS["khot_t9216_h7168_e256_k8"].scaled(2500)
    ids_np, wt_np, x, y = make_workload(w, device=DEV)
    ids = torch.from_numpy(ids_np).to(DEV)
    wt = torch.from_numpy(wt_np).to(DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(3):
            meta = moe.moe_prepare(ids, w.E)
            xd = moe.moe_dispatch_rows(x, w.k, meta.input_permutation, meta.output_permutation)
            out = moe.moe_combine(y, meta.output_permutation, wt)
    s.synchronize()
    ref = oracle.prepare(ids_np, w.E)
    np.testing.assert_array_equal(meta.output_permutation.cpu().numpy(), ref["output_perm"])
    np.testing.assert_array_equal(bits(xd), oracle.dispatch(bits(x), w.k, ref["input_perm"]))
    _combine_check(y, ref["output_perm"], wt_np, "bf16", out)


@pytest.mark.parametrize("S,E", [
    (4097, 511),            # one-launch path, widest expert range it takes (E + 1 = 512)
    (4097, 512),            # one expert more: the two-kernel path
    (32768, 511),           # 2 rounds, 32 blocks
    (40960, 255),           # last size at 1 round (80 rows of 256 staged counts)
    (40961, 255),           # first at 2 rounds
    (81920, 255),           # last size at 2 rounds
    (81921, 255),           # first at 3 rounds
    (1212416, 64),          # 148 blocks of 16 rounds: the last with input_permutation staged
    (303104, 64),           # 148 blocks of 4 rounds: input_permutation slot by slot
    (303105, 64),           # 5 rounds: input_permutation staged
    (1212417, 64),          # 17 rounds: input_permutation written slot by slot
    (2424832, 64),          # 32 rounds: the last with every round's id load unrolled
    (2424833, 64),          # 33 rounds: id loads four at a time
    (4849664, 64),          # the largest one-launch problem on 148 SMs (64 rounds)
    (4849665, 64),          # one slot more: the two-kernel path
])
def test_prepare_path_boundaries(S, E):
    """Sizes on each side of the rules that pick the prepare path and the
    one-launch path's rounds, with k = 1 (S tokens) and 2 % invalid ids."""
    rng = np.random.default_rng(S + E)
    ids = _ids_random(rng, S, 1, E, p_invalid=0.02, distinct=False)
    _check_prepare(ids, E, A=8)
