"""Pins for the CPU oracle: each check ties the oracle to something other
than itself — a library routine, a brute force, a closed form, an invariant
of the definition, or a hand-worked example — so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them.

Sources of the definitions: sglang PR #19058 "[jit_kernel] Add
prepare_moe_input JIT kernels", section "Changes" (prepare_moe_input,
shuffle_rows, apply_shuffle_mul_sum); TensorRT-LLM PR #9592 (expanded /
permuted index naming, FP8 block-scale path).  The e4m3 format facts (bias
7, max 448, subnormal step 2^-9, no infinities) are those of the OCP FP8
E4M3 format.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make_workload

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------------------
# scalar formats
# ---------------------------------------------------------------------------

def test_bf16_decode_exhaustive_vs_torch():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = oracle.bf16_to_f32(bits)
    np.testing.assert_array_equal(got.view(np.uint32)[~np.isnan(ref)], ref.view(np.uint32)[~np.isnan(ref)])
    assert np.isnan(got[np.isnan(ref)]).all()


def test_f16_decode_exhaustive_vs_numpy():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = oracle.f16_to_f32(bits)
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got.view(np.uint32)[ok], ref.view(np.uint32)[ok])
    assert np.isnan(got[~ok]).all()


def _f32_samples(n):
    """Random fp32 bit patterns plus values sitting exactly on rounding ties."""
    u = RNG.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    return f[np.isfinite(f)]


def test_f32_to_bf16_vs_torch():
    f = _f32_samples(2_000_000)
    # ties: low 16 bits exactly 0x8000, both parities of the kept bit
    tie = (RNG.integers(0, 1 << 16, size=100_000).astype(np.uint32) << 16) | 0x8000
    f = np.concatenate([f, tie.view(np.float32)])
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_bf16(f), ref)


def test_f32_to_f16_vs_numpy():
    f = _f32_samples(2_000_000)
    # values around the fp16 range: subnormals, ties at 13 dropped bits,
    # the overflow threshold 65520
    g = (RNG.standard_normal(500_000) * np.exp2(RNG.integers(-26, 17, 500_000))).astype(np.float32)
    ties = ((RNG.integers(0, 1 << 19, 100_000).astype(np.uint32) << 13) | 0x1000).view(np.float32)
    edges = np.array([65504, 65519.996, 65520, 65536, 2**-24, 2**-25, 3 * 2**-26, 2**-14,
                      2**-14 - 2**-25], np.float32)
    f = np.concatenate([f, g, ties, edges, -edges])
    f = f[np.isfinite(f)]
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_f16(f), ref)


def _e4m3_grid():
    """All finite e4m3 magnitudes, decoded by torch (library routine)."""
    codes = np.arange(0x7f, dtype=np.uint8)  # 0x00..0x7e
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()


def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_to_f32(codes)
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert np.isnan(got[~ok]).all() and set(codes[~ok].tolist()) == {0x7f, 0xff}


def test_e4m3_closed_forms():
    # hand-derived from the format: bias 7, 3 fraction bits, max 448
    cases = [  # (value, code); a list, since 0.0 and -0.0 are equal dict keys
        (448.0, 0x7E), (1e9, 0x7E), (464.0, 0x7E), (np.inf, 0x7E),     # saturate
        (-448.0, 0xFE), (-np.inf, 0xFE),
        (1.0, 0x38), (1.125, 0x39), (1.0625, 0x38),                    # tie 1+1/16 -> even (1.0)
        (1.1875, 0x3A),                                                # tie 1+3/16 -> even (1.25)
        (2.0 ** -6, 0x08), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),      # min normal, min subnormal, tie to 0
        (3 * 2.0 ** -10, 0x02),                                        # 1.5 steps -> 2 (even)
        (3 * 2.0 ** -11, 0x01), (0.0, 0x00), (-0.0, 0x80),
        (240.0, 0x77), (256.0, 0x78), (416.0, 0x7D), (432.0, 0x7E),    # 432 = tie 416|448 -> even 448
        (-3.5, 0xC6),
    ]
    got = oracle.f32_to_e4m3(np.array([v for v, _ in cases], np.float32))
    np.testing.assert_array_equal(got, np.array([c for _, c in cases], np.uint8))
    assert oracle.f32_to_e4m3(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_e4m3_encode_vs_torch_ties_and_random():
    grid = _e4m3_grid()
    # midpoints between neighbouring e4m3 values and their fp32 neighbours
    mids = ((grid[1:].astype(np.float64) + grid[:-1]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                           grid, np.nextafter(grid[1:], np.float32(0)), np.nextafter(grid, np.float32(1e9))])
    rnd = (RNG.standard_normal(3_000_000) * np.exp2(RNG.integers(-14, 10, 3_000_000))).astype(np.float32)
    f = np.concatenate([near, -near, rnd])
    f = f[np.abs(f) <= 448]  # torch maps magnitudes above 464 to NaN: compare inside the range only
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.f32_to_e4m3(f), ref)


def test_e4m3_roundtrip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    np.testing.assert_array_equal(oracle.f32_to_e4m3(oracle.e4m3_to_f32(codes)), codes)


# ---------------------------------------------------------------------------
# prepare
# ---------------------------------------------------------------------------

def test_prepare_hand_worked_example():
    # ids [[2,0],[1,2],[2,1]], E=3, k=2 -> slots i: e(0)=2 e(1)=0 e(2)=1 e(3)=2 e(4)=2 e(5)=1
    # expert 0 holds slot 1; expert 1 slots 2,5; expert 2 slots 0,3,4 (ascending)
    ids = np.array([[2, 0], [1, 2], [2, 1]], np.int32)
    m = oracle.prepare(ids, E=3, block_align=4)
    assert m["counts"].tolist() == [1, 2, 3]
    assert m["offsets"].tolist() == [0, 1, 3, 6]
    assert m["bso"].tolist() == [0, 4, 8, 12]
    assert m["input_perm"].tolist() == [1, 2, 5, 0, 3, 4]
    assert m["output_perm"].tolist() == [3, 0, 1, 4, 5, 2]
    assert m["n_invalid"] == 0


def test_prepare_hand_worked_invalid_and_duplicates():
    # a token may name an expert twice; ids -1 and 3 (E=3) are invalid
    ids = np.array([[1, 1], [-1, 0], [3, 1]], np.int32)
    m = oracle.prepare(ids, E=3)
    assert m["counts"].tolist() == [1, 3, 0]
    assert m["offsets"].tolist() == [0, 1, 4, 4]
    assert m["input_perm"].tolist() == [3, 0, 1, 5, -1, -1]
    assert m["output_perm"].tolist() == [1, 2, -1, 0, -1, 3]
    assert m["n_invalid"] == 2


@pytest.mark.parametrize("trial", range(60))
def test_prepare_vs_bruteforce_tiny(trial):
    rng = np.random.default_rng(trial)
    T = int(rng.integers(0, 9))
    k = int(rng.integers(1, 5))
    E = int(rng.integers(1, 7))
    A = int(rng.integers(1, 5))
    ids = rng.integers(-1, E + 1, size=(T, k)).astype(np.int32)  # duplicates and invalid ids included
    m = oracle.prepare(ids, E, A)
    b = oracle.brute_prepare(ids, E, A)
    for key in ("counts", "offsets", "bso", "input_perm", "output_perm"):
        assert np.asarray(m[key]).tolist() == list(b[key]), key
    assert m["n_invalid"] == b["n_invalid"]


def _check_prepare_invariants(ids, E, A, m):
    flat = ids.ravel()
    S = flat.size
    # library special cases
    np.testing.assert_array_equal(m["counts"], np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(m["offsets"][1:], np.cumsum(m["counts"]))
    ref_perm = torch.argsort(torch.from_numpy(flat.astype(np.int64)), stable=True).numpy()
    np.testing.assert_array_equal(m["input_perm"], ref_perm)
    # invariants
    assert m["offsets"][0] == 0 and m["offsets"][E] == S
    inp, outp = m["input_perm"], m["output_perm"]
    assert np.array_equal(np.sort(inp), np.arange(S))
    np.testing.assert_array_equal(outp[inp], np.arange(S))
    np.testing.assert_array_equal(inp[outp], np.arange(S))
    assert (np.diff(flat[inp]) >= 0).all()
    for e in range(E):
        seg = inp[m["offsets"][e]:m["offsets"][e + 1]]
        assert (np.diff(seg) > 0).all()
        assert (flat[seg] == e).all()
    pad = np.diff(m["bso"]) - m["counts"]
    assert (np.diff(m["bso"]) % A == 0).all() and (pad >= 0).all() and (pad < A).all()


@pytest.mark.parametrize("name", list(CONFIGS))
def test_prepare_invariants_on_workloads(name):
    w = CONFIGS[name]
    if w.S > 200_000:
        w = w.scaled(200_000 // w.k)
    ids, _, _, _ = make_workload(w, with_x=False, with_y=False)
    A = w.block_align if w.block_align > 1 else 128
    m = oracle.prepare(ids, w.E, A)
    _check_prepare_invariants(ids, w.E, A, m)
    m1 = oracle.prepare(ids, w.E, 1)
    np.testing.assert_array_equal(m1["bso"], m1["offsets"])


# ---------------------------------------------------------------------------
# dispatch
# ---------------------------------------------------------------------------

def test_dispatch_same_dtype_vs_index_select():
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(64)
    ids, _, x, _ = make_workload(w, with_y=False)
    m = oracle.prepare(ids, w.E)
    xb = x.view(torch.int16).numpy()
    got = oracle.dispatch(xb, w.k, m["input_perm"])
    ref = torch.from_numpy(xb).index_select(0, torch.from_numpy(m["input_perm"] // w.k).long()).numpy()
    np.testing.assert_array_equal(got, ref)
    # every token row appears exactly k times
    rows, mult = np.unique(got.view(np.dtype((np.void, got.shape[1] * 2))), return_counts=True)
    assert (mult == w.k).all() and rows.size == w.T


def test_dispatch_leaves_invalid_rows_untouched():
    ids = np.array([[0, 5], [1, 0]], np.int32)  # id 5 invalid with E=2
    m = oracle.prepare(ids, 2)
    x = np.array([[1, 2], [3, 4]], np.float32)
    out = np.full((4, 2), -7.0, np.float32)
    oracle.dispatch(x, 2, m["input_perm"], out)
    np.testing.assert_array_equal(out, [[1, 2], [3, 4], [3, 4], [-7, -7]])


# ---------------------------------------------------------------------------
# fp8 dispatch
# ---------------------------------------------------------------------------

def _fp8_case(T=48, H=512, E=16, k=4, dtype="bf16", seed=7):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(seed)).to(tdt)
    x[3, 128:256] = 0           # an all-zero block
    x[5, :128] *= 1e-3          # a block of tiny values
    return ids, x


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_dispatch_fp8_vs_torch_witness(dtype):
    T, H, E, k, A = 48, 512, 16, 4, 8
    ids, x = _fp8_case(T, H, E, k, dtype)
    m = oracle.prepare(ids, E, A)
    q, scales = oracle.dispatch_fp8(x.view(torch.int16).numpy().view(np.uint16), dtype, ids, m)
    xf = x.float().view(T, H // 128, 128)
    amax = xf.abs().amax(dim=2)                       # torch reduction
    s_ref = amax / 448.0                              # torch fp32 division
    safe = torch.where(s_ref == 0, torch.ones_like(s_ref), s_ref)
    q_tok = (xf / safe[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).view(T, H)
    q_tok[(s_ref == 0).repeat_interleave(128, dim=1)] = 0
    inp = m["input_perm"]
    np.testing.assert_array_equal(q, q_tok.numpy()[inp // k])
    e_of_p = ids.ravel()[inp]
    srow = m["bso"][e_of_p] + np.arange(T * k) - m["offsets"][e_of_p]
    np.testing.assert_array_equal(scales[srow], s_ref.numpy()[inp // k])
    # padding rows of the scale tensor were never written
    written = np.zeros(scales.shape[0], bool)
    written[srow] = True
    assert (scales[~written] == 0).all()


def test_dispatch_fp8_decode_error_bound_and_amax_code():
    T, H, E, k = 32, 1024, 8, 2
    ids, x = _fp8_case(T, H, E, k, "bf16", seed=11)
    m = oracle.prepare(ids, E, 1)
    q, scales = oracle.dispatch_fp8(x.view(torch.int16).numpy().view(np.uint16), "bf16", ids, m)
    xr = x.double().numpy()[m["input_perm"] // k]
    s = np.repeat(scales, 128, axis=1).astype(np.float64)
    dec = oracle.e4m3_to_f32(q).reshape(q.shape).astype(np.float64) * s
    # |x - decode(q) * s| <= half an e4m3 step of v = x / s (step 2^(e-3) for
    # v in [2^e, 2^(e+1)), 2^-9 below 2^-6), plus the fp32 rounding of x / s
    v = np.abs(xr / np.where(s == 0, 1, s))
    half_step = np.where(v >= 2.0 ** -6, np.exp2(np.floor(np.log2(np.maximum(v, 2.0 ** -6))) - 4), 2.0 ** -10)
    assert (np.abs(dec - xr) <= half_step * s + np.abs(xr) * 2.0 ** -23).all()
    # the element that attains amax encodes to +-448 exactly
    blocks = np.abs(xr).reshape(T * k, H // 128, 128)
    hit = blocks.argmax(axis=2)
    qb = q.reshape(T * k, H // 128, 128)
    codes = np.take_along_axis(qb, hit[..., None], axis=2)[..., 0]
    live = blocks.max(axis=2) > 0
    assert ((codes[live] & 0x7F) == 0x7E).all()


# ---------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------

def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype != torch.float32 else t.numpy()


def _from_bits(a, dtype):
    if dtype == "fp32":
        return torch.from_numpy(a)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    return torch.from_numpy(a.view(np.int16)).view(tdt)


def test_combine_hand_worked_example():
    # two tokens, k=2, H=3; y rows in dispatched order; weights powers of two
    y = torch.tensor([[1, 2, 3], [4, 5, 6], [8, 16, 32], [0.5, -1, 2]], dtype=torch.bfloat16)
    out_perm = np.array([2, 0, 3, 1], np.int32)      # token0 -> rows 2,0 ; token1 -> rows 3,1
    w = np.array([[0.5, 0.25], [2.0, 0.125]], np.float32)
    got = _from_bits(oracle.combine(_bits(y), "bf16", out_perm, w, "fp32"), "fp32")
    # token0: 0.5*[8,16,32] + 0.25*[1,2,3] = [4.25, 8.5, 16.75]
    # token1: 2*[0.5,-1,2] + 0.125*[4,5,6] = [1.5, -1.375, 4.75]
    assert got.tolist() == [[4.25, 8.5, 16.75], [1.5, -1.375, 4.75]]


@pytest.mark.parametrize("y_dtype,out_dtype", [("bf16", "bf16"), ("fp16", "fp16"), ("fp16", "fp32"),
                                               ("bf16", "fp32"), ("fp32", "bf16"), ("fp32", "fp32")])
def test_combine_identity_round_trip(y_dtype, out_dtype):
    """dispatch then combine with weights summing to 1 returns x."""
    T, H, E, k = 40, 256, 12, 4
    rng = np.random.default_rng(3)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[y_dtype]
    # values on the bf16 grid, so that every output dtype can hold x exactly
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).to(tdt)
    m = oracle.prepare(ids, E)
    y = oracle.dispatch(_bits(x), k, m["input_perm"])
    w = rng.random((T, k)).astype(np.float32)
    w /= w.sum(axis=1, keepdims=True)
    got = _from_bits(oracle.combine(y, y_dtype, m["output_perm"], w, out_dtype), out_dtype)
    if out_dtype == y_dtype and out_dtype != "fp32":
        assert torch.equal(got, x)
    elif out_dtype == "fp32":
        torch.testing.assert_close(got, x.float(), rtol=1e-6, atol=0)
    else:
        assert torch.equal(got, x.to(got.dtype))


def test_combine_one_hot_selects_row_exactly():
    T, H, k = 16, 128, 6
    rng = np.random.default_rng(9)
    y = torch.randn(T * k, H, generator=torch.Generator().manual_seed(1)).to(torch.float16)
    out_perm = rng.permutation(T * k).astype(np.int32)
    pick = rng.integers(0, k, T)
    w = np.zeros((T, k), np.float32)
    w[np.arange(T), pick] = 1.0
    got = _from_bits(oracle.combine(_bits(y), "fp16", out_perm, w, "fp16"), "fp16")
    ref = y[torch.from_numpy(out_perm.reshape(T, k)[np.arange(T), pick]).long()]
    assert torch.equal(got, ref)


def test_combine_within_fp64_error_bound():
    """|oracle - exact| <= k * 2^-24 * sum_j |w y| + half an output ulp."""
    w_ = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(24)
    ids, wt, _, y = make_workload(w_, with_x=False)
    m = oracle.prepare(ids, w_.E)
    got32 = oracle.combine(_bits(y), "bf16", m["output_perm"], wt, "fp32")
    yy = y.double().numpy()[m["output_perm"]].reshape(w_.T, w_.k, w_.H)
    exact = np.einsum("tk,tkh->th", wt.astype(np.float64), yy)
    mag = np.einsum("tk,tkh->th", np.abs(wt.astype(np.float64)), np.abs(yy))
    assert (np.abs(got32 - exact) <= w_.k * 2.0 ** -24 * mag + 1e-30).all()
    gotb = _from_bits(oracle.combine(_bits(y), "bf16", m["output_perm"], wt, "bf16"), "bf16")
    # the bf16 output is the fp32 result rounded once (torch RNE as witness)
    assert torch.equal(gotb, torch.from_numpy(got32).to(torch.bfloat16))


def test_combine_skips_invalid_slots():
    y = torch.tensor([[1.0, 2.0], [3.0, 4.0]], dtype=torch.float32)
    out_perm = np.array([1, -1, 0, -1], np.int32)
    w = np.array([[0.5, 100.0], [2.0, 100.0]], np.float32)
    got = oracle.combine(y.numpy(), "fp32", out_perm, w, "fp32")
    np.testing.assert_array_equal(got, [[1.5, 2.0], [2.0, 4.0]])


# ---------------------------------------------------------------------------
# grouped-GEMM metadata (problem sizes, tile-padded layout)
# ---------------------------------------------------------------------------

def test_problem_sizes_closed_form():
    counts = np.array([0, 5, 3, 9], np.int32)
    ps1, ps2 = oracle.problem_sizes(counts, 14336, 7168, 7168, 7168)
    np.testing.assert_array_equal(ps1, np.stack([counts, np.full(4, 14336), np.full(4, 7168)], 1))
    np.testing.assert_array_equal(ps2, np.stack([counts, np.full(4, 7168), np.full(4, 7168)], 1))


def test_tile_layout_hand_worked_example():
    # ids [[2,0],[1,2],[2,1]], E=3, tile 2: counts [1,2,3] pad to [2,2,4]
    # rows: expert 0 -> 0 (1 padding), expert 1 -> 2,3, expert 2 -> 4,5,6 (7 padding)
    ids = np.array([[2, 0], [1, 2], [2, 1]], np.int32)
    m = oracle.prepare(ids, 3)
    L = oracle.tile_layout(ids, m, 3, 2, 6)
    assert L["padded_offsets"].tolist() == [0, 2, 4, 8]
    assert L["num_tiles"] == 4 and L["total_padded"] == 8
    assert L["tile_group"].tolist() == [0, 1, 2, 2, -1, -1]
    assert L["tile_mn_limit"].tolist() == [1, 4, 7, 7, -1, -1]
    assert L["exp2perm"].tolist() == [4, 0, 2, 5, 6, 3]
    assert L["perm2exp"].tolist() == [1, -1, 2, 5, 0, 3, 4, -1, -1, -1, -1, -1]
    assert oracle.tile_layout(ids, m, 3, 2, 3) is None   # 6 rows cannot hold 8


@pytest.mark.parametrize("tile", [1, 7, 128])
@pytest.mark.parametrize("name", ["uniform_t4096_h7168_e256_k8", "zipf_fp8_t16384_h4096_e288_k8"])
def test_tile_layout_invariants(name, tile):
    w = CONFIGS[name].scaled(3000)
    ids, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids = ids.copy()
    ids[::53, 1] = -1
    m = oracle.prepare(ids, w.E)
    max_tiles = -(-w.S // tile) + w.E
    L = oracle.tile_layout(ids, m, w.E, tile, max_tiles)
    per_expert = -(-m["counts"] // tile)
    # library special case: the tile owners are each expert repeated once per tile
    np.testing.assert_array_equal(L["tile_group"][:L["num_tiles"]],
                                  np.repeat(np.arange(w.E), per_expert))
    assert (L["tile_group"][L["num_tiles"]:] == -1).all()
    np.testing.assert_array_equal(L["padded_offsets"][1:], np.cumsum(per_expert * tile))
    g = L["tile_group"][:L["num_tiles"]]
    np.testing.assert_array_equal(L["tile_mn_limit"][:L["num_tiles"]],
                                  L["padded_offsets"][g] + m["counts"][g])
    # the padded rows hold exactly the valid slots, each expert's in its own range, in order
    flat = ids.ravel()
    valid = (flat >= 0) & (flat < w.E)
    e2p = L["exp2perm"]
    assert (e2p[~valid] == -1).all()
    rows = e2p[valid]
    assert np.unique(rows).size == rows.size
    np.testing.assert_array_equal(L["perm2exp"][rows], np.nonzero(valid)[0])
    assert (np.delete(L["perm2exp"], rows) == -1).all()
    e = flat[valid]
    assert (rows >= L["padded_offsets"][e]).all() and (rows < L["padded_offsets"][e] + m["counts"][e]).all()
    np.testing.assert_array_equal(rows - L["padded_offsets"][e], m["output_perm"][valid] - m["offsets"][e])


# ---------------------------------------------------------------------------
# one rank's expert window, int64 ids, output memset
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("base,E", [(0, 256), (64, 32), (250, 16), (2**33, 40)])
def test_prepare_local_equals_prepare_of_shifted_ids(base, E):
    """The window [base, base+E) over int64 ids is prepare of ids - base with
    every id outside the window made invalid (a different code path)."""
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(700)
    ids32, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids = ids32.astype(np.int64) + (base - 64 if base >= 64 else 0)
    m = oracle.prepare_local(ids, base, E, 8)
    shifted = ids - base
    shifted[(shifted < 0) | (shifted >= E)] = -1
    r = oracle.prepare(shifted.astype(np.int32), E, 8)
    for key in ("counts", "offsets", "bso", "input_perm", "output_perm", "n_invalid"):
        np.testing.assert_array_equal(m[key], r[key])


def test_prepare_local_hand_worked_example():
    # window [10, 13): ids 10, 12 local (experts 0 and 2); 9, 13, -1 not local
    ids = np.array([[12, 9], [10, 13], [12, -1]], np.int64)
    m = oracle.prepare_local(ids, 10, 3)
    assert m["counts"].tolist() == [1, 0, 2]
    assert m["offsets"].tolist() == [0, 1, 1, 3]
    assert m["input_perm"].tolist() == [2, 0, 4, -1, -1, -1]
    assert m["output_perm"].tolist() == [1, -1, 0, -1, 2, -1]
    assert m["n_invalid"] == 3


def test_output_memset_zeroes_exactly_the_routed_tokens():
    rng = np.random.default_rng(4)
    T, k, H = 50, 4, 24
    out_perm = rng.integers(0, 10, size=T * k).astype(np.int32)
    out_perm[rng.random(T * k) < 0.6] = -1
    out = rng.standard_normal((T, H)).astype(np.float32)
    before = out.copy()
    oracle.output_memset(out, out_perm, k)
    routed = (out_perm.reshape(T, k) >= 0).any(axis=1)
    assert (out[routed] == 0).all()
    np.testing.assert_array_equal(out[~routed], before[~routed])
    assert routed.any() and (~routed).any()


# ---------------------------------------------------------------------------
# NVFP4 (E2M1 elements, one E4M3 scale per 16 elements)
# ---------------------------------------------------------------------------

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # codes 0..7, from the format


def test_e2m1_decode_all_codes():
    got = oracle.e2m1_to_f32(np.arange(16))
    np.testing.assert_array_equal(got[:8], E2M1_VALUES)
    np.testing.assert_array_equal(got[8:], [-v for v in E2M1_VALUES])


def test_e2m1_closed_forms():
    cases = [(0.25, 0), (0.26, 1), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6),
             (5.0, 6), (5.01, 7), (6.0, 7), (100.0, 7), (-0.75, 10), (-5.0, 14), (-0.0, 8)]
    got = oracle.f32_to_e2m1(np.array([v for v, _ in cases], np.float32))
    np.testing.assert_array_equal(got, np.array([c for _, c in cases], np.uint8))


def test_e2m1_encode_vs_bruteforce_nearest_even():
    """Nearest representable magnitude by brute force over the 8 values, ties
    to the even code (fraction bit 0), saturation at 6."""
    rng = np.random.default_rng(8)
    vals = np.array(E2M1_VALUES)
    mids = (vals[1:] + vals[:-1]) / 2
    f = np.concatenate([rng.uniform(-8, 8, 200_000), mids, -mids,
                        np.nextafter(mids.astype(np.float32), np.float32(0)),
                        np.nextafter(mids.astype(np.float32), np.float32(9))]).astype(np.float32)
    a = np.minimum(np.abs(f).astype(np.float64), 6.0)
    dist = np.abs(a[:, None] - vals[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = code | np.where(np.signbit(f), 8, 0)
    np.testing.assert_array_equal(oracle.f32_to_e2m1(f), code.astype(np.uint8))


def test_dispatch_nvfp4_decode_bound_and_layout():
    T, H, E, k, A = 40, 256, 8, 3, 4
    rng = np.random.default_rng(9)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    x[0, :16] = 0
    m = oracle.prepare(ids, E, A)
    q, sc = oracle.dispatch_nvfp4(x.view(torch.int16).numpy().view(np.uint16), "bf16", ids, m)
    xr = x.float().numpy()[m["input_perm"] // k]
    codes = np.stack([q & 0xF, q >> 4], axis=2).reshape(T * k, H)     # low nibble first
    vals = oracle.e2m1_to_f32(codes).reshape(T * k, H).astype(np.float64)
    e = ids.ravel()[m["input_perm"]]
    srow = m["bso"][e] + np.arange(T * k) - m["offsets"][e]
    d = oracle.e4m3_to_f32(sc[srow].ravel()).reshape(T * k, H // 16).astype(np.float64)
    dd = np.repeat(d, 16, axis=1)
    # the scale is e4m3(amax / 6): the amax element lands on +-6 or one e2m1 step below
    blocks = np.abs(xr).reshape(T * k, H // 16, 16)
    amax = blocks.max(axis=2)
    np.testing.assert_array_equal(sc[srow], oracle.f32_to_e4m3((amax / 6.0).astype(np.float32)).reshape(amax.shape))
    # every element within half an e2m1 step (of x / d) of its value, saturation aside
    v = np.abs(xr) / np.where(dd == 0, 1, dd)
    half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    ok = (np.abs(vals * dd - xr) <= half * dd * (1 + 1e-6) + 1e-30) | (v > 6)
    assert ok.all()
    # token 0's first block is all zero: scale byte 0 and codes 0 on each of its k rows
    rows0 = np.nonzero(m["input_perm"] // k == 0)[0]
    assert len(rows0) == k
    assert (sc[srow[rows0], 0] == 0).all() and (q[rows0, :8] == 0).all()


# ---------------------------------------------------------------------------
# Expert-parallel exchange: the receiving rank's layout
# ---------------------------------------------------------------------------

def test_ep_recv_layout_hand_worked():
    # 2 source ranks, 3 local experts.  Source 0 sends 2 rows of expert 0 and
    # 1 of expert 2 (received rows 0, 1 | 2); source 1 sends 1 row of expert
    # 0 and 3 of expert 1 (received rows 3 | 4, 5, 6).  Grouped by expert,
    # then source: expert 0 = rows 0, 1 (source 0), 3 (source 1); expert 1 =
    # rows 4, 5, 6; expert 2 = row 2.
    lay = oracle.ep_recv_layout(np.array([[2, 0, 1], [1, 3, 0]], np.int32))
    assert lay["recv_offsets"].tolist() == [0, 3, 7]
    assert lay["local_offsets"].tolist() == [0, 3, 6, 7]
    assert lay["local_to_recv"].tolist() == [0, 1, 3, 4, 5, 6, 2]
    assert lay["recv_to_local"].tolist() == [0, 1, 6, 2, 3, 4, 5]


@pytest.mark.parametrize("R,El,seed", [(1, 5, 0), (2, 3, 1), (4, 8, 2), (8, 1, 3), (3, 7, 4)])
def test_ep_recv_layout_invariants(R, El, seed):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 6, size=(R, El)).astype(np.int32)
    c[rng.random((R, El)) < 0.3] = 0
    lay = oracle.ep_recv_layout(c)
    n = int(c.sum())
    r2l, l2r = lay["recv_to_local"], lay["local_to_recv"]
    assert sorted(r2l.tolist()) == list(range(n)) and (r2l[l2r] == np.arange(n)).all()
    # every received row lands inside its local expert's grouped range, and
    # each (source, expert) run stays in order
    q = 0
    for s in range(R):
        for le in range(El):
            g = r2l[q:q + c[s, le]]
            assert (g >= lay["local_offsets"][le]).all() and (g < lay["local_offsets"][le + 1]).all()
            assert (np.diff(g) == 1).all()
            q += c[s, le]


@pytest.mark.parametrize("R,El,k,seed", [(2, 4, 2, 0), (4, 3, 3, 1), (3, 5, 1, 2)])
def test_ep_exchange_reproduces_the_global_prepare(R, El, k, seed):
    """Exchange + regroup on every rank equals one prepare over all ranks'
    tokens taken together (in rank order), restricted to the rank's expert
    window: the stable order expert, then global slot, is the order
    expert, then source rank, then the source's own slot order."""
    rng = np.random.default_rng(seed)
    E = R * El
    T = [int(rng.integers(0, 9)) for _ in range(R)]
    ids = [np.stack([rng.permutation(E)[:k] for _ in range(t)]).astype(np.int32)
           if t else np.zeros((0, k), np.int32) for t in T]
    for r in range(R):                       # a few invalid ids
        if T[r]:
            ids[r][0, 0] = -1
    metas = [oracle.prepare(i, E) for i in ids]
    g = oracle.prepare(np.concatenate(ids), E)
    tok0 = np.concatenate([[0], np.cumsum(T)])
    for dst in range(R):
        lo, hi = dst * El, (dst + 1) * El
        c = np.stack([m["counts"][lo:hi] for m in metas])
        lay = oracle.ep_recv_layout(c)
        # global slot index of every received row, source blocks in order
        recv = np.concatenate([tok0[s] * k + metas[s]["input_perm"][metas[s]["offsets"][lo]:
                                                                     metas[s]["offsets"][hi]]
                               for s in range(R)])
        assert np.array_equal(recv[lay["local_to_recv"]],
                              g["input_perm"][g["offsets"][lo]:g["offsets"][hi]])
        assert np.array_equal(lay["local_offsets"], g["offsets"][lo:hi + 1] - g["offsets"][lo])
