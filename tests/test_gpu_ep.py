"""Expert-parallel exchange on the GPU: the receive-layout kernel against
the oracle, the exchange of R ranks emulated on one GPU through the
library's kernels, and combine_permute_b200.ep over a one-rank NCCL group.

The emulation moves each source's row block to its destination with a
device copy (what the all-to-all does between GPUs), so every per-rank step
runs in the library's kernels: prepare, dispatch, the receive layout, the
regroup gathers and combine.  The result must be bit-exact against the
single-GPU answer of the oracle over all ranks' tokens taken together.
"""

import ctypes
import dataclasses
import socket

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
import oracle
from combine_permute_b200 import _lib
from tests._helpers import bits
from workloads import CONFIGS, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _counts(R, El, seed, zero_frac=0.3, hi=50):
    rng = np.random.default_rng(seed)
    c = rng.integers(0, hi, size=(R, El)).astype(np.int32)
    c[rng.random((R, El)) < zero_frac] = 0
    return c


@pytest.mark.parametrize("R,El,seed", [(1, 1, 0), (2, 128, 1), (8, 32, 2), (4, 288, 3),
                                       (64, 128, 4), (8, 1024, 5), (3, 7, 6)])
def test_recv_layout_matches_oracle(R, El, seed):
    c = _counts(R, El, seed, hi=30 if R * El > 2000 else 200)
    ref = oracle.ep_recv_layout(c)
    n = int(c.sum())
    lay = moe.moe_ep_recv_layout(torch.from_numpy(c).to(DEV), n)
    torch.cuda.synchronize()
    assert int(lay.num_recv.item()) == n
    for key in ("recv_offsets", "local_offsets", "recv_to_local", "local_to_recv"):
        assert np.array_equal(getattr(lay, key).cpu().numpy(), ref[key]), key


def test_recv_layout_empty_and_capacity_overflow():
    c = np.zeros((4, 16), np.int32)
    lay = moe.moe_ep_recv_layout(torch.from_numpy(c).to(DEV), 0)
    torch.cuda.synchronize()
    assert int(lay.num_recv.item()) == 0 and not lay.recv_offsets.any() and not lay.local_offsets.any()
    # too small a capacity: offsets and the count only, maps untouched
    c = _counts(4, 16, 9)
    n = int(c.sum())
    lib = _lib.load()
    i32 = dict(dtype=torch.int32, device=DEV)
    ro, lo, num = torch.empty(5, **i32), torch.empty(17, **i32), torch.empty(1, **i32)
    r2l, l2r = torch.full((n,), -5, **i32), torch.full((n,), -5, **i32)
    st = lib.moe_ep_recv_layout(torch.from_numpy(c).to(DEV).data_ptr(), 4, 16, n - 1,
                                ro.data_ptr(), lo.data_ptr(), r2l.data_ptr(), l2r.data_ptr(),
                                num.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    ref = oracle.ep_recv_layout(c)
    assert int(num.item()) == n and np.array_equal(ro.cpu().numpy(), ref["recv_offsets"])
    assert np.array_equal(lo.cpu().numpy(), ref["local_offsets"])
    assert (r2l == -5).all() and (l2r == -5).all()


@pytest.mark.parametrize("R,T,seed", [(2, 700, 0), (4, 1500, 1), (8, 300, 2)])
def test_exchange_of_emulated_ranks_matches_single_gpu(R, T, seed):
    """R ranks of the uniform workload's shape (E = 256 experts, top-8,
    H = 7168, bf16), each with its own tokens; rank r owns 256 / R experts."""
    base = CONFIGS["uniform_t4096_h7168_e256_k8"]
    E, k, H = base.E, base.k, base.H
    El = E // R
    ranks = []
    for r in range(R):
        w = dataclasses.replace(base, T=T + 37 * r, seed=seed * 100 + r, name=f"rank{r}")
        ids_np, wt_np, x, _ = make_workload(w, device=DEV, with_y=False)
        ids_np[::53, 0] = -1  # a few invalid ids
        meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), E)
        xd = moe.moe_dispatch_rows(x, k, meta.input_permutation, meta.output_permutation)
        ranks.append(dict(T=w.T, ids=ids_np, wt=wt_np, x=x, meta=meta, xd=xd,
                          bounds=meta.expert_offsets[::El].tolist()))
    # one-GPU answer over every rank's tokens (oracle)
    g = oracle.prepare(np.concatenate([r["ids"] for r in ranks]), E)
    xg = np.concatenate([bits(r["x"]) for r in ranks])
    want = oracle.dispatch(xg, k, g["input_perm"])
    S = sum(r["T"] for r in ranks) * k
    y_global = torch.randn(S, H, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    backs = [torch.zeros(r["T"] * k, H, dtype=torch.bfloat16, device=DEV) for r in ranks]
    for dst in range(R):
        counts = torch.stack([r["meta"].expert_counts[dst * El:(dst + 1) * El] for r in ranks])
        blocks = [r["xd"][r["bounds"][dst]:r["bounds"][dst + 1]] for r in ranks]
        recv = torch.cat(blocks)  # the all-to-all, as device copies
        lay = moe.moe_ep_recv_layout(counts.contiguous(), recv.shape[0])
        grouped = moe.moe_dispatch_rows(recv, 1, input_permutation=lay.local_to_recv)
        lo, hi = g["offsets"][dst * El], g["offsets"][(dst + 1) * El]
        assert np.array_equal(bits(grouped), want[lo:hi]), dst
        assert np.array_equal(lay.local_offsets.cpu().numpy(),
                              g["offsets"][dst * El:(dst + 1) * El + 1] - lo)
        # expert outputs of this window back to the sources' dispatched order
        y_recv = moe.moe_dispatch_rows(y_global[lo:hi].to(DEV).contiguous(), 1,
                                       input_permutation=lay.recv_to_local)
        q = 0
        for s, r in enumerate(ranks):
            m = r["bounds"][dst + 1] - r["bounds"][dst]
            backs[s][r["bounds"][dst]:r["bounds"][dst + 1]] = y_recv[q:q + m]
            q += m
    full = oracle.combine(bits(y_global), "bf16", g["output_perm"],
                          np.concatenate([r["wt"] for r in ranks]), "bf16")
    t0 = 0
    for s, r in enumerate(ranks):
        out = moe.moe_combine(backs[s], r["meta"].output_permutation,
                              torch.from_numpy(r["wt"]).to(DEV))
        assert np.array_equal(bits(out), full[t0:t0 + r["T"]]), s
        t0 += r["T"]


def test_ep_module_over_a_one_rank_nccl_group():
    import torch.distributed as dist
    from combine_permute_b200 import ep
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=DEV)
    try:
        w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(900)
        ids_np, wt_np, x, y = make_workload(w, device=DEV)
        grouped, local_offsets, handle = ep.ep_dispatch(x, torch.from_numpy(ids_np).to(DEV), w.E)
        out = ep.ep_combine(y, torch.from_numpy(wt_np).to(DEV), handle)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = oracle.prepare(ids_np, w.E)
    # one rank owns every expert: the grouped rows are the dispatched rows
    assert np.array_equal(bits(grouped), oracle.dispatch(bits(x), w.k, ref["input_perm"]))
    assert np.array_equal(local_offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(bits(out), oracle.combine(bits(y), "bf16", ref["output_perm"], wt_np,
                                                    "bf16"))


# ---------------------------------------------------------------------------
# The exchange as stores into the owners' buffers (moe_ep_peer_layout,
# moe_ep_dispatch_peer, moe_ep_combine_peer).  R ranks are emulated on one
# GPU: every rank's grouped buffer lives here, and each source's kernels get
# the array of all R buffer addresses, as a rank with the other GPUs' memory
# mapped in would.
# ---------------------------------------------------------------------------

def _emulated_ranks(R, T, seed, base_name="uniform_t4096_h7168_e256_k8", invalid_every=53):
    base = CONFIGS[base_name]
    ranks = []
    for r in range(R):
        w = dataclasses.replace(base, T=T + 29 * r, seed=seed * 100 + r, name=f"rank{r}")
        ids_np, wt_np, x, _ = make_workload(w, device=DEV, with_y=False)
        if invalid_every:
            ids_np[::invalid_every, 0] = -1
        ids = torch.from_numpy(ids_np).to(DEV)
        ranks.append(dict(w=w, T=w.T, ids_np=ids_np, ids=ids, wt=wt_np, x=x,
                          meta=moe.moe_prepare(ids, base.E)))
    return base, ranks


@pytest.mark.parametrize("R,T,seed", [(1, 500, 3), (2, 700, 4), (4, 1100, 5), (8, 300, 6)])
def test_peer_layout_matches_the_single_gpu_rows(R, T, seed):
    base, ranks = _emulated_ranks(R, T, seed)
    E, k = base.E, base.k
    El = E // R
    counts = torch.stack([r["meta"].expert_counts for r in ranks]).contiguous()
    g = oracle.prepare(np.concatenate([r["ids_np"] for r in ranks]), E)
    tok0 = 0
    for s, r in enumerate(ranks):
        lay = moe.moe_ep_peer_layout(counts, s, r["ids"], r["meta"])
        torch.cuda.synchronize()
        # slot i of rank s is global slot tok0*k + i; its owner's grouped buffer
        # is the single-GPU dispatched rows of the owner's expert window
        gi = tok0 * k + np.arange(r["T"] * k)
        P = g["output_perm"][gi]
        e = r["ids_np"].ravel()
        ok = P >= 0
        want_rank = np.where(ok, e // El, -1)
        want_row = np.where(ok, P - g["offsets"][np.clip(e // El, 0, R - 1) * El], -1)
        assert np.array_equal(lay.dest_rank.cpu().numpy(), want_rank)
        assert np.array_equal(lay.dest_row.cpu().numpy(), want_row)
        assert np.array_equal(lay.recv_rows.cpu().numpy(), np.diff(g["offsets"][::El]))
        assert np.array_equal(lay.local_offsets.cpu().numpy(),
                              g["offsets"][s * El:(s + 1) * El + 1] - g["offsets"][s * El])
        tok0 += r["T"]


@pytest.mark.parametrize("R,T,seed,ydt,odt", [(2, 700, 7, "bf16", "bf16"), (4, 900, 8, "bf16", "bf16"),
                                              (8, 400, 9, "bf16", "fp32")])
def test_peer_dispatch_and_combine_match_single_gpu(R, T, seed, ydt, odt):
    base, ranks = _emulated_ranks(R, T, seed)
    E, k, H = base.E, base.k, base.H
    El = E // R
    counts = torch.stack([r["meta"].expert_counts for r in ranks]).contiguous()
    lays = [moe.moe_ep_peer_layout(counts, s, r["ids"], r["meta"]) for s, r in enumerate(ranks)]
    rows = lays[0].recv_rows.tolist()
    sentinel = -3.0
    bufs = [torch.full((max(n, 1), H), sentinel, dtype=torch.bfloat16, device=DEV) for n in rows]
    for s, r in enumerate(ranks):
        moe.moe_ep_dispatch_peer(r["x"], k, lays[s], bufs)
    torch.cuda.synchronize()
    g = oracle.prepare(np.concatenate([r["ids_np"] for r in ranks]), E)
    want = oracle.dispatch(np.concatenate([bits(r["x"]) for r in ranks]), k, g["input_perm"])
    for d in range(R):
        lo, hi = g["offsets"][d * El], g["offsets"][(d + 1) * El]
        assert rows[d] == hi - lo
        assert np.array_equal(bits(bufs[d][:rows[d]]), want[lo:hi]), d
    # expert outputs: the single-GPU y rows of each owner's window, in its buffer
    TD = {"bf16": torch.bfloat16, "fp32": torch.float32}
    S = sum(r["T"] for r in ranks) * k
    y = torch.randn(S, H, generator=torch.Generator().manual_seed(seed)).to(TD[ydt])
    outs = [y[g["offsets"][d * El]:g["offsets"][(d + 1) * El]].to(DEV).contiguous() for d in range(R)]
    outs = [o if o.shape[0] else torch.zeros(1, H, dtype=TD[ydt], device=DEV) for o in outs]
    full = oracle.combine(bits(y), ydt, g["output_perm"], np.concatenate([r["wt"] for r in ranks]), odt)
    t0 = 0
    for s, r in enumerate(ranks):
        got = moe.moe_ep_combine_peer(outs, TD[ydt], H, lays[s], torch.from_numpy(r["wt"]).to(DEV),
                                      out_dtype=TD[odt])
        torch.cuda.synchronize()
        assert np.array_equal(bits(got), full[t0:t0 + r["T"]]), s
        t0 += r["T"]


def test_ep_peer_module_over_a_one_rank_nccl_group():
    import torch.distributed as dist
    from combine_permute_b200 import ep
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=DEV)
    try:
        w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(800)
        ids_np, wt_np, x, y = make_workload(w, device=DEV)
        buf = torch.empty((w.S, w.H), dtype=x.dtype, device=DEV)
        grouped, local_offsets, handle = ep.ep_dispatch_peer(x, torch.from_numpy(ids_np).to(DEV),
                                                             w.E, [buf])
        out = ep.ep_combine_peer([y], y.dtype, w.H, torch.from_numpy(wt_np).to(DEV), handle)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = oracle.prepare(ids_np, w.E)
    assert np.array_equal(bits(grouped), oracle.dispatch(bits(x), w.k, ref["input_perm"]))
    assert np.array_equal(local_offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(bits(out), oracle.combine(bits(y), "bf16", ref["output_perm"], wt_np,
                                                    "bf16"))


def test_peer_calls_take_a_prebuilt_buffer_table():
    """moe_ep_buffer_table built once (as for a CUDA graph) gives the same
    bytes as the list of buffers, and the peer dispatch records into a graph
    with it."""
    base, ranks = _emulated_ranks(2, 600, 11)
    E, k, H = base.E, base.k, base.H
    counts = torch.stack([r["meta"].expert_counts for r in ranks]).contiguous()
    r = ranks[0]
    lay = moe.moe_ep_peer_layout(counts, 0, r["ids"], r["meta"])
    rows = lay.recv_rows.tolist()
    want = [torch.full((n, H), -3.0, dtype=torch.bfloat16, device=DEV) for n in rows]
    moe.moe_ep_dispatch_peer(r["x"], k, lay, want)
    got = [torch.full((n, H), -3.0, dtype=torch.bfloat16, device=DEV) for n in rows]
    table = moe.moe_ep_buffer_table(got, DEV)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            moe.moe_ep_dispatch_peer(r["x"], k, lay, table)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(want, got):
        assert np.array_equal(bits(a), bits(b))
    wt = torch.from_numpy(r["wt"]).to(DEV)
    assert np.array_equal(bits(moe.moe_ep_combine_peer(want, torch.bfloat16, H, lay, wt)),
                          bits(moe.moe_ep_combine_peer(table, torch.bfloat16, H, lay, wt)))


def test_buffer_table_keeps_its_buffers_allocated():
    """The table refers to the tensors it was built from: dropping the
    caller's list and emptying torch's cache (as a graph capture does) leaves
    the memory it points to allocated, so the peer dispatch still has it."""
    import gc
    base, ranks = _emulated_ranks(2, 400, 12)
    counts = torch.stack([r["meta"].expert_counts for r in ranks]).contiguous()
    r = ranks[0]
    lay = moe.moe_ep_peer_layout(counts, 0, r["ids"], r["meta"])
    rows = lay.recv_rows.tolist()
    bufs = [torch.full((n, base.H), -3.0, dtype=torch.bfloat16, device=DEV) for n in rows]
    want = [b.clone() for b in bufs]
    moe.moe_ep_dispatch_peer(r["x"], base.k, lay, want)
    table = moe.moe_ep_buffer_table(bufs, DEV)
    kept = table._buffers
    del bufs
    gc.collect()
    torch.cuda.empty_cache()
    moe.moe_ep_dispatch_peer(r["x"], base.k, lay, table)
    torch.cuda.synchronize()
    for a, b in zip(want, kept):
        assert np.array_equal(bits(a), bits(b))
