"""The bounded waits give up, report, and leave the GPU usable.

Every wait in the library's kernels is bounded (about one second by
default).  These tests make a wait run out without faulting anything: a
wait limit of zero on the TMA dispatch, and prepare workspaces whose
counters were disturbed on the host (a barrier counter that can never reach
the block count, a tile ticket that hands tile 0 to a block that cannot be
scheduled while the first wave of tiles waits on it).  Each call must still
return, report through its status word (the dispatch error query, diag[1]),
and a following call with intact state must be bit-exact against the
oracle.
"""

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
import oracle
from tests._helpers import bits
from workloads import CONFIGS, make_workload

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _default_limits():
    moe.moe_set_wait_limits(-1, -1)
    yield
    moe.moe_set_wait_limits(-1, -1)


def _check_prepare(meta, ids_np, E):
    ref = oracle.prepare(ids_np, E)
    assert np.array_equal(meta.input_permutation.cpu().numpy(), ref["input_perm"])
    assert np.array_equal(meta.output_permutation.cpu().numpy(), ref["output_perm"])
    assert np.array_equal(meta.expert_offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(meta.expert_counts.cpu().numpy(), ref["counts"])
    assert meta.diag.cpu().tolist() == [ref["n_invalid"], 0]
    return ref


def test_dispatch_wait_gives_up_and_reports():
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(600)
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), w.E)
    assert int(moe.moe_dispatch_error().item()) == 0
    sentinel = torch.full((w.S, w.H), -7.0, dtype=x.dtype, device=DEV)

    moe.moe_set_wait_limits(-1, 0)  # every staged-chunk wait gives up at once
    out = sentinel.clone()
    moe.moe_dispatch_rows(x, w.k, meta.input_permutation, meta.output_permutation, out=out)
    err = moe.moe_dispatch_error()
    torch.cuda.synchronize(DEV)
    assert int(err.item()) == 1
    # every block stopped at its first chunk: no row was written
    assert torch.equal(out, sentinel)
    # the query cleared the word
    assert int(moe.moe_dispatch_error().item()) == 0

    moe.moe_set_wait_limits(-1, -1)
    out = sentinel.clone()
    moe.moe_dispatch_rows(x, w.k, meta.input_permutation, meta.output_permutation, out=out)
    err = moe.moe_dispatch_error()
    torch.cuda.synchronize(DEV)
    assert int(err.item()) == 0
    ref = oracle.prepare(ids_np, w.E)
    assert np.array_equal(bits(out), oracle.dispatch(bits(x), w.k, ref["input_perm"]))


def _ws(w):
    n = moe.moe_prepare_workspace_bytes(w.T, w.k, w.E)
    assert n > 0
    return torch.zeros(n, dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("wait_us", [-1, 0])
def test_prepare_grid_barrier_that_never_fills_gives_up(wait_us):
    # 32768 slots: the one-launch path (64 blocks and one grid barrier)
    w = CONFIGS["uniform_t4096_h7168_e256_k8"]
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids = torch.from_numpy(ids_np).to(DEV)
    ws = _ws(w)
    ws.view(torch.int32)[6] = 1 << 20  # barrier arrivals: the count never reads the block count
    moe.moe_set_wait_limits(wait_us, -1)
    meta = moe.moe_prepare(ids, w.E, workspace=ws)
    torch.cuda.synchronize(DEV)  # the kernel ended
    assert int(meta.diag[1].item()) == 1
    # the stream and the context are still usable: intact state, exact result
    moe.moe_set_wait_limits(-1, -1)
    meta = moe.moe_prepare(ids, w.E, workspace=_ws(w))
    torch.cuda.synchronize(DEV)
    _check_prepare(meta, ids_np, w.E)


def test_prepare_lookback_on_an_unscheduled_tile_gives_up():
    # above about 3.9 M slots of 256 experts prepare runs as two kernels of
    # 2048-slot tiles (more tiles than fit on the GPU at once) with a
    # decoupled look-back.  A ticket
    # word of 1 hands tile 0 to the block that takes the last ticket; the
    # first wave of resident tiles all wait on it and give up after the
    # default limit.
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(500000)  # 4 M slots
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    ids = torch.from_numpy(ids_np).to(DEV)
    ws = _ws(w)
    ws.view(torch.int32)[0] = 1
    meta = moe.moe_prepare(ids, w.E, workspace=ws)
    torch.cuda.synchronize(DEV)
    assert int(meta.diag[1].item()) == 1
    meta = moe.moe_prepare(ids, w.E, workspace=_ws(w))
    torch.cuda.synchronize(DEV)
    _check_prepare(meta, ids_np, w.E)
