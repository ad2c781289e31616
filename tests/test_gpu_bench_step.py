"""Parity of the step exactly as bench.py times it: bench.Step's buffers and
calls, captured as a CUDA graph of several consecutive steps and replayed,
on the full-size workloads; the results of the last replay are checked
against the oracle (metadata in full, dispatched rows and combined tokens
sampled, fp8 bytes and scales sampled)."""

import numpy as np
import pytest
import torch

import bench
import oracle
from workloads import CONFIGS

from _helpers import bits

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _replay_graph(step, n_steps=3, replays=2):
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(side):
        step.run()
        with torch.cuda.graph(g, stream=side):
            for _ in range(n_steps):
                step.run()
    for _ in range(replays):
        g.replay()
    torch.cuda.synchronize(DEV)
    del g


@pytest.mark.parametrize("name", ["tiny_t32_h4096_e256_k8", "uniform_t4096_h7168_e256_k8",
                                  "zipf_fp8_t16384_h4096_e288_k8"])
def test_graph_replayed_step_matches_oracle(name):
    w = CONFIGS[name]
    step = bench.Step(w, DEV)
    # poison every output first, so that a step that skipped work would show
    step.meta_bufs["input_permutation"].fill_(-7)
    step.meta_bufs["output_permutation"].fill_(-7)
    step.out.fill_(float("nan"))
    if step.fp8:
        step.xq.fill_(0xAB)
    else:
        step.xd.fill_(float("nan"))
    _replay_graph(step)

    A = step.A or 1
    ref = oracle.prepare(step.ids_np, w.E, A)
    mb = step.meta_bufs
    np.testing.assert_array_equal(mb["expert_offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(mb["input_permutation"].cpu().numpy(), ref["input_perm"])
    np.testing.assert_array_equal(mb["output_permutation"].cpu().numpy(), ref["output_perm"])

    rng = np.random.default_rng(7)
    toks = np.unique(rng.integers(0, w.T, min(w.T, 200)))
    slots = (toks[:, None] * w.k + np.arange(w.k)).ravel()
    rows = ref["output_perm"][slots]
    x_sub = bits(step.x[torch.from_numpy(toks).to(DEV)])
    sub_ids = step.ids_np[toks]
    sub_meta = dict(input_perm=np.arange(slots.size, dtype=np.int32),
                    offsets=np.zeros(w.E + 1, np.int32), bso=np.zeros(w.E + 1, np.int32))
    rows_t = torch.from_numpy(rows).long().to(DEV)
    if step.fp8:
        q_sub, sc_sub = oracle.dispatch_fp8(x_sub, "bf16", sub_ids, sub_meta,
                                            scales=np.zeros((slots.size, w.H // 128), np.float32))
        np.testing.assert_array_equal(step.xq[rows_t].cpu().numpy(), q_sub)
        e = step.ids_np.ravel()[slots]
        srow = ref["bso"][e] + rows - ref["offsets"][e]
        got_sc = step.scales[torch.from_numpy(srow).long().to(DEV)].cpu().numpy()
        np.testing.assert_array_equal(got_sc.view(np.uint32), sc_sub.view(np.uint32))
    else:
        # every sampled slot's dispatched row is its token's x row
        xd = bits(step.xd[rows_t])
        np.testing.assert_array_equal(xd, np.repeat(x_sub, w.k, axis=0))
    # combine of the sampled tokens: their k expert-output rows and weights
    y_rows = bits(step.y[rows_t])
    sub_perm = np.arange(slots.size, dtype=np.int32)
    want = oracle.combine(y_rows, w.y_dtype, sub_perm, step.wt_np[toks], w.out_dtype)
    got = bits(step.out[torch.from_numpy(toks).to(DEV)])
    np.testing.assert_array_equal(got, want)
