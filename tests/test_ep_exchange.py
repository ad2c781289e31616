"""Expert-parallel exchange between ranks (combine_permute_b200.ep), run as
CPU processes over gloo with world sizes 2 and 3.

The exchange logic of ep_dispatch / ep_combine (count exchange, per-rank
splits, the all-to-alls, the receive layout and the regroup) runs
unchanged; the per-rank steps are the oracle's, passed in as ``ops``, since
these processes have no GPU.  Every rank draws all ranks' seeded inputs, so
it can check its own result against the single-GPU answer over all tokens
taken together (in rank order):

* the rows it receives, grouped by local expert, are exactly the rows the
  one-GPU dispatch puts in its expert window, in the same order;
* the combined output of its tokens equals the one-GPU combine of those
  tokens, bit for bit (the k outputs are summed in slot order either way).
"""

import json
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
H = 64


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _from_bits(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """The per-rank steps of the exchange, on the CPU oracle (bf16 rows)."""

    def __init__(self, oracle):
        self.o = oracle

    def prepare(self, topk_ids, num_experts):
        m = self.o.prepare(topk_ids.numpy(), num_experts)
        return SimpleNamespace(expert_counts=torch.from_numpy(m["counts"]),
                               expert_offsets=torch.from_numpy(m["offsets"]),
                               input_permutation=torch.from_numpy(m["input_perm"]),
                               output_permutation=torch.from_numpy(m["output_perm"]))

    def dispatch(self, x, top_k, meta):
        return _from_bits(self.o.dispatch(_bits(x), top_k, meta.input_permutation.numpy()))

    def recv_layout(self, recv_counts, num_recv):
        lay = self.o.ep_recv_layout(recv_counts.numpy())
        return SimpleNamespace(**{k: torch.from_numpy(v) for k, v in lay.items()})

    def gather_rows(self, rows, index):
        return _from_bits(self.o.dispatch(_bits(rows), 1, index.numpy()))

    def combine(self, y, meta, weights, out_dtype):
        assert out_dtype == torch.bfloat16
        return _from_bits(self.o.combine(_bits(y), "bf16", meta.output_permutation.numpy(),
                                         weights.numpy(), "bf16"))


def _inputs(R, El, k, seed):
    """Every rank's tokens: ids over R*El experts (a few invalid), weights,
    x rows, and one expert-output row per global dispatched row."""
    rng = np.random.default_rng(seed)
    E = R * El
    T = [int(rng.integers(0, 40)) for _ in range(R)]
    ids, wts, xs = [], [], []
    for r in range(R):
        i = np.stack([rng.permutation(E)[:k] for _ in range(T[r])]).astype(np.int32) \
            if T[r] else np.zeros((0, k), np.int32)
        if T[r] > 2:
            i[1, 0] = -1
            i[2, k - 1] = E + 3
        ids.append(i)
        w = rng.random((T[r], k)).astype(np.float32)
        wts.append(w / np.maximum(w.sum(1, keepdims=True), 1e-6))
        xs.append(torch.randn(T[r], H, generator=torch.Generator().manual_seed(seed * 10 + r))
                  .to(torch.bfloat16))
    S = sum(T) * k
    y_global = torch.randn(S, H, generator=torch.Generator().manual_seed(seed + 77)).to(torch.bfloat16)
    return T, ids, wts, xs, y_global


def _worker(rank, world, El, k, seed, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from combine_permute_b200 import ep

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ops = OracleOps(oracle)
        T, ids, wts, xs, y_global = _inputs(world, El, k, seed)
        E = world * El
        grouped, local_offsets, handle = ep.ep_dispatch(xs[rank], torch.from_numpy(ids[rank]), E,
                                                        ops=ops)
        # the one-GPU answer over every rank's tokens
        g = oracle.prepare(np.concatenate(ids), E)
        xg = _bits(torch.cat(xs))
        lo, hi = g["offsets"][rank * El], g["offsets"][(rank + 1) * El]
        want_rows = oracle.dispatch(xg, k, g["input_perm"])[lo:hi]
        res = {"rows_equal": bool(np.array_equal(_bits(grouped), want_rows)),
               "offsets_equal": bool(np.array_equal(local_offsets.numpy(),
                                                    g["offsets"][rank * El:(rank + 1) * El + 1] - lo)),
               "n": int(grouped.shape[0])}
        # expert outputs of this rank's window are the global rows lo..hi
        out = ep.ep_combine(y_global[lo:hi].contiguous(), torch.from_numpy(wts[rank]), handle,
                            ops=ops)
        full = oracle.combine(_bits(y_global), "bf16", g["output_perm"], np.concatenate(wts), "bf16")
        t0 = sum(T[:rank])
        res["combine_equal"] = bool(np.array_equal(_bits(out), full[t0:t0 + T[rank]]))
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"ep_rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.parametrize("world,El,k,seed", [(2, 4, 3, 0), (2, 1, 1, 1), (3, 5, 4, 2)])
def test_ep_exchange_matches_the_single_gpu_path_gloo(tmp_path, world, El, k, seed):
    port = _free_port()
    mp.start_processes(_worker, args=(world, El, k, seed, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    total = 0
    for r in range(world):
        res = json.load(open(tmp_path / f"ep_rank{r}.json"))
        assert res["rows_equal"] and res["offsets_equal"] and res["combine_equal"], (r, res)
        total += res["n"]
    T, ids, _, _, _ = _inputs(world, El, k, seed)
    flat = np.concatenate(ids).ravel()
    assert total == int(((flat >= 0) & (flat < world * El)).sum())  # every valid slot, once
