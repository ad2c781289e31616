"""Host-side pieces of bench.py: the algorithmic byte counts behind every
roofline fraction (checked against the per-step byte table the method's
sizes give), the graph step count, the whole-job throughput and the rule
that a profile's traffic only counts for the sources it was taken on."""

import json

import pytest

import bench
from workloads import CONFIGS

MB = 1e6

# (dispatch, combine) minimal bytes per step in MB: every input read once,
# every output written once; x read once although written k times.
TABLE = {
    "tiny_t32_h4096_e256_k8": (2.36, 2.36),
    "uniform_t4096_h7168_e256_k8": (528.6, 528.7),
    "khot_t9216_h7168_e256_k8": (1189.4, 1189.7),
    "zipf_fp8_t16384_h4096_e288_k8": (688.4, 1209.0),
    "zipf_fp16_t131072_h2048_e64_k6": (3761.2, 4301.3),
}


@pytest.mark.parametrize("name", list(TABLE))
def test_algorithmic_bytes_match_the_table(name):
    b = bench.algorithmic_bytes(CONFIGS[name])
    d, c = TABLE[name]
    assert abs(b["dispatch"] / MB - d) < 0.05 + 1e-3 * d
    assert abs(b["combine"] / MB - c) < 0.05 + 1e-3 * c


def test_algorithmic_bytes_closed_form_uniform():
    w = CONFIGS["uniform_t4096_h7168_e256_k8"]
    S = w.T * w.k
    b = bench.algorithmic_bytes(w)
    assert b["dispatch"] == w.T * w.H * 2 + S * w.H * 2 + 4 * S
    assert b["combine"] == S * w.H * 2 + 8 * S + w.T * w.H * 2
    assert b["prepare"] == 4 * S + 4 * w.E + 4 * (w.E + 1) + 8 * S


@pytest.mark.parametrize("K,n", [(1, 1), (3, 3), (7, 7), (20, 10), (200, 10), (201, 3), (11, 1)])
def test_steps_per_graph_divides_K(K, n):
    assert bench.steps_per_graph(K) == n
    assert K % bench.steps_per_graph(K) == 0


def test_whole_job_throughput_counts_every_rank():
    # 2 ranks x 10 steps x 4096 tokens in 20 ms (the slowest rank's time)
    assert bench.whole_job_tokens_per_s(4096, 10, 2, 20.0) == pytest.approx(4096 * 20 / 0.02)


def test_traffic_counts_only_for_the_captured_sources(monkeypatch):
    key = "dispatch@uniform_t4096_h7168_e256_k8"
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        entry = json.load(f)["kernels"][key]
    monkeypatch.setattr(bench, "src_hash", lambda step: entry["src_hash"])
    assert bench.committed_traffic(key) == entry["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "src_hash", lambda step: "0" * 16)
    assert bench.committed_traffic(key) is None


def test_next_row_bytes_of_the_fp8_workload():
    """Worked by hand for T=16384, H=4096, E=288, k=8 (S = 131072): the NVFP4
    dispatch reads x once (16384 * 4096 * 2), writes 2048 code bytes and 256
    scale bytes per slot, reads the permutation (4 bytes a slot) and the two
    offset arrays (8 * 289)."""
    b = bench.next_row_bytes(CONFIGS["zipf_fp8_t16384_h4096_e288_k8"])
    assert b["dispatch_nvfp4"] == 134217728 + 131072 * 2304 + 524288 + 2312
    assert b["problem_sizes"] == 28 * 288


def test_net_of_events_shares_sum_to_the_event_free_step():
    # three calls timed with events (13.0 + 88.0 + 93.0 = 194 us) in a step
    # that takes 179.6 us without them: 14.4 us of events, 4.8 a call
    overhead, net = bench.net_of_events({"prepare": 13.0, "dispatch": 88.0, "combine": 93.0}, 179.6)
    assert abs(overhead - 14.4) < 1e-9
    assert abs(net["prepare"] - 8.2) < 1e-9 and abs(net["combine"] - 88.2) < 1e-9
    assert abs(sum(net.values()) - 179.6) < 1e-9
