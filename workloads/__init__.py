"""Seeded synthetic inputs for the MoE dispatch / combine path.

This package generates inputs only: top-k expert ids, router weights and
activation tensors.  It holds none of the path's arithmetic (no counting,
no prefix sums, no permutation, no gather, no reduce), so that the CPU
oracle and the CUDA path can both consume its output without sharing code.

Routing modes follow the benchmark design of the Mooncake RFC
"Comprehensive MoE / EP Kernel Benchmark Under Incast Traffic" (section
"Routing Modes": uniform, K-hot-expert incast, Zipfian); the shapes are the
pages' workloads (Mooncake PR #4581 "Performance Test": 32 tokens, hidden
4096, top-8 of 256; TensorRT-LLM PR #9592 description: max_num_tokens 9216,
num_slots 288).
"""

from .routing import (  # noqa: F401
    CONFIGS,
    Workload,
    RoutingSpec,
    seed_streams,
    make_routing,
    make_weights,
    make_activations,
    make_workload,
)
