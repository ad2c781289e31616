"""Seeded routing, router-weight and activation generators.

Recipe (every stream derives from one integer seed):

* ``numpy.random.SeedSequence(seed).spawn(4)`` gives four independent
  streams, in this order: expert ids, router logits, x, y.
* Expert ids: each token draws k *distinct* experts.  For the uniform and
  Zipf modes this is Gumbel-top-k over per-expert log-probabilities, which
  is the same distribution as drawing k times without replacement with
  probability proportional to popularity; the slot order is the draw order
  (largest perturbed log-probability first).
* Uniform: equal popularity over E experts (Mooncake RFC "Routing Modes",
  1. Uniform Routing).
* K-hot incast: for every slot, with probability ``hot_fraction`` the slot
  draws uniformly from the not-yet-used experts of the hot set
  ``{0, .., hot_experts-1}``, otherwise uniformly from the not-yet-used
  experts outside it (Mooncake RFC "Routing Modes", 2. K-Hot-Expert Incast:
  the hot set is the first experts, "--hot-fraction 0.90").  When one pool
  is exhausted the slot draws from the other.
* Zipf: a seeded random permutation ``perm`` of the experts ranks them;
  expert ``perm[r-1]`` has popularity ``r ** -s`` (Mooncake RFC "Routing
  Modes", 3. Zipfian Routing, "--zipf-alpha").
* Router weights: softmax over the k chosen slots of N(0,1) fp32 logits,
  computed in float64 and rounded once to fp32.  "Softmax renormalised over
  the top-k" is the same quantity, since the softmax over all experts
  restricted to k of them and renormalised equals the softmax of the k
  logits.
* Activations x [T,H] and expert outputs y [T*k,H]: N(0,1) drawn in fp32 by
  ``torch.randn`` with a ``torch.Generator`` seeded from the x / y stream on
  the requested device, then rounded to the storage dtype.  The CPU and CUDA
  generators give different values for the same seed; a parity test draws
  on one device and hands the same bits to both sides.

Nothing here counts, scans, sorts, gathers or reduces: that is the method's
arithmetic and lives in the oracle and in the CUDA library.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "CONFIGS",
    "Workload",
    "RoutingSpec",
    "seed_streams",
    "make_routing",
    "make_weights",
    "make_activations",
    "make_workload",
]


@dataclasses.dataclass(frozen=True)
class RoutingSpec:
    mode: str  # "uniform" | "khot" | "zipf"
    hot_experts: int = 8
    hot_fraction: float = 0.9
    zipf_s: float = 1.2


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic dispatch/combine problem.

    ``x_dtype`` is the activation dtype read by dispatch; ``dispatch_dtype``
    is what dispatch writes (equal to ``x_dtype`` or ``"fp8_e4m3"``);
    ``y_dtype`` / ``out_dtype`` are combine's input and output dtypes.
    ``block_align`` is the scale-row alignment A of the block-scale offsets
    (only used on the fp8 path).
    """

    name: str
    T: int
    H: int
    E: int
    k: int
    routing: RoutingSpec
    x_dtype: str = "bf16"
    dispatch_dtype: str = "bf16"
    y_dtype: str = "bf16"
    out_dtype: str = "bf16"
    block_align: int = 1
    seed: int = 0

    @property
    def S(self) -> int:
        return self.T * self.k

    def scaled(self, T: int, name: Optional[str] = None) -> "Workload":
        """Same routing and dtypes with a different token count."""
        return dataclasses.replace(self, T=T, name=name or f"{self.name}@T{T}")


# The five workloads of the path: a tiny decode-like batch, uniform routing
# on a DeepSeek-V3-sized layer, K-hot incast, Zipf routing with fp8
# dispatch, and a large fp16 -> fp32 batch.
CONFIGS = {
    "tiny_t32_h4096_e256_k8": Workload(
        "tiny_t32_h4096_e256_k8", T=32, H=4096, E=256, k=8,
        routing=RoutingSpec("uniform")),
    "uniform_t4096_h7168_e256_k8": Workload(
        "uniform_t4096_h7168_e256_k8", T=4096, H=7168, E=256, k=8,
        routing=RoutingSpec("uniform")),
    "khot_t9216_h7168_e256_k8": Workload(
        "khot_t9216_h7168_e256_k8", T=9216, H=7168, E=256, k=8,
        routing=RoutingSpec("khot", hot_experts=8, hot_fraction=0.9)),
    "zipf_fp8_t16384_h4096_e288_k8": Workload(
        "zipf_fp8_t16384_h4096_e288_k8", T=16384, H=4096, E=288, k=8,
        routing=RoutingSpec("zipf", zipf_s=1.2),
        dispatch_dtype="fp8_e4m3", block_align=128),
    "zipf_fp16_t131072_h2048_e64_k6": Workload(
        "zipf_fp16_t131072_h2048_e64_k6", T=131072, H=2048, E=64, k=6,
        routing=RoutingSpec("zipf", zipf_s=0.8),
        x_dtype="fp16", dispatch_dtype="fp16", y_dtype="fp16",
        out_dtype="fp32"),
}


def seed_streams(seed: int):
    """The four independent streams (ids, logits, x, y) of one seed."""
    return np.random.SeedSequence(seed).spawn(4)


def _gumbel_topk(rng: np.random.Generator, logp: np.ndarray, T: int, k: int) -> np.ndarray:
    """k distinct columns per row by Gumbel-top-k; draw order = slot order."""
    E = logp.shape[-1]
    g = rng.gumbel(size=(T, E)) + logp
    if k < E:
        part = np.argpartition(-g, k - 1, axis=1)[:, :k]
    else:
        part = np.broadcast_to(np.arange(E), (T, E)).copy()
    key = np.take_along_axis(g, part, axis=1)
    order = np.argsort(-key, axis=1, kind="stable")
    return np.take_along_axis(part, order, axis=1)


def make_routing(T: int, E: int, k: int, spec: RoutingSpec, rng: np.random.Generator) -> np.ndarray:
    """[T, k] int32 expert ids, distinct within each token."""
    if k > E:
        raise ValueError("top-k larger than the number of experts")
    if T == 0:
        return np.zeros((0, k), dtype=np.int32)
    if spec.mode == "uniform":
        ids = _gumbel_topk(rng, np.zeros(E), T, k)
    elif spec.mode == "zipf":
        perm = rng.permutation(E)
        logp = np.empty(E)
        logp[perm] = -spec.zipf_s * np.log(np.arange(1, E + 1, dtype=np.float64))
        ids = _gumbel_topk(rng, logp, T, k)
    elif spec.mode == "khot":
        h = spec.hot_experts
        if not 0 < h < E:
            raise ValueError("hot set must be a proper, non-empty subset")
        n_hot_max = min(k, h)
        n_cold_max = min(k, E - h)
        # The hot pool in a uniformly random order, the cold pool likewise;
        # slot j takes the next unused element of the pool it draws from.
        hot_order = _gumbel_topk(rng, np.zeros(h), T, n_hot_max)
        cold_order = h + _gumbel_topk(rng, np.zeros(E - h), T, n_cold_max)
        u = rng.random(size=(T, k))
        ids = np.empty((T, k), dtype=np.int64)
        used_hot = np.zeros(T, dtype=np.int64)
        used_cold = np.zeros(T, dtype=np.int64)
        rows = np.arange(T)
        for j in range(k):
            want_hot = u[:, j] < spec.hot_fraction
            take_hot = np.where(want_hot, used_hot < n_hot_max, used_cold >= n_cold_max)
            hi = np.minimum(used_hot, n_hot_max - 1)
            ci = np.minimum(used_cold, n_cold_max - 1)
            ids[:, j] = np.where(take_hot, hot_order[rows, hi], cold_order[rows, ci])
            used_hot += take_hot
            used_cold += ~take_hot
    else:
        raise ValueError(f"unknown routing mode {spec.mode!r}")
    return np.ascontiguousarray(ids, dtype=np.int32)


def make_weights(T: int, k: int, rng: np.random.Generator) -> np.ndarray:
    """[T, k] fp32 router weights: softmax over the k chosen N(0,1) logits."""
    logits = rng.standard_normal(size=(T, k))
    z = np.exp(logits - logits.max(axis=1, keepdims=True)) if T else logits
    w = z / z.sum(axis=1, keepdims=True) if T else z
    return np.ascontiguousarray(w, dtype=np.float32)


_TORCH_DTYPES = {"bf16": "bfloat16", "fp16": "float16", "fp32": "float32"}


def torch_dtype(name: str):
    import torch
    return getattr(torch, _TORCH_DTYPES[name])


def make_activations(shape, dtype: str, seed_seq: np.random.SeedSequence, device="cpu"):
    """N(0,1) fp32 drawn by torch.randn on ``device``, rounded to ``dtype``."""
    import torch
    seed = int(seed_seq.generate_state(1, dtype=np.uint64)[0] >> 1)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    rows, cols = shape
    out = torch.empty((rows, cols), dtype=torch_dtype(dtype), device=device)
    # Draw in row chunks so that the fp32 temporary stays bounded; the
    # generator's state carries over, so the chunking is part of the recipe.
    chunk = max(1, (1 << 28) // max(cols, 1))
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        out[r0:r1] = torch.randn((r1 - r0, cols), generator=gen, device=device,
                                 dtype=torch.float32).to(out.dtype)
    return out


def make_workload(w: Workload, device="cpu", with_x=True, with_y=True):
    """ids [T,k] int32 and weights [T,k] fp32 (numpy), x [T,H], y [T*k,H] (torch)."""
    s_ids, s_logits, s_x, s_y = seed_streams(w.seed)
    ids = make_routing(w.T, w.E, w.k, w.routing, np.random.Generator(np.random.PCG64(s_ids)))
    weights = make_weights(w.T, w.k, np.random.Generator(np.random.PCG64(s_logits)))
    x = make_activations((w.T, w.H), w.x_dtype, s_x, device) if with_x else None
    y = make_activations((w.S, w.H), w.y_dtype, s_y, device) if with_y else None
    return ids, weights, x, y
