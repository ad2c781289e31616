"""CPU oracle for the MoE dispatch / combine path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library under
``combine_permute_b200`` never does, and this package imports nothing from
it.  Everything here is a plain restatement of what the pages say each
step computes:

* ``prepare``: sglang PR #19058, "Changes", item 1 (prepare_moe_input:
  tokens per expert, prefix-sum expert offsets, optional FP8 block-scale
  offsets, input / output permutations).
* ``dispatch``: same page, item 2 (shuffle_rows, a dtype-agnostic row
  gather).
* ``dispatch_fp8``: the FP8 block-scale MoE path of TensorRT-LLM PR #9592
  (run_moe_fp8_block_scales), with 1x128 blocks and scale = amax / 448.
* ``combine``: sglang PR #19058, item 3 (apply_shuffle_mul_sum: gather,
  scale by the router weight, reduce with fp32 accumulation).
* ``dispatch_nvfp4``: the B200 NVFP4 MoE path of TensorRT-LLM PR #9592
  (run_moe_nvfp4, scaling_vector_size = 16): E2M1 codes, one E4M3 scale per
  16 elements.
* ``problem_sizes`` and ``tile_layout``: the grouped-GEMM metadata that
  follows prepare (sglang's problem_sizes1/2; TensorRT-LLM's moe_sort
  outputs).
* ``ep_recv_layout``: the receiving rank's side of the expert-parallel
  exchange between GPUs (Mooncake PR #4581, dispatch / combine across
  ranks; TensorRT-LLM PR #9592, all-to-all communication and the local
  expert window): where each received row goes in the expert-grouped
  layout.
* ``prepare_local`` and ``output_memset``: one rank's expert window
  (local_expert_offset / num_local_experts) over int64 ids, and
  moe_output_memset_inplace (TensorRT-LLM PR #9592; Mooncake PR #4581 for
  the int64 top-k index type).

The arithmetic lives in ``moe_oracle.c`` (built with gcc, ``-O2
-ffp-contract=off``, single-threaded).  ``brute_prepare`` is a second,
pure-Python statement of the metadata step for tiny inputs, built on a
stable ``sorted`` instead of the per-expert scan.
"""

from __future__ import annotations

import contextlib
import ctypes
import os

import numpy as np

from .build import build_oracle, oracle_lib_path

__all__ = [
    "F32", "F16", "BF16", "lib", "prepare", "dispatch", "dispatch_fp8",
    "combine", "brute_prepare", "problem_sizes", "tile_layout", "prepare_local",
    "output_memset", "dispatch_nvfp4", "f32_to_e2m1", "e2m1_to_f32", "f32_to_bf16", "f32_to_f16", "f16_to_f32",
    "bf16_to_f32", "f32_to_e4m3", "e4m3_to_f32", "openmp", "threads", "ep_recv_layout",
]

F32, F16, BF16 = 0, 1, 2
_DT = {"fp32": F32, "fp16": F16, "bf16": BF16}

_lib = None
_i32p = ctypes.POINTER(ctypes.c_int32)
_vp = ctypes.c_void_p


_omp_lib = None
_use_omp = False


@contextlib.contextmanager
def openmp():
    """Within this block the oracle's calls run on its OpenMP build, which
    shares the dispatch and combine row loops among the host cores (same
    results; prepare stays one thread).  For the benchmark's CPU baseline."""
    global _use_omp
    prev = _use_omp
    _use_omp = True
    try:
        yield threads(True)
    finally:
        _use_omp = prev


def threads(openmp_build: bool = False) -> int:
    """Threads the oracle's row loops use: 1, or the OpenMP build's count."""
    return int(_load(openmp_build).oracle_threads())


def lib():
    """The oracle shared library (built on first use if it is missing)."""
    return _load(_use_omp)


def _load(openmp_build: bool):
    global _lib, _omp_lib
    if (_omp_lib if openmp_build else _lib) is None:
        path = oracle_lib_path(openmp_build)
        if not os.path.exists(path):
            build_oracle(openmp=openmp_build)
        L = ctypes.CDLL(path)
        L.oracle_threads.restype = ctypes.c_int
        L.oracle_threads.argtypes = []
        L.oracle_prepare.restype = ctypes.c_int64
        L.oracle_prepare.argtypes = [_vp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, _vp, _vp, _vp, _vp, _vp]
        L.oracle_dispatch.restype = None
        L.oracle_dispatch.argtypes = [_vp, ctypes.c_int64, ctypes.c_int32, _vp, ctypes.c_int64, _vp]
        L.oracle_dispatch_fp8.restype = None
        L.oracle_dispatch_fp8.argtypes = [_vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int32, _vp, _vp, _vp, _vp, ctypes.c_int64,
                                          _vp, _vp]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [_vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int32, _vp, _vp, _vp, ctypes.c_int]
        L.oracle_prepare_local_i64.restype = ctypes.c_int64
        L.oracle_prepare_local_i64.argtypes = [_vp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64,
                                               ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp]
        L.oracle_output_memset.restype = None
        L.oracle_output_memset.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _vp]
        L.oracle_dispatch_nvfp4.restype = None
        L.oracle_dispatch_nvfp4.argtypes = [_vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int32, _vp, _vp, _vp, _vp, ctypes.c_int64,
                                            _vp, _vp]
        L.oracle_ep_recv_layout.restype = ctypes.c_int64
        L.oracle_ep_recv_layout.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32] + [_vp] * 4
        L.oracle_e2m1_to_f32.restype = ctypes.c_float
        L.oracle_e2m1_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_problem_sizes.restype = None
        L.oracle_problem_sizes.argtypes = [_vp, ctypes.c_int32] + [ctypes.c_int32] * 4 + [_vp, _vp]
        L.oracle_tile_layout.restype = ctypes.c_int
        L.oracle_tile_layout.argtypes = [_vp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.c_int32, _vp, _vp, _vp, ctypes.c_int32] + [_vp] * 7
        for name in ["oracle_f32_to_e2m1_n", "oracle_f32_to_e4m3_n", "oracle_f32_to_bf16_n", "oracle_f32_to_f16_n",
                     "oracle_f16_to_f32_n", "oracle_bf16_to_f32_n", "oracle_e4m3_to_f32_n"]:
            fn = getattr(L, name)
            fn.restype = None
            fn.argtypes = [_vp, ctypes.c_int64, _vp]
        if openmp_build:
            _omp_lib = L
        else:
            _lib = L
    return _omp_lib if openmp_build else _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def prepare(ids: np.ndarray, E: int, block_align: int = 1):
    """Routing metadata of ids [T,k] int32.

    Returns a dict with counts [E], offsets [E+1], bso [E+1] (block-scale
    offsets with alignment ``block_align``), input_perm [T*k],
    output_perm [T*k] (all int32) and n_invalid (ids outside [0, E)).
    """
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    S = T * k
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    bso = np.zeros(E + 1, np.int32)
    inp = np.zeros(S, np.int32)
    outp = np.zeros(S, np.int32)
    n_bad = lib().oracle_prepare(_ptr(ids), T, k, E, block_align, _ptr(counts), _ptr(offsets),
                                 _ptr(bso), _ptr(inp), _ptr(outp))
    return dict(counts=counts, offsets=offsets, bso=bso, input_perm=inp, output_perm=outp,
                n_invalid=int(n_bad))


def dispatch(x: np.ndarray, k: int, input_perm: np.ndarray, out: np.ndarray | None = None):
    """Same-dtype dispatch: out[p] = x[input_perm[p] // k] (rows with -1 untouched)."""
    x = np.ascontiguousarray(x)
    input_perm = np.ascontiguousarray(input_perm, dtype=np.int32)
    S = input_perm.shape[0]
    if out is None:
        out = np.zeros((S,) + x.shape[1:], dtype=x.dtype)
    row_bytes = x.dtype.itemsize * int(np.prod(x.shape[1:]))
    lib().oracle_dispatch(_ptr(x), row_bytes, k, _ptr(input_perm), S, _ptr(out))
    return out


def dispatch_fp8(x_bits: np.ndarray, x_dtype: str, ids: np.ndarray, meta: dict,
                 q: np.ndarray | None = None, scales: np.ndarray | None = None):
    """FP8 E4M3 1x128 block-scale dispatch.

    ``x_bits`` is [T,H] uint16 holding bf16 or fp16 bit patterns.  Returns
    (q [S,H] uint8, scales [bso[E], H/128] fp32).  Arrays passed in are
    written in place, so untouched rows keep their previous contents.
    """
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, H = x_bits.shape
    k = ids.shape[1]
    S = T * k
    nb = H // 128
    if q is None:
        q = np.zeros((S, H), np.uint8)
    if scales is None:
        scales = np.zeros((int(meta["bso"][-1]), nb), np.float32)
    lib().oracle_dispatch_fp8(_ptr(x_bits), _DT[x_dtype], T, H, k, _ptr(ids),
                              _ptr(meta["input_perm"]), _ptr(meta["offsets"]), _ptr(meta["bso"]),
                              S, _ptr(q), _ptr(scales))
    return q, scales


def combine(y_bits: np.ndarray, y_dtype: str, output_perm: np.ndarray, w: np.ndarray,
            out_dtype: str):
    """out[t] = round(sum_j w[t,j] * y[output_perm[t*k+j]]) in fp32, j ascending.

    ``y_bits`` holds the raw storage ([S,H] uint16 for bf16/fp16, float32
    for fp32).  Returns raw storage of the output dtype.
    """
    y_bits = np.ascontiguousarray(y_bits)
    w = np.ascontiguousarray(w, dtype=np.float32)
    output_perm = np.ascontiguousarray(output_perm, dtype=np.int32)
    T, k = w.shape
    H = y_bits.shape[1]
    out = np.zeros((T, H), np.float32 if out_dtype == "fp32" else np.uint16)
    lib().oracle_combine(_ptr(y_bits), _DT[y_dtype], T, H, k, _ptr(output_perm), _ptr(w),
                         _ptr(out), _DT[out_dtype])
    return out


def prepare_local(ids: np.ndarray, base: int, E: int, block_align: int = 1):
    """Routing metadata of the experts [base, base + E) from int64 ids [T,k];
    slots outside the window are excluded like invalid ids."""
    ids = np.ascontiguousarray(ids, dtype=np.int64)
    T, k = ids.shape
    S = T * k
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    bso = np.zeros(E + 1, np.int32)
    inp = np.zeros(S, np.int32)
    outp = np.zeros(S, np.int32)
    n_bad = lib().oracle_prepare_local_i64(_ptr(ids), T, k, base, E, block_align, _ptr(counts),
                                           _ptr(offsets), _ptr(bso), _ptr(inp), _ptr(outp))
    return dict(counts=counts, offsets=offsets, bso=bso, input_perm=inp, output_perm=outp,
                n_invalid=int(n_bad))


def output_memset(out: np.ndarray, output_perm: np.ndarray, k: int):
    """Zero (in place) the rows of tokens with at least one routed slot."""
    assert out.flags["C_CONTIGUOUS"]
    output_perm = np.ascontiguousarray(output_perm, dtype=np.int32)
    T = out.shape[0]
    lib().oracle_output_memset(_ptr(out), out.nbytes // max(T, 1), T, k, _ptr(output_perm))
    return out


def dispatch_nvfp4(x_bits: np.ndarray, x_dtype: str, ids: np.ndarray, meta: dict,
                   q: np.ndarray | None = None, scales: np.ndarray | None = None):
    """NVFP4 dispatch (see moe_oracle.c): (q [S, H/2] packed E2M1 codes,
    scales [bso[E], H/16] E4M3 bytes).  Arrays passed in are written in place."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, H = x_bits.shape
    k = ids.shape[1]
    S = T * k
    if q is None:
        q = np.zeros((S, H // 2), np.uint8)
    if scales is None:
        scales = np.zeros((int(meta["bso"][-1]), H // 16), np.uint8)
    lib().oracle_dispatch_nvfp4(_ptr(x_bits), _DT[x_dtype], T, H, k, _ptr(ids),
                                _ptr(meta["input_perm"]), _ptr(meta["offsets"]), _ptr(meta["bso"]),
                                S, _ptr(q), _ptr(scales))
    return q, scales


def f32_to_e2m1(a):
    return _conv("oracle_f32_to_e2m1_n", a, np.float32, np.uint8)


def e2m1_to_f32(codes):
    return np.array([lib().oracle_e2m1_to_f32(int(c)) for c in np.asarray(codes).ravel()], np.float32)


def problem_sizes(counts: np.ndarray, n1: int, k1: int, n2: int, k2: int):
    """(M, N, K) of the two grouped GEMMs per expert: [E,3] int32 each."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    E = counts.size
    ps1 = np.zeros((E, 3), np.int32)
    ps2 = np.zeros((E, 3), np.int32)
    lib().oracle_problem_sizes(_ptr(counts), E, n1, k1, n2, k2, _ptr(ps1), _ptr(ps2))
    return ps1, ps2


def tile_layout(ids: np.ndarray, meta: dict, E: int, tile: int, max_tiles: int):
    """Tile-padded grouped-GEMM layout (see moe_oracle.c).  Returns a dict,
    or None when max_tiles * tile cannot hold the padded rows."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    out = dict(padded_offsets=np.zeros(E + 1, np.int32), tile_group=np.zeros(max_tiles, np.int32),
               tile_mn_limit=np.zeros(max_tiles, np.int32), exp2perm=np.zeros(T * k, np.int32),
               perm2exp=np.zeros(max_tiles * tile, np.int32), num_tiles=np.zeros(1, np.int32),
               total_padded=np.zeros(1, np.int32))
    rc = lib().oracle_tile_layout(_ptr(ids), T, k, E, tile, _ptr(meta["counts"]), _ptr(meta["offsets"]),
                                  _ptr(meta["output_perm"]), max_tiles, _ptr(out["padded_offsets"]),
                                  _ptr(out["tile_group"]), _ptr(out["tile_mn_limit"]), _ptr(out["exp2perm"]),
                                  _ptr(out["perm2exp"]), _ptr(out["num_tiles"]), _ptr(out["total_padded"]))
    if rc != 0:
        return None
    out["num_tiles"] = int(out["num_tiles"][0])
    out["total_padded"] = int(out["total_padded"][0])
    return out


def brute_prepare(ids, E: int, block_align: int = 1):
    """Pure-Python metadata for tiny inputs (a second statement of prepare).

    The dispatched order is ``sorted`` over (expert, token, slot) tuples of
    the valid slots, which is the stable order by expert id.
    """
    ids = [[int(v) for v in row] for row in ids]
    T = len(ids)
    k = len(ids[0]) if T else 0
    keyed = sorted((e, t, j) for t in range(T) for j, e in enumerate(ids[t]) if 0 <= e < E)
    input_perm = [t * k + j for (_, t, j) in keyed] + [-1] * (T * k - len(keyed))
    output_perm = [-1] * (T * k)
    for p, (_, t, j) in enumerate(keyed):
        output_perm[t * k + j] = p
    counts = [sum(1 for (e, _, _) in keyed if e == x) for x in range(E)]
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    bso = [0]
    for c in counts:
        bso.append(bso[-1] + -(-c // block_align) * block_align)
    return dict(counts=counts, offsets=offsets, bso=bso, input_perm=input_perm,
                output_perm=output_perm, n_invalid=T * k - len(keyed))


def _conv(name, arr, in_dtype, out_dtype):
    a = np.ascontiguousarray(np.asarray(arr, dtype=in_dtype).ravel())
    out = np.empty(a.shape, dtype=out_dtype)
    getattr(lib(), name)(_ptr(a), a.size, _ptr(out))
    return out


def f32_to_bf16(a):
    return _conv("oracle_f32_to_bf16_n", a, np.float32, np.uint16)


def f32_to_f16(a):
    return _conv("oracle_f32_to_f16_n", a, np.float32, np.uint16)


def f32_to_e4m3(a):
    return _conv("oracle_f32_to_e4m3_n", a, np.float32, np.uint8)


def bf16_to_f32(a):
    return _conv("oracle_bf16_to_f32_n", a, np.uint16, np.float32)


def f16_to_f32(a):
    return _conv("oracle_f16_to_f32_n", a, np.uint16, np.float32)


def e4m3_to_f32(a):
    return _conv("oracle_e4m3_to_f32_n", a, np.uint8, np.float32)


def ep_recv_layout(counts: np.ndarray):
    """Receive layout of one rank in the expert-parallel exchange.

    ``counts`` [R, El] int32: rows source rank s sends for local expert le.
    Returns recv_offsets [R+1], local_offsets [El+1], recv_to_local [N] and
    local_to_recv [N] (int32), N = counts.sum().
    """
    c = np.ascontiguousarray(counts, dtype=np.int32)
    R, El = c.shape
    n = int(c.astype(np.int64).sum())
    ro = np.zeros(R + 1, np.int32)
    lo = np.zeros(El + 1, np.int32)
    r2l = np.zeros(n, np.int32)
    l2r = np.zeros(n, np.int32)
    got = lib().oracle_ep_recv_layout(_ptr(c), R, El, _ptr(ro), _ptr(lo), _ptr(r2l), _ptr(l2r))
    assert got == n
    return dict(recv_offsets=ro, local_offsets=lo, recv_to_local=r2l, local_to_recv=l2r)
