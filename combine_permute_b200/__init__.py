"""Single-GPU MoE dispatch / combine for B200 (sm_100a).

Python face of libmoe.so.  The functions carry the C ABI's names and take
torch CUDA tensors; they check shapes and types, allocate outputs with torch
when none are given (torch is the device-memory and stream plumbing here),
and call the library on the current CUDA stream.  Every step runs in the
library's CUDA kernels; if libmoe.so is missing, calls raise.

    meta = moe_prepare(topk_ids, num_experts)                 # routing metadata
    xd = moe_dispatch_rows(x, k, meta.input_permutation,
                           meta.output_permutation)           # expert-grouped rows
    out = moe_combine(y, meta.output_permutation, weights)    # weighted k-way sum
"""

from __future__ import annotations

from typing import NamedTuple, Optional

import torch

from . import _lib
from ._lib import MoeError  # noqa: F401

__all__ = [
    "MoeError",
    "PrepareResult",
    "moe_prepare",
    "moe_prepare_workspace_bytes",
    "moe_dispatch_rows",
    "moe_dispatch_error",
    "moe_set_wait_limits",
    "moe_dispatch_rows_fp8",
    "moe_dispatch_rows_nvfp4",
    "moe_combine",
    "moe_prepare_dispatch",
    "moe_version",
    "moe_problem_sizes",
    "moe_tile_layout",
    "moe_prepare_local",
    "moe_output_memset",
    "moe_ep_recv_layout",
    "EpRecvLayout",
    "moe_ep_peer_layout",
    "EpPeerLayout",
    "moe_ep_dispatch_peer",
    "moe_ep_combine_peer",
    "moe_ep_buffer_table",
    "TileLayout",
    "library_path",
]

_DTYPES = {
    torch.float32: _lib.MOE_F32,
    torch.float16: _lib.MOE_F16,
    torch.bfloat16: _lib.MOE_BF16,
}


class TileLayout(NamedTuple):
    padded_offsets: torch.Tensor                # [E+1]
    tile_idx_to_group_idx: torch.Tensor         # [max_tiles]
    tile_idx_to_mn_limit: torch.Tensor          # [max_tiles]
    expanded_idx_to_permuted_idx: torch.Tensor  # [T*k]
    permuted_idx_to_expanded_idx: torch.Tensor  # [max_tiles * tile_size]
    num_non_exiting_tiles: torch.Tensor         # [1] (-1: max_tiles too small)
    total_num_padded_tokens: torch.Tensor       # [1]


class EpRecvLayout(NamedTuple):
    recv_offsets: torch.Tensor    # [R+1] int32
    local_offsets: torch.Tensor   # [El+1] int32
    recv_to_local: torch.Tensor   # [N] int32
    local_to_recv: torch.Tensor   # [N] int32
    num_recv: torch.Tensor        # [1] int32


class EpPeerLayout(NamedTuple):
    dest_rank: torch.Tensor       # [T*k] int32: rank owning each slot's expert (-1: none)
    dest_row: torch.Tensor        # [T*k] int32: the slot's row in that rank's grouped buffer
    recv_rows: torch.Tensor       # [R] int32: rows of each rank's grouped buffer
    local_offsets: torch.Tensor   # [El+1] int32: this rank's grouped expert offsets


class PrepareResult(NamedTuple):
    expert_counts: torch.Tensor        # [E] int32
    expert_offsets: torch.Tensor       # [E+1] int32
    blockscale_offsets: Optional[torch.Tensor]  # [E+1] int32 or None
    input_permutation: torch.Tensor    # [T*k] int32
    output_permutation: torch.Tensor   # [T*k] int32
    diag: torch.Tensor                 # [2] int32: invalid ids, wait gave up


def library_path() -> str:
    return _lib.LIB_PATH


def moe_version() -> int:
    return int(_lib.load().moe_version())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=None, shape=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t


def _dtype_code(dt: torch.dtype) -> int:
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    return _DTYPES[dt]


# One prepare workspace per (device, stream), zeroed once when allocated;
# the library maintains it between calls.
_WORKSPACES: dict = {}


def _workspace(device: torch.device, nbytes: int) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return None
    key = (device, torch.cuda.current_stream(device).cuda_stream)
    ws = _WORKSPACES.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _WORKSPACES[key] = ws
    return ws


def _drop_workspace(device: torch.device, status: int) -> None:
    """After a failed launch the cached workspace may hold a half-written
    call's words; the library needs it all-zero again, so forget it."""
    if status == _lib.MOE_ERR_CUDA:
        _WORKSPACES.pop((device, torch.cuda.current_stream(device).cuda_stream), None)


def moe_prepare_workspace_bytes(num_tokens: int, top_k: int, num_experts: int) -> int:
    return int(_lib.load().moe_prepare_workspace_bytes(num_tokens, top_k, num_experts))


def _alloc_meta(device, S, E, with_bso, expert_counts, expert_offsets, blockscale_offsets,
                input_permutation, output_permutation, diag):
    i32 = dict(dtype=torch.int32, device=device)
    ec = expert_counts if expert_counts is not None else torch.empty(E, **i32)
    eo = expert_offsets if expert_offsets is not None else torch.empty(E + 1, **i32)
    bs = blockscale_offsets
    if with_bso and bs is None:
        bs = torch.empty(E + 1, **i32)
    ip = input_permutation if input_permutation is not None else torch.empty(S, **i32)
    op = output_permutation if output_permutation is not None else torch.empty(S, **i32)
    dg = diag if diag is not None else torch.empty(2, **i32)
    _need(ec, "expert_counts", torch.int32, (E,), device)
    _need(eo, "expert_offsets", torch.int32, (E + 1,), device)
    if bs is not None:
        _need(bs, "blockscale_offsets", torch.int32, (E + 1,), device)
    _need(ip, "input_permutation", torch.int32, (S,), device)
    _need(op, "output_permutation", torch.int32, (S,), device)
    _need(dg, "diag", torch.int32, (2,), device)
    return PrepareResult(ec, eo, bs, ip, op, dg)


def moe_prepare(topk_ids: torch.Tensor, num_experts: int, *, blockscale_align: Optional[int] = None,
                expert_counts=None, expert_offsets=None, blockscale_offsets=None,
                input_permutation=None, output_permutation=None, diag=None,
                workspace: Optional[torch.Tensor] = None) -> PrepareResult:
    """Routing metadata of topk_ids [T, k] int32 (see include/moe.h).

    Block-scale offsets are produced when ``blockscale_align`` is given.
    """
    _need(topk_ids, "topk_ids", torch.int32)
    if topk_ids.dim() != 2:
        raise ValueError("topk_ids must be [T, k]")
    T, k = topk_ids.shape
    dev = topk_ids.device
    with torch.cuda.device(dev):
        meta = _alloc_meta(dev, T * k, num_experts, blockscale_align is not None, expert_counts,
                           expert_offsets, blockscale_offsets, input_permutation,
                           output_permutation, diag)
        need = moe_prepare_workspace_bytes(T, k, num_experts) if T * k > 0 else 0
        if workspace is None:
            workspace = _workspace(dev, need)
        elif need:
            _need(workspace, "workspace", device=dev)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = _lib.load().moe_prepare(
            topk_ids.data_ptr(), T, k, num_experts, meta.expert_counts.data_ptr(),
            meta.expert_offsets.data_ptr(), _ptr(meta.blockscale_offsets),
            blockscale_align or 1, meta.input_permutation.data_ptr(),
            meta.output_permutation.data_ptr(), meta.diag.data_ptr(), _ptr(workspace), ws_bytes,
            _stream(dev))
        _drop_workspace(dev, st)
    _lib.check("moe_prepare", st)
    return meta


def moe_dispatch_rows(x: torch.Tensor, top_k: int, input_permutation: Optional[torch.Tensor] = None,
                      output_permutation: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[p] = x[input_permutation[p] // k] (see include/moe.h)."""
    _need(x, "x")
    if x.dim() != 2:
        raise ValueError("x must be [T, H]")
    T, H = x.shape
    S = T * top_k
    dev = x.device
    for name, t in (("input_permutation", input_permutation),
                    ("output_permutation", output_permutation)):
        if t is not None:
            _need(t, name, torch.int32, (S,), dev)
    if out is None:
        out = torch.empty((S, H), dtype=x.dtype, device=dev)
    _need(out, "out", x.dtype, (S, H), dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_dispatch_rows(x.data_ptr(), _dtype_code(x.dtype), T, H, top_k,
                                           _ptr(input_permutation), _ptr(output_permutation),
                                           out.data_ptr(), _stream(dev))
    _lib.check("moe_dispatch_rows", st)
    return out


def moe_dispatch_error(device=None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Enqueues the read-and-clear of the TMA dispatch's error word on the
    current stream of ``device``; returns the int32 [1] device tensor it is
    written to (1: a bounded wait gave up since the last query, rows are
    incomplete; 0 otherwise).  See include/moe.h."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = torch.empty(1, dtype=torch.int32, device=dev)
    _need(out, "out", torch.int32, (1,), dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_dispatch_error(out.data_ptr(), _stream(dev))
    _lib.check("moe_dispatch_error", st)
    return out


def moe_set_wait_limits(prepare_wait_us: int = -1, dispatch_polls: int = -1) -> None:
    """Limits of the library's bounded waits (negative: the default), for
    tests of the failure reporting.  See include/moe.h."""
    _lib.check("moe_set_wait_limits",
               _lib.load().moe_set_wait_limits(int(prepare_wait_us), int(dispatch_polls)))


def moe_dispatch_rows_fp8(x: torch.Tensor, top_k: int, output_permutation: torch.Tensor,
                          expert_offsets: torch.Tensor, blockscale_offsets: torch.Tensor, *,
                          blockscale_align: int = 1, out_q: Optional[torch.Tensor] = None,
                          out_scales: Optional[torch.Tensor] = None):
    """FP8 E4M3 1x128 block-scale dispatch.  Returns (out_q uint8 [T*k, H],
    out_scales fp32 [rows, H/128]).

    Without ``out_scales`` the scale tensor is allocated with the upper bound
    T*k + E*(blockscale_align - 1) rows (no device-to-host read).
    """
    _need(x, "x")
    T, H = x.shape
    k = top_k
    E = expert_offsets.numel() - 1
    S = T * k
    dev = x.device
    _need(output_permutation, "output_permutation", torch.int32, (S,), dev)
    _need(expert_offsets, "expert_offsets", torch.int32, (E + 1,), dev)
    _need(blockscale_offsets, "blockscale_offsets", torch.int32, (E + 1,), dev)
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("fp8 dispatch reads bf16 or fp16 activations")
    if out_q is None:
        out_q = torch.empty((S, H), dtype=torch.uint8, device=dev)
    if out_q.dtype == torch.float8_e4m3fn:
        out_q = out_q.view(torch.uint8)
    _need(out_q, "out_q", torch.uint8, (S, H), dev)
    if out_scales is None:
        out_scales = torch.empty((S + E * (blockscale_align - 1), H // 128), dtype=torch.float32,
                                 device=dev)
    _need(out_scales, "out_scales", torch.float32, None, dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_dispatch_rows_fp8(
            x.data_ptr(), _dtype_code(x.dtype), T, H, k, E, output_permutation.data_ptr(),
            expert_offsets.data_ptr(), blockscale_offsets.data_ptr(), out_q.data_ptr(),
            out_scales.data_ptr(), _stream(dev))
    _lib.check("moe_dispatch_rows_fp8", st)
    return out_q, out_scales


def moe_dispatch_rows_nvfp4(x: torch.Tensor, top_k: int, output_permutation: torch.Tensor,
                            expert_offsets: torch.Tensor, blockscale_offsets: torch.Tensor, *,
                            blockscale_align: int = 1, out_q: Optional[torch.Tensor] = None,
                            out_scales: Optional[torch.Tensor] = None):
    """NVFP4 dispatch (E2M1 codes two per byte, one E4M3 scale byte per 16
    elements; see include/moe.h).  Returns (out_q uint8 [T*k, H/2],
    out_scales uint8 [rows, H/16]).

    Without ``out_scales`` the scale tensor is allocated with the upper bound
    T*k + E*(blockscale_align - 1) rows (no device-to-host read).
    """
    _need(x, "x")
    T, H = x.shape
    k = top_k
    E = expert_offsets.numel() - 1
    S = T * k
    dev = x.device
    _need(output_permutation, "output_permutation", torch.int32, (S,), dev)
    _need(expert_offsets, "expert_offsets", torch.int32, (E + 1,), dev)
    _need(blockscale_offsets, "blockscale_offsets", torch.int32, (E + 1,), dev)
    if x.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("nvfp4 dispatch reads bf16 or fp16 activations")
    if H % 16:
        raise ValueError("nvfp4 dispatch needs a hidden size that is a multiple of 16")
    if out_q is None:
        out_q = torch.empty((S, H // 2), dtype=torch.uint8, device=dev)
    _need(out_q, "out_q", torch.uint8, (S, H // 2), dev)
    if out_scales is None:
        out_scales = torch.empty((S + E * (blockscale_align - 1), H // 16), dtype=torch.uint8,
                                 device=dev)
    if out_scales.dtype == torch.float8_e4m3fn:
        out_scales = out_scales.view(torch.uint8)
    _need(out_scales, "out_scales", torch.uint8, None, dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_dispatch_rows_nvfp4(
            x.data_ptr(), _dtype_code(x.dtype), T, H, k, E, output_permutation.data_ptr(),
            expert_offsets.data_ptr(), blockscale_offsets.data_ptr(), out_q.data_ptr(),
            out_scales.data_ptr(), _stream(dev))
    _lib.check("moe_dispatch_rows_nvfp4", st)
    return out_q, out_scales


def moe_combine(y: torch.Tensor, output_permutation: torch.Tensor, weights: torch.Tensor, *,
                out_dtype: Optional[torch.dtype] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[t] = sum_j weights[t, j] * y[output_permutation[t*k + j]] (fp32
    accumulation, see include/moe.h)."""
    _need(y, "y")
    _need(weights, "weights", torch.float32)
    T, k = weights.shape
    S, H = y.shape
    dev = y.device
    if S != T * k:
        raise ValueError("y must have T*k rows")
    _need(output_permutation, "output_permutation", torch.int32, (S,), dev)
    _need(weights, "weights", torch.float32, (T, k), dev)
    if out is None:
        out = torch.empty((T, H), dtype=out_dtype or y.dtype, device=dev)
    _need(out, "out", None, (T, H), dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_combine(y.data_ptr(), _dtype_code(y.dtype), T, H, k,
                                     output_permutation.data_ptr(), weights.data_ptr(),
                                     out.data_ptr(), _dtype_code(out.dtype), _stream(dev))
    _lib.check("moe_combine", st)
    return out


def moe_prepare_dispatch(topk_ids: torch.Tensor, num_experts: int, x: torch.Tensor, *,
                         blockscale_align: Optional[int] = None, out: Optional[torch.Tensor] = None,
                         expert_counts=None, expert_offsets=None, blockscale_offsets=None,
                         input_permutation=None, output_permutation=None, diag=None):
    """moe_prepare + moe_dispatch_rows in one launch for tiny batches.
    Returns (PrepareResult, dispatched rows)."""
    _need(topk_ids, "topk_ids", torch.int32)
    _need(x, "x")
    T, k = topk_ids.shape
    H = x.shape[1]
    dev = x.device
    _need(x, "x", None, (T, H), dev)
    meta = _alloc_meta(dev, T * k, num_experts, blockscale_align is not None, expert_counts,
                       expert_offsets, blockscale_offsets, input_permutation, output_permutation,
                       diag)
    if out is None:
        out = torch.empty((T * k, H), dtype=x.dtype, device=dev)
    _need(out, "out", x.dtype, (T * k, H), dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_prepare_dispatch(
            topk_ids.data_ptr(), T, k, num_experts, meta.expert_counts.data_ptr(),
            meta.expert_offsets.data_ptr(), _ptr(meta.blockscale_offsets), blockscale_align or 1,
            meta.input_permutation.data_ptr(), meta.output_permutation.data_ptr(),
            meta.diag.data_ptr(), x.data_ptr(), _dtype_code(x.dtype), H, out.data_ptr(),
            _stream(dev))
    _lib.check("moe_prepare_dispatch", st)
    return meta, out


def moe_problem_sizes(expert_counts: torch.Tensor, n1: int, k1: int, n2: int, k2: int):
    """(M, N, K) per expert of the two grouped GEMMs: two [E, 3] int32 tensors."""
    _need(expert_counts, "expert_counts", torch.int32)
    E = expert_counts.numel()
    dev = expert_counts.device
    ps1 = torch.empty((E, 3), dtype=torch.int32, device=dev)
    ps2 = torch.empty((E, 3), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_problem_sizes(expert_counts.data_ptr(), E, n1, k1, n2, k2,
                                           ps1.data_ptr(), ps2.data_ptr(), _stream(dev))
    _lib.check("moe_problem_sizes", st)
    return ps1, ps2


def moe_tile_layout(meta: PrepareResult, top_k: int, tile_size: int,
                    max_tiles: Optional[int] = None) -> TileLayout:
    """Tile-padded grouped-GEMM layout from moe_prepare's results (see
    include/moe.h).  Without ``max_tiles`` the always-sufficient bound
    ceil(T*k / tile) + min(E, T*k) is used."""
    E = meta.expert_counts.numel()
    S = meta.output_permutation.numel()
    T = S // top_k
    dev = meta.expert_counts.device
    if max_tiles is None:
        max_tiles = max(1, -(-S // tile_size) + min(E, S))
    i32 = dict(dtype=torch.int32, device=dev)
    out = TileLayout(torch.empty(E + 1, **i32), torch.empty(max_tiles, **i32),
                     torch.empty(max_tiles, **i32), torch.empty(S, **i32),
                     torch.empty(max_tiles * tile_size, **i32), torch.empty(1, **i32),
                     torch.empty(1, **i32))
    with torch.cuda.device(dev):
        st = _lib.load().moe_tile_layout(
            T, top_k, E, tile_size, meta.expert_counts.data_ptr(), meta.expert_offsets.data_ptr(),
            _ptr(meta.output_permutation) if S else None, max_tiles,
            *[_ptr(t) if t.numel() else None for t in out], _stream(dev))
    _lib.check("moe_tile_layout", st)
    return out


def moe_prepare_local(topk_ids: torch.Tensor, local_expert_offset: int, num_local_experts: int, *,
                      blockscale_align: Optional[int] = None,
                      workspace: Optional[torch.Tensor] = None) -> PrepareResult:
    """Routing metadata of one rank's experts [offset, offset + n) from int32
    or int64 ids [T, k]; other slots are excluded (see include/moe.h)."""
    if topk_ids.dtype not in (torch.int32, torch.int64):
        raise ValueError("topk_ids must be int32 or int64")
    _need(topk_ids, "topk_ids")
    T, k = topk_ids.shape
    E = num_local_experts
    dev = topk_ids.device
    with torch.cuda.device(dev):
        meta = _alloc_meta(dev, T * k, E, blockscale_align is not None, None, None, None, None,
                           None, None)
        need = moe_prepare_workspace_bytes(T, k, E) if T * k > 0 else 0
        if workspace is None:
            workspace = _workspace(dev, need)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        id_type = _lib.MOE_I64 if topk_ids.dtype == torch.int64 else _lib.MOE_I32
        st = _lib.load().moe_prepare_local(
            _ptr(topk_ids) if T * k else None, id_type, T, k, local_expert_offset, E,
            meta.expert_counts.data_ptr(), meta.expert_offsets.data_ptr(),
            _ptr(meta.blockscale_offsets), blockscale_align or 1,
            _ptr(meta.input_permutation) if T * k else None,
            _ptr(meta.output_permutation) if T * k else None, meta.diag.data_ptr(),
            _ptr(workspace), ws_bytes, _stream(dev))
        _drop_workspace(dev, st)
    _lib.check("moe_prepare_local", st)
    return meta


def moe_output_memset(out: torch.Tensor, output_permutation: torch.Tensor, top_k: int) -> torch.Tensor:
    """Zero (in place) the rows of tokens with at least one routed slot."""
    _need(out, "out")
    T, H = out.shape
    _need(output_permutation, "output_permutation", torch.int32, (T * top_k,), out.device)
    with torch.cuda.device(out.device):
        st = _lib.load().moe_output_memset(out.data_ptr(), _dtype_code(out.dtype), T, H, top_k,
                                           output_permutation.data_ptr(), _stream(out.device))
    _lib.check("moe_output_memset", st)
    return out


def moe_ep_recv_layout(recv_expert_counts: torch.Tensor, num_recv: int) -> EpRecvLayout:
    """Receiving rank's layout of the expert-parallel exchange (see
    include/moe.h).  ``recv_expert_counts`` [R, El] int32 on the GPU;
    ``num_recv`` = its sum (the caller knows it from the count exchange),
    which sizes the two row maps."""
    _need(recv_expert_counts, "recv_expert_counts", torch.int32)
    if recv_expert_counts.dim() != 2:
        raise ValueError("recv_expert_counts must be [num_ranks, num_local_experts]")
    R, El = recv_expert_counts.shape
    dev = recv_expert_counts.device
    i32 = dict(dtype=torch.int32, device=dev)
    lay = EpRecvLayout(torch.empty(R + 1, **i32), torch.empty(El + 1, **i32),
                       torch.empty(num_recv, **i32), torch.empty(num_recv, **i32),
                       torch.empty(1, **i32))
    with torch.cuda.device(dev):
        st = _lib.load().moe_ep_recv_layout(
            recv_expert_counts.data_ptr(), R, El, num_recv, lay.recv_offsets.data_ptr(),
            lay.local_offsets.data_ptr(), _ptr(lay.recv_to_local) if num_recv else None,
            _ptr(lay.local_to_recv) if num_recv else None, lay.num_recv.data_ptr(), _stream(dev))
    _lib.check("moe_ep_recv_layout", st)
    return lay


def moe_ep_peer_layout(all_expert_counts: torch.Tensor, rank: int, topk_ids: torch.Tensor,
                       meta: PrepareResult) -> EpPeerLayout:
    """Every slot's destination rank and row in the owners' grouped buffers
    (see include/moe.h).  ``all_expert_counts`` [R, E] int32 holds every
    rank's expert counts; ``meta`` is this rank's moe_prepare over all E
    experts of ``topk_ids`` [T, k]."""
    _need(all_expert_counts, "all_expert_counts", torch.int32)
    if all_expert_counts.dim() != 2:
        raise ValueError("all_expert_counts must be [num_ranks, num_experts]")
    R, E = all_expert_counts.shape
    T, k = topk_ids.shape
    dev = topk_ids.device
    _need(topk_ids, "topk_ids", torch.int32, (T, k), dev)
    i32 = dict(dtype=torch.int32, device=dev)
    lay = EpPeerLayout(torch.empty(T * k, **i32), torch.empty(T * k, **i32), torch.empty(R, **i32),
                       torch.empty(E // R + 1 if R and E % R == 0 else 1, **i32))
    with torch.cuda.device(dev):
        st = _lib.load().moe_ep_peer_layout(
            all_expert_counts.data_ptr(), R, rank, E, topk_ids.data_ptr(), T, k,
            meta.expert_offsets.data_ptr(), meta.output_permutation.data_ptr(),
            lay.dest_rank.data_ptr(), lay.dest_row.data_ptr(), lay.recv_rows.data_ptr(),
            lay.local_offsets.data_ptr(), _stream(dev))
    _lib.check("moe_ep_peer_layout", st)
    return lay


def moe_ep_buffer_table(buffers, device) -> torch.Tensor:
    """The device array of the ranks' buffer addresses that moe_ep_dispatch_peer
    and moe_ep_combine_peer read (int64 [R] on ``device``), from tensors or raw
    device addresses valid in this process (another GPU's memory mapped in).
    Building it copies from the host; a caller that records the exchange in a
    CUDA graph builds it once beforehand and passes it in place of the list.
    The table holds references to the tensors it was built from, so that
    their memory stays allocated while the table exists (torch may otherwise
    hand freed blocks back to the driver, e.g. when a graph capture begins);
    raw addresses stay the caller's to keep valid."""
    ptrs = [b.data_ptr() if isinstance(b, torch.Tensor) else int(b) for b in buffers]
    table = torch.tensor(ptrs, dtype=torch.int64).to(device)
    table._buffers = [b for b in buffers if isinstance(b, torch.Tensor)]
    return table


def _pointer_array(buffers, dev) -> torch.Tensor:
    if isinstance(buffers, torch.Tensor):  # a table from moe_ep_buffer_table
        _need(buffers, "buffer table", torch.int64, (buffers.numel(),), dev)
        return buffers
    return moe_ep_buffer_table(buffers, dev)


def moe_ep_dispatch_peer(x: torch.Tensor, top_k: int, layout: EpPeerLayout, recv_buffers) -> None:
    """Stores every row of x [T, H] into the grouped buffers of the ranks
    owning its experts (``recv_buffers``: one per rank, tensors or device
    addresses, or their moe_ep_buffer_table; see include/moe.h)."""
    _need(x, "x")
    T, H = x.shape
    dev = x.device
    R = layout.recv_rows.numel()
    if len(recv_buffers) != R:
        raise ValueError(f"{len(recv_buffers)} buffers for {R} ranks")
    ptrs = _pointer_array(recv_buffers, dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_ep_dispatch_peer(
            x.data_ptr(), _dtype_code(x.dtype), T, H, top_k, layout.dest_rank.data_ptr(),
            layout.dest_row.data_ptr(), ptrs.data_ptr(), layout.recv_rows.data_ptr(), R,
            _stream(dev))
    _lib.check("moe_ep_dispatch_peer", st)
    ptrs.record_stream(torch.cuda.current_stream(dev))


def moe_ep_combine_peer(out_buffers, y_dtype: torch.dtype, hidden: int, layout: EpPeerLayout,
                        weights: torch.Tensor, *, out_dtype: Optional[torch.dtype] = None,
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[t] = sum_j weights[t, j] * (expert output of slot (t, j), read from
    its owner's buffer ``out_buffers[rank]``, or through their
    moe_ep_buffer_table), fp32 accumulation in slot order (see
    include/moe.h)."""
    _need(weights, "weights", torch.float32)
    T, k = weights.shape
    dev = weights.device
    R = layout.recv_rows.numel()
    if len(out_buffers) != R:
        raise ValueError(f"{len(out_buffers)} buffers for {R} ranks")
    if out is None:
        out = torch.empty((T, hidden), dtype=out_dtype or y_dtype, device=dev)
    _need(out, "out", None, (T, hidden), dev)
    ptrs = _pointer_array(out_buffers, dev)
    with torch.cuda.device(dev):
        st = _lib.load().moe_ep_combine_peer(
            ptrs.data_ptr(), layout.recv_rows.data_ptr(), R, _dtype_code(y_dtype), T, hidden, k,
            layout.dest_rank.data_ptr(), layout.dest_row.data_ptr(), weights.data_ptr(),
            out.data_ptr(), _dtype_code(out.dtype), _stream(dev))
    _lib.check("moe_ep_combine_peer", st)
    ptrs.record_stream(torch.cuda.current_stream(dev))
    return out
