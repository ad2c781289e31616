"""Host-side tests of the C ABI: libmoe.so loads without a GPU, exports
every symbol include/moe.h declares, and rejects invalid arguments on the
host (returning a status, launching nothing).  No compute call is made.
"""

import ctypes
import os
import re
import subprocess

import pytest

from combine_permute_b200 import _lib
from combine_permute_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = 0, 1, 2, 3, 4
F32, F16, BF16, FP8 = 0, 1, 2, 3
P = 0x100000  # a non-null, 256-byte aligned stand-in pointer (never dereferenced)


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_binding_binds():
    assert declared_symbols() == sorted(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_[a-z0-9_]+)\b", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)
    # the library carries nothing of the oracle
    assert "oracle" not in out


def test_library_is_built_for_sm100a_only():
    from combine_permute_b200 import build as b
    assert b.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "--use_fast_math" not in b.NVCC_FLAGS  # IEEE division on the fp8 path


def test_status_strings_and_version(lib):
    for s in range(5):
        assert lib.moe_status_string(s).decode().startswith("MOE_")
    assert b"unknown" in lib.moe_status_string(99)
    assert lib.moe_version() >= 10000


def test_workspace_bytes(lib):
    assert lib.moe_prepare_workspace_bytes(32, 8, 256) == 0          # single-block path
    assert lib.moe_prepare_workspace_bytes(512, 8, 256) == 0         # 4096 slots: still one block
    a = lib.moe_prepare_workspace_bytes(513, 8, 256)                 # tiled path
    b = lib.moe_prepare_workspace_bytes(1 << 20, 6, 256)
    assert a > 0 and b > a and a % 256 == 0 and b % 256 == 0
    assert lib.moe_prepare_workspace_bytes(-1, 8, 256) == 0


def _prepare(lib, ids=P, T=4, k=2, E=8, counts=P, offsets=P, bso=None, A=1, inp=P, outp=P,
             diag=None, ws=None, ws_bytes=0):
    return lib.moe_prepare(ids, T, k, E, counts, offsets, bso, A, inp, outp, diag, ws, ws_bytes,
                           None)


def test_prepare_validation(lib):
    assert _prepare(lib, T=-1) == INVALID
    assert _prepare(lib, k=0) == INVALID
    assert _prepare(lib, E=0) == INVALID
    assert _prepare(lib, E=1025) == UNSUPPORTED
    assert _prepare(lib, ids=None) == INVALID
    assert _prepare(lib, counts=None) == INVALID
    assert _prepare(lib, offsets=None) == INVALID
    assert _prepare(lib, inp=None) == INVALID
    assert _prepare(lib, outp=None) == INVALID
    # an empty batch needs neither ids nor permutations (torch gives NULL for
    # empty tensors); it still launches, so only the argument check is tested
    assert _prepare(lib, T=0, ids=None, inp=None, outp=None, E=0) == INVALID
    assert _prepare(lib, bso=P, A=0) == INVALID
    assert _prepare(lib, T=1 << 28, k=8) == UNSUPPORTED              # T*k = 2^31
    # above one tile the workspace is required, large enough and aligned
    need = lib.moe_prepare_workspace_bytes(140000, 8, 8)
    assert need > 0
    assert _prepare(lib, T=140000, k=8, ws=None) == WORKSPACE
    assert _prepare(lib, T=140000, k=8, ws=P, ws_bytes=need - 1) == WORKSPACE
    assert _prepare(lib, T=140000, k=8, ws=P + 16, ws_bytes=need) == WORKSPACE


def test_dispatch_validation(lib):
    d = lib.moe_dispatch_rows
    assert d(P, F32, -1, 64, 2, P, P, P, None) == INVALID
    assert d(P, F32, 4, 64, 0, P, P, P, None) == INVALID
    assert d(P, FP8, 4, 64, 2, P, P, P, None) == INVALID             # fp8 is not a copy dtype
    assert d(P, BF16, 4, 12, 2, P, P, P, None) == INVALID            # 24-byte rows
    assert d(P, F32, 4, 6, 2, P, P, P, None) == INVALID              # 24-byte rows
    assert d(None, BF16, 4, 64, 2, P, P, P, None) == INVALID
    assert d(P, BF16, 4, 64, 2, None, None, P, None) == INVALID      # no permutation
    assert d(P, BF16, 4, 64, 2, P, P, None, None) == INVALID
    assert d(P + 8, BF16, 4, 64, 2, P, P, P, None) == INVALID        # misaligned x
    assert d(P, BF16, 4, 64, 2, P, P, P + 4, None) == INVALID        # misaligned out
    assert d(None, BF16, 0, 64, 2, None, None, None, None) == OK      # empty batch: nothing to do


def test_dispatch_fp8_validation(lib):
    f = lib.moe_dispatch_rows_fp8
    args = dict(x=P, dt=BF16, T=4, H=256, k=2, E=8, op=P, off=P, bso=P, q=P, sc=P)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["x"], a["dt"], a["T"], a["H"], a["k"], a["E"], a["op"], a["off"], a["bso"],
                 a["q"], a["sc"], None)

    assert call(dt=F32) == UNSUPPORTED
    assert call(H=200) == INVALID                                    # H % 128 != 0
    assert call(E=0) == INVALID
    for key in ("x", "op", "off", "bso", "q", "sc"):
        assert call(**{key: None}) == INVALID, key
    assert call(q=P + 8) == INVALID
    assert call(sc=P + 2) == INVALID
    assert call(T=0, x=None) == OK


def test_dispatch_nvfp4_validation(lib):
    f = lib.moe_dispatch_rows_nvfp4
    args = dict(x=P, dt=BF16, T=4, H=256, k=2, E=8, op=P, off=P, bso=P, q=P, sc=P)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["x"], a["dt"], a["T"], a["H"], a["k"], a["E"], a["op"], a["off"], a["bso"],
                 a["q"], a["sc"], None)

    assert call(dt=F32) == UNSUPPORTED
    assert call(dt=FP8) == UNSUPPORTED
    assert call(H=24) == INVALID                                     # H % 16 != 0
    assert call(H=0) == INVALID
    assert call(E=0) == INVALID
    assert call(k=0) == INVALID
    for key in ("x", "op", "off", "bso", "q", "sc"):
        assert call(**{key: None}) == INVALID, key
    assert call(x=P + 8) == INVALID                                  # x needs 16 bytes
    assert call(q=P + 4) == INVALID                                  # codes need 8 bytes
    assert call(T=0, x=None, q=None) == OK


def test_prepare_local_and_memset_validation(lib):
    pl = lib.moe_prepare_local
    assert pl(P, 2, 4, 2, 0, 8, P, P, None, 1, P, P, None, None, 0, None) == INVALID   # bad id type
    assert pl(P, 1, 4, 2, 0, 0, P, P, None, 1, P, P, None, None, 0, None) == INVALID   # no experts
    assert pl(P, 1, 4, 2, 0, 2000, P, P, None, 1, P, P, None, None, 0, None) == UNSUPPORTED
    assert pl(P, 1, 1000, 8, 5, 8, P, P, None, 1, P, P, None, None, 0, None) == WORKSPACE
    om = lib.moe_output_memset
    assert om(P, FP8, 4, 64, 2, P, None) == INVALID
    assert om(P, BF16, 4, 12, 2, P, None) == INVALID                   # 24-byte rows
    assert om(None, BF16, 4, 64, 2, P, None) == INVALID
    assert om(P + 4, BF16, 4, 64, 2, P, None) == INVALID
    assert om(None, BF16, 0, 64, 2, None, None) == OK


def test_tile_layout_validation(lib):
    tl = lib.moe_tile_layout
    args = [4, 2, 8, 16, P, P, P, 4, P, P, P, P, P, P, P, None]
    bad = list(args); bad[3] = 0
    assert tl(*bad) == INVALID                                       # tile size 0
    bad = list(args); bad[7] = 0
    assert tl(*bad) == INVALID                                       # no tiles
    bad = list(args); bad[7] = 1 << 20; bad[3] = 1 << 12
    assert tl(*bad) == UNSUPPORTED                                   # rows past 2^31
    bad = list(args); bad[6] = None
    assert tl(*bad) == INVALID                                       # no permutation
    assert lib.moe_problem_sizes(None, 8, 1, 1, 1, 1, P, P, None) == INVALID


def test_combine_validation(lib):
    c = lib.moe_combine
    assert c(P, BF16, -1, 64, 2, P, P, P, BF16, None) == INVALID
    assert c(P, FP8, 4, 64, 2, P, P, P, BF16, None) == INVALID
    assert c(P, BF16, 4, 64, 2, P, P, P, FP8, None) == INVALID
    assert c(P, F32, 4, 6, 2, P, P, P, BF16, None) == INVALID         # 24-byte y rows
    assert c(P, BF16, 4, 4, 2, P, P, P, F32, None) == INVALID         # 8-byte y rows
    assert c(None, BF16, 4, 64, 2, P, P, P, BF16, None) == INVALID
    assert c(P, BF16, 4, 64, 2, None, P, P, BF16, None) == INVALID
    assert c(P, BF16, 4, 64, 2, P, None, P, BF16, None) == INVALID
    assert c(P, BF16, 4, 64, 2, P, P, None, BF16, None) == INVALID
    assert c(P, BF16, 4, 64, 2, P, P + 2, P, BF16, None) == INVALID   # misaligned weights
    assert c(P, BF16, 0, 64, 2, None, None, None, BF16, None) == OK


def test_prepare_dispatch_validation(lib):
    f = lib.moe_prepare_dispatch
    assert f(P, 513, 8, 8, P, P, None, 1, P, P, None, P, BF16, 64, P, None) == UNSUPPORTED  # > 4096 slots
    assert f(P, 4, 2, 2000, P, P, None, 1, P, P, None, P, BF16, 64, P, None) == UNSUPPORTED
    assert f(P, 4, 2, 8, P, P, None, 1, P, P, None, P, BF16, 12, P, None) == INVALID
    assert f(P, 4, 2, 8, P, P, None, 1, P, P, None, None, BF16, 64, P, None) == INVALID
    assert f(P, 4, 2, 8, None, P, None, 1, P, P, None, P, BF16, 64, P, None) == INVALID
    assert f(P, 4, 2, 8, P, P, P, 0, P, P, None, P, BF16, 64, P, None) == INVALID


def test_product_code_never_touches_the_oracle():
    """The library and its binding neither import, load nor name the oracle;
    the oracle imports nothing of the library."""
    pkg = os.path.join(ROOT, "combine_permute_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"\boracle", text), fn
    for fn in os.listdir(os.path.join(ROOT, "oracle")):
        if fn.endswith((".py", ".c")):
            text = open(os.path.join(ROOT, "oracle", fn)).read()
            assert not re.search(r"^\s*(import|from)\s+combine_permute_b200", text, re.M), fn
            assert "libmoe" not in text and "moe.h" not in text, fn


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libmoe.so"))
    with pytest.raises(RuntimeError, match="no non-CUDA fallback"):
        _lib.load()


def test_valid_call_without_gpu_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = lib.moe_combine(P, BF16, 4, 64, 2, P, P, P, BF16, None)
    assert st == CUDA


def test_dispatch_error_and_wait_limits_validation(lib):
    # the error query needs somewhere to write; the limits call never fails
    assert lib.moe_dispatch_error(None, None) == INVALID
    assert lib.moe_set_wait_limits(0, 0) == OK
    assert lib.moe_set_wait_limits(-1, -1) == OK  # back to the defaults


def test_ep_peer_validation(lib):
    # layout: ranks, rank index, experts divisible by ranks, pointers
    def layout(R=2, rank=0, E=8, T=4, k=2, counts=P, ids=P, offs=P, outp=P, dr=P, drow=P, rr=P,
               lo=P):
        return lib.moe_ep_peer_layout(counts, R, rank, E, ids, T, k, offs, outp, dr, drow, rr, lo,
                                      None)
    assert layout(R=0) == INVALID
    assert layout(rank=2) == INVALID and layout(rank=-1) == INVALID
    assert layout(E=7) == INVALID
    assert layout(E=2048) == UNSUPPORTED
    assert layout(counts=None) == INVALID and layout(dr=None) == INVALID
    # dispatch into peer buffers: row size, alignment, pointers
    assert lib.moe_ep_dispatch_peer(P, BF16, 4, 4, 2, P, P, P, P, 2, None) == INVALID  # 8-byte rows
    assert lib.moe_ep_dispatch_peer(P + 8, BF16, 4, 64, 2, P, P, P, P, 2, None) == INVALID
    assert lib.moe_ep_dispatch_peer(P, BF16, 4, 64, 2, P, P, None, P, 2, None) == INVALID
    assert lib.moe_ep_dispatch_peer(P, FP8, 4, 64, 2, P, P, P, P, 2, None) == INVALID
    assert lib.moe_ep_dispatch_peer(P, BF16, 0, 64, 2, None, None, None, None, 2, None) == OK
    # combine from peer buffers (every call here returns before launching)
    assert lib.moe_ep_combine_peer(None, P, 2, BF16, 4, 64, 2, P, P, P, P, BF16, None) == INVALID
    assert lib.moe_ep_combine_peer(P, P, 0, BF16, 4, 64, 2, P, P, P, P, BF16, None) == INVALID
    assert lib.moe_ep_combine_peer(P, P, 2, BF16, 4, 4, 2, P, P, P, P, BF16, None) == INVALID
