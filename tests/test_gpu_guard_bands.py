"""Every output of every entry point is a view into a larger buffer whose
guard bands before and after hold a sentinel; after the call the bands must
be unchanged (no write lands outside its output).  Sizes cover the small,
single-block and tiled prepare paths."""

import numpy as np
import pytest
import torch

import combine_permute_b200 as moe
from workloads import CONFIGS, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
BAND = 256  # bytes of guard before and after each output (keeps 16-byte alignment)


class Guarded:
    """Output views with sentinel guard bands, checked by check()."""

    def __init__(self):
        self.bufs = []

    def __call__(self, shape, dtype, sentinel):
        n = int(np.prod(shape))
        esz = torch.empty((), dtype=dtype).element_size()
        g = BAND // esz
        buf = torch.full((n + 2 * g,), sentinel, dtype=dtype, device=DEV)
        self.bufs.append((buf, g, n, sentinel))
        return buf[g:g + n].view(shape)

    def check(self):
        torch.cuda.synchronize()
        for buf, g, n, sentinel in self.bufs:
            host = buf.cpu()
            for band in (host[:g], host[g + n:]):
                if band.dtype.is_floating_point and np.isnan(sentinel):
                    assert torch.isnan(band.float()).all()
                else:
                    assert (band == sentinel).all()


@pytest.mark.parametrize("T", [40, 300, 700])
def test_outputs_stay_inside_their_buffers(T):
    w = CONFIGS["zipf_fp8_t16384_h4096_e288_k8"].scaled(T)
    ids_np, wt_np, x, y = make_workload(w, device=DEV)
    ids = torch.from_numpy(ids_np).to(DEV)
    wt = torch.from_numpy(wt_np).to(DEV)
    S, E, H, k, A = w.S, w.E, w.H, w.k, 16
    gd = Guarded()
    i32 = torch.int32
    meta = moe.moe_prepare(ids, E, blockscale_align=A,
                           expert_counts=gd((E,), i32, -5), expert_offsets=gd((E + 1,), i32, -5),
                           blockscale_offsets=gd((E + 1,), i32, -5),
                           input_permutation=gd((S,), i32, -5),
                           output_permutation=gd((S,), i32, -5), diag=gd((2,), i32, -5))
    rows = int(meta.blockscale_offsets[-1].item())
    moe.moe_dispatch_rows(x, k, meta.input_permutation, meta.output_permutation,
                          out=gd((S, H), torch.bfloat16, float("nan")))
    moe.moe_dispatch_rows(x, k, meta.input_permutation, None,
                          out=gd((S, H), torch.bfloat16, float("nan")))
    moe.moe_dispatch_rows_fp8(x, k, meta.output_permutation, meta.expert_offsets,
                              meta.blockscale_offsets, out_q=gd((S, H), torch.uint8, 0xAB),
                              out_scales=gd((rows, H // 128), torch.float32, float("nan")))
    moe.moe_dispatch_rows_nvfp4(x, k, meta.output_permutation, meta.expert_offsets,
                                meta.blockscale_offsets, out_q=gd((S, H // 2), torch.uint8, 0xAB),
                                out_scales=gd((rows, H // 16), torch.uint8, 0xCD))
    for odt in (torch.bfloat16, torch.float32):
        moe.moe_combine(y, meta.output_permutation, wt, out=gd((T, H), odt, float("nan")))
    out = gd((T, H), torch.bfloat16, float("nan"))
    out.fill_(1.0)
    moe.moe_output_memset(out, meta.output_permutation, k)
    gd.check()


def test_tiny_one_launch_and_window_outputs_stay_inside():
    w = CONFIGS["tiny_t32_h4096_e256_k8"]
    ids_np, _, x, _ = make_workload(w, device=DEV, with_y=False)
    S, E, k = w.S, w.E, w.k
    gd = Guarded()
    i32 = torch.int32
    moe.moe_prepare_dispatch(torch.from_numpy(ids_np).to(DEV), E, x,
                             out=gd((S, w.H), torch.bfloat16, float("nan")),
                             expert_counts=gd((E,), i32, -5),
                             expert_offsets=gd((E + 1,), i32, -5),
                             input_permutation=gd((S,), i32, -5),
                             output_permutation=gd((S,), i32, -5), diag=gd((2,), i32, -5))
    gd.check()


def test_grouped_gemm_metadata_outputs_stay_inside():
    w = CONFIGS["uniform_t4096_h7168_e256_k8"].scaled(900)
    ids_np, _, _, _ = make_workload(w, with_x=False, with_y=False)
    meta = moe.moe_prepare(torch.from_numpy(ids_np).to(DEV), w.E)
    S, E, tile = w.S, w.E, 64
    max_tiles = -(-S // tile) + min(E, S)
    gd = Guarded()
    i32 = torch.int32
    lib = moe._lib.load()
    bufs = [gd((E + 1,), i32, -5), gd((max_tiles,), i32, -5), gd((max_tiles,), i32, -5),
            gd((S,), i32, -5), gd((max_tiles * tile,), i32, -5), gd((1,), i32, -5),
            gd((1,), i32, -5)]
    st = lib.moe_tile_layout(w.T, w.k, E, tile, meta.expert_counts.data_ptr(),
                             meta.expert_offsets.data_ptr(), meta.output_permutation.data_ptr(),
                             max_tiles, *[b.data_ptr() for b in bufs],
                             torch.cuda.current_stream(DEV).cuda_stream)
    assert st == moe._lib.MOE_OK
    ps1, ps2 = gd((E, 3), i32, -5), gd((E, 3), i32, -5)
    st = lib.moe_problem_sizes(meta.expert_counts.data_ptr(), E, 2048, 7168, 7168, 2048,
                               ps1.data_ptr(), ps2.data_ptr(),
                               torch.cuda.current_stream(DEV).cuda_stream)
    assert st == moe._lib.MOE_OK
    gd.check()
