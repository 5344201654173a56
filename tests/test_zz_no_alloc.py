"""mf_block_stats_noalloc: block statistics for callers that cannot allocate.

A serving engine that has handed all free HBM to its KV-cache pool, or a host
program with a fixed memory plan, cannot give the library a workspace.  This
entry point takes its scratch from an array the library keeps in device
memory.  The test calls it through the C ABI twice in a row, on two different
contexts, and checks each result against mf_block_stats with a caller
workspace.  Both run the same deterministic kernels, so the results must be
equal bit for bit, which also shows that every scratch word a call reads was
written by that call.  It lives in a file of its own that pytest collects
last.
"""
import ctypes as C

import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb
from cross_model_attention_block_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    f = lib.mf_block_stats_noalloc
    f.restype = C.c_int
    f.argtypes = [C.c_void_p] * 6
    return f


@pytest.mark.parametrize("cases", [[
    dict(lengths=[700, 300], Hs=40, d=128, B=128, dtype="bf16"),
    dict(lengths=[257, 64, 1000], Hs=8, d=128, B=64, dtype="bf16"),
]])
def test_noalloc_stats_match_the_workspace_entry_point(cases):
    lib = mfb.load_library()
    f = _noalloc(lib)
    for case in cases:  # two calls in a row share the library's scratch array
        w, x = synth.small_case(case["lengths"], case["Hs"], 4, 2, case["d"], case["B"], 0.9,
                                dtype=case["dtype"])
        ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width,
                               w.torch_dtype)
        Q, K = x.Q.cuda(), x.K.cuda()
        lse_ref, mass_ref = mfb.block_stats(ctx, Q, K)
        _, nblocks = ctx.layout_sizes()
        lse = torch.full_like(lse_ref, float("nan"))
        mass = torch.full((nblocks,), float("nan"), dtype=torch.float32, device="cuda")
        d = ctx.desc()
        st = f(C.byref(d), Q.data_ptr(), K.data_ptr(), lse.data_ptr(), mass.data_ptr(),
               torch.cuda.current_stream().cuda_stream)
        assert st == mfb.MF_OK, lib.mf_last_error().decode()
        mfb.sync_status()
        assert torch.equal(lse, lse_ref)
        assert torch.equal(mass, mass_ref[:nblocks])


def test_noalloc_rejects_a_context_beyond_its_scratch():
    lib = mfb.load_library()
    f = _noalloc(lib)
    g = lib.mf_block_stats_noalloc_max_workspace
    g.restype = C.c_size_t
    limit = g()
    assert limit == 8 << 20
    # 64 heads x 32768 tokens at B = 64: 64 * 131328 * 4 bytes of partial masses > 8 MiB
    ctx = mfb.Context.make([32768], 64, 128, 64, 2.0, 256, torch.bfloat16)
    d = ctx.desc()
    st = f(C.byref(d), 16, 16, 16, 16, None)
    assert st == mfb.MF_ERR_WORKSPACE
    assert "8 MiB" in lib.mf_last_error().decode()
