"""Host-side checks of the C ABI: exports, layout sizes, argument validation,
and the prefix-hash index (no GPU needed; nothing here launches a kernel)."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mapflow.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mf_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert "mf_mapped_av" in names and len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(mfb.EXPORTED) <= set(names)
    assert lib.mf_version().decode().startswith("mapflow")


def _sizes_py(lengths, B):
    nqb = sum((L + B - 1) // B for L in lengths)
    nbl = sum(((L + B - 1) // B) * ((L + B - 1) // B + 1) // 2 for L in lengths)
    return nqb, nbl


@pytest.mark.parametrize("lengths,B", [([512], 64), ([8192], 64), ([32768], 128),
                                       ([1, 63, 64, 65, 0, 1000], 64), ([130, 7], 128)])
def test_layout_sizes(lib, lengths, B):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    assert mfb.layout_sizes(cu, B) == _sizes_py(lengths, B)


def test_layout_sizes_rejects_bad_input(lib):
    with pytest.raises(mfb.MapflowError) as e:
        mfb.layout_sizes(np.array([0, 100], np.int32), 32)
    assert e.value.status == mfb.MF_ERR_UNSUPPORTED
    with pytest.raises(mfb.MapflowError) as e:
        mfb.layout_sizes(np.array([0, 100, 50], np.int32), 64)
    assert e.value.status == mfb.MF_ERR_INVALID_ARG
    with pytest.raises(mfb.MapflowError) as e:
        mfb.layout_sizes(np.array([0, 512 * 64 + 1], np.int32), 64)
    assert e.value.status == mfb.MF_ERR_UNSUPPORTED


def _desc(Hs=4, d=64, B=64, cu=(0, 512), dt=mfb.MF_F32):
    host = np.array(cu, dtype=np.int32)
    dsc = mfb.AttnDesc(len(cu) - 1, 0x1000, host.ctypes.data, Hs, d, B, 0.0, 256, dt)
    return dsc, host


def test_null_is_accepted_only_for_empty_buffers(lib):
    """Empty buffers may be NULL (a batch without tokens): the calls then get
    past the argument checks (here, with no GPU, to MF_ERR_CUDA); the same
    NULL with tokens present is MF_ERR_INVALID_ARG."""
    P = C.c_void_p
    empty, _h0 = _desc(cu=(0, 0, 0))
    full, _h1 = _desc(cu=(0, 100))
    ws = P(256)
    need = lib.mf_block_stats_workspace(C.byref(empty))
    assert lib.mf_block_stats(C.byref(empty), None, None, None, None, ws, need, None) == \
        mfb.MF_ERR_CUDA
    assert lib.mf_block_stats(C.byref(full), None, None, None, None, ws, 1 << 20, None) == \
        mfb.MF_ERR_INVALID_ARG
    # no query blocks: only row_ptr must exist
    cache0 = mfb.CsrCache(0, 0, 16, None, None, None, None, 4, 64, mfb.MF_F32, 2, 0x1000)
    need = lib.mf_select_extract_workspace(C.byref(empty))
    assert lib.mf_select_extract(C.byref(empty), None, None, None, None, 0.9,
                                 C.byref(cache0), ws, need, None) == mfb.MF_ERR_CUDA
    cache1 = mfb.CsrCache(2, 0, 16, None, None, None, None, 4, 64, mfb.MF_F32, 1, 0x1000)
    assert lib.mf_select_extract(C.byref(full), P(16), P(16), P(16), P(16), 0.9,
                                 C.byref(cache1), ws, 1 << 20, None) == mfb.MF_ERR_INVALID_ARG
    v0 = mfb.VDesc(None, None, 16, 0, 0, 2, 64)
    assert lib.mf_mapped_av(C.byref(cache0), C.byref(empty), 4, P(16), C.byref(v0), None,
                            ws, 1 << 20, None) == mfb.MF_ERR_CUDA
    assert lib.mf_mapped_av(C.byref(cache0), C.byref(empty), 4, None, C.byref(v0), None,
                            ws, 1 << 20, None) == mfb.MF_ERR_INVALID_ARG  # W is never empty


def test_argument_errors_return_before_any_launch(lib):
    dsc, host = _desc()
    P = C.c_void_p
    # NULL descriptor
    assert lib.mf_block_stats(None, P(16), P(16), P(16), P(16), P(256), 1 << 20, None) == \
        mfb.MF_ERR_INVALID_ARG
    # unsupported head dim / Hs
    for bad in (dict(d=96), dict(Hs=65), dict(B=32)):
        b, h = _desc(**bad)
        st = lib.mf_block_stats(C.byref(b), P(16), P(16), P(16), P(16), P(256), 1 << 20, None)
        assert st == mfb.MF_ERR_UNSUPPORTED, bad
        assert lib.mf_last_error().decode()
    # NULL inputs
    assert lib.mf_block_stats(C.byref(dsc), None, P(16), P(16), P(16), P(256), 1 << 20,
                              None) == mfb.MF_ERR_INVALID_ARG
    # workspace too small or misaligned
    need = lib.mf_block_stats_workspace(C.byref(dsc))
    assert need > 0
    assert lib.mf_block_stats(C.byref(dsc), P(16), P(16), P(16), P(16), P(256), need - 1,
                              None) == mfb.MF_ERR_WORKSPACE
    assert lib.mf_block_stats(C.byref(dsc), P(16), P(16), P(16), P(16), P(257), need,
                              None) == mfb.MF_ERR_WORKSPACE
    # select: tau must be positive; cache must match the descriptor
    cache = mfb.CsrCache(8, 36, 16, 16, 16, 16, 16, 4, 64, mfb.MF_F32, 1, 0x1000)
    ws = lib.mf_select_extract_workspace(C.byref(dsc))
    assert lib.mf_select_extract(C.byref(dsc), P(16), P(16), P(16), P(16), 0.0,
                                 C.byref(cache), P(256), ws, None) == mfb.MF_ERR_INVALID_ARG
    bad = mfb.CsrCache(8, 36, 16, 16, 16, 16, 16, 5, 64, mfb.MF_F32, 1, 0x1000)
    assert lib.mf_select_extract(C.byref(dsc), P(16), P(16), P(16), P(16), 0.9,
                                 C.byref(bad), P(256), ws, None) == mfb.MF_ERR_INVALID_ARG
    wrong_rows = mfb.CsrCache(9, 36, 16, 16, 16, 16, 16, 4, 64, mfb.MF_F32, 1, 0x1000)
    assert lib.mf_select_extract(C.byref(dsc), P(16), P(16), P(16), P(16), 0.9,
                                 C.byref(wrong_rows), P(256), ws, None) == mfb.MF_ERR_INVALID_ARG
    # mapped AV: Hr must be a multiple of Hkv; page size rule
    v = mfb.VDesc(16, None, 16, 0, 0, 3, 64)
    assert lib.mf_mapped_av(C.byref(cache), C.byref(dsc), 4, P(16), C.byref(v), P(16),
                            P(256), 1 << 20, None) == mfb.MF_ERR_INVALID_ARG
    assert lib.mf_mapped_av_workspace(C.byref(cache), C.byref(dsc), 4, C.byref(v)) == 0
    v = mfb.VDesc(16, 16, 8, 64, 10, 2, 64)
    assert lib.mf_mapped_av(C.byref(cache), C.byref(dsc), 4, P(16), C.byref(v), P(16),
                            P(256), 1 << 20, None) == mfb.MF_ERR_INVALID_ARG
    # bf16, d = 128 runs on the tensor-core kernel, which needs a workspace
    dsc2, host2 = _desc(Hs=40, d=128, B=128, cu=(0, 1000), dt=mfb.MF_BF16)
    cache2 = mfb.CsrCache(8, 36, 16, 16, 16, 16, 16, 40, 128, mfb.MF_BF16, 1, 0x1000)
    v2 = mfb.VDesc(16, None, 16, 0, 0, 8, 128)
    need = lib.mf_mapped_av_workspace(C.byref(cache2), C.byref(dsc2), 32, C.byref(v2))
    assert need >= 63 * 4096 * 8  # V regrouped per 16 keys: ceil(1000/16) images
    assert lib.mf_mapped_av(C.byref(cache2), C.byref(dsc2), 32, P(16), C.byref(v2), P(16),
                            P(256), need - 1, None) == mfb.MF_ERR_WORKSPACE


def test_cache_layout_helpers_match_the_header_formula():
    """tests/parity.py's stored <-> logical transforms follow the C header."""
    from tests import parity as par
    for Hs, B in ((8, 64), (40, 128)):
        y = np.arange(Hs * B * B, dtype=np.float64).reshape(Hs, B, B)
        st = par.logical_to_stored(y, Hs, B)
        np.testing.assert_array_equal(par.stored_to_logical(st, Hs, B), y)
        flat = st.reshape(-1)
        rng = np.random.default_rng(0)
        for _ in range(300):
            h, i, j = int(rng.integers(Hs)), int(rng.integers(B)), int(rng.integers(B))
            line = (((j // 16) * (B // 8) + i // 8) * 2 + (i % 8) // 4) * Hs + h
            m = (i % 4) * 16 + j % 16
            off = line * 64 + ((m // 8) ^ (h % 8)) * 8 + m % 8
            assert flat[off] == y[h, i, j]


# ----------------------------------------------------------- prefix hashing

def test_prefix_hash_chains_over_the_prefix(lib):
    rng = np.random.default_rng(2)
    toks = rng.integers(0, 150000, size=1000).astype(np.int32)
    h = mfb.prefix_hash(toks, 64)
    assert h.shape == (16, 2)
    assert len({tuple(x) for x in h}) == 16
    np.testing.assert_array_equal(h, mfb.prefix_hash(toks, 64))
    # a prefix hashes to the same leading blocks
    np.testing.assert_array_equal(mfb.prefix_hash(toks[:640], 64), h[:10])
    # changing token 300 changes block 4 and every later block, not earlier ones
    t2 = toks.copy()
    t2[300] += 1
    h2 = mfb.prefix_hash(t2, 64)
    np.testing.assert_array_equal(h2[:4], h[:4])
    assert np.all(h2[4:, 0] != h[4:, 0]) and np.all(h2[4:, 1] != h[4:, 1])
    # the seed changes everything; swapping two tokens in a block changes it
    assert np.all(mfb.prefix_hash(toks, 64, seed=1) != h)
    t3 = toks.copy()
    t3[[5, 6]] = t3[[6, 5]]
    assert np.all(mfb.prefix_hash(t3, 64)[:, 0] != h[:, 0])


def test_index_longest_prefix_and_misses(lib):
    rng = np.random.default_rng(3)
    ctx = rng.integers(0, 1000, size=640).astype(np.int32)
    h = mfb.prefix_hash(ctx, 64)
    ix = mfb.PrefixIndex()
    c0 = mfb.CsrCache(10, 55, 0x10, 0x20, 0x30, 0x40, 0x50, 4, 64, mfb.MF_BF16, 1, 0x60)
    ix.insert(h, sender_layer=3, seq=0, cache_struct=c0)
    assert len(ix) == 10
    # a receiver context sharing 6 blocks and then diverging
    q = np.concatenate([ctx[:400], rng.integers(1000, 2000, size=300).astype(np.int32)])
    got = ix.lookup(mfb.prefix_hash(q, 64), 3)
    assert got is not None
    cache, seq, matched = got
    assert matched == 6 and seq == 0 and cache.values == 0x50 and cache.row_ptr == 0x10
    # the full context matches every block; other layer or other text misses
    assert ix.lookup(h, 3)[2] == 10
    assert ix.lookup(h, 4) is None
    assert ix.lookup(mfb.prefix_hash(ctx[::-1].copy(), 64), 3) is None
    assert ix.lookup(h[:0], 3) is None


def test_index_same_key_newest_wins(lib):
    """Two states under one key (a forced collision): the newer one is kept."""
    h = mfb.prefix_hash(np.arange(256, dtype=np.int32), 64)
    ix = mfb.PrefixIndex()
    a = mfb.CsrCache(4, 10, 1, 2, 3, 4, 5, 4, 64, mfb.MF_BF16, 1, 6)
    b = mfb.CsrCache(4, 10, 11, 12, 13, 14, 15, 4, 64, mfb.MF_BF16, 2, 16)
    ix.insert(h, 0, 0, a)
    ix.insert(h, 0, 1, b)
    cache, seq, matched = ix.lookup(h, 0)
    assert (cache.values, seq, matched) == (15, 1, 4)
    assert len(ix) == 4


def test_selftest_timeout_rejects_bad_limits(lib):
    assert lib.mf_selftest_timeout(0, None) == mfb.MF_ERR_INVALID_ARG
    assert lib.mf_selftest_timeout(5000, None) == mfb.MF_ERR_INVALID_ARG


def test_mapped_av_range_rejects_bad_ranges(lib):
    dsc, host = _desc()
    P = C.c_void_p
    cache = mfb.CsrCache(8, 36, 16, 16, 16, 16, 16, 4, 64, mfb.MF_F32, 1, 0x1000)
    v = mfb.VDesc(16, None, 16, 0, 0, 2, 64)
    for lo, hi in ((-1, 3), (0, 9), (5, 3)):
        st = lib.mf_mapped_av_range(C.byref(cache), C.byref(dsc), 4, P(16), C.byref(v), P(16),
                                    lo, hi, P(256), 1 << 20, None)
        assert st == mfb.MF_ERR_INVALID_ARG, (lo, hi)


def test_fused_kernel_plan_fits_every_supported_shape(lib):
    """The tensor-core fused kernel's shared-memory plan, for every shape it
    accepts: within the 227 KB a CTA may use, operand rings on 1 KB
    boundaries (128-byte-swizzled operands), at least double-buffered."""
    seen_kg = set()
    for Hs in range(8, 65, 8):
        for Hr in (16, 32):
            for G in (2, 4, 8):
                Hkv = Hr // G
                pl = mfb.mapped_av_plan(Hs, Hr, Hkv)
                kg = pl["groups_per_stage"]
                seen_kg.add(kg)
                assert kg in (1, 2)
                assert pl["smem_bytes"] <= 227 * 1024, (Hs, Hr, Hkv, pl)
                assert pl["map_stages"] >= 2 and pl["v_stages"] >= 2
                # V ring first, then map ring, mixed-map ring, W^T, barriers
                assert pl["off_map"] == pl["v_stages"] * kg * 4096 * Hkv
                assert pl["off_map"] % 1024 == 0
                assert pl["off_map"] + pl["map_stages"] * kg * Hs * 256 <= pl["off_mt"]
                assert pl["off_mt"] % 16 == 0 and pl["off_mt"] < pl["off_w"] < pl["off_bar"]
                assert pl["off_bar"] % 8 == 0
    assert seen_kg == {1, 2}
    # 32-key stages where they fit, 16-key stages for big V images or big maps
    assert mfb.mapped_av_plan(40, 32, 8)["groups_per_stage"] == 2
    assert mfb.mapped_av_plan(40, 32, 16)["groups_per_stage"] == 1
    assert mfb.mapped_av_plan(64, 32, 8)["groups_per_stage"] == 1
    with pytest.raises(mfb.MapflowError) as e:
        mfb.mapped_av_plan(40, 24, 8)
    assert e.value.status == mfb.MF_ERR_UNSUPPORTED


def test_every_bf16_workload_runs_the_tensor_core_kernels(lib):
    """mf_path_info on the workloads' shapes: all three stages of every bf16
    workload run on the tensor cores; the float32 one runs the scalar
    kernels; a sequence past 256 key blocks drops the statistics to the
    scalar two-pass kernel."""
    from cross_model_attention_block_b200 import synth
    for name, w in synth.workloads().items():
        ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width,
                               w.torch_dtype, device="cpu")
        got = mfb.path_info(ctx, w.Hr, w.Hkv)
        want = w.dtype == "bf16"
        assert got == {"stats_tc": want, "extract_tc": want, "mapped_av_tc": want}, name
    long = mfb.Context.make([257 * 64], 32, 128, 64, 2.0, 256, torch.bfloat16, device="cpu")
    assert mfb.path_info(long, 32, 8) == {"stats_tc": False, "extract_tc": True,
                                          "mapped_av_tc": True}
    odd = mfb.Context.make([1000], 12, 128, 64, 2.0, 256, torch.bfloat16, device="cpu")
    assert mfb.path_info(odd, 32, 8)["mapped_av_tc"] is False      # Hs not a multiple of 8
    assert mfb.path_info(odd, 24, 8)["mapped_av_tc"] is False      # Hr not 16 or 32
    with pytest.raises(mfb.MapflowError):
        mfb.path_info(odd, 30, 8)                                  # Hr not a multiple of Hkv


def test_range_forms_reject_bad_ranges_before_any_launch(lib):
    """The statistics and selection range forms check the range on the host."""
    import ctypes as C
    ctx = mfb.Context.make([300, 200], 8, 128, 64, 2.0, 256, torch.bfloat16, device="cpu")
    d = ctx.desc()
    nqb, _ = ctx.layout_sizes()
    for lo, hi in ((-1, 2), (3, 2), (0, nqb + 1)):
        st = lib.mf_block_stats_range(C.byref(d), 16, 16, 16, 16, lo, hi, 256, 1 << 20, None)
        assert st == mfb.MF_ERR_INVALID_ARG
        assert "range" in lib.mf_last_error().decode()
        cs = mfb.CsrCache(nqb, 10, 16, 16, 16, 16, 16, 8, 64, mfb.MF_BF16, 2, 16)
        st = lib.mf_select_extract_range(C.byref(d), 16, 16, 16, 16, 0.9, C.byref(cs), lo, hi,
                                         256, 1 << 20, None)
        assert st == mfb.MF_ERR_INVALID_ARG
        assert "range" in lib.mf_last_error().decode()


@pytest.mark.parametrize("starts,msg", [
    ([64, 128, 500], "from 0"),
    ([0, 128, 128, 500], "increase"),
    ([0, 100, 500], "block boundary"),
    ([0, 128, 320, 500], "crosses"),
    ([0, 128, 500], "crosses"),
], ids=["not_from_zero", "not_increasing", "unaligned", "crosses_seq_end", "seq_without_round"])
def test_round_layout_rejected_before_any_launch(lib, starts, msg):
    """Rounds must run from 0 to ntok, start every sequence, start on block
    boundaries of their sequence and end inside it (two sequences, 300 + 200
    tokens, B = 64)."""
    ctx = mfb.Context.make([300, 200], 8, 128, 64, 2.0, 256, torch.bfloat16, device="cpu")
    mass = torch.zeros(ctx.layout_sizes()[1])
    with pytest.raises(mfb.MapflowError) as e:
        mfb.select_rounds(ctx, mass, starts, 0.9, cache=mfb.Cache(ctx, device="cpu"))
    assert e.value.status == mfb.MF_ERR_INVALID_ARG
    assert msg in str(e.value)


def test_cache_tier_checks_layouts_and_ranges(lib):
    """mf_cache_fetch / mf_cache_offload reject mismatched layouts and bad
    ranges before any copy."""
    ctx = mfb.Context.make([300], 8, 128, 64, 2.0, 256, torch.bfloat16, device="cpu")
    a = mfb.Cache(ctx, device="cpu")
    ctx2 = mfb.Context.make([300], 4, 128, 64, 2.0, 256, torch.bfloat16, device="cpu")
    b = mfb.Cache(ctx2, device="cpu")
    with pytest.raises(mfb.MapflowError) as e:
        mfb.cache_fetch(a, b, (0, 1))
    assert e.value.status == mfb.MF_ERR_INVALID_ARG and "differ" in str(e.value)
    with pytest.raises(mfb.MapflowError) as e:
        mfb.cache_offload(a, b)
    assert e.value.status == mfb.MF_ERR_INVALID_ARG
    with pytest.raises(mfb.MapflowError) as e:
        mfb.cache_fetch(a, mfb.Cache(ctx, device="cpu"), (2, 99))
    assert "range" in str(e.value)
    # arrays may be NULL only where they are empty
    rp = np.zeros(1, np.int64)
    none = mfb.CsrCache(0, 0, rp.ctypes.data, None, None, None, None, 8, 64, mfb.MF_BF16, 1,
                        0x1000)
    assert lib.mf_cache_fetch(C.byref(none), C.byref(none), 0, 0, None) == mfb.MF_OK
    holes = mfb.CsrCache(0, 4, rp.ctypes.data, None, None, None, None, 8, 64, mfb.MF_BF16, 1,
                         0x1000)
    assert lib.mf_cache_fetch(C.byref(holes), C.byref(holes), 0, 0, None) == \
        mfb.MF_ERR_INVALID_ARG


def test_overlap_chunk_ranges_cover_the_rows():
    from cross_model_attention_block_b200 import overlap as ov
    for nqb in (0, 1, 5, 128, 256):
        for chunks in (1, 3, 8, 300):
            r = ov.chunk_ranges(nqb, chunks)
            covered = [g for a, b in r for g in range(a, b)]
            assert covered == list(range(nqb))
            assert all(a < b for a, b in r)
