"""The partitioned path on one GPU: the ranges every rank would run, executed
one after another through the C ABI range entry points, give the result of
one call bit for bit (statistics, kept sets and probability blocks, O).
Each query block's work depends only on its own rows and the keys before
them, so a rank needs no data from another rank's ranges."""
import numpy as np
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb
from cross_model_attention_block_b200 import partition as part
from cross_model_attention_block_b200 import synth
from tests import parity as par

pytestmark = pytest.mark.gpu


def _run_ranks(ctx, Q, K, V, W, Hr, Hkv, tau, rank_ranges):
    nqb, nblocks = ctx.layout_sizes()
    lse = torch.full((ctx.Hs, ctx.ntok), float("nan"), device="cuda")
    mass = torch.full((max(nblocks, 1),), float("nan"), device="cuda")
    O = torch.full((ctx.ntok, Hr, ctx.d), 7.0, dtype=ctx.dtype, device="cuda")
    caches = []
    for ranges in rank_ranges:
        for a, b in ranges:
            mfb.block_stats(ctx, Q, K, lse=lse, mass=mass, qb_range=(a, b))
            c = mfb.Cache(ctx, capacity=ctx.range_blocks(a, b))
            mfb.select_extract(ctx, Q, K, lse, mass, tau, cache=c, qb_range=(a, b))
            mfb.mapped_av(c, Hr, W, V, Hkv, O=O, qb_range=(a, b))
            caches.append((a, b, c))
    mfb.sync_status()
    return lse, mass, O, caches


def _check_equal(full, got, nqb):
    lse_f, mass_f, cache_f, O_f = full
    lse, mass, O, caches = got
    assert torch.equal(lse, lse_f)
    assert torch.equal(mass, mass_f)
    assert torch.equal(O, O_f)
    rp_f, ci_f = par.kept_sets(cache_f)
    vals_f = cache_f.values_view()
    covered = []
    for a, b, c in caches:
        rp, ci = par.kept_sets(c)
        vv = c.values_view()
        assert rp[a] == 0 and rp[b] == rp[-1] == c.nnz       # rows outside are empty
        for g in range(a, b):
            assert list(ci[rp[g]:rp[g + 1]]) == list(ci_f[rp_f[g]:rp_f[g + 1]])
        n = c.nnz
        assert torch.equal(vv[:n], vals_f[rp_f[a]:rp_f[a] + n])
        covered += list(range(a, b))
    assert sorted(covered) == list(range(nqb))


@pytest.mark.parametrize("case,world", [
    (dict(lengths=[1000], Hs=16, Hr=16, Hkv=8, d=128, B=64, tau=0.9), 3),
    (dict(lengths=[1000, 333, 700], Hs=40, Hr=32, Hkv=8, d=128, B=64, tau=0.95), 4),
    (dict(lengths=[1100], Hs=8, Hr=32, Hkv=8, d=128, B=128, tau=0.9), 2),
    (dict(lengths=[500, 260], Hs=4, Hr=2, Hkv=2, d=64, B=64, tau=0.9, dtype="f32"), 3),
], ids=["bf16_b64_w3", "bf16_varlen_w4", "bf16_b128_w2", "f32_w3"])
def test_rank_ranges_in_sequence_equal_one_call(case, world):
    w, x = synth.small_case(**case)
    ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width, w.torch_dtype)
    Q, K, V, W = x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda()
    full = par.run_gpu(ctx, Q, K, V, W, w.Hkv, w.tau)
    nqb, _ = ctx.layout_sizes()
    rr = [part.zigzag_ranges(nqb, world, r) for r in range(world)]
    _check_equal(full, _run_ranks(ctx, Q, K, V, W, w.Hr, w.Hkv, w.tau, rr), nqb)


def test_zigzag_ranks_on_the_32k_workload_equal_one_call():
    """The launch configuration of `bench.py --gpus 8`, one rank after another."""
    w = synth.workloads()["large_bf16_n32768"]
    x = synth.single_layer(w)
    ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width, w.torch_dtype)
    Q, K, V, W = x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda()
    full = par.run_gpu(ctx, Q, K, V, W, w.Hkv, w.tau)
    nqb, _ = ctx.layout_sizes()
    rr = [part.zigzag_ranges(nqb, 8, r) for r in range(8)]
    got = _run_ranks(ctx, Q, K, V, W, w.Hr, w.Hkv, w.tau, rr)
    _check_equal(full, got, nqb)
    # and sampled query blocks of the rank-assembled output against the oracle
    par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau,
                             (got[0], got[1], full[2], got[2]), [(0, 15), (0, 240)],
                             torch.bfloat16, check_values=False, label="zigzag ranks 32K")
