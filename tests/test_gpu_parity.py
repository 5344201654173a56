"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small cases are compared on every query block (several tiles, ragged tails,
empty sequences); the full-size workloads are compared on sampled query
blocks that the oracle computes one by one, in the same launch configuration
the benchmark uses.
"""
import numpy as np
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb
from cross_model_attention_block_b200 import synth
from tests import parity as par

pytestmark = pytest.mark.gpu


def _ctx_of(w, dtype=None):
    dt = dtype or w.torch_dtype
    return mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width, dt)


def _small(lengths, Hs, Hr, Hkv, d, B, tau, dtype="bf16", band_bias=2.0, band_width=256,
           seed=0):
    w, x = synth.small_case(lengths, Hs, Hr, Hkv, d, B, tau, dtype=dtype, band_bias=band_bias,
                            band_width=band_width, seed=seed)
    ctx = _ctx_of(w)
    gpu = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(), Hkv, tau)
    return w, x, ctx, gpu


@pytest.mark.parametrize("case", [
    dict(lengths=[300, 1000, 64, 129, 1], Hs=8, Hr=8, Hkv=2, d=128, B=64, tau=0.9),
    dict(lengths=[1000, 130], Hs=40, Hr=32, Hkv=8, d=128, B=128, tau=0.95),
    dict(lengths=[700], Hs=32, Hr=32, Hkv=8, d=128, B=64, tau=0.95),
    dict(lengths=[333, 65], Hs=4, Hr=4, Hkv=4, d=64, B=64, tau=0.9),
    dict(lengths=[200, 77], Hs=3, Hr=6, Hkv=3, d=128, B=128, tau=0.9, dtype="f32"),
    dict(lengths=[100, 0, 70], Hs=5, Hr=4, Hkv=2, d=64, B=64, tau=0.8, dtype="f32"),
    # 12 sender heads: tensor-core statistics and extraction with a partial
    # last head group (8 + 4); the fused step runs the scalar kernel
    dict(lengths=[700, 257], Hs=12, Hr=8, Hkv=4, d=128, B=128, tau=0.95),
    dict(lengths=[450, 1], Hs=12, Hr=8, Hkv=4, d=128, B=64, tau=0.9),
    # empty sequences between non-empty ones, all three stages on the tensor cores
    dict(lengths=[0, 300, 0, 129], Hs=8, Hr=16, Hkv=4, d=128, B=64, tau=0.9),
], ids=["bf16_b64_varlen", "bf16_b128_hs40", "bf16_b64_hs32", "bf16_d64",
        "f32_d128_b128", "f32_empty_seq", "bf16_b128_hs12", "bf16_b64_hs12",
        "bf16_empty_seqs_tc"])
def test_small_cases_every_block(case):
    w, x, ctx, gpu = _small(**case)
    dt = w.torch_dtype
    n, ex, worst = par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu,
                                            par.all_picks(ctx), dt, label="small cases")
    assert ex <= max(1, n // 50)


def test_batch_without_tokens():
    """Every sequence empty: the three calls launch nothing, report no error
    and return an empty cache and an empty O."""
    w, x = synth.small_case([0, 0], 8, 16, 4, 128, 64, 0.9)
    ctx = _ctx_of(w)
    lse, mass, cache, O = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(),
                                      w.Hkv, w.tau)
    mfb.sync_status()
    assert cache.nnz == 0 and O.shape[0] == 0 and lse.numel() == 0


def test_tiny_f32_workload_every_block():
    w = synth.workloads()["tiny_f32_n512"]
    x = synth.single_layer(w)
    ctx = _ctx_of(w)
    gpu = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(), w.Hkv, w.tau)
    n, ex, worst = par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu,
                                            par.all_picks(ctx), torch.float32, label=w.name)
    assert n == 8 and ex == 0 and worst <= 1e-4


def test_tau_one_keeps_every_causal_block():
    w, x, ctx, gpu = _small([260, 64], 4, 4, 2, 128, 64, 1.0)
    cache = gpu[2]
    nqb, nblocks = ctx.layout_sizes()
    assert cache.nnz == nblocks
    rp, ci = par.kept_sets(cache)
    g = 0
    for L in (260, 64):
        for qb in range((L + 63) // 64):
            assert list(ci[rp[g]:rp[g + 1]]) == list(range(qb + 1))
            g += 1


def test_capacity_overflow_is_reported():
    w, x = synth.small_case([400], 4, 4, 2, 128, 64, 0.99)
    ctx = _ctx_of(w)
    Q, K = x.Q.cuda(), x.K.cuda()
    lse, mass = mfb.block_stats(ctx, Q, K)
    cache = mfb.Cache(ctx, capacity=5)
    mfb.select_extract(ctx, Q, K, lse, mass, 0.99, cache=cache)
    mfb.mapped_av(cache, 4, x.W.cuda(), x.V.cuda(), 2)
    with pytest.raises(mfb.MapflowError) as e:
        mfb.sync_status()
    assert e.value.status == mfb.MF_ERR_CAPACITY
    mfb.sync_status()  # the status word was cleared by the read


def test_mid_workload_every_block():
    w = synth.workloads()["mid_bf16_n8192"]
    x = synth.single_layer(w)
    ctx = _ctx_of(w)
    gpu = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(), w.Hkv, w.tau)
    picks = par.all_picks(ctx)
    n, ex, worst = par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu,
                                            picks, torch.bfloat16, check_values=False,
                                            label=w.name)
    assert n == 128 and ex <= 2
    # extracted values on a subset
    par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu,
                             [(0, 0), (0, 1), (0, 63), (0, 127)], torch.bfloat16)


def test_large_workload_sampled():
    w = synth.workloads()["large_bf16_n32768"]
    x = synth.single_layer(w)
    ctx = _ctx_of(w)
    gpu = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(), w.Hkv, w.tau)
    picks = [(0, 0), (0, 1), (0, 2), (0, 77), (0, 128), (0, 254), (0, 255)]
    n, ex, worst = par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu,
                                            picks, torch.bfloat16, label=w.name)
    assert ex <= 1
    # properties that hold at any size: every row keeps its diagonal block, the
    # row pointers are consistent, every output is finite
    cache, O = gpu[2], gpu[3]
    rp, ci = par.kept_sets(cache)
    nqb = 256
    assert rp[0] == 0 and np.all(np.diff(rp) >= 1) and rp[-1] == cache.nnz
    for g in range(nqb):
        row = ci[rp[g]:rp[g + 1]]
        assert row[-1] == g and np.all(np.diff(row) > 0)
    assert torch.isfinite(O.float()).all()


def test_long_b64_sequence_past_256_key_blocks():
    """One 16,500-token sequence at B = 64 (258 key blocks): the statistics
    take the scalar two-pass kernel (the tensor-core one keeps per-block
    partials for at most 256 key blocks in TMEM) while extraction and the
    fused kernel stay on the tensor cores, with block-map entries past 256.
    Sampled query blocks, the last ones included, against the oracle."""
    w, x = synth.small_case([16500], 8, 16, 4, 128, 64, 0.95)
    ctx = _ctx_of(w)
    assert mfb.path_info(ctx, w.Hr, w.Hkv) == {"stats_tc": False, "extract_tc": True,
                                                "mapped_av_tc": True}
    gpu = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(), w.Hkv, w.tau)
    picks = [(0, 0), (0, 1), (0, 128), (0, 255), (0, 256), (0, 257)]
    n, ex, worst = par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu,
                                            picks, torch.bfloat16, label="long B = 64")
    assert n == len(picks) and ex <= 1
    assert torch.isfinite(gpu[3].float()).all()


def test_multi_receiver_workload_as_specified():
    """One sender state of 8 layers, each compressed once, serves receiver r1
    (6 layers) and receiver r2 (4 layers) through the layer table; every
    receiver layer is compared with the oracle on sampled query blocks, and
    the extracted values are compared on the first layer."""
    w = synth.workloads()["multi_receiver_n16384"]
    ctx = _ctx_of(w)
    assert w.sender_layers == 8 and [r[1] for r in w.receivers] == [6, 4]
    sender = {}
    for sl in range(w.sender_layers):
        Q, K = synth.sender_layer(w, sl)
        Qd, Kd = Q.cuda(), K.cuda()
        lse, mass = mfb.block_stats(ctx, Qd, Kd)
        cache = mfb.select_extract(ctx, Qd, Kd, lse, mass, w.tau)
        mfb.sync_status()
        sender[sl] = (Q, K, lse, mass, cache)
        del Qd, Kd
    served = set()
    nqb = (w.lengths[0] + w.B - 1) // w.B
    for rec, (name, nl, table) in enumerate(w.receivers):
        for layer in range(nl):
            sl = table[layer]
            served.add(sl)
            V, W = synth.receiver_layer(w, rec, layer)
            Q, K, lse, mass, cache = sender[sl]
            O = mfb.mapped_av(cache, w.Hr, W.cuda(), V.cuda(), w.Hkv)
            mfb.sync_status()
            picks = [(0, 0), (0, 1 + (37 * (rec * 6 + layer)) % (nqb - 2)), (0, nqb - 1)]
            par.compare_query_blocks(ctx, Q, K, V, W, w.Hkv, w.tau, (lse, mass, cache, O),
                                     picks, torch.bfloat16,
                                     check_values=(rec == 0 and layer == 0),
                                     label=f"{w.name} {name}")
    assert served == {0, 1, 2, 4, 5, 6}
    # sender layers no receiver reads (3, 7) were compressed all the same:
    # check their statistics and selection through one receiver layer's V and W
    V, W = synth.receiver_layer(w, 0, 0)
    for sl in sorted(set(range(w.sender_layers)) - served):
        Q, K, lse, mass, cache = sender[sl]
        O = mfb.mapped_av(cache, w.Hr, W.cuda(), V.cuda(), w.Hkv)
        mfb.sync_status()
        par.compare_query_blocks(ctx, Q, K, V, W, w.Hkv, w.tau, (lse, mass, cache, O),
                                 [(0, 3), (0, nqb - 1)], torch.bfloat16, check_values=False,
                                 label=f"{w.name} unread sender layers")


def test_varlen_paged_workload_sampled():
    w = synth.workloads()["varlen_paged_64seq"]
    x = synth.single_layer(w)
    pool, table = synth.paged_v(x.V, w.lengths, synth.page_rng(w))
    ctx = _ctx_of(w)
    Q, K = x.Q.cuda(), x.K.cuda()
    gpu = par.run_gpu(ctx, Q, K, None, x.W.cuda(), w.Hkv, w.tau, page_table=table.cuda(),
                      Vpool=pool.cuda())
    lens = np.array(w.lengths)
    longest, shortest = int(np.argmax(lens)), int(np.argmin(lens))
    picks = [(0, 0), (shortest, (lens[shortest] - 1) // 64), (longest, (lens[longest] - 1) // 64),
             (longest, 100), (17, 5), (63, (lens[63] - 1) // 64)]
    par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, gpu, picks,
                             torch.bfloat16, label=w.name)
    # paged V gives exactly the contiguous result
    O_c = mfb.mapped_av(gpu[2], w.Hr, x.W.cuda(), x.V.cuda(), w.Hkv)
    mfb.sync_status()
    assert torch.equal(O_c, gpu[3])


@pytest.mark.parametrize("case", [
    dict(lengths=[300, 200], Hs=40, Hr=32, Hkv=8, B=64, tau=0.9),
    dict(lengths=[390], Hs=40, Hr=32, Hkv=8, B=128, tau=0.9),
    dict(lengths=[257, 31], Hs=32, Hr=16, Hkv=4, B=64, tau=0.8),
    dict(lengths=[160], Hs=16, Hr=16, Hkv=8, B=128, tau=0.95),
    # 16-key stages: V images of 16 KV heads, or 64 sender heads, leave no
    # room for two 32-key stages in shared memory
    dict(lengths=[270], Hs=40, Hr=32, Hkv=16, B=64, tau=0.9),
    dict(lengths=[200, 77], Hs=64, Hr=32, Hkv=8, B=128, tau=0.9),
], ids=["hs40_b64", "hs40_b128", "hs32_g4_b64", "hs16_g2_b128", "hs40_kv16_b64_16key",
        "hs64_b128_16key"])
def test_mapped_av_on_an_oracle_built_cache(case):
    """The fused kernel alone: cache (CSR + probability blocks) written from the
    oracle, O compared with the oracle's."""
    from oracle import mapflow_oracle as orc
    w, x = synth.small_case(case["lengths"], case["Hs"], case["Hr"], case["Hkv"], 128,
                            case["B"], case["tau"])
    res, O_ref = orc.run_layer(x.Q, x.K, x.V, x.W, w.lengths, w.Hkv, w.B, w.tau,
                               w.band_bias, w.band_width, want_values=True)
    ctx = _ctx_of(w)
    cache = mfb.Cache(ctx)
    rows, cols, vals = [0], [], []
    g = 0
    for s, r in enumerate(res):
        for qb in sorted(r):
            rec = r[qb]
            for kb in rec["kept"]:
                cols.append(int(kb))
                blk = np.zeros((w.Hs, w.B, w.B))
                v = rec["values"][int(kb)]
                blk[:, : v.shape[1], :] = v
                vals.append(blk)
            rows.append(rows[-1] + len(rec["kept"]))
            cache.qb_seq[g] = s
            cache.qb_idx[g] = qb
            g += 1
    cache.row_ptr.copy_(torch.tensor(rows, dtype=torch.int64))
    cache.col_idx[: len(cols)].copy_(torch.tensor(cols, dtype=torch.int32))
    vv = cache.values_view()
    stored = np.stack([par.logical_to_stored(v, w.Hs, w.B) for v in vals])
    vv[: len(vals)].copy_(torch.from_numpy(stored).to(torch.bfloat16))
    O = mfb.mapped_av(cache, w.Hr, x.W.cuda(), x.V.cuda(), w.Hkv)
    mfb.sync_status()
    O = O.double().cpu().numpy()
    err = np.abs(O - O_ref).max() / np.abs(O_ref).max()
    assert err <= 2e-2, err
