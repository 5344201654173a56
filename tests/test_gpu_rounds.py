"""Round-level selection (the Round Attention page, "方法详解": a watershed
layer's attention keeps, per conversation round, the earlier rounds that
matter) through the C ABI, against the CPU oracle: kept rounds and blocks of
every query block, the extracted blocks of every later layer, and its O."""
import numpy as np
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb
from cross_model_attention_block_b200 import synth
from oracle import mapflow_oracle as orc
from tests import parity as par

pytestmark = pytest.mark.gpu

NEAR_TAU = 1e-4


def check_rounds(m, gpu_rounds, tau):
    """'' if the kept rounds equal the oracle's, 'near_tau' if the oracle's
    cumulative fraction at the cut lies within 1e-4 of tau; raises otherwise."""
    want = orc.select_rounds(m, tau)
    if list(want) == list(gpu_rounds):
        return ""
    q = len(m) - 1
    order = sorted(range(q), key=lambda r: (-m[r], r))
    fr = np.cumsum([m[q]] + [m[r] for r in order]) / m.sum()
    k = len(want) - 1
    near = [abs(fr[k] - tau)] + ([abs(fr[k - 1] - tau)] if k >= 1 else [])
    if min(near) < NEAR_TAU:
        return "near_tau"
    raise AssertionError(f"kept rounds differ: oracle {list(want)} gpu {list(gpu_rounds)}")


def run_case(lengths, rounds, Hs, Hr, Hkv, B, tau, nlayers, watershed, dtype="bf16", seed=0,
             picks_o=None, label="rounds"):
    """rounds: per sequence, round starts within it (then its length)."""
    d = 128 if dtype == "bf16" else 64
    ctx = mfb.Context.make(lengths, Hs, d, B, 2.0, 256, torch.float32 if dtype == "f32"
                           else torch.bfloat16)
    layers = []
    for l in range(nlayers):
        rng = np.random.default_rng(seed + 100 * l)
        Q, K = synth.sender_qk(lengths, Hs, d, dtype, rng)
        V, W = synth.receiver_vw(sum(lengths), Hr, Hkv, Hs, d, dtype, rng)
        layers.append((Q, K, V, W))
    cu = synth.cu_seqlens(lengths)
    starts = [int(cu[s]) + r for s, st in enumerate(rounds) for r in st[:-1]] + [int(cu[-1])]
    Qw, Kw = layers[watershed][0].cuda(), layers[watershed][1].cuda()
    _, mass = mfb.block_stats(ctx, Qw, Kw)
    cache = mfb.select_rounds(ctx, mass, starts, tau)
    mfb.sync_status()
    rp, ci = par.kept_sets(cache)
    nq = [(L + B - 1) // B for L in lengths]
    cu_qb = np.concatenate([[0], np.cumsum(nq)])
    f64 = par.f64
    n_ex = 0
    # kept rounds and blocks of every query block
    oracle = {}
    for s, L in enumerate(lengths):
        if L == 0:
            continue
        s0 = int(cu[s])
        Qs, Ks = f64(layers[watershed][0][s0:s0 + L]), f64(layers[watershed][1][s0:s0 + L])
        st = rounds[s]
        for q in range(len(st) - 1):
            m = orc.round_mass(Qs, Ks, st, q, 2.0, 256)
            qbs = range(st[q] // B, (st[q + 1] + B - 1) // B)
            for qb in qbs:
                g = int(cu_qb[s] + qb)
                kept_g = ci[rp[g]:rp[g + 1]]
                got_r = sorted({orc.round_of_token(st, int(kb) * B) for kb in kept_g})
                ex = check_rounds(m, got_r, tau)
                n_ex += ex != ""
                # the blocks are exactly those of the GPU's kept rounds up to qb
                assert list(kept_g) == list(orc.round_kept_blocks(got_r, st, qb, B))
                oracle[(s, qb)] = kept_g
    par.record(label, par.Result(len(oracle), n_ex, 0, 0.0))
    # every layer from the watershed on: extraction over the selection, then O
    tol = par.o_tol(ctx.dtype)
    for l in range(watershed, nlayers):
        Q, K, V, W = layers[l]
        lse, _ = mfb.block_stats(ctx, Q.cuda(), K.cuda())
        mfb.extract(ctx, Q.cuda(), K.cuda(), lse, cache)
        O = mfb.mapped_av(cache, Hr, W.cuda(), V.cuda(), Hkv)
        mfb.sync_status()
        vals = cache.values_view()
        Wf = f64(W)
        for (s, qb), kept_g in oracle.items():
            if picks_o is not None and (s, qb) not in picks_o:
                continue
            s0, L = int(cu[s]), lengths[s]
            i0, i1 = qb * B, min(L, (qb + 1) * B)
            _, P, _ = orc.query_block(f64(Q[s0:s0 + i1]), f64(K[s0:s0 + i1]), qb, B, 2.0, 256)
            g = int(cu_qb[s] + qb)
            for e, kb in zip(range(rp[g], rp[g + 1]), kept_g):
                got = par.stored_to_logical(f64(vals[e]), Hs, B)
                ref = np.zeros((Hs, B, B))
                hi = min(P.shape[2], (kb + 1) * B)
                ref[:, : i1 - i0, : hi - kb * B] = P[:, :, kb * B:hi]
                if ctx.dtype == torch.float32:
                    np.testing.assert_allclose(got, ref, rtol=2e-5, atol=1e-7)
                else:
                    np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-6)
            O_o = orc.mapped_av(orc.mixed_map(P, np.array(kept_g), Wf, B),
                                f64(V[s0:s0 + i1]), Hkv)
            err = np.abs(f64(O[s0 + i0:s0 + i1]) - O_o).max() / max(np.abs(O_o).max(), 1e-30)
            assert err <= tol, f"layer {l} seq {s} qb {qb}: rel err {err:.3e}"
    return n_ex, len(oracle)


@pytest.mark.parametrize("case", [
    dict(lengths=[640, 384], rounds=[[0, 128, 192, 448, 640], [0, 256, 384]], Hs=16, Hr=16,
         Hkv=8, B=64, tau=0.7, nlayers=3, watershed=1),
    dict(lengths=[700, 0, 300], rounds=[[0, 128, 384, 512, 700], [], [0, 300]], Hs=40, Hr=32,
         Hkv=8, B=128, tau=0.6, nlayers=2, watershed=0),
    dict(lengths=[520, 200], rounds=[[0, 64, 256, 320, 520], [0, 64, 128, 200]], Hs=4, Hr=2,
         Hkv=2, B=64, tau=0.75, nlayers=2, watershed=1, dtype="f32"),
], ids=["bf16_b64", "bf16_b128_empty_seq", "f32_b64"])
def test_round_selection_every_query_block(case):
    n_ex, n = run_case(**case, label="rounds small cases")
    assert n_ex <= max(1, n // 50)


def test_round_selection_keeps_everything_at_tau_one():
    lengths = [500]
    ctx = mfb.Context.make(lengths, 8, 128, 64, 2.0, 256, torch.bfloat16)
    Q, K = synth.sender_qk(lengths, 8, 128, "bf16", np.random.default_rng(1))
    _, mass = mfb.block_stats(ctx, Q.cuda(), K.cuda())
    cache = mfb.select_rounds(ctx, mass, [0, 64, 192, 500], 1.0)
    mfb.sync_status()
    rp, ci = par.kept_sets(cache)
    for qb in range(8):
        assert list(ci[rp[qb]:rp[qb + 1]]) == list(range(qb + 1))


def test_multi_turn_workload():
    """8K tokens in 17 rounds, 4 sender layers, watershed layer 1: kept rounds
    of every query block; values and O of layers 1-3 on sampled blocks."""
    w = synth.workloads()["multi_turn_rounds_n8192"]
    ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width, w.torch_dtype)
    st = w.rounds[0]
    layers = [synth.sender_layer(w, l) + synth.receiver_layer(w, 0, l)
              for l in range(w.sender_layers)]
    Qw, Kw = layers[w.watershed][0].cuda(), layers[w.watershed][1].cuda()
    _, mass = mfb.block_stats(ctx, Qw, Kw)
    cache = mfb.select_rounds(ctx, mass, st, w.tau)
    mfb.sync_status()
    rp, ci = par.kept_sets(cache)
    Qs, Ks = par.f64(layers[w.watershed][0]), par.f64(layers[w.watershed][1])
    n_ex = 0
    nqb = w.lengths[0] // w.B
    for q in range(len(st) - 1):
        m = orc.round_mass(Qs, Ks, st, q, w.band_bias, w.band_width)
        for qb in range(st[q] // w.B, (st[q + 1] + w.B - 1) // w.B):
            kept = ci[rp[qb]:rp[qb + 1]]
            got_r = sorted({orc.round_of_token(st, int(kb) * w.B) for kb in kept})
            n_ex += check_rounds(m, got_r, w.tau) != ""
            assert list(kept) == list(orc.round_kept_blocks(got_r, st, qb, w.B))
    par.record(w.name, par.Result(nqb, n_ex, 0, 0.0))
    assert n_ex <= 1
    assert cache.nnz < nqb * (nqb + 1) // 2          # rounds were dropped
    picks = [0, 37, 90, nqb - 1]
    for l in range(w.watershed, w.sender_layers):
        Q, K, V, W = layers[l]
        lse, _ = mfb.block_stats(ctx, Q.cuda(), K.cuda())
        mfb.extract(ctx, Q.cuda(), K.cuda(), lse, cache)
        O = mfb.mapped_av(cache, w.Hr, W.cuda(), V.cuda(), w.Hkv)
        mfb.sync_status()
        vals = cache.values_view()
        for qb in picks:
            i0, i1 = qb * w.B, (qb + 1) * w.B
            _, P, _ = orc.query_block(par.f64(Q[:i1]), par.f64(K[:i1]), qb, w.B, w.band_bias,
                                      w.band_width)
            kept = ci[rp[qb]:rp[qb + 1]]
            e = rp[qb + 1] - 1                                # the diagonal block
            got = par.stored_to_logical(par.f64(vals[e]), w.Hs, w.B)
            np.testing.assert_allclose(got, P[:, :, qb * w.B:i1], rtol=2 ** -8, atol=1e-6)
            O_o = orc.mapped_av(orc.mixed_map(P, np.array(kept), par.f64(W), w.B),
                                par.f64(V[:i1]), w.Hkv)
            err = np.abs(par.f64(O[i0:i1]) - O_o).max() / np.abs(O_o).max()
            assert err <= 2e-2, f"layer {l} qb {qb}: {err:.3e}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_extract_on_a_given_csr_equals_select_extract(dtype):
    """mf_extract over the CSR that mf_select_extract built writes the same
    probability blocks, bit for bit."""
    w, x = synth.small_case([700, 130], 8, 8, 2, 128 if dtype == "bf16" else 64, 64, 0.9,
                            dtype=dtype)
    ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width, w.torch_dtype)
    Q, K = x.Q.cuda(), x.K.cuda()
    lse, mass = mfb.block_stats(ctx, Q, K)
    cache = mfb.select_extract(ctx, Q, K, lse, mass, w.tau)
    mfb.sync_status()
    n = cache.nnz
    ref = cache.values_view()[:n].clone()
    cache.values.zero_()
    mfb.extract(ctx, Q, K, lse, cache)
    mfb.sync_status()
    assert torch.equal(cache.values_view()[:n], ref)
