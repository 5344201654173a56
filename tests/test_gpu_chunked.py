"""Chunked prefill and prefix-partial reuse (the fused kernel over a range of
query blocks), through the C ABI."""
import numpy as np
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb
from cross_model_attention_block_b200 import synth
from tests import parity as par

pytestmark = pytest.mark.gpu


def _case(lengths, Hs, Hr, Hkv, d, B, tau, dtype="bf16"):
    w, x = synth.small_case(lengths, Hs, Hr, Hkv, d, B, tau, dtype=dtype)
    ctx = mfb.Context.make(w.lengths, w.Hs, w.d, w.B, w.band_bias, w.band_width, w.torch_dtype)
    gpu = par.run_gpu(ctx, x.Q.cuda(), x.K.cuda(), x.V.cuda(), x.W.cuda(), Hkv, tau)
    return w, x, ctx, gpu


@pytest.mark.parametrize("args", [
    dict(lengths=[300, 200, 77], Hs=40, Hr=32, Hkv=8, d=128, B=64, tau=0.9),    # 32-key stages
    dict(lengths=[390, 130], Hs=16, Hr=16, Hkv=8, d=128, B=128, tau=0.95),
    dict(lengths=[200, 90], Hs=4, Hr=2, Hkv=2, d=64, B=64, tau=0.9, dtype="f32"),  # scalar kernel
], ids=["bf16_b64", "bf16_b128", "f32_b64"])
def test_chunked_prefill_equals_one_call(args):
    w, x, ctx, (lse, mass, cache, O_full) = _case(**args)
    nqb = cache.nqb
    W, V = x.W.cuda(), x.V.cuda()
    O = torch.full_like(O_full, 7.0)
    cuts = [0, 1, max(2, nqb // 2), nqb - 1, nqb]
    for a, b in zip(cuts[:-1], cuts[1:]):
        mfb.mapped_av(cache, w.Hr, W, V, w.Hkv, O=O, qb_range=(a, b))
    mfb.sync_status()
    assert torch.equal(O, O_full)  # every CTA computes its rows the same way
    # and the rows the ranges wrote are the oracle's
    par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, (lse, mass, cache, O),
                             par.all_picks(ctx), w.torch_dtype, check_values=False,
                             label="chunked ranges")


def test_range_writes_only_its_rows():
    w, x, ctx, (lse, mass, cache, O_full) = _case([300, 200], 40, 32, 8, 128, 64, 0.9)
    O = torch.full_like(O_full, 7.0)
    mfb.mapped_av(cache, w.Hr, x.W.cuda(), x.V.cuda(), w.Hkv, O=O, qb_range=(2, 6))
    mfb.sync_status()
    # global query blocks 2..5: rows 128..299 of sequence 0 and rows 0..63 of sequence 1
    rows = torch.zeros(O.shape[0], dtype=torch.bool)
    rows[128:300] = True
    rows[300:364] = True
    assert torch.equal(O[rows], O_full[rows])
    assert bool((O[~rows] == 7.0).all())
    par.compare_query_blocks(ctx, x.Q, x.K, x.V, x.W, w.Hkv, w.tau, (lse, mass, cache, O),
                             [(0, 2), (0, 3), (0, 4), (1, 0)], w.torch_dtype,
                             check_values=False, label="chunked ranges")
    with pytest.raises(mfb.MapflowError):
        mfb.mapped_av(cache, w.Hr, x.W.cuda(), x.V.cuda(), w.Hkv, O=O, qb_range=(3, 99))


def test_prefix_partial_reuse_through_the_index():
    """A receiver whose context shares a prefix with the sender's reuses the
    sender's cache for the shared query blocks: those rows equal the rows of
    the full run over the same map with the receiver's V."""
    B, P = 64, 170  # 2 whole shared blocks, then the contexts diverge
    w, x, ctx, (lse, mass, cache, O_sender) = _case([300], 40, 32, 8, 128, B, 0.9)
    rng = np.random.default_rng(5)
    sender_tokens = rng.integers(0, 50000, size=300).astype(np.int32)
    receiver_tokens = np.concatenate([sender_tokens[:P],
                                      rng.integers(50000, 60000, size=140).astype(np.int32)])
    ix = mfb.PrefixIndex()
    ix.insert(mfb.prefix_hash(sender_tokens, B), sender_layer=0, seq=0, cache_struct=cache.struct())
    hit = ix.lookup(mfb.prefix_hash(receiver_tokens, B), 0)
    assert hit is not None
    _, seq, matched = hit
    assert (seq, matched) == (0, P // B)
    # the receiver's own V on the shared prefix (rows past it are never read)
    Vr = torch.randn(x.V.shape, generator=torch.Generator().manual_seed(9)).to(x.V.dtype).cuda()
    O_ref = mfb.mapped_av(cache, w.Hr, x.W.cuda(), Vr, w.Hkv)
    O = torch.full_like(O_ref, 7.0)
    mfb.mapped_av(cache, w.Hr, x.W.cuda(), Vr, w.Hkv, O=O, qb_range=(0, matched))
    mfb.sync_status()
    n = matched * B
    assert torch.equal(O[:n], O_ref[:n])
    assert bool((O[n:] == 7.0).all())
    # the oracle on the receiver's side: the sender's map over the shared
    # prefix (the receiver's rows there attend only to prefix keys) times the
    # receiver's own V
    par.compare_query_blocks(ctx, x.Q, x.K, Vr.cpu(), x.W, w.Hkv, w.tau,
                             (lse, mass, cache, O), [(0, qb) for qb in range(matched)],
                             w.torch_dtype, check_values=False, label="prefix reuse")
