"""The host-memory cache tier and the receiver prefill that overlaps the cache
fetch with the early-layer recompute (article, second component), through
the C ABI: offload and fetch move the cache exactly, and the overlapped and
serial prefills both give O equal bit for bit to the fused kernel run on the
device-resident cache."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from cross_model_attention_block_b200 import mapflow as mfb
from cross_model_attention_block_b200 import overlap as ov
from cross_model_attention_block_b200 import synth
from tests import parity as par

pytestmark = pytest.mark.gpu


def _sender_cache(lengths, Hs, B, tau, seed):
    ctx = mfb.Context.make(lengths, Hs, 128, B, 2.0, 256, torch.bfloat16)
    Q, K = synth.sender_qk(lengths, Hs, 128, "bf16", np.random.default_rng(seed))
    Q, K = Q.cuda(), K.cuda()
    lse, mass = mfb.block_stats(ctx, Q, K)
    cache = mfb.select_extract(ctx, Q, K, lse, mass, tau)
    mfb.sync_status()
    return ctx, cache


def test_offload_and_fetch_move_the_cache_exactly():
    ctx, dev = _sender_cache([700, 300], 16, 64, 0.9, 1)
    nnz = dev.nnz
    host = mfb.Cache(ctx, capacity=nnz, device="cpu", pin=True)
    mfb.cache_offload(dev, host)
    torch.cuda.synchronize()
    assert torch.equal(host.row_ptr, dev.row_ptr.cpu())
    assert torch.equal(host.col_idx[:nnz], dev.col_idx[:nnz].cpu())
    assert torch.equal(host.values_view()[:nnz], dev.values_view()[:nnz].cpu())
    back = mfb.Cache(ctx, capacity=nnz)
    back.values.fill_(float("nan"))
    for r in ov.chunk_ranges(dev.nqb, 3):
        mfb.cache_fetch(host, back, r)
    torch.cuda.synchronize()
    assert torch.equal(back.row_ptr, dev.row_ptr)
    assert torch.equal(back.values_view()[:nnz], dev.values_view()[:nnz])
    with pytest.raises(mfb.MapflowError):          # the source must be host memory
        mfb.cache_fetch(dev, back, (0, 2))


@pytest.mark.parametrize("serial", [False, True], ids=["overlapped", "serial"])
def test_prefill_equals_the_device_resident_run(serial):
    lengths, Hs, Hr, Hkv, B = [1000, 450], 40, 32, 8, 64
    ctx, dev0 = _sender_cache(lengths, Hs, B, 0.9, 2)
    ctx1, dev1 = _sender_cache(lengths, Hs, B, 0.9, 3)
    ntok = sum(lengths)
    mapped, refs = [], []
    rng = np.random.default_rng(4)
    for dev in (dev0, dev1):
        V, W = synth.receiver_vw(ntok, Hr, Hkv, Hs, 128, "bf16", rng)
        V, W = V.cuda(), W.cuda()
        refs.append(mfb.mapped_av(dev, Hr, W, V, Hkv))
        host = mfb.Cache(ctx, capacity=dev.nnz, device="cpu", pin=True)
        mfb.cache_offload(dev, host)
        target = mfb.Cache(ctx, capacity=dev.nnz)
        target.values.zero_()
        mapped.append(ov.MappedLayer(host, target, W, V, torch.full_like(refs[-1], 7.0)))
    torch.cuda.synchronize()
    # stand-in for the receiver's own first layers: dense causal attention
    q = torch.randn(1, Hr, ntok, 128, device="cuda", dtype=torch.bfloat16)
    kv = torch.randn(1, Hkv, ntok, 128, device="cuda", dtype=torch.bfloat16)
    outs = []
    recompute = [lambda: outs.append(F.scaled_dot_product_attention(q, kv, kv, is_causal=True,
                                                                    enable_gqa=True))] * 2
    ov.prefill(recompute, mapped, Hr, Hkv, chunks=4, serial=serial)
    mfb.sync_status()
    for m, ref in zip(mapped, refs):
        assert torch.equal(m.O, ref)
    assert len(outs) == 2
    # and the first layer's rows against the oracle on sampled query blocks
    Q, K = synth.sender_qk(lengths, Hs, 128, "bf16", np.random.default_rng(2))
    lse, mass = mfb.block_stats(ctx, Q.cuda(), K.cuda())
    par.compare_query_blocks(ctx, Q, K, mapped[0].V.cpu(), mapped[0].W.cpu(), Hkv, 0.9,
                             (lse, mass, dev0, mapped[0].O), [(0, 0), (0, 15), (1, 7)],
                             torch.bfloat16, check_values=False, label="overlapped prefill")
