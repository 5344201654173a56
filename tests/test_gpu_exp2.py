"""The statistics kernel's FMA-pipe exp2, through the C ABI, against CUDA's exp2f."""
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb


@pytest.mark.gpu
def test_exp2_fma_matches_cuda_exp2f(lib):
    g = torch.Generator(device="cuda").manual_seed(0)
    x = torch.rand(1 << 20, device="cuda", generator=g) * -125.0
    special = torch.tensor([0.0, -1e-7, -0.5, -0.49999, -1.0, -24.5, -100.0, -125.0],
                           device="cuda")
    x = torch.cat([x, special, -torch.arange(126, device="cuda", dtype=torch.float32)])
    y = mfb.exp2_fma_eval(x)
    ref = torch.exp2(x.double())
    rel = (y.double() / ref - 1.0).abs().max().item()
    assert rel < 4e-6, rel
    lo = mfb.exp2_fma_eval(torch.tensor([-126.0, -300.0, float("-inf")], device="cuda"))
    assert bool((lo > 0).all()) and bool((lo < 2.0 ** -124).all())
    mfb.sync_status()
