"""Failure detection without a GPU fault: a bounded device wait on a barrier
that nothing completes gives up, the status word reports MF_ERR_TIMEOUT, and
the context keeps working."""
import pytest
import torch

from cross_model_attention_block_b200 import mapflow as mfb


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives(lib):
    mfb.sync_status()  # clean slate
    mfb.selftest_timeout(20)
    with pytest.raises(mfb.MapflowError) as e:
        mfb.sync_status()
    assert e.value.status == mfb.MF_ERR_TIMEOUT
    # the status word was cleared and the device still runs kernels
    mfb.sync_status()
    x = -torch.arange(64, dtype=torch.float32, device="cuda") / 8
    y = mfb.exp2_fma_eval(x)
    assert torch.allclose(y, torch.exp2(x), rtol=1e-5, atol=0)
    mfb.sync_status()
