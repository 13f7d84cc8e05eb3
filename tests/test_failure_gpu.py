"""Failure path without a GPU fault: a bounded in-kernel wait that nothing
satisfies gives up after its limit, the kernel returns, the host reads
FA_ERR_TIMEOUT, and the context stays usable for the next call."""

import time

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def test_bounded_wait_reports_timeout_and_context_survives():
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK          # clean start
    t0 = time.time()
    assert fa.fa_debug_wait_timeout(50000) == fa.FA_OK    # 50 ms limit
    assert fa.fa_last_device_error() == fa.FA_ERR_TIMEOUT
    assert time.time() - t0 < 10.0
    assert fa.fa_last_device_error() == fa.FA_OK          # the word was cleared
    # the context still works
    x = synth.attention_inputs(1, 1, 64, 64, 1, device="cuda", with_dout=False)
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert fa.fa_last_device_error() == fa.FA_OK
