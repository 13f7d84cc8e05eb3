"""BNHD (token-major [B, N, H, d]) tensors through the packed entry points.

A [B, N, H, d] tensor is the packed [T, H, d] layout with T = B N and every
sequence N tokens long ("Flash Attention 再学习", Flash Attention v2: rows,
heads and batches are independent problems, so the layout only changes the
addressing). fa_fwd_varlen / fa_bwd_varlen with cu_seqlens = 0, N, 2N, ...
must give what fa_fwd / fa_bwd give on the same values in [B, H, N, d]: the
same kernels walk the same key blocks per row, so the forward agrees to the
last bit; the backward's dQ sums CTA partials in HBM in an order that varies
from run to run, so the gradients agree to fp32 rounding.
"""

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _bnhd(t):
    """[B, H, N, d] -> token-major [B * N, H, d] (a BNHD tensor, flattened)."""
    B, H, N, d = t.shape
    return t.permute(0, 2, 1, 3).contiguous().view(B * N, H, d)


def _bhnd(t, B, N):
    T, H, d = t.shape
    return t.view(B, N, H, d).permute(0, 2, 1, 3)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bnhd_through_the_packed_entry_points(d, causal):
    B, H, N = 3, 4, 300
    x = synth.attention_inputs(B, H, N, d, 77 + d + causal, device="cuda")
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    q, k, v, do = (_bnhd(x[n]) for n in ("q", "k", "v", "do"))

    o_ref, l_ref = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    o, lse = fa.fa_fwd_varlen(q, k, v, cu, cu, N, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    assert torch.equal(_bhnd(o, B, N), o_ref)
    # L: [H, T] packed against [B, H, N]
    assert torch.equal(lse.view(H, B, N).permute(1, 0, 2), l_ref)

    g_ref = fa.fa_bwd(x["q"], x["k"], x["v"], o_ref, l_ref, x["do"], causal=causal)
    g = fa.fa_bwd_varlen(q, k, v, o, lse, do, cu, cu, N, N, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    for name, got, ref in zip(("dQ", "dK", "dV"), g, g_ref):
        got = _bhnd(got, B, N)
        scale = float(ref.abs().max())
        err = float((got - ref).abs().max())
        assert err <= 1e-5 * max(scale, 1.0), f"{name}: {err:.3e} against {scale:.3e}"
