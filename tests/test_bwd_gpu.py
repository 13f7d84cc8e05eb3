"""Backward parity: fa_bwd (sm_100a kernels, through the C ABI) vs the float64
oracle's analytic gradients on the same seeded bf16 inputs, with the forward
output and statistic taken from fa_fwd as a user would chain them; plus a
bit-exact causal check and guard regions."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import GRAD_TOL, assert_close_abs, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _fwd_bwd(x, causal):
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    dq, dk, dv = fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return o, lse, dq, dk, dv


def _check(x, dq, dk, dv, causal, heads=None):
    sl = (slice(None), slice(None)) if heads is None else (0, heads)
    q, k, v, do = (f64(x[n][sl]) for n in ("q", "k", "v", "do"))
    dq_r, dk_r, dv_r, _ = oracle.attention_bwd(q, k, v, do, causal=causal)
    e = [assert_close_abs(f64(dq[sl]), dq_r, GRAD_TOL, "dQ"),
         assert_close_abs(f64(dk[sl]), dk_r, GRAD_TOL, "dK"),
         assert_close_abs(f64(dv[sl]), dv_r, GRAD_TOL, "dV")]
    return e


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 300])
def test_ragged_shapes(N, d, causal):
    x = synth.attention_inputs(1, 2, N, d, 9000 + N + d, device="cuda")
    _, _, dq, dk, dv = _fwd_bwd(x, causal)
    _check(x, dq, dk, dv, causal)


def test_gpt2_small_shape_causal():
    """B=8, H=12, N=1024, d=64, causal, seed 1001: every gradient element."""
    x = synth.attention_inputs(8, 12, 1024, 64, 1001, device="cuda")
    _, _, dq, dk, dv = _fwd_bwd(x, True)
    _check(x, dq, dk, dv, True)


def test_long_sequence_two_heads():
    """B=1, H=16, N=16384, d=128, causal, seed 1002 (the benchmark launch):
    all 16 heads run; heads 0 and 11 are checked element by element."""
    x = synth.attention_inputs(1, 16, 16384, 128, 1002, device="cuda")
    _, _, dq, dk, dv = _fwd_bwd(x, True)
    for h in (0, 11):
        _check(x, dq, dk, dv, True, heads=slice(h, h + 1))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [5, 300])
def test_causal_one_hot_dv_bit_exact(N, d):
    """Scores that grow by >= 181 nats per key make P one-hot on the diagonal
    (causal): dV must equal dO bit for bit; a leaked mask or a wrong row/column
    index adds other rows of dO."""
    q = torch.zeros((1, 1, N, d))
    k = torch.zeros((1, 1, N, d))
    q[..., 0] = 16.0
    q[..., 1] = 16.0
    j = torch.arange(N, dtype=torch.float32)
    k[0, 0, :, 0] = 128.0 * (j % 256)
    k[0, 0, :, 1] = 32768.0 * torch.div(j, 256, rounding_mode="floor")
    g = torch.Generator().manual_seed(4)
    v = torch.randn((1, 1, N, d), generator=g)
    do = torch.randn((1, 1, N, d), generator=g)
    x = {n: t.to(torch.bfloat16).cuda() for n, t in (("q", q), ("k", k), ("v", v), ("do", do))}
    _, _, dq, dk, dv = _fwd_bwd(x, True)
    assert torch.equal(dv, x["do"].float())
    # dS is zero up to rounding (dP_ii = D_i): dQ and dK vanish
    assert float(dq.abs().max()) < 1e-3 and float(dk.abs().max()) < 1e-3


def test_guard_regions_and_workspace():
    B, H, N, d = 1, 2, 200, 64
    x = synth.attention_inputs(B, H, N, d, 21, device="cuda")
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    n = B * H * N * d
    pad = 1024
    bufs = [torch.full((n + 2 * pad,), 5.0, device="cuda") for _ in range(3)]
    dq, dk, dv = (b[pad:pad + n].view(B, H, N, d) for b in bufs)
    ws_n = fa.fa_bwd_workspace_bytes(B, H, N, d)
    wbuf = torch.full((ws_n + 2 * pad,), 0x3C, dtype=torch.uint8, device="cuda")
    fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=True, dq=dq, dk=dk, dv=dv,
              workspace=wbuf[pad:pad + ws_n])
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:pad] == 5.0) and torch.all(b[-pad:] == 5.0)
    assert torch.all(wbuf[:pad] == 0x3C) and torch.all(wbuf[-pad:] == 0x3C)
    _check(x, dq, dk, dv, True)


def test_repeated_calls_match():
    """dQ is accumulated with floating-point reductions whose order varies from
    run to run; two runs agree to rounding, dK and dV exactly."""
    x = synth.attention_inputs(1, 4, 1000, 128, 22, device="cuda")
    _, _, dq1, dk1, dv1 = _fwd_bwd(x, True)
    _, _, dq2, dk2, dv2 = _fwd_bwd(x, True)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert float((dq1 - dq2).abs().max()) < 1e-4
