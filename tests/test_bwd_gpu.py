"""Backward parity: fa_bwd (sm_100a kernels, through the C ABI) vs the float64
oracle's analytic gradients on the same seeded bf16 inputs.

fa_bwd's inputs include the forward's O, which crosses the interface as bf16,
and D_i = sum_c dO_ic O_ic is computed from it. The expected gradients are
therefore the oracle's textbook backward with D taken from the oracle's own O
rounded to bf16 (oracle.round_bf16); that is what the backward computes from
the inputs it is given. Two kinds of test:
  * contract: fa_bwd gets the oracle's bf16-rounded O and fp32 L directly;
  * chained: fa_fwd then fa_bwd, as a user runs them.
The difference to the exact gradient (D from unrounded O) is reported by the
chained tests and bounded there by the error the bf16 O can carry into D.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import GRAD_TOL, assert_close_abs, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _oracle_fwd_io(x, causal, sl=(slice(None), slice(None))):
    """Oracle O (rounded to bf16, as the interface carries it) and L."""
    o_ref, l_ref = oracle.attention_fwd(f64(x["q"][sl]), f64(x["k"][sl]), f64(x["v"][sl]),
                                        causal=causal)
    return oracle.round_bf16(o_ref), l_ref


def _expected(x, causal, o_in, sl=(slice(None), slice(None))):
    q, k, v, do = (f64(x[n][sl]) for n in ("q", "k", "v", "do"))
    return oracle.attention_bwd(q, k, v, do, causal=causal, o=o_in)[:3]


def _check(got, exp):
    return [assert_close_abs(f64(g), e, GRAD_TOL, n)
            for g, e, n in zip(got, exp, ("dQ", "dK", "dV"))]


def _contract(x, causal):
    o_in, l_ref = _oracle_fwd_io(x, causal)
    o_t = torch.from_numpy(o_in).to(torch.bfloat16).cuda()      # exact: already on the bf16 grid
    l_t = torch.from_numpy(l_ref).float().cuda()
    grads = fa.fa_bwd(x["q"], x["k"], x["v"], o_t, l_t, x["do"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    _check(grads, _expected(x, causal, o_in))


def _chained(x, causal):
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    grads = fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return grads


def _exact_gap_bound(x, causal, o_ref_exact, sl=(slice(None), slice(None))):
    """How far D built from a bf16 O can move dQ and dK: with
    |dD_i| <= sum_c |dO_ic| ulp_bf16(O_ic) (one ulp covers the rounding plus the
    forward's own error), dQ_i moves by <= scale |dD_i| sum_j P_ij |K_j| and dK_j
    by <= scale sum_i P_ij |dD_i| |Q_i|."""
    q, k, v, do = (f64(x[n][sl]) for n in ("q", "k", "v", "do"))
    n, d = q.shape[-2:]
    sc = 1.0 / math.sqrt(d)
    a = np.abs(o_ref_exact)
    _, e = np.frexp(np.where(a > 0, a, 1.0))
    ulp = np.exp2(e - 8.0)
    dd = (np.abs(do) * ulp).sum(-1)
    q2, k2, dd2 = q.reshape(-1, n, d), k.reshape(-1, n, d), dd.reshape(-1, n)
    bq, bk = np.zeros_like(q2), np.zeros_like(k2)
    for h in range(q2.shape[0]):
        _, _, p = oracle.attention_rows(q2[h], np.arange(n), k2[h], k2[h], causal)
        bq[h] = sc * dd2[h][:, None] * (p @ np.abs(k2[h]))
        bk[h] = sc * (p.T @ (dd2[h][:, None] * np.abs(q2[h])))
    return bq.reshape(q.shape), bk.reshape(k.shape)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 256, 300])
def test_contract_ragged_shapes(N, d, causal):
    x = synth.attention_inputs(1, 2, N, d, 9000 + N + d, device="cuda")
    _contract(x, causal)


def test_contract_gpt2_small_shape():
    """B=8, H=12, N=1024, d=64, causal, seed 1001: every gradient element."""
    _contract(synth.attention_inputs(8, 12, 1024, 64, 1001, device="cuda"), True)


def test_contract_long_sequence_two_heads():
    """N=16384, d=128, causal, seed 1002, two heads (B=1, H=2)."""
    _contract(synth.attention_inputs(1, 2, 16384, 128, 1002, device="cuda"), True)


def test_chained_gpt2_small_shape():
    """fa_fwd -> fa_bwd on B=8, H=12, N=1024, d=64, causal, seed 1001; also
    bounds the gap to the exact gradient (D from unrounded O)."""
    x = synth.attention_inputs(8, 12, 1024, 64, 1001, device="cuda")
    dq, dk, dv = _chained(x, True)
    o_ex, _ = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), causal=True)
    _check((dq, dk, dv), _expected(x, True, oracle.round_bf16(o_ex)))
    ex = oracle.attention_bwd(*(f64(x[n]) for n in ("q", "k", "v", "do")), causal=True)
    bq, bk = _exact_gap_bound(x, True, o_ex)
    assert np.all(np.abs(f64(dq) - ex[0]) <= GRAD_TOL + bq)
    assert np.all(np.abs(f64(dk) - ex[1]) <= GRAD_TOL + bk)
    assert_close_abs(f64(dv), ex[2], GRAD_TOL, "dV (exact)")


def test_chained_long_sequence_full_launch():
    """B=1, H=16, N=16384, d=128, causal, seed 1002 (the benchmark launch):
    all 16 heads run; heads 0 and 11 are checked element by element."""
    x = synth.attention_inputs(1, 16, 16384, 128, 1002, device="cuda")
    dq, dk, dv = _chained(x, True)
    for h in (0, 11):
        sl = (0, slice(h, h + 1))
        o_in, _ = _oracle_fwd_io(x, True, sl)
        _check((dq[sl], dk[sl], dv[sl]), _expected(x, True, o_in, sl))


def _diag_staircase(N, d):
    """q_i . k_j / sqrt(d) = 1024 (j - i) / sqrt(d) exactly (>= 90 nats per key),
    every value exact in bf16 and fp16: row i's largest visible score is 0 at
    j = i, so P is one-hot on the diagonal and L_i = 0 exactly."""
    q = torch.zeros((1, 1, N, d))
    k = torch.zeros((1, 1, N, d))
    i = torch.arange(N, dtype=torch.float32)
    q[0, 0, :, 0] = 16.0
    q[0, 0, :, 1] = 16.0
    k[0, 0, :, 0] = 64.0 * (i % 64)
    k[0, 0, :, 1] = 4096.0 * torch.div(i, 64, rounding_mode="floor")
    q[0, 0, :, 2] = -64.0 * (i % 64)
    q[0, 0, :, 3] = -4096.0 * torch.div(i, 64, rounding_mode="floor")
    k[0, 0, :, 2] = 16.0
    k[0, 0, :, 3] = 16.0
    return q, k


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [5, 300, 700])
def test_causal_one_hot_dv_bit_exact(N, d):
    """P one-hot on the diagonal (causal): dV must equal dO bit for bit; a
    leaked mask or a wrong row/column index adds other rows of dO."""
    q, k = _diag_staircase(N, d)
    s = (q[0, 0].double() @ k[0, 0].double().T) / math.sqrt(d)
    jj, ii = np.meshgrid(np.arange(N), np.arange(N))
    assert np.allclose(s.numpy(), 1024.0 * (jj - ii) / math.sqrt(d))
    g = torch.Generator().manual_seed(4)
    v = torch.randn((1, 1, N, d), generator=g)
    do = torch.randn((1, 1, N, d), generator=g)
    x = {n: t.to(torch.bfloat16).cuda() for n, t in (("q", q), ("k", k), ("v", v), ("do", do))}
    dq, dk, dv = _chained(x, True)
    assert torch.equal(dv, x["do"].float())
    # dS_ii = P_ii (dP_ii - D_i) is zero up to fp32 rounding: dP_ii and D_i sum
    # the same d products dO_ic V_ic (O_i = V_i) in different orders, so
    # |dS_ii| <= 2 (d + 2) 2^-24 sum_c |dO_ic V_ic| (twice that for an
    # accumulator that truncates), and dQ_i = scale dS_ii K_i, dK_i =
    # scale dS_ii Q_i (one-hot P: row i meets column i only)
    sc = 1.0 / math.sqrt(d)
    ds = 4.0 * (d + 2) * 2.0 ** -24 * (x["do"][0, 0].double() * x["v"][0, 0].double()).abs().sum(-1)
    bq = sc * ds * k[0, 0].double().abs().max(-1).values.cuda()
    bk = sc * ds * q[0, 0].double().abs().max(-1).values.cuda()
    assert torch.all(dq[0, 0].double().abs().max(-1).values <= bq)
    assert torch.all(dk[0, 0].double().abs().max(-1).values <= bk)


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
    o_ex, _ = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), causal=True)
    _check((dq, dk, dv), _expected(x, True, oracle.round_bf16(o_ex)))


def test_repeated_calls_match():
    """dQ is accumulated with floating-point reductions whose order varies from
    run to run; two runs agree to rounding, dK and dV exactly."""
    x = synth.attention_inputs(1, 4, 1000, 128, 22, device="cuda")
    dq1, dk1, dv1 = _chained(x, True)
    dq2, dk2, dv2 = _chained(x, True)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert float((dq1 - dq2).abs().max()) < 1e-4
