"""fa_fwd_dropout / fa_bwd_dropout vs the float64 oracle (oracle.dropout),
through the C ABI: the keep mask bit for bit in both kernels, O, L and the
gradients within the stated tolerances, p = 0 reducing to the plain calls."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import GRAD_TOL, O_TOL, assert_bf16_close, assert_close_abs, assert_lse_close, f64
from oracle.dropout import attention_dropout, attention_dropout_bwd, drop_threshold, keep_mask

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _keep_scale(p):
    return 256.0 / (256 - drop_threshold(p))


def _one_hot_rows(B, H, N, d):
    """Row i = 2^(i div d) e_(i mod d): a sum over rows i = c, c + d, ... of
    kept/dropped weights reads back as the bits of an integer."""
    x = torch.zeros((B, H, N, d), dtype=torch.float32)
    i = torch.arange(N)
    x[:, :, i, i % d] = torch.exp2((i // d).float())
    return x.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_forward_keep_mask_bit_exact(p):
    """K = 0 makes P uniform (P = 1, l = N); with V_j = 2^(j div 128) e_(j mod 128),
    O_ic * N / s equals sum_m Z[i, c + 128 m] 2^m exactly, so every keep bit of
    the kernel is read back and compared with the oracle's mask."""
    B, H, N, d = 2, 3, 384, 128
    g = torch.Generator().manual_seed(77)
    q = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).cuda()
    k = torch.zeros_like(q)
    v = _one_hot_rows(B, H, N, d)
    seed, off = 0x5EED0000DEADBEEF, 3
    o, _ = fa.fa_fwd_dropout(q, k, v, p, seed, off)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    code = np.rint(f64(o) * N / _keep_scale(p)).astype(np.int64)      # [B, H, N, 128]
    assert code.min() >= 0 and code.max() <= 7
    got = np.stack([(code >> m) & 1 for m in range(N // d)], axis=-2).reshape(B, H, N, N)
    want = keep_mask(B, H, N, p, seed, off)
    assert np.array_equal(got.astype(bool), want)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_backward_keep_mask_bit_exact(p, d):
    """The backward regenerates the mask with keys on the lanes (one Philox call
    per 16 keys and query, shared across 16 lanes by shuffles). K = 0 and
    dO_i = 2^(i div d) e_(i mod d) make dV_jc * N / s = sum_m Z[c + d m, j] 2^m."""
    B, H, N = 2, 3, 384
    g = torch.Generator().manual_seed(78)
    q = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).cuda()
    k = torch.zeros_like(q)
    v = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).cuda()
    do = _one_hot_rows(B, H, N, d)
    seed, off = 12345, 0
    o, lse = fa.fa_fwd_dropout(q, k, v, p, seed, off)
    _, _, dv = fa.fa_bwd_dropout(q, k, v, o, lse, do, p, seed, off)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    x = f64(dv) * N / _keep_scale(p)                                    # [B, H, N keys, d]
    code = np.rint(x).astype(np.int64)
    assert np.abs(x - code).max() < 0.05 and code.min() >= 0 and code.max() < 2 ** (N // d)
    # bit m of code[b, h, j, c] is Z[query c + d m, key j]
    got = np.stack([(code >> m) & 1 for m in range(N // d)], axis=-2)   # [B, H, j, m, c]
    got = got.reshape(B, H, N, N).transpose(0, 1, 3, 2)                 # [B, H, i, j]
    assert np.array_equal(got.astype(bool), keep_mask(B, H, N, p, seed, off))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_p_zero_is_fa_fwd_and_fa_bwd(d, causal):
    x = synth.attention_inputs(1, 2, 300, d, 4100 + d + causal, device="cuda")
    o, lse = fa.fa_fwd_dropout(x["q"], x["k"], x["v"], 0.0, 1, 0, causal=causal)
    o2, l2 = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    # dK and dV are summed inside one CTA: bit-equal; dQ is reduced across
    # CTAs in an order that varies from run to run: equal to rounding
    dq1, dk1, dv1 = fa.fa_bwd_dropout(x["q"], x["k"], x["v"], o, lse, x["do"], 0.0, 1, 0,
                                      causal=causal)
    dq2, dk2, dv2 = fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert float((dq1 - dq2).abs().max()) < 1e-5


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 200, 513])
@pytest.mark.parametrize("p", [0.1, 0.3])
def test_forward_parity(p, N, d, causal):
    B, H = 1, 2
    x = synth.attention_inputs(B, H, N, d, 4200 + N + d, device="cuda", with_dout=False)
    seed, off = 99 + N, 5
    o, lse = fa.fa_fwd_dropout(x["q"], x["k"], x["v"], p, seed, off, causal=causal)
    _, l_plain = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, l_ref = attention_dropout(f64(x["q"]), f64(x["k"]), f64(x["v"]), p, seed, off, causal)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)
    assert torch.equal(lse, l_plain)                    # L is that of the undropped scores


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [17, 129, 300])
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_backward_contract(p, N, causal, d):
    """Gradients from the oracle's own (bf16-rounded) O and L, as fa_bwd's tests."""
    B, H = 1, 2
    x = synth.attention_inputs(B, H, N, d, 4300 + N + causal + d, device="cuda")
    seed, off = 2024, 1
    q, k, v, do = (f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, l_ref = attention_dropout(q, k, v, p, seed, off, causal)
    o_in = oracle.round_bf16(o_ref)
    o_t = torch.from_numpy(o_in).to(torch.bfloat16).cuda()
    l_t = torch.from_numpy(l_ref).float().cuda()
    grads = fa.fa_bwd_dropout(x["q"], x["k"], x["v"], o_t, l_t, x["do"], p, seed, off,
                              causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    exp = attention_dropout_bwd(q, k, v, do, p, seed, off, causal, o=o_in)[:3]
    for g, e, n in zip(grads, exp, ("dQ", "dK", "dV")):
        assert_close_abs(f64(g), e, GRAD_TOL, n)


def test_chained_two_heads_n2048_causal():
    """fwd then bwd through the kernels, B = 1, H = 2, N = 2048, p = 0.1."""
    B, H, N, d, p = 1, 2, 2048, 128, 0.1
    x = synth.attention_inputs(B, H, N, d, 4400, device="cuda")
    seed, off = 31337, 9
    o, lse = fa.fa_fwd_dropout(x["q"], x["k"], x["v"], p, seed, off, causal=True)
    grads = fa.fa_bwd_dropout(x["q"], x["k"], x["v"], o, lse, x["do"], p, seed, off, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    q, k, v, do = (f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, l_ref = attention_dropout(q, k, v, p, seed, off, True)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)
    # D from the kernel's bf16 O: compare against the oracle fed that same O
    exp = attention_dropout_bwd(q, k, v, do, p, seed, off, True, o=f64(o))[:3]
    for g, e, n in zip(grads, exp, ("dQ", "dK", "dV")):
        assert_close_abs(f64(g), e, GRAD_TOL, n)


def test_forward_full_size_sampled_rows():
    """B = 1, H = 16, N = 16384, d = 128, causal, p = 0.1 (the timed dropout
    workload): 12 sampled query rows of 3 heads against the definition."""
    B, H, N, d, p = 1, 16, 16384, 128, 0.1
    x = synth.attention_inputs(B, H, N, d, 1002, device="cuda", with_dout=False)
    seed, off = 1002, 0
    o, lse = fa.fa_fwd_dropout(x["q"], x["k"], x["v"], p, seed, off, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    rows = np.array([0, 1, 127, 128, 4095, 9000, 16255, 16256, 16383, 777, 12000, 15000])
    inv_q = _keep_scale(p)
    for h in (0, 7, 15):
        qh, kh, vh = (f64(x[n][0, h]) for n in ("q", "k", "v"))
        _, l_ref, pr = oracle.attention_rows(qh[rows], rows, kh, vh, True)
        z = keep_mask(B, H, N, p, seed, off, rows=rows)[0, h]
        o_ref = ((pr * z) @ vh) * inv_q
        assert_bf16_close(f64(o[0, h])[rows], o_ref, O_TOL, f"O head {h}")
        assert_lse_close(f64(lse[0, h])[rows], l_ref)
    assert math.isfinite(float(lse.float().abs().max()))
