"""FP8 path: fa_fp8_prepare (rotation by an orthogonal R, per-64-row e4m3
block quantisation) and fa_fwd_fp8, through the C ABI.

What is compared. The pages' FP8 method quantises Q R, K R and V to e4m3 with
one scale per block; that quantisation is part of the method, and on the FP8
workload (0.1% of entries scaled by 50, so nearly every 64 x 128 block holds
outliers) it alone moves O by up to ~15 against unquantised attention, even
when every later step is exact (float64 emulation). So:
  * fa_fp8_prepare is checked code by code against the oracle's rotation and
    e4m3 block quantiser (rare one-step differences where the fp32 rotation
    lands on a rounding boundary);
  * fa_fwd_fp8 runs on the oracle's codes and scales and is checked against the
    float64 forward on the dequantised inputs. It then differs by rounding P'
    to e4m3 for the P.V product: per element |dO| <= 5e-2 + 2^-4 (P |V|)
    (relative e4m3 rounding of each weight) plus half a bf16 ulp of the
    output; L is checked to 1e-3 relative;
  * the chained fa_fp8_prepare -> fa_fwd_fp8 result is held to the same bound
    against the oracle's quantised inputs, widened only by the first-order
    effect of the one-step code differences (computed from the oracle);
  * without outliers the whole chain meets the plain 5e-2 against unquantised
    attention; with them the gap to unquantised attention is recorded (the
    CPU pin in tests/test_precision_readings.py shows the quantisation alone
    exceeds 5e-2 there).
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import FP8_TOL, assert_lse_close, bf16_half_ulp, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _e4m3_to_f64(t):
    return t.view(torch.float8_e4m3fn).to("cpu", torch.float64).numpy()


def _prepare(B, H, N, seed, d=128):  # GPU prepare (codes checked against the oracle's)
    x = synth.fp8_inputs(B, H, N, d, seed, device="cuda")
    r64 = synth.orthogonal_matrix(d, 2003)
    R = torch.from_numpy(r64).float().cuda()
    out = fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R)
    torch.cuda.synchronize()
    return x, r64.astype(np.float32).astype(np.float64), out


def _oracle_quantised(x, r32):
    """The oracle's rotation + block quantisation of the whole batch: e4m3
    codes (as uint8 bytes for the kernel) and fp32 scales, plus the dequantised
    float64 tensors the expected values are computed from."""
    out = {}
    for name, rot in (("q", True), ("k", True), ("v", False)):
        src = f64(x[name])
        if rot:
            src = src @ r32
        vals, scales = oracle.fp8_block_quantize(src)
        codes = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).cuda()
        out[name] = (codes, torch.from_numpy(scales).float().cuda(),
                     oracle.dequantize_blocks_e4m3(vals, scales.astype(np.float32)))
    return out


def _check_rows(o, lse, deq, b, h, rows, causal):
    """|dO| <= 5e-2 + 2^-4 (P|V|) + half a bf16 ulp against the float64
    forward on the dequantised inputs the kernel consumed."""
    qd, kd, vd = (deq[n][2][b, h] for n in ("q", "k", "v"))
    o_ref, l_ref, p = oracle.attention_rows(qd[rows], rows, kd, vd, causal)
    bound = FP8_TOL + 2.0 ** -4 * (p @ np.abs(vd)) + bf16_half_ulp(o_ref)
    got = f64(o[b, h, rows])
    diff = np.abs(got - o_ref)
    assert np.all(np.isfinite(got))
    assert np.all(diff <= bound), f"b{b} h{h}: worst excess {float((diff - bound).max()):.3e}"
    assert_lse_close(f64(lse[b, h, rows]), l_ref)
    return float(diff.max())


def _fwd_on_oracle_codes(deq, causal):
    (q8, sq, _), (k8, sk, _), (v8, sv, _) = (deq[n] for n in ("q", "k", "v"))
    o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
def test_prepare_matches_oracle_quantiser(d):
    B, H, N = 1, 3, 300
    x, r32, (q8, k8, v8, sq, sk, sv) = _prepare(B, H, N, 31, d)
    for name, t8, sc, rot in (("q", q8, sq, True), ("k", k8, sk, True), ("v", v8, sv, False)):
        src = f64(x[name])
        if rot:
            src = src @ r32
        vals, scales = oracle.fp8_block_quantize(src)
        np.testing.assert_allclose(f64(sc), scales, rtol=1e-5)
        got = _e4m3_to_f64(t8)
        # rotation rounding on the GPU (fp32 accumulation) may move a value across an e4m3
        # rounding boundary: allow rare one-step differences, nothing else
        diff = got != vals
        assert diff.mean() < 2e-3, f"{name}: {diff.mean():.2e} of codes differ"
        step = np.abs(vals) * 2.0 ** -3 + 2.0 ** -9
        assert np.all(np.abs(got - vals)[diff] <= step[diff] * 1.01)


def _code_flip_bound(x, r32, deq, b, h, rows):
    """How far O_rows can move when the GPU's fp32 rotation and fp32 scale put
    an element on the other side of an e4m3 rounding boundary than the
    oracle's float64 ones (the one-step code differences
    test_prepare_matches_oracle_quantiser allows), or scale it by a slightly
    different fp32 block scale. From the oracle alone, and worst-case (so
    loose wherever an outlier sits near an ambiguous element):
      * an element y = x / s is ambiguous when y - e and y + e round to
        different codes, e = the error bound of the GPU's rotation over s,
        plus 2^-18 |y| for the scale. The rotation (d = 128) runs on the
        tensor core with x exact in bf16 and R split into bf16 terms hi + lo:
        the split leaves |R - hi - lo| <= 2^-18 |R|, and the fp32
        accumulation of the 2 d products, each step taken as truncating
        (2^-23 of the partial sum), adds at most 2 d 2^-23: together
        (2^-18 + 2 d 2^-23) sum_c |x_c R_c|;
        its dequantised value can then move by the difference of those codes
        times s, and every element by 2^-18 of itself (the scale);
      * with |dS_ij| <= scale (sum_c dq_ic |k_jc| + |q_ic| dk_jc) <= delta_i
        for every key j, each P_ij changes by a factor within e^(+-2 delta_i),
        so O_i moves by at most (e^(2 delta_i) - 1) max_j |V_j - O_i| +
        e^(2 delta_i) sum_j P_ij |dV_j| (max norms over the head dimension)."""
    d = 128
    moves = {}
    for name, rot in (("q", True), ("k", True), ("v", False)):
        src = f64(x[name][b, h])
        xe = src @ r32 if rot else src
        err_x = ((2.0 ** -18 + 2 * d * 2.0 ** -23) * (np.abs(src) @ np.abs(r32)) if rot
                 else 0.0 * xe)
        vals, scales = oracle.fp8_block_quantize(xe)
        srow = np.repeat(scales, 64)[: xe.shape[0]][:, None]
        y = xe / srow
        e = err_x / srow + 2.0 ** -18 * np.abs(y)
        flip = np.abs(oracle.quantize_e4m3(y + e) - oracle.quantize_e4m3(y - e)) * srow
        moves[name] = flip + 2.0 ** -18 * np.abs(vals) * srow
    qd, kd, vd = (deq[n][2][b, h] for n in ("q", "k", "v"))
    o_ref, _, p = oracle.attention_rows(qd[rows], rows, kd, vd, False)
    sc = 1.0 / np.sqrt(d)
    delta = sc * (moves["q"][rows] @ np.abs(kd).T + np.abs(qd[rows]) @ moves["k"].T).max(-1)
    spread = np.abs(vd).max() + np.abs(o_ref).max(-1)                   # >= max_j |V_j - O_i|
    grow = np.exp(2.0 * delta)
    return ((grow - 1.0) * spread)[:, None] + grow[:, None] * (p @ moves["v"])


def test_fp8_config_sampled_rows(record_property):
    """B=4, H=16, N=4096, d=128, no mask, seed 1003: 0.1% outliers x50, R from
    seed 2003. fa_fwd_fp8 runs on the oracle's e4m3 codes and scales (so both
    sides see identical quantised inputs); sampled rows of 8 heads. The chained
    fa_fp8_prepare -> fa_fwd_fp8 result is held to the same bound against the
    float64 forward on the oracle's dequantised inputs, plus the first-order
    effect of the one-step code differences the GPU's fp32 rotation may make
    (_code_flip_bound); its gap to unquantised attention is recorded."""
    B, H, N = 4, 16, 4096
    x = synth.fp8_inputs(B, H, N, 128, 1003, device="cuda")
    r32 = synth.orthogonal_matrix(128, 2003).astype(np.float32).astype(np.float64)
    deq = _oracle_quantised(x, r32)
    o, lse = _fwd_on_oracle_codes(deq, False)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 1, N - 1], rng.choice(N, 200, replace=False)]))
    heads = ((0, 0), (0, 7), (1, 3), (1, 15), (2, 9), (3, 0), (3, 8), (3, 15))
    for b, h in heads:
        _check_rows(o, lse, deq, b, h, rows, False)
    # chained path (the GPU's own prepare)
    R = torch.from_numpy(r32).float().cuda()
    o2, lse2 = fa.fa_fwd_fp8(*fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R), causal=False)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    gap, over = 0.0, 0
    for b, h in heads:
        qd, kd, vd = (deq[n][2][b, h] for n in ("q", "k", "v"))
        o_ref, l_ref, p = oracle.attention_rows(qd[rows], rows, kd, vd, False)
        tight = FP8_TOL + 2.0 ** -4 * (p @ np.abs(vd)) + bf16_half_ulp(o_ref)
        bound = tight + _code_flip_bound(x, r32, deq, b, h, rows)
        got = f64(o2[b, h, rows])
        assert np.all(np.isfinite(got))
        diff = np.abs(got - o_ref)
        assert np.all(diff <= bound), f"chained b{b} h{h}: worst excess {float((diff - bound).max()):.3e}"
        over += int((diff > tight).any(-1).sum())
        assert_lse_close(f64(lse2[b, h, rows]), l_ref, rtol=FP8_TOL)
        o_ex, _, _ = oracle.attention_rows(f64(x["q"][b, h, rows]), rows, f64(x["k"][b, h]),
                                           f64(x["v"][b, h]), False)
        gap = max(gap, float(np.abs(got - o_ex).max()))
    # code differences are rare (a few elements per head): nearly every row
    # must meet the tight bound itself
    assert over <= 0.01 * len(heads) * len(rows), over
    # the pages' block quantisation alone moves O by whole units on this input
    # (tests/test_precision_readings.py); recorded, not a kernel property
    record_property("chained_max_abs_gap_to_unquantised_attention", gap)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 257, 640])
def test_fp8_ragged_shapes(N, causal, d):
    B, H = 1, 2
    x = synth.fp8_inputs(B, H, N, d, 40 + N, device="cuda")
    r32 = synth.orthogonal_matrix(d, 2003).astype(np.float32).astype(np.float64)
    deq = _oracle_quantised(x, r32)
    o, lse = _fwd_on_oracle_codes(deq, causal)
    for h in range(H):
        _check_rows(o, lse, deq, 0, h, np.arange(N), causal)


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_without_outliers_meets_plain_tolerance(d):
    """Gaussian inputs without outliers: against unquantised attention the
    FP8 result stays within the plain 5e-2 (+ half a bf16 ulp)."""
    B, H, N = 1, 4, 2048
    x = synth.attention_inputs(B, H, N, d, 1005, device="cuda", with_dout=False)
    R = torch.from_numpy(synth.orthogonal_matrix(d, 2003)).float().cuda()
    q8, k8, v8, sq, sk, sv = fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R)
    o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=False)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]))
    diff = np.abs(f64(o) - o_ref)
    assert np.all(diff <= FP8_TOL + bf16_half_ulp(o_ref)), float(diff.max())
    assert_lse_close(f64(lse), l_ref, rtol=FP8_TOL)
