"""Backward over bf16's whole range: inputs far from magnitude 1.

The backward's tensor-core operands are fp16 copies of the bf16 inputs, each
tensor multiplied by a power of two chosen from its largest magnitude (fp16
has 5 exponent bits against bf16's 8). Two kinds of check:

  * oracle parity at training-like magnitudes: dO scaled by 2^-20 and 2^-24
    (a loss averaged over many tokens), and a call that holds values above
    fp16's largest (65504) and below its smallest normal (2^-14) at once.
    Expected gradients come from oracle.attention_bwd on the same scaled
    inputs; the bar is the 1e-2 tolerance times the power of two by which
    that gradient scales.
  * equivariance: multiplying Q by 2^a and K by 2^-a leaves the scores
    unchanged, and V by 2^b, dO by 2^c scale O, D and the gradients by
    exact powers of two. A power-of-two input scale must then change the
    results by exactly that power of two, bit for bit (dQ, whose reductions
    run in a varying order, to rounding): the library's arithmetic does not
    depend on the binade of its inputs.

A test that scales Q and K by the same factor changes the scores, so it is a
different softmax; at 2^8 each the scores and L reach ~3e5, where the fp32
rounding of S and L alone moves the recomputed P enough to miss 1e-2 on dV,
whatever the kernel does (the CPU pin in tests/test_precision_readings.py
shows it). The tests here keep S fixed.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import GRAD_TOL, assert_close_abs, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _scaled(x, a=0, b=0, c=0):
    """Q 2^a, K 2^-a, V 2^b, dO 2^c (exact on bf16 values in range)."""
    y = {"q": x["q"] * 2.0 ** a, "k": x["k"] * 2.0 ** -a, "v": x["v"] * 2.0 ** b,
         "do": x["do"] * 2.0 ** c}
    for n in ("q", "k", "v", "do"):
        assert y[n].dtype == torch.bfloat16
        assert torch.all(torch.isfinite(y[n]))
    return y


def _factors(a, b, c):
    """Powers of two by which dQ, dK, dV scale: dS goes with dO V (2^(b+c)),
    dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO."""
    return 2.0 ** (b + c - a), 2.0 ** (b + c + a), 2.0 ** c


def _run(x, causal):
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    g = fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return o, lse, g


def _oracle_check(x, causal, factors, sl=(slice(None), slice(None))):
    """fa_bwd on the oracle's bf16 O and L vs oracle.attention_bwd, every
    element, with the tolerance scaled like each gradient."""
    q, k, v, do = (f64(x[n][sl]) for n in ("q", "k", "v", "do"))
    o_ref, l_ref = oracle.attention_fwd(q, k, v, causal=causal)
    o_in = oracle.round_bf16(o_ref)
    exp = oracle.attention_bwd(q, k, v, do, causal=causal, o=o_in)[:3]
    o_t = torch.from_numpy(o_in).to(torch.bfloat16).cuda()
    l_t = torch.from_numpy(l_ref).float().cuda()
    xs = {n: x[n][sl].contiguous() for n in ("q", "k", "v", "do")}
    got = fa.fa_bwd(xs["q"], xs["k"], xs["v"], o_t, l_t, xs["do"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    for g, e, f, n in zip(got, exp, factors, ("dQ", "dK", "dV")):
        assert_close_abs(f64(g), e, GRAD_TOL * f, n)


SCALINGS = [
    (0, 0, -20),    # dO 2^-20: dO of order 1e-6, gradients too
    (0, 0, -24),    # dO 2^-24: every dO entry below fp16's smallest normal
    (16, 16, -24),  # Q and V up to ~3e5 (> 65504), K and dO below 2^-14
]


@pytest.mark.parametrize("a,b,c", SCALINGS)
def test_gpt2_small_shape_scaled_vs_oracle(a, b, c):
    """B=8, H=12, N=1024, d=64, causal, seed 1001, with scaled inputs."""
    x = _scaled(synth.attention_inputs(8, 12, 1024, 64, 1001, device="cuda"), a, b, c)
    _oracle_check(x, True, _factors(a, b, c))


@pytest.mark.parametrize("a,b,c", SCALINGS)
def test_long_sequence_slice_scaled_vs_oracle(a, b, c):
    """B=1, H=16, N=16384, d=128, causal, seed 1002: head 3, scaled inputs."""
    x = _scaled(synth.attention_inputs(1, 16, 16384, 128, 1002, device="cuda"), a, b, c)
    _oracle_check(x, True, _factors(a, b, c), (slice(0, 1), slice(3, 4)))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("a,b,c", SCALINGS + [(60, 100, -100), (-40, -60, 90)])
def test_power_of_two_equivariance(d, a, b, c):
    """fa_fwd -> fa_bwd on scaled inputs equals the unscaled run times the
    exact power of two, bit for bit for O, L, dK and dV. The last two
    scalings put V at ~1e30 and dO at ~1e-30, and V at ~1e-18 and dO at ~1e27."""
    base = synth.attention_inputs(2, 3, 700, d, 31 + d, device="cuda")
    o0, l0, (dq0, dk0, dv0) = _run(base, True)
    x = _scaled(base, a, b, c)
    o1, l1, (dq1, dk1, dv1) = _run(x, True)
    fq, fk, fv = _factors(a, b, c)
    assert torch.equal(l1, l0)
    assert torch.equal(o1, (o0.double() * 2.0 ** b).to(torch.bfloat16))
    assert torch.equal(dk1.double(), dk0.double() * fk)
    assert torch.equal(dv1.double(), dv0.double() * fv)
    rel = ((dq1.double() / fq - dq0.double()).abs().max() / dq0.double().abs().max()).item()
    assert rel < 1e-5


def test_inconsistent_lse_is_reported():
    """dS is scaled to stay below 2^15 when L is the logsumexp of the scores;
    an L that is not (P = exp(S - L) far above 1) overflows the fp16 dS
    operand, and the backward reports it as FA_ERR_UNSUPPORTED."""
    x = synth.attention_inputs(1, 1, 128, 64, 23, device="cuda")
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=False)
    fa.fa_bwd(x["q"], x["k"], x["v"], o, lse - 40.0, x["do"], causal=False)
    assert fa.fa_last_device_error() == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_last_device_error() == fa.FA_OK
    fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=False)
    assert fa.fa_last_device_error() == fa.FA_OK
