"""fa_bwd_fp8 (the backward of the FP8 forward) through the C ABI, against
oracle.attention_fp8_bwd on the oracle's own e4m3 codes and block scales.

The contract: gradients with respect to the forward's unrotated inputs,
straight through the e4m3 block quantisation and back through the rotation R.
The kernel runs its products on fp16 operands (the e4m3 codes are fp16 values
exactly) and applies every block scale in fp32. The bound, per element, is
derived from that arithmetic (with a factor 2 of slack on each term):
  dV_jc:  2^-10 sum_i P_ij |dO_ic|                      (P rounded to fp16)
  dK'_jc: scale sum_i e_ij |Q'_ic|,  dQ'_ic: scale sum_j e_ij |K'_jc|, with
          e_ij = 2^-10 |dS_ij| + 2^-20 P_ij (|dP_ij| + |D_i|)
          (dS rounded to fp16; fp32 sums in dP and D)
  dQ = dQ' R^T, dK = dK' R^T: the bound vector b of a row maps to b |R|^T
          (the kernel's rotation, on split bf16 terms, adds a relative error
          near 2^-16 of |dQ'| |R|^T, far inside the 2^-10 term);
plus 1e-3 absolute. O and L are the oracle's (the forward's outputs are
checked by tests/test_fp8_gpu.py).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _inputs(B, H, N, seed, d=128):
    x = synth.fp8_inputs(B, H, N, d, seed, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    x["do"] = torch.randn((B, H, N, d), generator=g, device="cuda").to(torch.bfloat16)
    r32 = synth.orthogonal_matrix(d, 2003).astype(np.float32).astype(np.float64)
    codes = {}
    for name, rot in (("q", True), ("k", True), ("v", False)):
        src = f64(x[name])
        vals, scales = oracle.fp8_block_quantize(src @ r32 if rot else src)
        codes[name] = (vals, scales.astype(np.float32).astype(np.float64))
    return x, r32, codes


def _run(x, r32, codes, causal, heads):
    """Oracle forward (O bf16-rounded, L) on the dequantised codes, then the
    kernel on the codes; returns the GPU gradients and the expected ones for
    the listed (b, h) heads."""
    B, H, N, d = x["q"].shape
    deq = {n: oracle.dequantize_blocks_e4m3(*codes[n]) for n in codes}
    to8 = lambda v: torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).cuda()
    dev = dict(
        q8=to8(codes["q"][0]), k8=to8(codes["k"][0]), v8=to8(codes["v"][0]),
        sq=torch.from_numpy(codes["q"][1]).float().cuda(),
        sk=torch.from_numpy(codes["k"][1]).float().cuda(),
        sv=torch.from_numpy(codes["v"][1]).float().cuda())
    # the heads that are not checked take the FP8 forward's own O and L (only
    # so that every head of the launch does realistic work); the checked heads
    # take the oracle's
    o_t, l_t = fa.fa_fwd_fp8(dev["q8"], dev["k8"], dev["v8"], dev["sq"], dev["sk"], dev["sv"],
                             causal=causal)
    o_in = {}
    for b, h in heads:
        o_ref, l_ref = oracle.attention_fwd(deq["q"][b, h], deq["k"][b, h], deq["v"][b, h],
                                            causal=causal)
        o_in[(b, h)] = oracle.round_bf16(o_ref)
        o_t[b, h] = torch.from_numpy(o_in[(b, h)]).to(torch.bfloat16).cuda()
        l_t[b, h] = torch.from_numpy(l_ref).float().cuda()
    R = torch.from_numpy(r32).float().cuda()
    got = fa.fa_bwd_fp8(dev["q8"], dev["k8"], dev["v8"], dev["sq"], dev["sk"], dev["sv"], R,
                        o_t, l_t, x["do"], causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return got, deq, o_in


def _check_head(got, deq, o_in, do, r32, codes, b, h, causal):
    d = r32.shape[0]
    sc = 1.0 / math.sqrt(d)
    q, k, v = (deq[n][b, h] for n in ("q", "k", "v"))
    g = do[b, h]
    exp = oracle.attention_fp8_bwd(*(c[b, h] for c in (codes["q"][0], codes["q"][1],
                                                       codes["k"][0], codes["k"][1],
                                                       codes["v"][0], codes["v"][1])),
                                   r32, g, o_in[(b, h)], causal)
    n = q.shape[0]
    _, _, p = oracle.attention_rows(q, np.arange(n), k, v, causal)
    dp = g @ v.T
    dd = (g * o_in[(b, h)]).sum(-1)
    ds = p * (dp - dd[:, None])
    e = 2.0 ** -10 * np.abs(ds) + 2.0 ** -20 * p * (np.abs(dp) + np.abs(dd)[:, None])
    b_dv = 2.0 ** -10 * (p.T @ np.abs(g))
    b_dk = (sc * (e.T @ np.abs(q))) @ np.abs(r32).T
    b_dq = (sc * (e @ np.abs(k))) @ np.abs(r32).T
    for name, gt, ref, bound in (("dQ", got[0], exp[0], b_dq), ("dK", got[1], exp[1], b_dk),
                                 ("dV", got[2], exp[2], b_dv)):
        x = f64(gt[b, h])
        assert np.all(np.isfinite(x)), name
        diff = np.abs(x - ref)
        lim = 1e-3 + 2.0 * bound
        assert np.all(diff <= lim), (f"{name} b{b} h{h}: worst excess "
                                     f"{float((diff - lim).max()):.3e}, max err {float(diff.max()):.3e}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [64, 100, 300, 513])
def test_ragged_shapes(N, causal, d):
    x, r32, codes = _inputs(1, 2, N, 60 + N + causal, d)
    heads = [(0, 0), (0, 1)]
    got, deq, o_in = _run(x, r32, codes, causal, heads)
    for b, h in heads:
        _check_head(got, deq, o_in, f64(x["do"]), r32, codes, b, h, causal)


def test_fp8_config_two_heads():
    """The FP8 workload's shape (B=4, H=16, N=4096, d=128, no mask, seed 1003,
    0.1% outliers x50): the whole launch runs; heads (0, 0) and (3, 15) are
    checked element by element."""
    x, r32, codes = _inputs(4, 16, 4096, 1003)
    heads = [(0, 0), (3, 15)]
    got, deq, o_in = _run(x, r32, codes, False, heads)
    for b, h in heads:
        _check_head(got, deq, o_in, f64(x["do"]), r32, codes, b, h, False)


@pytest.mark.parametrize("d", [64, 128])
def test_identity_rotation_and_unit_scales_match_fa_bwd(d):
    """Codes on the e4m3 grid with every scale 1 and R = I: the FP8 backward
    is fa_bwd on the same values (dK, dV to fp32 rounding of differently
    scaled operands, dQ likewise)."""
    B, H, N = 1, 2, 200
    g = torch.Generator().manual_seed(91)
    vals = {n: oracle.quantize_e4m3(torch.randn((B, H, N, d), generator=g).double().numpy() * 0.5)
            for n in ("q", "k", "v")}
    do = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).cuda()
    bf = {n: torch.from_numpy(v).to(torch.bfloat16).cuda() for n, v in vals.items()}
    assert all(np.array_equal(f64(bf[n]), vals[n]) for n in vals)     # exact in bf16 too
    to8 = lambda v: torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).cuda()
    ones = torch.ones((B, H, (N + 63) // 64), device="cuda")
    eye = torch.eye(d, device="cuda")
    for causal in (False, True):
        o, lse = fa.fa_fwd(bf["q"], bf["k"], bf["v"], causal=causal)
        ref = fa.fa_bwd(bf["q"], bf["k"], bf["v"], o, lse, do, causal=causal)
        got = fa.fa_bwd_fp8(to8(vals["q"]), to8(vals["k"]), to8(vals["v"]), ones, ones, ones, eye,
                            o, lse, do, causal=causal)
        torch.cuda.synchronize()
        assert fa.fa_last_device_error() == fa.FA_OK
        for a, r in zip(got, ref):
            scale = float(r.abs().max())
            assert float((a - r).abs().max()) <= 1e-5 * max(scale, 1.0)
