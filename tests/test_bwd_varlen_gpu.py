"""fa_bwd_varlen vs the float64 oracle's attention_varlen_bwd (packed
variable-length batches, unequal lengths, grouped KV heads, bottom-right
causal), through the C ABI. As for fa_bwd, the contract tests feed the
oracle's O rounded to bf16 and its L, and the gradients are compared with the
oracle's backward built from that O; max-abs 1e-2 on dQ, dK, dV."""

import numpy as np
import pytest
import torch

import oracle
from helpers import GRAD_TOL, assert_close_abs, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _case(lens_q, lens_k, H, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    tq, tk = max(int(cu_q[-1]), 1), max(int(cu_k[-1]), 1)
    t = {n: torch.randn(shape, generator=g).to(torch.bfloat16)
         for n, shape in (("q", (tq, H, d)), ("k", (tk, Hkv, d)), ("v", (tk, Hkv, d)),
                          ("do", (tq, H, d)))}
    return {n: x.cuda() for n, x in t.items()}, cu_q, cu_k


def _contract(x, cu_q, cu_k, causal, **kw):
    q, k, v, do = (f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, l_ref = oracle.attention_varlen(q, k[:cu_k[-1]], v[:cu_k[-1]], cu_q, cu_k, causal)
    o_in = oracle.round_bf16(o_ref)
    o_t = torch.from_numpy(o_in).to(torch.bfloat16).cuda()
    l_t = torch.from_numpy(l_ref).float().cuda()
    grads = fa.fa_bwd_varlen(x["q"], x["k"], x["v"], o_t, l_t, x["do"],
                             torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                             int(np.diff(cu_q).max()), int(max(np.diff(cu_k).max(), 1)),
                             causal=causal, **kw)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    exp = oracle.attention_varlen_bwd(q, k[:cu_k[-1]], v[:cu_k[-1]], do, cu_q, cu_k, causal,
                                      o=o_in)
    nq, nk = int(cu_q[-1]), int(cu_k[-1])
    for g, e, n, rows in zip(grads, exp, ("dQ", "dK", "dV"), (nq, nk, nk)):
        assert_close_abs(f64(g)[:rows], e[:rows], GRAD_TOL, n)
    return grads


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_fa_bwd(causal, d):
    """Equal lengths, H = Hkv: dK and dV agree with fa_bwd on the [B, H, N, d]
    view bit for bit; dQ (summed by reductions in varying order) to rounding."""
    B, H, N = 2, 4, 300
    x, cu_q, cu_k = _case([N] * B, [N] * B, H, H, d, 700 + causal)
    o, lse = fa.fa_fwd_varlen(x["q"], x["k"], x["v"], torch.from_numpy(cu_q).cuda(),
                              torch.from_numpy(cu_k).cuda(), N, causal=causal)
    g1 = fa.fa_bwd_varlen(x["q"], x["k"], x["v"], o, lse, x["do"], torch.from_numpy(cu_q).cuda(),
                          torch.from_numpy(cu_k).cuda(), N, N, causal=causal)
    bhnd = lambda t: t.view(B, N, H, d).permute(0, 2, 1, 3).contiguous()
    lse_b = lse.view(H, B, N).permute(1, 0, 2).contiguous()
    g2 = fa.fa_bwd(bhnd(x["q"]), bhnd(x["k"]), bhnd(x["v"]), bhnd(o), lse_b, bhnd(x["do"]),
                   causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    assert torch.equal(bhnd(g1[1]), g2[1]) and torch.equal(bhnd(g1[2]), g2[2])
    assert float((bhnd(g1[0]) - g2[0]).abs().max()) < 1e-4


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_cross_lengths_gqa(causal, d):
    """Unequal lengths both ways, tails off the 64 / 128 grid, a sequence with
    no queries (its dK, dV are 0) and one with no keys, 8 query heads on 2 KV
    heads; bottom-right causal includes queries that see no key."""
    lens_q = [17, 128, 200, 0, 300, 1, 64, 90]
    lens_k = [40, 128, 129, 50, 300, 500, 0, 33]
    x, cu_q, cu_k = _case(lens_q, lens_k, 8, 2, d, 710 + causal + d)
    _, dk, dv = _contract(x, cu_q, cu_k, causal)
    k0, k1 = int(cu_k[3]), int(cu_k[4])                  # the sequence without queries
    assert torch.all(dk[k0:k1] == 0) and torch.all(dv[k0:k1] == 0)


@pytest.mark.parametrize("d", [64, 128])
def test_long_mixed_batch(d):
    """8 sequences, lengths U[1, 2048] (queries = keys), 8 heads on 4 KV heads,
    causal: every gradient element."""
    rng = np.random.default_rng(720)
    lens = rng.integers(1, 2049, 8).tolist()
    x, cu_q, cu_k = _case(lens, lens, 8, 4, d, 720 + d)
    _contract(x, cu_q, cu_k, True)


def test_guard_regions():
    lens_q, lens_k = [70, 130], [200, 90]
    x, cu_q, cu_k = _case(lens_q, lens_k, 4, 2, 128, 730)
    pad = 4096
    tq, tk = x["q"].shape[0], x["k"].shape[0]
    bufs = [torch.full((n + 2 * pad,), 5.0, device="cuda") for n in (tq * 4 * 128, tk * 2 * 128,
                                                                      tk * 2 * 128)]
    dq = bufs[0][pad:-pad].view(tq, 4, 128)
    dk = bufs[1][pad:-pad].view(tk, 2, 128)
    dv = bufs[2][pad:-pad].view(tk, 2, 128)
    _contract(x, cu_q, cu_k, True, dq=dq, dk=dk, dv=dv)
    for b in bufs:
        assert torch.all(b[:pad] == 5.0) and torch.all(b[-pad:] == 5.0)
