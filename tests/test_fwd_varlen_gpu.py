"""fa_fwd_varlen (packed variable-length batches, unequal query / key lengths,
grouped KV heads, bottom-right causal) vs the float64 oracle's
attention_varlen, through the C ABI.

Tolerances as for fa_fwd: |O - O_ref| <= 1e-2 + half a bf16 ulp of O_ref per
element, |dL| <= 1e-3 max(|L|, 1); a query that sees no key must give O = 0
exactly and L = -inf.
"""

import numpy as np
import pytest
import torch

import oracle
from helpers import O_TOL, assert_bf16_close, assert_lse_close, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _case(lens_q, lens_k, H, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q = torch.randn((int(cu_q[-1]), H, d), generator=g).to(torch.bfloat16)
    k = torch.randn((max(int(cu_k[-1]), 1), Hkv, d), generator=g).to(torch.bfloat16)
    v = torch.randn((max(int(cu_k[-1]), 1), Hkv, d), generator=g).to(torch.bfloat16)
    return q.cuda(), k.cuda(), v.cuda(), cu_q, cu_k


def _run(q, k, v, cu_q, cu_k, causal, **kw):
    o, lse = fa.fa_fwd_varlen(q, k, v, torch.from_numpy(cu_q).cuda(),
                              torch.from_numpy(cu_k).cuda(), int(np.diff(cu_q).max()),
                              causal=causal, **kw)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return o, lse


def _check(q, k, v, cu_q, cu_k, causal, o, lse):
    o_ref, l_ref = oracle.attention_varlen(f64(q), f64(k)[:cu_k[-1]], f64(v)[:cu_k[-1]],
                                           cu_q, cu_k, causal)
    got_o, got_l = f64(o), f64(lse)
    empty = np.isneginf(l_ref)
    assert np.all(np.isneginf(got_l[empty])), "rows without keys must have L = -inf"
    assert np.all(got_o.transpose(1, 0, 2)[empty] == 0), "rows without keys must have O = 0"
    assert_bf16_close(got_o, o_ref, O_TOL, "O")
    assert_lse_close(got_l[~empty], l_ref[~empty])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_equal_lengths_bit_match_fa_fwd(d, causal):
    """Equal lengths, H = Hkv: the same kernel arithmetic as fa_fwd on the
    [B, H, N, d] view, so the outputs agree bit for bit."""
    B, H, N = 3, 4, 300
    q, k, v, cu_q, cu_k = _case([N] * B, [N] * B, H, H, d, 500 + d)
    o, lse = _run(q, k, v, cu_q, cu_k, causal)
    bhnd = lambda t: t.view(B, N, H, d).permute(0, 2, 1, 3).contiguous()
    o2, l2 = fa.fa_fwd(bhnd(q), bhnd(k), bhnd(v), causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(bhnd(o), o2)
    assert torch.equal(lse.view(H, B, N).permute(1, 0, 2), l2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_cross_lengths_gqa(d, causal):
    """Unequal query / key lengths (both ways), tails that are not multiples
    of 128, single-token queries, an empty key sequence, 8 query heads on 2 KV
    heads; bottom-right causal includes queries that see no key."""
    lens_q = [1, 17, 128, 129, 300, 513, 40, 200, 5]
    lens_k = [1, 300, 128, 64, 300, 200, 0, 513, 129]
    q, k, v, cu_q, cu_k = _case(lens_q, lens_k, 8, 2, d, 600 + d + causal)
    o, lse = _run(q, k, v, cu_q, cu_k, causal)
    _check(q, k, v, cu_q, cu_k, causal, o, lse)


def test_decode_shaped_batch():
    """Lq = 1 per sequence (the newest token, causal): every key is visible."""
    lens_k = [16, 700, 4096, 1, 2049]
    q, k, v, cu_q, cu_k = _case([1] * 5, lens_k, 32, 8, 128, 610)
    o, lse = _run(q, k, v, cu_q, cu_k, True)
    _check(q, k, v, cu_q, cu_k, True, o, lse)


def test_long_mixed_batch_sampled():
    """16 sequences with lengths drawn from U[1, 4096] (queries = keys),
    H = 16 on 4 KV heads, d = 128, causal; sampled heads checked in full."""
    rng = np.random.default_rng(611)
    lens = rng.integers(1, 4097, 16).tolist()
    q, k, v, cu_q, cu_k = _case(lens, lens, 16, 4, 128, 611)
    o, lse = _run(q, k, v, cu_q, cu_k, True)
    for h in (0, 5, 15):
        sl = slice(h, h + 1)
        hk = h // 4
        _check(q[:, sl].contiguous(), k[:, hk:hk + 1].contiguous(), v[:, hk:hk + 1].contiguous(),
               cu_q, cu_k, True, o[:, sl], lse[sl])


def test_guard_regions():
    """Sentinels around O and L stay untouched (packed writes stay in bounds)."""
    lens_q, lens_k = [130, 7, 260], [100, 300, 260]
    H, Hkv, d = 4, 4, 128
    q, k, v, cu_q, cu_k = _case(lens_q, lens_k, H, Hkv, d, 612)
    Tq, pad = q.shape[0], 4096
    ob = torch.full((Tq * H * d + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    lb = torch.full((H * Tq + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = ob[pad:pad + Tq * H * d].view(Tq, H, d)
    lse = lb[pad:pad + H * Tq].view(H, Tq)
    _run(q, k, v, cu_q, cu_k, True, o=o, lse=lse)
    assert torch.all(ob[:pad] == 7.0) and torch.all(ob[-pad:] == 7.0)
    assert torch.all(lb[:pad] == 7.0) and torch.all(lb[-pad:] == 7.0)
    _check(q, k, v, cu_q, cu_k, True, o, lse)


def test_inconsistent_lengths_are_reported():
    """A query length above max_seqlen_q is caught on the device: that
    sequence is skipped, the rest computed, FA_ERR_INVALID_ARG reported."""
    lens = [64, 300]
    q, k, v, cu_q, cu_k = _case(lens, lens, 2, 2, 64, 613)
    o = torch.full_like(q, 3.0)
    lse = torch.full((2, q.shape[0]), 3.0, device="cuda")
    fa.fa_fwd_varlen(q, k, v, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(), 100,
                     causal=False, o=o, lse=lse)
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
    assert torch.all(o[64:] == 3.0)            # the skipped sequence is untouched
    o_ref, _ = oracle.attention_varlen(f64(q)[:64], f64(k)[:64], f64(v)[:64],
                                       cu_q[:2], cu_k[:2], False)
    assert_bf16_close(f64(o[:64]), o_ref, O_TOL, "O")
