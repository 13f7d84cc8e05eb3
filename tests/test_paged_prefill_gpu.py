"""fa_paged_prefill (chunks of queries over a paged KV cache, bottom-right
causal) vs the float64 oracle's paged_prefill, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
from helpers import O_TOL, assert_bf16_close, assert_lse_close, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _case(chunks, ctxs, hq, hkv, d, seed):
    rng = np.random.default_rng(seed)
    nb = [-(-c // 16) for c in ctxs]
    n_phys = sum(nb) + 5
    perm = rng.permutation(n_phys).astype(np.int32)
    table = np.zeros((len(ctxs), max(nb) + 2), dtype=np.int32)
    p = 0
    for s, n in enumerate(nb):
        table[s, :n] = perm[p:p + n]
        p += n
    if len(ctxs) > 1 and min(nb[:2]) > 1:
        table[1, 0] = table[0, 0]                     # a block shared by two sequences
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn((n_phys, hkv, 16, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((n_phys, hkv, 16, d), generator=g).to(torch.bfloat16)
    cu_q = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = torch.randn((int(cu_q[-1]), hq, d), generator=g).to(torch.bfloat16)
    return q.cuda(), kc.cuda(), vc.cuda(), table, cu_q, np.array(ctxs, dtype=np.int32)


def _run(q, kc, vc, table, cu_q, ctx, causal=True):
    o, lse = fa.fa_paged_prefill(q, kc, vc, torch.from_numpy(table).cuda(),
                                 torch.from_numpy(cu_q).cuda(), torch.from_numpy(ctx).cuda(),
                                 int(np.diff(cu_q).max()), causal=causal)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_chunks_over_paged_cache(d, causal):
    chunks = [1, 17, 128, 129, 300, 64]
    ctxs = [40, 17, 700, 129, 1000, 2050]
    q, kc, vc, tab, cu_q, ctx = _case(chunks, ctxs, 32, 8, d, 900 + d + causal)
    o, lse = _run(q, kc, vc, tab, cu_q, ctx, causal)
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, l_ref = oracle.paged_prefill(f64(q), f64(kc), f64(vc), tab, cu_q, ctx, causal)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)


def test_single_token_chunks_match_paged_decode():
    """Chunks of one token: the same quantity as paged_attn_decode."""
    ctxs = [40, 700, 4096, 1, 2049]
    q, kc, vc, tab, cu_q, ctx = _case([1] * 5, ctxs, 32, 8, 128, 910)
    o, lse = _run(q, kc, vc, tab, cu_q, ctx)
    od, ld = fa.paged_attn_decode(q, kc, vc, torch.from_numpy(tab).cuda(),
                                  torch.from_numpy(ctx).cuda(), max(ctxs))
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    assert float((o.float() - od.float()).abs().max()) <= 2 * O_TOL
    o_ref, _ = oracle.paged_prefill(f64(q), f64(kc), f64(vc), tab, cu_q, ctx)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")


def test_bad_table_entry_is_reported_not_dereferenced():
    q, kc, vc, tab, cu_q, ctx = _case([32, 16], [100, 64], 8, 2, 128, 920)
    tab[1, 2] = 10 ** 6
    _run(q, kc, vc, tab, cu_q, ctx)
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
