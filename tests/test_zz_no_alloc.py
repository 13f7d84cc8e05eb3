"""The allocation-free decode entry point (paged_attn_decode_noalloc).

Some callers cannot allocate device memory on their decode path (an engine
that fixes its memory plan at start-up, or code that must not pay cudaMalloc's
implicit synchronisation). For them the library keeps the decode's split
partials in a 16 MiB array of its own. This file checks, through the C ABI,
that two calls in a row give the same results as the workspace-taking
paged_attn_decode on the same inputs, and that the calls allocate nothing
through torch. It is collected last so that a failure here cannot hide any
other test's result.
"""

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _case(num_seqs, lo, hi, seed):
    lay = synth.paged_decode_layout(num_seqs, 16, lo, hi, seed)
    q, kc, vc = synth.paged_decode_tensors(num_seqs, 32, 8, 128, 16, lay["num_phys"], seed,
                                           device="cuda")
    tab = torch.from_numpy(lay["block_table"]).cuda()
    lens = torch.from_numpy(lay["context_lens"]).cuda()
    return q, kc, vc, tab, lens, hi


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [_case(16, 100, 8192, 301), _case(6, 1, 20000, 302)]
    # the limit admits both cases
    for q, _, _, _, _, max_ctx in cases:
        need = fa.paged_attn_decode_workspace_bytes(q.shape[0], 32, 128, max_ctx)
        assert need <= 16 << 20
    refs = []
    for q, kc, vc, tab, lens, max_ctx in cases:
        refs.append(fa.paged_attn_decode(q, kc, vc, tab, lens, max_ctx))
    outs = [(torch.empty_like(c[0]), torch.empty(c[0].shape[:2], device="cuda")) for c in cases]
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    for (q, kc, vc, tab, lens, max_ctx), (o, lse) in zip(cases, outs):   # two calls in a row
        fa.paged_attn_decode_noalloc(q, kc, vc, tab, lens, max_ctx, o, lse)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    assert fa.fa_last_device_error() == fa.FA_OK
    # the same split and combine kernels run on the same splits: only the
    # partials' home differs, so the results are identical bit for bit
    for (o_ref, l_ref), (o, lse) in zip(refs, outs):
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, l_ref)


def test_noalloc_rejects_requests_over_the_limit():
    q, kc, vc, tab, lens, _ = _case(4, 100, 400, 303)
    o = torch.empty_like(q)
    with pytest.raises(fa.FAError) as e:
        # 64 sequences x 32 heads x 32 splits of partials do not fit in 16 MiB;
        # every other argument passes the checks (the call is rejected before
        # anything is read: a table width of 2048 entries is only declared)
        fa.lib()
        status = fa.lib().paged_attn_decode_noalloc(
            fa._ptr(q), fa._ptr(kc), fa._ptr(vc), kc.shape[0], fa._ptr(tab), 2048,
            fa._ptr(lens), fa._ptr(o), None, 64, 32, 8, 128, 16, 32768, fa._stream())
        fa._check("paged_attn_decode_noalloc", status)
    assert e.value.status == fa.FA_ERR_WORKSPACE
