"""Paged decode parity: paged_attn_decode (through the C ABI) vs the float64
oracle's paged_decode on the same seeded inputs, plus bit-exact block-table
indexing and guard regions."""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import O_TOL, assert_bf16_close, assert_close_abs, assert_lse_close, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")

HQ, HKV, D, BS = 32, 8, 128, 16


def _inputs(num_seqs, lo, hi, seed, share_frac=0.10, extra_blocks=0):
    lay = synth.paged_decode_layout(num_seqs, BS, lo, hi, seed, share_frac=share_frac,
                                    extra_blocks=extra_blocks)
    q, kc, vc = synth.paged_decode_tensors(num_seqs, HQ, HKV, D, BS, lay["num_phys"], seed,
                                           device="cuda")
    return lay, q, kc, vc


def _oracle_for(seqs, lay, q, kc, vc):
    """Oracle on a subset of sequences: hand it the blocks those sequences
    use (copied to the host) with their table rows remapped."""
    lens = lay["context_lens"][seqs]
    tab = lay["block_table"][seqs]
    nblk = (lens + BS - 1) // BS
    used = np.unique(np.concatenate([tab[i, :nblk[i]] for i in range(len(seqs))]))
    remap = {int(p): i for i, p in enumerate(used)}
    tab2 = np.zeros_like(tab)
    for i in range(len(seqs)):
        tab2[i, :nblk[i]] = [remap[int(p)] for p in tab[i, :nblk[i]]]
    idx = torch.from_numpy(used.astype(np.int64)).cuda()
    return oracle.paged_decode(f64(q[torch.from_numpy(np.asarray(seqs)).cuda()]),
                               f64(kc[idx]), f64(vc[idx]), tab2, lens, block_size=BS)


def _run(lay, q, kc, vc, max_ctx=None):
    tab = torch.from_numpy(lay["block_table"]).cuda()
    lens = torch.from_numpy(lay["context_lens"]).cuda()
    max_ctx = int(lay["context_lens"].max()) if max_ctx is None else max_ctx
    o, lse = fa.paged_attn_decode(q, kc, vc, tab, lens, max_ctx)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return o, lse


def test_paged_decode_full_config_sampled():
    """64 sequences, Hq 32 / Hkv 8, d 128, contexts uniform on [512, 32768],
    shuffled table, 4-way sibling prefix sharing; every head of 12 sampled
    sequences (siblings included) checked against the oracle."""
    lay, q, kc, vc = _inputs(64, 512, 32768, 1004)
    o, lse = _run(lay, q, kc, vc, max_ctx=32768)
    seqs = [0, 1, 2, 3, 17, 30, 31, 40, 47, 52, 60, 63]
    o_ref, l_ref = _oracle_for(seqs, lay, q, kc, vc)
    assert_bf16_close(f64(o[seqs]), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse[seqs]), l_ref)


@pytest.mark.parametrize("lens", [[1, 15, 16, 17], [1023, 1024, 1025, 2049],
                                  [33, 100, 1, 5000]])
def test_short_and_boundary_contexts(lens):
    """Contexts at block and split boundaries (1 block = 16 tokens, 1 split =
    64 blocks), all sequences checked."""
    n = len(lens)
    lay = synth.paged_decode_layout(n, BS, 1, 1, seed=77, share_frac=0.0)
    # rebuild the layout with the requested lengths
    nblk = [(x + BS - 1) // BS for x in lens]
    total = sum(nblk)
    perm = np.random.default_rng(8).permutation(total + 5)
    tab = np.zeros((n, max(nblk)), dtype=np.int32)
    pos = 0
    for i in range(n):
        tab[i, :nblk[i]] = perm[pos:pos + nblk[i]]
        pos += nblk[i]
    lay = {"context_lens": np.array(lens, dtype=np.int32), "block_table": tab,
           "num_phys": total + 5}
    q, kc, vc = synth.paged_decode_tensors(n, HQ, HKV, D, BS, total + 5, 78, device="cuda")
    o, lse = _run(lay, q, kc, vc)
    o_ref, l_ref = _oracle_for(list(range(n)), lay, q, kc, vc)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)


def test_fully_shared_table():
    """All four siblings map every block to the same physical blocks: their
    outputs differ only through their own queries."""
    lens = np.array([3000, 3000, 3000, 3000], dtype=np.int32)
    nb = (3000 + BS - 1) // BS
    tab = np.tile(np.random.default_rng(2).permutation(nb).astype(np.int32), (4, 1))
    lay = {"context_lens": lens, "block_table": tab, "num_phys": nb}
    q, kc, vc = synth.paged_decode_tensors(4, HQ, HKV, D, BS, nb, 79, device="cuda")
    q[1] = q[0]
    o, lse = _run(lay, q, kc, vc)
    assert torch.equal(o[0], o[1]) and torch.equal(lse[0], lse[1])
    o_ref, l_ref = _oracle_for([0, 1, 2, 3], lay, q, kc, vc)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)


def test_block_table_bit_exact():
    """Per (sequence, query head) one target token's logit exceeds all others
    by > 2000 nats, so O must equal that token's V row bit for bit: any error
    in table lookup, slot arithmetic, GQA head mapping or split bounds picks
    another row."""
    lay, q, kc, vc = _inputs(16, 40, 3000, 91, share_frac=0.0, extra_blocks=7)
    lens = lay["context_lens"]
    tab = lay["block_table"]
    rng = np.random.default_rng(92)
    q.zero_()
    kc.zero_()
    targets = np.zeros((16, HQ), dtype=np.int64)
    for s in range(16):
        for h in range(HQ):
            kvh, hh = h // 4, h % 4
            t = int(rng.integers(0, lens[s]))
            # one coordinate per grouped head so the 4 heads' targets do not interact
            while any(targets[s, kvh * 4 + g] == t for g in range(hh)):
                t = int(rng.integers(0, lens[s]))
            targets[s, h] = t
            q[s, h, hh] = 16.0
            kc[tab[s, t // BS], kvh, t % BS, hh] = 2000.0
    o, lse = _run(lay, q, kc, vc)
    for s in range(16):
        for h in range(HQ):
            t = targets[s, h]
            assert torch.equal(o[s, h], vc[tab[s, t // BS], h // 4, t % BS]), (s, h, t)


def test_optional_lse_and_guard_regions():
    lay, q, kc, vc = _inputs(8, 100, 5000, 93)
    S = 8
    pad = 2048
    obuf = torch.full((2 * pad + S * HQ * D,), 3.0, dtype=torch.bfloat16, device="cuda")
    o = obuf[pad:pad + S * HQ * D].view(S, HQ, D)
    tab = torch.from_numpy(lay["block_table"]).cuda()
    lens = torch.from_numpy(lay["context_lens"]).cuda()
    max_ctx = int(lay["context_lens"].max())
    ws_bytes = fa.paged_attn_decode_workspace_bytes(S, HQ, D, max_ctx)
    wbuf = torch.full((ws_bytes + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    o2, lse = fa.paged_attn_decode(q, kc, vc, tab, lens, max_ctx, o=o, want_lse=False,
                                   workspace=wbuf[pad:pad + ws_bytes])
    torch.cuda.synchronize()
    assert lse is None
    assert torch.all(obuf[:pad] == 3.0) and torch.all(obuf[-pad:] == 3.0)
    assert torch.all(wbuf[:pad] == 0x5A) and torch.all(wbuf[-pad:] == 0x5A)
    o_ref, _ = _oracle_for(list(range(S)), lay, q, kc, vc)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")


def test_many_items_per_cta():
    """More work items than resident CTAs (each CTA walks several items,
    with empty splits in between): every sequence checked."""
    lay, q, kc, vc = _inputs(40, 1, 5000, 94)
    o, lse = _run(lay, q, kc, vc, max_ctx=5000)
    seqs = list(range(40))
    o_ref, l_ref = _oracle_for(seqs, lay, q, kc, vc)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)


# ------------------------------------------ query groups of 1..8, d 64 / 128
GROUPS = [(8, 8), (16, 8), (32, 8), (64, 8), (24, 3), (7, 1)]   # groups 1, 2, 4, 8, 8, 7


def _general(num_seqs, Hq, Hkv, d, lo, hi, seed, share_frac=0.10):
    lay = synth.paged_decode_layout(num_seqs, BS, lo, hi, seed, share_frac=share_frac)
    q, kc, vc = synth.paged_decode_tensors(num_seqs, Hq, Hkv, d, BS, lay["num_phys"], seed,
                                           device="cuda")
    return lay, q, kc, vc


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", GROUPS)
def test_query_groups_and_head_dims(Hq, Hkv, d):
    """Hq / Hkv from 1 to 8 query heads per KV head and d in {64, 128}: every
    head of 12 sequences with contexts U[1, 3000] against the oracle (which
    maps query head h to KV head h // (Hq / Hkv))."""
    lay, q, kc, vc = _general(12, Hq, Hkv, d, 1, 3000, 500 + Hq + d)
    o, lse = _run(lay, q, kc, vc)
    o_ref, l_ref = _oracle_for(list(range(12)), lay, q, kc, vc)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse), l_ref)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8), (64, 8)])
def test_block_table_bit_exact_groups(Hq, Hkv, d):
    """The dominant-logit check of test_block_table_bit_exact for other query
    groups and d = 64: query head hh of a group uses coordinate hh, so the G
    heads of one KV head pick their own target tokens independently."""
    S = 10
    G = Hq // Hkv
    lay = synth.paged_decode_layout(S, BS, 40, 2000, 95 + Hq + d, share_frac=0.0, extra_blocks=5)
    q, kc, vc = synth.paged_decode_tensors(S, Hq, Hkv, d, BS, lay["num_phys"], 96, device="cuda")
    lens, tab = lay["context_lens"], lay["block_table"]
    rng = np.random.default_rng(97)
    q.zero_()
    kc.zero_()
    targets = np.zeros((S, Hq), dtype=np.int64)
    for s in range(S):
        for h in range(Hq):
            kvh, hh = h // G, h % G
            t = int(rng.integers(0, lens[s]))
            while any(targets[s, kvh * G + g] == t for g in range(hh)):
                t = int(rng.integers(0, lens[s]))
            targets[s, h] = t
            q[s, h, hh] = 16.0
            kc[tab[s, t // BS], kvh, t % BS, hh] = 2000.0
    o, lse = _run(lay, q, kc, vc)
    for s in range(S):
        for h in range(Hq):
            t = targets[s, h]
            assert torch.equal(o[s, h], vc[tab[s, t // BS], h // G, t % BS]), (s, h, t)


@pytest.mark.parametrize("bad", [0, -3, None])
def test_context_length_outside_range_is_reported(bad):
    """context_lens[s] must lie in [1, max_ctx]; a length outside it (None:
    max_ctx + 1) is reported through the device error word
    (FA_ERR_INVALID_ARG), never silently accepted. The reads stay inside the
    table and the workspace."""
    lay, q, kc, vc = _inputs(4, 100, 4000, 98)
    max_ctx = lay["block_table"].shape[1] * BS
    lens = lay["context_lens"].copy()
    lens[2] = max_ctx + 1 if bad is None else bad
    tab = torch.from_numpy(lay["block_table"]).cuda()
    o, lse = fa.paged_attn_decode(q, kc, vc, tab, torch.from_numpy(lens).cuda(), max_ctx)
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
    assert fa.fa_last_device_error() == fa.FA_OK
    # the other sequences are unaffected
    keep = [0, 1, 3]
    o_ref, l_ref = _oracle_for(keep, lay, q, kc, vc)
    assert_bf16_close(f64(o[keep]), o_ref, O_TOL, "O")
    assert_lse_close(f64(lse[keep]), l_ref)
