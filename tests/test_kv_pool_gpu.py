"""The block pool driving a real paged cache on the GPU: a prompt, a 3-way
fork (parallel samples), appends that trigger copy-on-write of the shared
partial block (applied with fa_kv_copy_blocks), a freed sequence whose blocks
are reused, then paged_attn_decode through the pool's tables compared with
attention over each sequence's logical tokens (oracle.attention_varlen, one
query per sequence, which sees every key)."""

import numpy as np
import pytest
import torch

import oracle
from helpers import O_TOL, assert_bf16_close, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")

HQ, HKV, D, BS = 32, 8, 128, 16


class Cache:
    """Device caches written through the pool, plus each sequence's logical
    K / V rows on the host (what attention should see)."""

    def __init__(self, pool, num_blocks, seed):
        self.pool = pool
        self.k = torch.zeros((num_blocks, HKV, BS, D), dtype=torch.bfloat16, device="cuda")
        self.v = torch.zeros_like(self.k)
        self.rows = {}
        self.g = torch.Generator().manual_seed(seed)

    def append(self, seq, n, check_copy=False):
        start = self.pool.seq_len(seq)
        st, copies = self.pool.append(seq, n)
        assert st == fa.FA_OK
        if copies:
            src = torch.tensor([c[0] for c in copies], dtype=torch.int32, device="cuda")
            dst = torch.tensor([c[1] for c in copies], dtype=torch.int32, device="cuda")
            fa.kv_copy_blocks(self.k, self.v, src, dst)
            torch.cuda.synchronize()
            if check_copy:                     # bit-exact copy of both caches
                for s_, d_ in copies:
                    assert torch.equal(self.k[d_], self.k[s_]) and torch.equal(self.v[d_], self.v[s_])
        table, _ = self.pool.block_tables([seq])
        kr = torch.randn((n, HKV, D), generator=self.g).to(torch.bfloat16)
        vr = torch.randn((n, HKV, D), generator=self.g).to(torch.bfloat16)
        for i in range(n):
            pos = start + i
            blk, slot = table[0][pos // BS], pos % BS
            self.k[blk, :, slot] = kr[i].cuda()
            self.v[blk, :, slot] = vr[i].cuda()
        self.rows.setdefault(seq, [[], []])
        self.rows[seq][0].append(kr)
        self.rows[seq][1].append(vr)
        return copies

    def fork(self, parent, child):
        assert self.pool.fork(parent, child) == fa.FA_OK
        self.rows[child] = [list(self.rows[parent][0]), list(self.rows[parent][1])]

    def free(self, seq):
        assert self.pool.free(seq) == fa.FA_OK
        del self.rows[seq]


def test_decode_through_pool_with_forks_and_copy_on_write():
    pool = fa.KVPool(96, BS, 8, 64)
    c = Cache(pool, 96, 800)
    assert pool.add(0) == fa.FA_OK
    c.append(0, 40)                                   # blocks 0, 1, 2 (block 2 holds 8)
    for child in (1, 2, 3):
        c.fork(0, child)
    assert pool.refcount(2) == 4
    cows = [c.append(s, 5, check_copy=True) for s in (1, 2, 3)]
    assert all(len(x) == 1 and x[0][0] == 2 for x in cows)      # each copied the shared block
    assert c.append(0, 5) == []                       # the last holder writes in place
    c.append(1, 37)                                   # crosses block boundaries
    c.free(2)
    assert pool.add(4) == fa.FA_OK
    c.append(4, 300)                                  # reuses the freed blocks
    seqs = [0, 1, 3, 4]
    table, lens = pool.block_tables(seqs)
    g = torch.Generator().manual_seed(801)
    q = torch.randn((len(seqs), HQ, D), generator=g).to(torch.bfloat16).cuda()
    o, lse = fa.paged_attn_decode(q, c.k, c.v, torch.tensor(table, dtype=torch.int32).cuda(),
                                  torch.tensor(lens, dtype=torch.int32).cuda(), max(lens))
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    kl = [torch.cat(c.rows[s][0]) for s in seqs]
    vl = [torch.cat(c.rows[s][1]) for s in seqs]
    assert [x.shape[0] for x in kl] == lens
    cu_q = np.arange(len(seqs) + 1, dtype=np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o_ref, l_ref = oracle.attention_varlen(f64(q), f64(torch.cat(kl)), f64(torch.cat(vl)), cu_q,
                                           cu_k, causal=True)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    np.testing.assert_allclose(f64(lse), l_ref.T, rtol=1e-3, atol=1e-3)


def test_copy_blocks_rejects_out_of_range_ids():
    k = torch.randn((4, HKV, BS, D), device="cuda").to(torch.bfloat16)
    v = torch.randn_like(k)
    k0, v0 = k.clone(), v.clone()
    src = torch.tensor([0, 7], dtype=torch.int32, device="cuda")
    dst = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    fa.kv_copy_blocks(k, v, src, dst)
    assert fa.fa_last_device_error() == fa.FA_ERR_INVALID_ARG
    assert torch.equal(k[1], k0[0]) and torch.equal(v[1], v0[0])    # the valid pair is copied
    assert torch.equal(k[2], k0[2]) and torch.equal(v[2], v0[2])    # the bad one is skipped
