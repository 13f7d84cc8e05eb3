"""Paged KV block pool: the reference model (oracle.kv_pool) pinned by a
hand-traced golden scenario and by invariants, and the C++ pool in libfa.so
(fa_kv_* entry points, host only) matched against the model operation by
operation. No GPU is needed; tests/test_kv_pool_gpu.py covers the device copy
and decoding through the pool's tables."""

import ctypes
import json
import os
import random

import pytest

from oracle.kv_pool import INVALID, NO_BLOCKS, OK, KVPoolModel

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_pool_parallel_sampling.json")


def _apply(pool, step):
    op = step["op"]
    if op == "add":
        return pool.add(step["seq"]), None
    if op == "fork":
        return pool.fork(step["parent"], step["child"]), None
    if op == "free":
        return pool.free(step["seq"]), None
    st, copies = pool.append(step["seq"], step["n"])
    return st, [list(c) for c in copies]


def test_model_golden_parallel_sampling():
    g = json.load(open(GOLDEN))
    m = KVPoolModel(**g["pool"])
    for step in g["steps"]:
        st, copies = _apply(m, step)
        assert st == step["status"], step
        if copies is not None:
            assert copies == step["copies"], step
    for s, t in g["final"]["tables"].items():
        assert m.table(int(s)) == t
    for s, n in g["final"]["lens"].items():
        assert m.seq_len(int(s)) == n
    assert m.ref == g["final"]["refcounts"]
    assert m.num_free() == g["final"]["num_free"]


def _random_ops(seed, n_ops, pool):
    rng = random.Random(seed)
    for _ in range(n_ops):
        r = rng.random()
        s = rng.randrange(pool["max_seqs"])
        if r < 0.15:
            yield {"op": "add", "seq": s}
        elif r < 0.3:
            yield {"op": "fork", "parent": s, "child": rng.randrange(pool["max_seqs"])}
        elif r < 0.4:
            yield {"op": "free", "seq": s}
        else:
            yield {"op": "append", "seq": s, "n": rng.choice([0, 1, 1, 1, 2, 3, 7, 16, 33])}


POOL = {"num_blocks": 64, "block_size": 16, "max_seqs": 12, "max_blocks_per_seq": 24}


def test_model_invariants_under_random_operations():
    """Reference counts equal the number of table entries naming the block;
    free blocks are those at zero; tables hold ceil(len / block_size) blocks;
    after an append the sequence's partially filled last block is not shared
    (so the tokens it receives are written only to this sequence)."""
    m = KVPoolModel(**POOL)
    for step in _random_ops(11, 4000, POOL):
        st, _ = _apply(m, step)
        assert st in (OK, INVALID, NO_BLOCKS)
        count = [0] * POOL["num_blocks"]
        for s, (length, blocks) in m.seqs.items():
            assert len(blocks) == -(-length // POOL["block_size"])
            for b in blocks:
                count[b] += 1
        assert count == m.ref
        assert m.num_free() == sum(1 for c in count if c == 0)
        if step["op"] == "append" and st == OK and step["n"] > 0:
            length, blocks = m.seqs[step["seq"]]
            if length % POOL["block_size"]:
                assert m.ref[blocks[-1]] == 1


# ------------------------------------------------------------- C++ pool
fa = pytest.importorskip("exact_attention_102_b200")


class _Native:
    """The C++ pool through the C ABI, shaped like the model."""

    def __init__(self, num_blocks, block_size, max_seqs, max_blocks_per_seq):
        self.p = fa.KVPool(num_blocks, block_size, max_seqs, max_blocks_per_seq)

    def add(self, s):
        return self.p.add(s)

    def fork(self, a, b):
        return self.p.fork(a, b)

    def free(self, s):
        return self.p.free(s)

    def append(self, s, n):
        return self.p.append(s, n)


def test_native_golden_parallel_sampling():
    g = json.load(open(GOLDEN))
    n = _Native(**g["pool"])
    for step in g["steps"]:
        st, copies = _apply(n, step)
        assert st == step["status"], step
        if copies is not None:
            assert copies == step["copies"], step
    seqs = [int(s) for s in g["final"]["tables"]]
    tables, lens = n.p.block_tables(seqs)
    for i, s in enumerate(seqs):
        t = g["final"]["tables"][str(s)]
        assert tables[i][:len(t)] == t and lens[i] == g["final"]["lens"][str(s)]
    assert [n.p.refcount(b) for b in range(8)] == g["final"]["refcounts"]
    assert n.p.num_free() == g["final"]["num_free"]


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_native_matches_model_operation_by_operation(seed):
    m, n = KVPoolModel(**POOL), _Native(**POOL)
    for step in _random_ops(seed, 3000, POOL):
        assert _apply(n, step) == _apply(m, step), step
        assert n.p.num_free() == m.num_free()
    seqs = sorted(m.seqs)
    if seqs:
        tables, lens = n.p.block_tables(seqs)
        for i, s in enumerate(seqs):
            assert lens[i] == m.seq_len(s)
            assert tables[i][:len(m.table(s))] == m.table(s)
    assert [n.p.refcount(b) for b in range(POOL["num_blocks"])] == m.ref


def test_native_rejects_bad_pools():
    L = fa.lib()
    out = ctypes.c_void_p(0)
    assert L.fa_kv_pool_create(0, 16, 4, 4, ctypes.byref(out)) == fa.FA_ERR_INVALID_ARG
    assert L.fa_kv_pool_create(8, 16, 4, 4, None) == fa.FA_ERR_INVALID_ARG
    p = fa.KVPool(4, 16, 2, 4)
    assert p.refcount(99) == -1 and p.seq_len(1) == -1
    assert p.add(5) == fa.FA_ERR_INVALID_ARG
