"""Reference model of the paged KV-cache block pool (test infrastructure only).

"FlashAttention系列优化" (johneyzheng.top), section PagedAttention: the KV cache
of a sequence is cut into fixed-size blocks; a block table maps the
sequence's logical blocks to physical blocks, which are allocated on demand as
tokens arrive; sequences (parallel samples of one prompt) share physical
blocks by mapping logical blocks to the same physical block; sharing is made
safe by a reference count per physical block and copy-on-write.

The pages give the mechanism, not a policy. This model fixes the plainest one,
and the C++ pool must match it operation for operation:

* the free block handed out is always the lowest-numbered free block;
* ``append(seq, n)`` reserves slots for n tokens after the sequence's last
  token. If its last block is partially filled and shared (reference count
  > 1), that block is copied first (copy-on-write): a new block is taken, the
  pair (old, new) is reported for the device copy, the old block loses one
  reference. Then new blocks are taken for the remaining tokens, in order.
  The operation is all-or-nothing: without enough free blocks (or beyond the
  table width) nothing changes;
* ``fork(parent, child)``: the child maps the parent's blocks (each block
  gains a reference) and has its length;
* ``free(seq)``: each of its blocks loses a reference; a block at zero is free.

Status values follow fa_status: 0 ok, 1 invalid argument, 5 out of blocks.
"""

OK, INVALID, NO_BLOCKS = 0, 1, 5


class KVPoolModel:
    def __init__(self, num_blocks, block_size, max_seqs, max_blocks_per_seq):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_seqs = max_seqs
        self.max_blocks = max_blocks_per_seq
        self.ref = [0] * num_blocks
        self.seqs = {}                      # seq id -> [length, [physical blocks]]

    # -- queries
    def num_free(self):
        return sum(1 for r in self.ref if r == 0)

    def _take(self):
        b = min(i for i, r in enumerate(self.ref) if r == 0)   # lowest free block
        self.ref[b] = 1
        return b

    def seq_len(self, s):
        return self.seqs[s][0] if s in self.seqs else -1

    def table(self, s):
        return list(self.seqs[s][1])

    # -- operations
    def add(self, s):
        if not 0 <= s < self.max_seqs or s in self.seqs:
            return INVALID
        self.seqs[s] = [0, []]
        return OK

    def fork(self, parent, child):
        if parent not in self.seqs or not 0 <= child < self.max_seqs or child in self.seqs:
            return INVALID
        length, blocks = self.seqs[parent]
        for b in blocks:
            self.ref[b] += 1
        self.seqs[child] = [length, list(blocks)]
        return OK

    def free(self, s):
        if s not in self.seqs:
            return INVALID
        for b in self.seqs.pop(s)[1]:
            self.ref[b] -= 1
        return OK

    def append(self, s, n):
        """Returns (status, copies) with copies a list of (src, dst) blocks."""
        if s not in self.seqs or n < 0:
            return INVALID, []
        length, blocks = self.seqs[s]
        new_len = length + n
        need = -(-new_len // self.block_size)
        if need > self.max_blocks:
            return INVALID, []
        cow = n > 0 and length % self.block_size != 0 and self.ref[blocks[-1]] > 1
        if need - len(blocks) + (1 if cow else 0) > self.num_free():
            return NO_BLOCKS, []
        copies = []
        if cow:
            old = blocks[-1]
            new = self._take()
            self.ref[old] -= 1
            blocks[-1] = new
            copies.append((old, new))
        while len(blocks) < need:
            blocks.append(self._take())
        self.seqs[s][0] = new_len
        return OK, copies
