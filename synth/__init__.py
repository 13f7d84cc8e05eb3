"""Seeded synthetic inputs shared by the tests, the bench and smoke().

This module draws random numbers and lays out index structures. It holds
none of the attention arithmetic: no scores, softmax, products or
quantisation live here. Both the CUDA path and the float64 oracle consume
what it produces (the oracle as float64 copies of the same bf16 values).

Recipes (shapes and value distributions of the workloads the pages talk
about; all seeded):
  * attention tensors: Q, K, V, dO ~ N(0, 1), drawn as float32 in the fixed
    order Q, K, V, dO from one generator, then rounded to bf16 (RNE);
  * FP8 workload: the same, then each entry independently (probability
    1e-3) multiplied by 50 before bf16 rounding (outliers);
  * orthogonal matrix for incoherent processing: QR of a seeded d x d
    standard-normal float64 matrix with the signs fixed so diag(R) > 0;
  * paged decode: context lengths uniform on [lo, hi] (integers, inclusive);
    sequences in groups of 4 siblings (parallel sampling) that share a
    prefix of full blocks (about 10% of a group's blocks; never the last,
    partial block); physical block ids are a seeded random permutation.
"""

from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "attention_inputs",
    "fp8_inputs",
    "orthogonal_matrix",
    "paged_decode_layout",
    "paged_decode_tensors",
    "to_f64",
]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def attention_inputs(B, H, N, d, seed, device="cpu", with_dout=True, outlier_p=0.0,
                     outlier_scale=50.0):
    """Q, K, V (and dO) as bf16 [B, H, N, d] tensors on ``device``.

    Drawn as float32 N(0,1) in the order Q, K, V, dO from one generator;
    ``outlier_p`` > 0 multiplies each entry independently with that
    probability by ``outlier_scale`` (drawn right after the tensor itself).
    """
    g = _gen(seed, device)
    names = ["q", "k", "v"] + (["do"] if with_dout else [])
    out = {}
    for name in names:
        x = torch.randn((B, H, N, d), generator=g, device=device, dtype=torch.float32)
        if outlier_p > 0:
            sel = torch.rand((B, H, N, d), generator=g, device=device) < outlier_p
            x = torch.where(sel, x * outlier_scale, x)
        out[name] = x.to(torch.bfloat16)
    return out


def packed_inputs(lens_q, lens_k, H, Hkv, d, seed, device="cpu"):
    """A packed variable-length batch: Q [Tq, H, d], K and V [Tk, Hkv, d] bf16
    (token-major, N(0,1) drawn as float32 in the order Q, K, V from one
    generator) and the int32 sequence starts cu_q, cu_k (numpy, [B + 1])."""
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    g = _gen(seed, device)
    out = {}
    for name, shape in (("q", (int(cu_q[-1]), H, d)), ("k", (max(int(cu_k[-1]), 1), Hkv, d)),
                        ("v", (max(int(cu_k[-1]), 1), Hkv, d))):
        out[name] = torch.randn(shape, generator=g, device=device,
                                dtype=torch.float32).to(torch.bfloat16)
    out["cu_q"], out["cu_k"] = cu_q, cu_k
    return out


def packed_lengths(n, lo, hi, seed):
    """n sequence lengths, integers uniform on [lo, hi], seeded."""
    return np.random.default_rng(seed).integers(lo, hi + 1, n).astype(np.int64).tolist()


def fp8_inputs(B, H, N, d, seed, device="cpu"):
    """The FP8 workload: N(0,1) with 0.1% of entries scaled by 50, bf16."""
    return attention_inputs(B, H, N, d, seed, device=device, with_dout=False,
                            outlier_p=1e-3, outlier_scale=50.0)


def orthogonal_matrix(d, seed):
    """Seeded random orthogonal d x d matrix (float64 numpy).

    QR factorisation of a standard-normal matrix, columns' signs chosen so
    that the triangular factor has a positive diagonal (the factorisation is
    then unique, so the matrix is a function of the seed alone).
    """
    rng = np.random.default_rng(int(seed))
    a = rng.standard_normal((d, d))
    qm, rm = np.linalg.qr(a)
    return qm * np.sign(np.diag(rm))[None, :]


def paged_decode_layout(num_seqs, block_size, ctx_lo, ctx_hi, seed, group=4,
                        share_frac=0.10, extra_blocks=0, table_blocks=None):
    """Index structure of a paged KV cache with parallel-sampling sharing.

    Returns dict with numpy arrays:
      context_lens [S] int32, block_table [S, max_blocks] int32 (entries
      past a sequence's last block are 0, a valid id that must never be
      read), num_phys (physical blocks allocated), shared_blocks (logical
      blocks that map to a block some sibling also maps to) and total_blocks.
    Sequences are grouped by ``group`` consecutive ids (siblings sampled from
    one prompt). Siblings share the first s_g full blocks where
    s_g = min(round(share_frac * mean blocks of the group), min blocks of the
    group - 1) (so the last, partially filled block is always private).
    ``extra_blocks`` unused physical blocks are added (spread by the
    permutation) so ids are not dense. The table has ``table_blocks``
    columns (default ceil(ctx_hi / block_size), enough for any length the
    recipe can draw).
    """
    rng = np.random.default_rng(int(seed))
    lens = rng.integers(ctx_lo, ctx_hi + 1, size=num_seqs).astype(np.int64)
    nblk = (lens + block_size - 1) // block_size
    max_blocks = int(nblk.max())
    if table_blocks is None:
        table_blocks = (ctx_hi + block_size - 1) // block_size
    table_blocks = max(int(table_blocks), max_blocks)
    logical = []   # per sequence: list of "allocation ids"
    next_id = 0
    shared = 0
    for g0 in range(0, num_seqs, group):
        members = list(range(g0, min(num_seqs, g0 + group)))
        nb = nblk[members]
        s_g = 0
        if len(members) > 1:
            s_g = int(min(round(share_frac * float(nb.mean())), int(nb.min()) - 1))
            s_g = max(s_g, 0)
        prefix = list(range(next_id, next_id + s_g))
        next_id += s_g
        for s in members:
            own = list(range(next_id, next_id + int(nblk[s]) - s_g))
            next_id += int(nblk[s]) - s_g
            logical.append(prefix + own)
            if len(members) > 1:
                shared += s_g
    num_phys = next_id + int(extra_blocks)
    perm = rng.permutation(num_phys).astype(np.int64)
    table = np.zeros((num_seqs, table_blocks), dtype=np.int32)
    for s, ids in enumerate(logical):
        table[s, :len(ids)] = perm[np.asarray(ids, dtype=np.int64)]
    return {
        "context_lens": lens.astype(np.int32),
        "block_table": table,
        "num_phys": int(num_phys),
        "shared_blocks": int(shared),
        "total_blocks": int(nblk.sum()),
    }


def paged_decode_tensors(num_seqs, Hq, Hkv, d, block_size, num_phys, seed, device="cpu"):
    """q [S, Hq, d] and k/v caches [P, Hkv, block_size, d], bf16 N(0,1)."""
    g = _gen(seed, device)
    q = torch.randn((num_seqs, Hq, d), generator=g, device=device).to(torch.bfloat16)
    shape = (num_phys, Hkv, block_size, d)
    k = torch.empty(shape, dtype=torch.bfloat16, device=device)
    v = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # fill in slabs so no full-size float32 temporary is ever needed
    slab = max(1, (1 << 26) // (Hkv * block_size * d))
    for dst in (k, v):
        for p0 in range(0, num_phys, slab):
            p1 = min(num_phys, p0 + slab)
            dst[p0:p1] = torch.randn((p1 - p0,) + shape[1:], generator=g,
                                     device=device).to(torch.bfloat16)
    return q, k, v


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a (bf16 / fp32) tensor, on the host."""
    return t.detach().to("cpu", torch.float64).numpy()
