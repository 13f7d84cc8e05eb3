"""Attention with dropout on the probabilities, float64 (oracle; test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may use this module; it shares no code with the CUDA path.

[FA-v1v2v3] (91haoming.cn repost), section FlashAttention v1, "注意力實現改進":
with tiling and recomputation, the matmuls, the softmax, the optional mask and
dropout all run inside one kernel. The pages stop there; what dropout computes and where its random
numbers come from are fixed here (the plainest readings, also listed in the
design notes):

* dropout acts on the attention probabilities: with P = softmax(scale*QK^T
  [+causal mask]) and a keep mask Z (1 = kept),
      O = (P o Z) V / q,      q = 1 - t/256 the keep probability;
  L (the logsumexp) is that of the undropped scores;
* the drop threshold t is a byte: t = floor(256*p + 1/2), 0 <= t <= 255;
  an element is kept iff its random byte is >= t (drop probability t/256);
* the random byte of element (b, h, i, j) of a [B, H, N, N] problem (query
  i, key j) is byte (j mod 16) of the 128-bit output of Philox4x32-10 with
      counter = (j div 16, i, b*H + h, offset),  key = (seed mod 2^32, seed div 2^32),
  bytes numbered from the least significant byte of output word 0 to the most
  significant byte of word 3;
* Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and
  Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC 2011): ten rounds of
  two 32 x 32 -> 64-bit multiplications by 0xD2511F53 and 0xCD9E8D57, the
  bijection (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
  hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)), and the key advanced by the Weyl
  constants (0x9E3779B9, 0xBB67AE85) between rounds.

Backward (textbook, with Z fixed): dV = (P o Z)^T dO / q; dP = Z o (dO V^T) / q;
D_i = sum_c dO_ic O_ic (the dropped O; equals sum_j P_ij dP_ij);
dS = P o (dP - D 1^T); dQ = scale dS K; dK = scale dS^T Q.

Pins: the published Philox4x32-10 known-answer vectors, p = 0 reducing to
the plain forward, keep frequencies per byte position, unbiasedness of O
over offsets (E[O] equals the undropped O), central finite differences of the
backward with the mask fixed, and the identity for D.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import ROW_CHUNK, _scale, attention_rows

_M0, _M1 = 0xD2511F53, 0xCD9E8D57
_W0, _W1 = 0x9E3779B9, 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(counter, key):
    """Philox4x32-10 of uint32 counters [..., 4] under key (k0, k1).

    Salmon et al., SC 2011: per round, (hi0, lo0) = M0 * c0 and (hi1, lo1) =
    M1 * c2 as 64-bit products; the new counter is (hi1 ^ c1 ^ k0, lo1,
    hi0 ^ c3 ^ k1, lo0); then k0 += 0x9E3779B9, k1 += 0xBB67AE85 (mod 2^32).
    Returns uint32 [..., 4]. Pinned by the published known-answer vectors.
    """
    ctr = np.asarray(counter, dtype=np.uint64)
    c0, c1, c2, c3 = (ctr[..., n] & _MASK32 for n in range(4))
    k0 = np.uint64(int(key[0]) & 0xFFFFFFFF)
    k1 = np.uint64(int(key[1]) & 0xFFFFFFFF)
    for _ in range(10):
        p0 = c0 * np.uint64(_M0)          # both factors < 2^32: no wrap
        p1 = c2 * np.uint64(_M1)
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK32)
        k0 = (k0 + np.uint64(_W0)) & _MASK32
        k1 = (k1 + np.uint64(_W1)) & _MASK32
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def drop_threshold(p: float) -> int:
    """The byte threshold t = floor(256 p + 1/2); valid for 0 <= p with t <= 255."""
    if not (p >= 0.0):
        raise ValueError("dropout probability must be >= 0")
    t = int(math.floor(256.0 * p + 0.5))
    if t > 255:
        raise ValueError("dropout probability rounds to 256/256: nothing would be kept")
    return t


def keep_prob(t: int) -> float:
    return 1.0 - t / 256.0


def random_bytes(bh: int, rows, cols, seed: int, offset: int):
    """The random byte of every element (rows[r], cols[c]) of slice bh: uint8 [R, C].

    One Philox4x32-10 output per element (counter (j div 16, i, bh, offset)),
    of which byte j mod 16 is taken: the definition, with no sharing of calls.
    """
    rows = np.asarray(rows, dtype=np.uint64)
    cols = np.asarray(cols, dtype=np.uint64)
    ii, jj = np.meshgrid(rows, cols, indexing="ij")
    ctr = np.stack([jj >> np.uint64(4), ii, np.full_like(ii, bh), np.full_like(ii, offset)], axis=-1)
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    u = (jj & np.uint64(15)).astype(np.int64)
    w = np.take_along_axis(words, (u >> 2)[..., None], axis=-1)[..., 0].astype(np.uint64)
    return ((w >> (np.uint64(8) * (u & 3).astype(np.uint64))) & np.uint64(0xFF)).astype(np.uint8)


def keep_mask(B: int, H: int, N: int, p: float, seed: int, offset: int, rows=None):
    """Keep mask Z [B, H, R, N] (bool) of a [B, H, N, N] problem; rows default to all."""
    t = drop_threshold(p)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    z = np.empty((B, H, len(rows), N), dtype=bool)
    for b in range(B):
        for h in range(H):
            z[b, h] = random_bytes(b * H + h, rows, np.arange(N), seed, offset) >= t
    return z


def _probs(q_rows, row_idx, k, v, causal, scale):
    """(P, L) of selected rows: the plain forward definition (attention_rows)."""
    _, lse, pr = attention_rows(q_rows, row_idx, k, v, causal, scale)
    return pr, lse


def attention_dropout(q, k, v, p, seed, offset, causal=False, scale=None):
    """Forward with dropout on P: q, k, v [B, H, N, d] float64.

    Returns (O [B, H, N, d], L [B, H, N]): O = (P o Z) V / keep_prob, L the
    logsumexp of the undropped (scaled, masked) scores.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, d = q.shape
    t = drop_threshold(p)
    inv_q = 1.0 / keep_prob(t)
    o = np.empty(q.shape[:-1] + (v.shape[-1],))
    lse = np.empty(q.shape[:-1])
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, ROW_CHUNK):
                rows = np.arange(r0, min(N, r0 + ROW_CHUNK))
                pr, lr = _probs(q[b, h, rows], rows, k[b, h], v[b, h], causal, scale)
                z = random_bytes(b * H + h, rows, np.arange(N), seed, offset) >= t
                o[b, h, rows] = ((pr * z) @ v[b, h]) * inv_q
                lse[b, h, rows] = lr
    return o, lse


def attention_dropout_bwd(q, k, v, do, p, seed, offset, causal=False, scale=None, o=None):
    """Gradients of the dropout forward with the mask fixed: (dQ, dK, dV, D).

    dV = (P o Z)^T dO / keep_prob, dP = Z o (dO V^T) / keep_prob,
    D_i = sum_c dO_ic O_ic, dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q.
    ``o`` (optional) supplies the O used for D; by default the oracle's own.
    """
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, H, N, d = q.shape
    sc = _scale(d, scale)
    t = drop_threshold(p)
    inv_q = 1.0 / keep_prob(t)
    if o is None:
        o, _ = attention_dropout(q, k, v, p, seed, offset, causal, scale)
    o = np.asarray(o, dtype=np.float64)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dd = np.empty(q.shape[:-1])
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, ROW_CHUNK):
                rows = np.arange(r0, min(N, r0 + ROW_CHUNK))
                pr, _ = _probs(q[b, h, rows], rows, k[b, h], v[b, h], causal, scale)
                z = random_bytes(b * H + h, rows, np.arange(N), seed, offset) >= t
                g = do[b, h, rows]
                dv[b, h] += ((pr * z).T @ g) * inv_q
                dp = (g @ v[b, h].T) * z * inv_q
                di = (g * o[b, h, rows]).sum(axis=1)
                ds = pr * (dp - di[:, None])
                dq[b, h, rows] = sc * (ds @ k[b, h])
                dk[b, h] += sc * (ds.T @ q[b, h, rows])
                dd[b, h, rows] = di
    return dq, dk, dv, dd
