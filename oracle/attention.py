"""Plain float64 definitions of exact attention (oracle; test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may use this module. Nothing here is blocked, fused or reordered beyond
what the definitions state; each function cites the passage it restates.

Sources (web pages on FlashAttention and PagedAttention):
  [FA-series]  "FlashAttention系列优化" (johneyzheng.top): sections
               FlashAttentionV1 (safe / online softmax), FlashAttentionV2
               (delayed rescaling), FlashAttentionV3 (block quantisation,
               incoherent processing), PagedAttention (block table, sharing).
  [FA-v1v2v3]  FlashAttention v1/v2/v3 overview (91haoming.cn repost):
               "注意力實現改進" (standard attention: S = QK^T, P = softmax(S),
               O = PV, "Algorithm 0"), "前向傳播改進" (store only the
               logsumexp L = m + log l), "FP8 低精度計算" (per-block scales).
  [FA-relearn] "Flash Attention 再学习" (jibinghu.github.io): 3-pass safe
               softmax, backward by recomputation.

Readings where the pages are silent (each also listed in the design notes):
  * softmax scale is 1/sqrt(d) and is part of S (the pages' torch example
    omits it; every other call here uses it unless ``scale`` is given);
  * L is the natural-log logsumexp of the scaled scores;
  * causal: query i sees key j iff j <= i (N_q == N_k, top-left aligned);
  * the backward is the textbook softmax gradient (the pages' gradient
    formulas were images and did not survive).
"""

from __future__ import annotations

import math

import numpy as np

# Rows of S materialised at once: 1024 x 16384 float64 = 128 MB. Chunking
# rows does not change the definition (every row is independent).
ROW_CHUNK = 1024


def _scale(d: int, scale):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def attention_rows(q_rows, row_idx, k, v, causal, scale=None):
    """Forward definition for selected query rows of one head.

    q_rows: [R, d] float64 queries; row_idx: [R] their positions (used only by
    the causal mask); k, v: [Nk, d]. Returns (O [R, d], L [R], P [R, Nk]).

    [FA-v1v2v3] "注意力實現改進": S = scale * Q K^T, P = softmax(S), O = P V,
    computed the way [FA-relearn] lays out the 3-pass safe softmax:
    pass 1 the row max m, pass 2 l = sum_j exp(S_j - m), pass 3 P = exp(S-m)/l.
    L = m + log l ([FA-v1v2v3] "前向傳播改進").
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q_rows.shape[-1]
    s = _scale(d, scale) * (q_rows @ k.T)
    if causal:
        keys = np.arange(k.shape[0])[None, :]
        s = np.where(keys <= np.asarray(row_idx)[:, None], s, -np.inf)
    if s.shape[1] == 0:                        # no keys at all
        s = np.full((s.shape[0], 1), -np.inf)
        v = np.zeros((1, v.shape[-1]))
    m = s.max(axis=1)                          # pass 1: row max
    # a row that sees no key (possible only for the packed, unequal-length
    # form): P = 0, O = 0, L = -inf
    empty = m == -np.inf
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe[:, None])            # masked entries give exp(-inf) = 0
    l = e.sum(axis=1)                          # pass 2: row sum
    p = e / np.where(empty, 1.0, l)[:, None]   # pass 3: normalise
    o = p @ v
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return o, lse, p


def attention_fwd(q, k, v, causal=False, scale=None):
    """Exact attention forward over [..., N, d] float64 tensors.

    Returns (O [..., N, d], L [..., N]). Leading dims (batch, head) are
    independent problems. Rows are processed in chunks of ``ROW_CHUNK``.
    Pinned by: the tiled online recurrence (oracle.online), rows of P summing
    to 1, constant V, key permutation, uniform logits, golden fixtures.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    q2 = q.reshape(-1, n, d)
    k2 = k.reshape(-1, k.shape[-2], d)
    v2 = v.reshape(-1, v.shape[-2], v.shape[-1])
    o = np.empty(q2.shape[:-1] + (v2.shape[-1],), dtype=np.float64)
    lse = np.empty(q2.shape[:-1], dtype=np.float64)
    for bh in range(q2.shape[0]):
        for r0 in range(0, n, ROW_CHUNK):
            rows = np.arange(r0, min(n, r0 + ROW_CHUNK))
            ob, lb, _ = attention_rows(q2[bh, rows], rows, k2[bh], v2[bh], causal, scale)
            o[bh, rows] = ob
            lse[bh, rows] = lb
    return o.reshape(lead + (n, v2.shape[-1])), lse.reshape(lead + (n,))


def attention_block_sparse(q, k, v, block_mask, causal=False, block=128, scale=None):
    """Exact attention restricted by a block mask, float64, [..., N, d] inputs.

    [FA-v1v2v3] FlashAttention v1 "實現效果" names block-sparse FlashAttention:
    query i sees key j only if the mask keeps their (i // block, j // block)
    pair (and j <= i when causal). block_mask: [nb, nb] or [..., nb, nb] of
    0 / 1. A query that sees no key has O = 0 and L = -inf (as in
    attention_varlen). Returns (O [..., N, d], L [..., N])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    bm = np.broadcast_to(np.asarray(block_mask) != 0, lead + np.asarray(block_mask).shape[-2:])
    qf, kf, vf = q.reshape(-1, n, d), k.reshape(-1, n, d), v.reshape(-1, n, d)
    bmf = bm.reshape(-1, *bm.shape[-2:])
    blk = np.arange(n) // block
    o = np.zeros_like(qf)
    lse = np.full(qf.shape[:2], -np.inf)
    for h in range(qf.shape[0]):
        allowed = bmf[h][blk[:, None], blk[None, :]]
        if causal:
            allowed = allowed & (np.arange(n)[None, :] <= np.arange(n)[:, None])
        s = _scale(d, scale) * (qf[h] @ kf[h].T)
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=1)                          # 3-pass safe softmax, empty rows kept at 0
        empty = m == -np.inf
        e = np.exp(s - np.where(empty, 0.0, m)[:, None])
        l = e.sum(axis=1)
        o[h] = (e / np.where(empty, 1.0, l)[:, None]) @ vf[h]
        with np.errstate(divide="ignore"):
            lse[h] = np.where(empty, -np.inf, m + np.log(np.where(empty, 1.0, l)))
    return o.reshape(q.shape), lse.reshape(lead + (n,))


def attention_varlen(q, k, v, cu_q, cu_k, causal=False, scale=None):
    """Exact attention over a packed batch of variable-length sequences.

    q: [Tq, H, d], k, v: [Tk, Hkv, d] (token-major); cu_q, cu_k: [B + 1]
    sequence starts. Sequence b is queries cu_q[b]..cu_q[b+1]-1 against keys
    cu_k[b]..cu_k[b+1]-1; query head h reads KV head h // (H // Hkv). Every
    (sequence, head) is an independent instance of the forward definition
    ([FA-relearn] "Flash Attention v2", thread blocks over batch and heads).
    The pages define the causal mask only for equal lengths (query i sees keys
    j <= i); for Lq queries and Lk keys it is read aligned to the bottom right,
    query i seeing keys j <= i + Lk - Lq, which is the equal-length mask when
    Lq = Lk and the decoding rule (the newest token sees every cached key) when
    Lq = 1. A query seeing no key has O = 0 and L = -inf.
    Returns (O [Tq, H, d], L [H, Tq]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    cu_q = np.asarray(cu_q)
    cu_k = np.asarray(cu_k)
    tq, h, d = q.shape
    hkv = k.shape[1]
    group = h // hkv
    o = np.zeros_like(q)
    lse = np.full((h, tq), -np.inf)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        lq, lk = q1 - q0, k1 - k0
        if lq == 0:
            continue
        pos = np.arange(lq) + (lk - lq)          # causal position of each query among the keys
        for hh in range(h):
            ob, lb, _ = attention_rows(q[q0:q1, hh], pos, k[k0:k1, hh // group],
                                       v[k0:k1, hh // group], causal, scale)
            o[q0:q1, hh] = ob
            lse[hh, q0:q1] = lb
    return o, lse


def attention_varlen_bwd(q, k, v, do, cu_q, cu_k, causal=False, scale=None, o=None):
    """Gradients of attention_varlen: per (sequence, query head) the textbook
    backward of attention_bwd (D from ``o`` when given, as fa_bwd receives O),
    with a KV head's dK, dV summed over the query heads that read it.
    Returns (dQ [Tq, H, d], dK [Tk, Hkv, d], dV [Tk, Hkv, d])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    tq, h, d = q.shape
    hkv = k.shape[1]
    group = h // hkv
    sc = _scale(d, scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        lq, lk = q1 - q0, k1 - k0
        if lq == 0 or lk == 0:
            continue
        pos = np.arange(lq) + (lk - lq)
        for hh in range(h):
            kh, vh = k[k0:k1, hh // group], v[k0:k1, hh // group]
            qh, gh = q[q0:q1, hh], do[q0:q1, hh]
            o_h, _, p = attention_rows(qh, pos, kh, vh, causal, scale)
            if o is not None:
                o_h = np.asarray(o, dtype=np.float64)[q0:q1, hh]
            dp = gh @ vh.T
            dd = (gh * o_h).sum(axis=1)
            ds = p * (dp - dd[:, None])
            dq[q0:q1, hh] = sc * ds @ kh
            dk[k0:k1, hh // group] += sc * ds.T @ qh
            dv[k0:k1, hh // group] += p.T @ gh
    return dq, dk, dv


def attention_bwd(q, k, v, do, causal=False, scale=None, o=None):
    """Analytic gradients of exact attention, float64.

    Returns (dQ, dK, dV, D) for O = softmax(scale*QK^T [+mask]) V and upstream
    gradient dO. The textbook softmax gradient with P rebuilt from the
    statistics, as [FA-relearn] "backward" and [FA-v1v2v3] (recompute S and P
    from the stored softmax statistics) describe:
        dV = P^T dO
        dP = dO V^T
        D_i = sum_c dO_ic O_ic        (= sum_j P_ij dP_ij)
        dS = P o (dP - D 1^T)
        dQ = scale * dS K,   dK = scale * dS^T Q
    ``o`` (optional) supplies O for D; by default the oracle's own O is used.
    Pinned by central finite differences and the identity for D.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    lead = q.shape[:-2]
    n, d = q.shape[-2:]
    sc = _scale(d, scale)
    q2, k2, v2, do2 = (x.reshape(-1, x.shape[-2], x.shape[-1]) for x in (q, k, v, do))
    o2 = None if o is None else np.asarray(o, dtype=np.float64).reshape(q2.shape[0], n, -1)
    dq = np.zeros_like(q2)
    dk = np.zeros_like(k2)
    dv = np.zeros_like(v2)
    dd = np.empty(q2.shape[:-1], dtype=np.float64)
    for bh in range(q2.shape[0]):
        for r0 in range(0, n, ROW_CHUNK):
            rows = np.arange(r0, min(n, r0 + ROW_CHUNK))
            ob, _, p = attention_rows(q2[bh, rows], rows, k2[bh], v2[bh], causal, scale)
            if o2 is not None:
                ob = o2[bh, rows]
            g = do2[bh, rows]
            dv[bh] += p.T @ g
            dp = g @ v2[bh].T
            di = (g * ob).sum(axis=1)
            ds = p * (dp - di[:, None])
            dq[bh, rows] = sc * (ds @ k2[bh])
            dk[bh] += sc * (ds.T @ q2[bh, rows])
            dd[bh, rows] = di
    return (dq.reshape(q.shape), dk.reshape(k.shape), dv.reshape(v.shape),
            dd.reshape(lead + (n,)))


def round_bf16(x):
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits (1 implicit + 7 stored) and float32's
    exponent range. Used to model tensors that cross the library's interface
    as bf16 (the forward's O, which the backward's D_i = sum_c dO_ic O_ic
    reads). Pinned by torch's float32 -> bfloat16 cast.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))       # a = f * 2^ex, f in [0.5, 1)
    step = np.exp2(ex.astype(np.float64) - 8.0)     # spacing of 8-bit significands
    r = a / step
    rq = np.floor(r)
    frac = r - rq
    rq = rq + ((frac > 0.5) | ((frac == 0.5) & (np.mod(rq, 2.0) == 1.0)))
    return np.where(a > 0, np.sign(x) * rq * step, x)


def combine_partials(o_parts, lse_parts):
    """Merge attention partials computed over disjoint key sets.

    o_parts: [S, ..., d] (each normalised over its own keys), lse_parts:
    [S, ...]. Follows from the definition L = log sum_j exp(S_j)
    ([FA-v1v2v3] "前向傳播改進"): L = log sum_s exp(L_s) and
    O = sum_s exp(L_s - L) O_s. Parts with L_s = -inf (no keys) weigh 0.
    Pinned by: splitting keys into any chunks and merging equals the unsplit
    forward.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m[None])
    tot = w.sum(axis=0)
    lse = m + np.log(tot)
    o = (w[..., None] * o_parts).sum(axis=0) / tot[..., None]
    return o, lse


def paged_decode(q, k_cache, v_cache, block_table, context_lens, block_size=16, scale=None):
    """Single-token decode over a paged KV cache, float64.

    q: [S, Hq, d]; k_cache, v_cache: [P, Hkv, block_size, d] (physical
    blocks); block_table: [S, max_blocks] int; context_lens: [S] int.
    Returns (O [S, Hq, d], L [S, Hq]).

    [FA-series] "PagedAttention": a block table maps each sequence's logical
    blocks to physical blocks; token t of sequence s sits in physical block
    table[s][t // block_size] at slot t % block_size. The gathered keys and
    values then enter the forward definition unmasked (the query is the newest
    token and sees all ctx_s tokens). Query head h reads KV head
    h // (Hq // Hkv) (contiguous grouping). Pinned by: equality with the
    forward on the contiguous sequence, and shared blocks giving identical
    results to private copies.
    """
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache)
    v_cache = np.asarray(v_cache)
    s_n, hq, d = q.shape
    hkv = k_cache.shape[1]
    group = hq // hkv
    o = np.empty((s_n, hq, d), dtype=np.float64)
    lse = np.empty((s_n, hq), dtype=np.float64)
    for s in range(s_n):
        n = int(context_lens[s])
        t = np.arange(n)
        phys = np.asarray(block_table[s])[t // block_size]
        slot = t % block_size
        for h in range(hq):
            kv = h // group
            ks = np.asarray(k_cache[phys, kv, slot], dtype=np.float64)
            vs = np.asarray(v_cache[phys, kv, slot], dtype=np.float64)
            ob, lb, _ = attention_rows(q[s, h][None], np.array([n - 1]), ks, vs, False, scale)
            o[s, h] = ob[0]
            lse[s, h] = lb[0]
    return o, lse


def paged_prefill(q, k_cache, v_cache, block_table, cu_q, context_lens, causal=True,
                  block_size=16, scale=None):
    """A chunk of queries per sequence over a paged KV cache, float64.

    q: [Tq, Hq, d] packed chunks (sequence s owns rows cu_q[s]..cu_q[s+1]-1);
    k_cache, v_cache: [P, Hkv, block_size, d]; block_table: [S, max_blocks];
    context_lens: [S], the tokens in the cache for each sequence, the chunk's
    own tokens included (they are its last Lq positions). The keys of sequence
    s are gathered through the table exactly as in ``paged_decode``
    ([FA-series] "PagedAttention"), then the chunk attends to them with the
    packed form's bottom-right causal rule (``attention_varlen``): chunk query i
    sits at position ctx - Lq + i and sees keys j <= ctx - Lq + i. For Lq = 1
    this is the decode. Returns (O [Tq, Hq, d], L [Hq, Tq])."""
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache)
    v_cache = np.asarray(v_cache)
    hkv = k_cache.shape[1]
    n_seq = len(cu_q) - 1
    lens = [int(context_lens[s]) for s in range(n_seq)]
    cu_k = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    keys = np.zeros((max(int(cu_k[-1]), 1), hkv, q.shape[-1]))
    vals = np.zeros_like(keys)
    for s in range(n_seq):
        t = np.arange(lens[s])
        phys = np.asarray(block_table[s])[t // block_size]
        keys[cu_k[s]:cu_k[s + 1]] = np.asarray(k_cache[phys, :, t % block_size], dtype=np.float64)
        vals[cu_k[s]:cu_k[s + 1]] = np.asarray(v_cache[phys, :, t % block_size], dtype=np.float64)
    return attention_varlen(q, keys, vals, cu_q, cu_k, causal, scale)


# ---------------------------------------------------------------------------
# FP8 (e4m3) block quantisation for the diagnostic FP8 oracle.
# [FA-series] FlashAttentionV3 "block quantization": one scaling factor per
# block of Q, K, V; [FA-v1v2v3] "FP8 低精度計算": per-block rather than
# per-tensor scaling. Reading: blocks are 64 token rows x full d, scale =
# amax / 448 (the largest finite e4m3 value), round to nearest even with
# saturation, scale 1 for an all-zero block.

E4M3_MAX = 448.0


def quantize_e4m3(x):
    """Round float64 values to the nearest e4m3 (FN variant) value, ties to even,
    saturating at +-448. Returns float64 values that are exactly representable.

    e4m3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; normal numbers
    2^(e-7) * (1 + m/8) for e in 1..15 (e=15 only m<=6), subnormals
    2^-6 * m/8. Pinned by torch's float8_e4m3fn cast on the same values.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # exponent of the binade holding a (frexp is exact: a = f * 2^x, f in
    # [0.5, 1)); the subnormal range shares 2^-6's spacing
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex.astype(np.float64) - 1.0, -6.0)
    step = np.exp2(e - 3.0)                    # spacing of representable values
    r = a / step
    # round half to even on the integer grid of multiples of step
    rq = np.floor(r)
    frac = r - rq
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(rq, 2.0) == 1.0))
    rq = rq + up
    y = np.minimum(rq * step, E4M3_MAX)
    return np.sign(x) * y


def fp8_block_quantize(x, block_rows=64):
    """Per-(64-row block) e4m3 quantisation of [..., N, d].

    Returns (values float64 [..., N, d] on the e4m3 grid, scales [..., ceil(N/64)])
    with x ~= values * scale per block. scale = amax(block) / 448, or 1 when
    the block is all zero.
    """
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-2]
    nb = (n + block_rows - 1) // block_rows
    vals = np.empty_like(x)
    scales = np.empty(x.shape[:-2] + (nb,), dtype=np.float64)
    for b in range(nb):
        sl = slice(b * block_rows, min(n, (b + 1) * block_rows))
        blk = x[..., sl, :]
        amax = np.abs(blk).max(axis=(-2, -1))
        s = np.where(amax > 0, amax / E4M3_MAX, 1.0)
        scales[..., b] = s
        vals[..., sl, :] = quantize_e4m3(blk / s[..., None, None])
    return vals, scales


def dequantize_blocks_e4m3(vals, scales, block_rows=64):
    """Inverse of the block scaling: vals * scale of the row's block."""
    vals = np.asarray(vals, dtype=np.float64)
    scales = np.asarray(scales, dtype=np.float64)
    n = vals.shape[-2]
    rs = np.repeat(scales, block_rows, axis=-1)[..., :n]
    return vals * rs[..., None]


def attention_fp8_bwd(q_vals, sq, k_vals, sk, v_vals, sv, R, do, o, causal=False,
                      block_rows=64, scale=None):
    """Gradients of the FP8 attention forward with respect to its unrotated
    inputs Q, K and its input V, float64.

    [FA-series] FlashAttentionV3 / FP低精度 and [FA-v1v2v3] "FP8 低精度計算":
    the FP8 forward attends over Q' = Q R and K' = K R (R orthogonal, so
    Q' K'^T = Q K^T) and V, each quantised to e4m3 with one scale per block of
    64 rows. The pages give no FP8 backward. Reading (the plainest one that
    makes it the backward of that forward): the quantisation is treated as the
    identity (straight through), so the gradients are the textbook ones of
    attention over the dequantised tensors Qh = q_vals * sq, Kh = k_vals * sk,
    Vh = v_vals * sv (blocks of ``block_rows`` rows), with D built from the
    forward's O, then carried back through the rotation:
        (dQh, dKh, dVh) = attention_bwd(Qh, Kh, Vh, dO, o=O)
        dQ = dQh R^T,  dK = dKh R^T,  dV = dVh
    (dQ'/dQ = R: d/dQ f(Q R) = (df/dQ') R^T). Inputs: e4m3 values (float64 on
    the e4m3 grid) [..., N, d], scales [..., ceil(N/64)], R [d, d], dO and O
    [..., N, d]. Returns (dQ, dK, dV). Pinned by torch autograd through the
    rotation and the block dequantisation in tests/test_oracle_pins.py.
    """
    qh = dequantize_blocks_e4m3(q_vals, sq, block_rows)
    kh = dequantize_blocks_e4m3(k_vals, sk, block_rows)
    vh = dequantize_blocks_e4m3(v_vals, sv, block_rows)
    dqh, dkh, dvh, _ = attention_bwd(qh, kh, vh, do, causal=causal, scale=scale, o=o)
    r = np.asarray(R, dtype=np.float64)
    return dqh @ r.T, dkh @ r.T, dvh
