"""Pins of the dropout oracle (CPU): the generator against its published
known-answer vectors, the keep mask against the generator's definition and
its statistics, the forward against the plain forward (p = 0) and against its
expectation, the backward against central finite differences."""

import json
import math
import os

import numpy as np
import pytest

from oracle import attention_fwd
from oracle.dropout import (attention_dropout, attention_dropout_bwd, drop_threshold, keep_mask,
                            keep_prob, philox4x32_10, random_bytes)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")


def _hex(ws):
    return [int(w, 16) for w in ws]


def test_philox_known_answer_vectors():
    kat = json.load(open(GOLDEN))["vectors"]
    for v in kat:
        out = philox4x32_10(np.array(_hex(v["counter"]), dtype=np.uint64), _hex(v["key"]))
        assert [int(x) for x in out] == _hex(v["out"])


def test_philox_vectorised_over_leading_dims():
    # the same vectors embedded in a batch under one key give the same words
    kat = json.load(open(GOLDEN))["vectors"]
    ctr = np.array([_hex(v["counter"]) for v in kat] * 3, dtype=np.uint64).reshape(3, 3, 4)
    out = philox4x32_10(ctr, (0, 0))
    ref = philox4x32_10(np.array(_hex(kat[0]["counter"]), dtype=np.uint64), (0, 0))
    assert (out[:, 0] == ref).all()
    assert [int(x) for x in out[1, 0]] == _hex(kat[0]["out"])


def test_random_bytes_follow_the_counter_layout():
    # element (i, j): byte j mod 16 of Philox((j div 16, i, bh, offset), seed words)
    seed, off, bh = 0x0123456789ABCDEF, 7, 5
    rows, cols = np.array([0, 3, 130]), np.array([0, 1, 15, 16, 37, 255])
    got = random_bytes(bh, rows, cols, seed, off)
    for a, i in enumerate(rows):
        for c, j in enumerate(cols):
            w = philox4x32_10(np.array([j // 16, i, bh, off], dtype=np.uint64),
                              (seed & 0xFFFFFFFF, seed >> 32))
            byte = (int(w[(j % 16) // 4]) >> (8 * (j % 4))) & 0xFF
            assert got[a, c] == byte


def test_threshold_rounding_and_limits():
    assert drop_threshold(0.0) == 0
    assert drop_threshold(0.1) == 26            # 25.6 -> 26
    assert drop_threshold(0.5) == 128
    assert drop_threshold(255 / 256) == 255
    with pytest.raises(ValueError):
        drop_threshold(1.0)
    with pytest.raises(ValueError):
        drop_threshold(-0.1)


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_keep_frequency_per_byte_position(p):
    # every byte of the 16 a call yields is uniform: keep rate 1 - t/256 at each
    t = drop_threshold(p)
    z = keep_mask(2, 2, 512, p, seed=1234, offset=0)
    q = keep_prob(t)
    for u in range(16):
        col = z[..., u::16]
        n = col.size
        assert abs(col.mean() - q) < 5 * math.sqrt(q * (1 - q) / n)
    # neighbouring keys and queries are uncorrelated
    zf = z.astype(np.float64)
    for a, b in ((zf[..., :-1], zf[..., 1:]), (zf[..., :-1, :], zf[..., 1:, :])):
        c = np.corrcoef(a.ravel(), b.ravel())[0, 1]
        assert abs(c) < 5 / math.sqrt(a.size)


def test_distinct_streams_for_heads_offsets_and_seeds():
    base = keep_mask(1, 2, 64, 0.5, seed=1, offset=0)
    assert (base[0, 0] != base[0, 1]).mean() > 0.4
    assert (base != keep_mask(1, 2, 64, 0.5, seed=1, offset=1)).mean() > 0.4
    assert (base != keep_mask(1, 2, 64, 0.5, seed=1 + (1 << 32), offset=0)).mean() > 0.4


def _inputs(B, H, N, d, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal((B, H, N, d)) for _ in range(4)]


@pytest.mark.parametrize("causal", [False, True])
def test_p_zero_is_the_plain_forward(causal):
    q, k, v, _ = _inputs(1, 2, 40, 8, 3)
    o, lse = attention_dropout(q, k, v, 0.0, seed=9, offset=0, causal=causal)
    o_ref, l_ref = attention_fwd(q, k, v, causal)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, l_ref)


def test_lse_is_the_undropped_logsumexp():
    q, k, v, _ = _inputs(1, 1, 32, 8, 4)
    _, lse = attention_dropout(q, k, v, 0.5, seed=9, offset=0, causal=True)
    assert np.array_equal(lse, attention_fwd(q, k, v, True)[1])


def test_forward_is_unbiased_over_offsets():
    # E_Z[(P o Z) V / q] = P V; the sample mean over independent offsets stays
    # within 6 standard errors, where Var = sum_j (P_ij V_jc)^2 (1 - q) / q
    q_, k, v, _ = _inputs(1, 1, 24, 4, 5)
    p, n = 0.25, 200
    q = keep_prob(drop_threshold(p))
    o_ref, _ = attention_fwd(q_, k, v)
    mean = np.mean([attention_dropout(q_, k, v, p, 77, off)[0] for off in range(n)], axis=0)
    s = 1.0 / math.sqrt(q_.shape[-1])
    logits = s * q_[0, 0] @ k[0, 0].T
    pr = np.exp(logits - logits.max(1, keepdims=True))
    pr /= pr.sum(1, keepdims=True)
    var = ((pr[:, :, None] * v[0, 0][None]) ** 2).sum(1) * (1 - q) / q
    assert (np.abs(mean[0, 0] - o_ref[0, 0]) <= 6 * np.sqrt(var / n) + 1e-12).all()
    # a missing 1/q would be off by (1 - q) |O|: far outside the bound
    assert (np.abs(mean[0, 0] * q - o_ref[0, 0]) > 6 * np.sqrt(var / n)).any()


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    B, H, N, d = 1, 2, 6, 4
    q, k, v, g = _inputs(B, H, N, d, 6)
    p, seed, off = 0.3, 11, 2

    def f(qq, kk, vv):
        return (attention_dropout(qq, kk, vv, p, seed, off, causal)[0] * g).sum()

    dq, dk, dv, _ = attention_dropout_bwd(q, k, v, g, p, seed, off, causal)
    h = 1e-6
    for x, dx in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            x[idx] += h
            fp = f(q, k, v)
            x[idx] -= 2 * h
            fm = f(q, k, v)
            x[idx] += h
            num[idx] = (fp - fm) / (2 * h)
        assert np.abs(num - dx).max() <= 1e-6 * max(1.0, np.abs(dx).max())


def test_delta_identity_with_dropout():
    # D_i = sum_c dO_ic O_ic equals sum_j P_ij dP_ij with dP = Z o (dO V^T) / q
    q, k, v, g = _inputs(1, 1, 20, 8, 8)
    p, seed, off = 0.2, 5, 0
    o, _ = attention_dropout(q, k, v, p, seed, off)
    _, _, _, dd = attention_dropout_bwd(q, k, v, g, p, seed, off)
    s = 1.0 / math.sqrt(8)
    logits = s * q[0, 0] @ k[0, 0].T
    pr = np.exp(logits - logits.max(1, keepdims=True))
    pr /= pr.sum(1, keepdims=True)
    z = keep_mask(1, 1, 20, p, seed, off)[0, 0]
    dp = z * (g[0, 0] @ v[0, 0].T) / keep_prob(drop_threshold(p))
    assert np.allclose(dd[0, 0], (pr * dp).sum(1), rtol=0, atol=1e-12)


def test_forward_brute_force_loops():
    # tiny causal case in plain loops: one Philox call per element, the
    # softmax by its definition, kept terms summed and divided by q
    B, H, N, d = 1, 2, 20, 4
    q_, k, v, _ = _inputs(B, H, N, d, 12)
    p, seed, off = 0.4, 0xABCDEF0123, 6
    t = drop_threshold(p)
    qk = keep_prob(t)
    o, lse = attention_dropout(q_, k, v, p, seed, off, causal=True)
    s = 1.0 / math.sqrt(d)
    for h in range(H):
        for i in range(N):
            logits = [s * sum(q_[0, h, i, c] * k[0, h, j, c] for c in range(d)) for j in range(i + 1)]
            m = max(logits)
            l = sum(math.exp(x - m) for x in logits)
            acc = [0.0] * d
            for j in range(i + 1):
                w = philox4x32_10(np.array([j // 16, i, h, off], dtype=np.uint64),
                                  (seed & 0xFFFFFFFF, seed >> 32))
                byte = (int(w[(j % 16) // 4]) >> (8 * (j % 4))) & 0xFF
                if byte >= t:
                    for c in range(d):
                        acc[c] += math.exp(logits[j] - m) / l * v[0, h, j, c]
            assert np.allclose(o[0, h, i], [a / qk for a in acc], rtol=0, atol=1e-12)
            assert abs(lse[0, h, i] - (m + math.log(l))) < 1e-12
