"""Tiled one-pass online-softmax forward (oracle cross-check; test infrastructure).

An independent second implementation of the forward, used only to pin
``oracle.attention.attention_fwd``. It follows the recurrence the pages
describe, in their order and notation, written out here from the
description rather than from any printed listing:

  "FlashAttention系列优化" (johneyzheng.top), FlashAttentionV1: the online
  softmax keeps a running max m_j = max(m_{j-1}, x_j) and a running
  denominator d_j = d_{j-1} e^{m_{j-1} - m_j} + e^{x_j - m_j}.
  Same page, FlashAttentionV2: Q blocks form the outer loop, K/V blocks the
  inner loop; the block output is kept unnormalised and rescaled,
  O^(2) = diag(e^{m^(1) - m^(2)}) O^(1) + e^{S^(2) - m^(2)} V^(2), and
  diag(l)^-1 is applied once after the last block.
  "Flash Attention 再学习" (jibinghu.github.io): the 1-pass form with the
  adjustment factor e^{m_{i-1} - m_i} applied to the running sum and output.

Block sizes Br x Bc are free parameters: the result must not depend on them
beyond rounding.
"""

from __future__ import annotations

import math

import numpy as np


def tiled_online_fwd(q, k, v, br, bc, causal=False, scale=None):
    """One head: q [N, d], k [Nk, d], v [Nk, dv] float64 -> (O [N, dv], L [N])."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, d = q.shape
    nk = k.shape[0]
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros((n, v.shape[1]))
    lse = np.zeros(n)
    for i0 in range(0, n, br):                      # outer loop over Q blocks
        qi = q[i0:i0 + br]
        rows = np.arange(i0, i0 + qi.shape[0])
        m = np.full(qi.shape[0], -np.inf)           # running max
        l = np.zeros(qi.shape[0])                   # running sum
        acc = np.zeros((qi.shape[0], v.shape[1]))   # unnormalised output
        for j0 in range(0, nk, bc):                 # inner loop over K/V blocks
            kj = k[j0:j0 + bc]
            vj = v[j0:j0 + bc]
            s = sc * (qi @ kj.T)
            if causal:
                cols = np.arange(j0, j0 + kj.shape[0])
                s = np.where(cols[None, :] <= rows[:, None], s, -np.inf)
            m_new = np.maximum(m, s.max(axis=1))
            # a row that has seen only masked keys keeps m = -inf; its factor
            # and its probabilities are defined as 1 and 0 (no contribution)
            live = np.isfinite(m_new)
            alpha = np.where(live, np.exp(np.where(live, m - m_new, 0.0)), 1.0)
            p = np.where(live[:, None], np.exp(s - np.where(live, m_new, 0.0)[:, None]), 0.0)
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ vj
            m = m_new
        out[i0:i0 + qi.shape[0]] = acc / l[:, None]  # diag(l)^-1 once, at the end
        lse[i0:i0 + qi.shape[0]] = m + np.log(l)
    return out, lse
