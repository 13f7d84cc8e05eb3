"""fa_fwd_block_sparse (128 x 128 block mask) vs the float64 oracle's
attention_block_sparse, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import O_TOL, assert_bf16_close, assert_lse_close, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _mask(nb, density, seed, shape=None):
    rng = np.random.default_rng(seed)
    m = (rng.random(shape if shape else (nb, nb)) < density).astype(np.uint8)
    return m


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_bit_matches_fa_fwd(causal):
    """Every block kept: the same arithmetic as fa_fwd, block by block."""
    x = synth.attention_inputs(1, 3, 700, 128, 950 + causal, device="cuda", with_dout=False)
    nb = 6
    o, lse = fa.fa_fwd_block_sparse(x["q"], x["k"], x["v"],
                                    torch.ones((nb, nb), dtype=torch.uint8, device="cuda"),
                                    causal=causal)
    o2, l2 = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("density", [0.3, 0.7])
def test_random_masks(density, d, causal):
    """Per-head masks with empty query blocks (O = 0, L = -inf) and tiles of
    a CTA that see different key blocks; N not a multiple of 128."""
    B, H, N = 1, 3, 1000
    nb = 8
    x = synth.attention_inputs(B, H, N, d, 960 + d, device="cuda", with_dout=False)
    m = _mask(nb, density, int(density * 10) + d + causal, (B, H, nb, nb))
    m[0, 0, 3, :] = 0                                # a query block with no key block
    o, lse = fa.fa_fwd_block_sparse(x["q"], x["k"], x["v"], torch.from_numpy(m).cuda(),
                                    causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, l_ref = oracle.attention_block_sparse(f64(x["q"]), f64(x["k"]), f64(x["v"]), m, causal)
    empty = np.isneginf(l_ref)
    got_l = f64(lse)
    assert np.all(np.isneginf(got_l[empty])) and np.all(f64(o)[empty] == 0)
    assert_bf16_close(f64(o), o_ref, O_TOL, "O")
    assert_lse_close(got_l[~empty], l_ref[~empty])


def test_shared_mask_long_sequence_sampled():
    """One mask for all heads, N = 8192, d = 128, causal, density 0.25."""
    B, H, N, d = 1, 4, 8192, 128
    nb = N // 128
    x = synth.attention_inputs(B, H, N, d, 970, device="cuda", with_dout=False)
    m = _mask(nb, 0.25, 971)
    np.fill_diagonal(m, 1)                            # every query sees its own block
    o, lse = fa.fa_fwd_block_sparse(x["q"], x["k"], x["v"], torch.from_numpy(m).cuda(),
                                    causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    rng = np.random.default_rng(972)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 150, replace=False)]))
    for h in (0, 3):
        o_ref, l_ref = oracle.attention_block_sparse(f64(x["q"][0, h]), f64(x["k"][0, h]),
                                                     f64(x["v"][0, h]), m, causal=True)
        assert_bf16_close(f64(o[0, h, rows]), o_ref[rows], O_TOL, "O")
        assert_lse_close(f64(lse[0, h, rows]), l_ref[rows])
