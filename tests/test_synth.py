"""Seeded input generators: determinism and the structure the recipes state."""

import numpy as np
import torch

import synth


def test_attention_inputs_deterministic_and_bf16():
    a = synth.attention_inputs(1, 2, 33, 64, seed=1000)
    b = synth.attention_inputs(1, 2, 33, 64, seed=1000)
    for k in ("q", "k", "v", "do"):
        assert a[k].dtype == torch.bfloat16 and a[k].shape == (1, 2, 33, 64)
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["q"], a["k"])
    x = synth.to_f64(a["q"])
    assert abs(x.mean()) < 0.1 and 0.9 < x.std() < 1.1


def test_fp8_inputs_have_outliers():
    x = synth.to_f64(synth.fp8_inputs(1, 4, 1024, 128, seed=1003)["q"])
    frac = (np.abs(x) > 8).mean()
    assert 3e-4 < frac < 2e-3


def test_orthogonal_matrix():
    r = synth.orthogonal_matrix(128, 2003)
    np.testing.assert_allclose(r.T @ r, np.eye(128), atol=1e-12)
    np.testing.assert_array_equal(r, synth.orthogonal_matrix(128, 2003))


def test_paged_layout_structure():
    lay = synth.paged_decode_layout(64, 16, 512, 32768, seed=1004)
    lens, tab = lay["context_lens"], lay["block_table"]
    assert lens.min() >= 512 and lens.max() <= 32768
    nblk = (lens + 15) // 16
    used = []
    for s in range(64):
        row = tab[s, :nblk[s]]
        assert row.min() >= 0 and row.max() < lay["num_phys"]
        used.append(row)
    allids = np.concatenate(used)
    # every physical block is used, shared ones exactly by 4 siblings
    ids, cnt = np.unique(allids, return_counts=True)
    assert len(ids) == lay["num_phys"]
    assert set(np.unique(cnt)) <= {1, 4}
    frac = lay["shared_blocks"] / lay["total_blocks"]
    assert 0.07 < frac < 0.13
    # the last (possibly partial) block of every sequence is private
    last = {int(tab[s, nblk[s] - 1]) for s in range(64)}
    assert all(cnt[np.searchsorted(ids, i)] == 1 for i in last)
    # siblings share a prefix
    for g in range(0, 64, 4):
        s_g = 0
        while all(tab[g + j, s_g] == tab[g, s_g] for j in range(4)) and s_g < nblk[g:g + 4].min():
            s_g += 1
        assert s_g >= 1
