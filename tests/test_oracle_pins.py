"""Pins for the float64 oracle (CPU only).

Each test ties an oracle function to something other than itself: a
hand-derived golden value, a closed form, an invariant of the definition,
an independent implementation (the tiled online recurrence), a library
routine (torch's float64 attention and autograd, torch's e4m3 cast) or
central finite differences. Chosen so that a dropped scale, a wrong sign or
index, a transposed operand, an off-by-one causal mask or a wrong log base
fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth


def _num(x):
    """Golden JSON numbers: plain floats or closed-form strings."""
    if isinstance(x, str):
        table = {"ln3": math.log(3.0), "ln4": math.log(4.0), "ln8": math.log(8.0),
                 "1/3": 1.0 / 3.0, "1.5ln3": 1.5 * math.log(3.0)}
        return table[x]
    if isinstance(x, list):
        return [_num(y) for y in x]
    return float(x)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- golden ---

@pytest.mark.parametrize("name", ["fwd_two_keys.json", "fwd_causal_three.json"])
def test_fwd_golden(golden_dir, name):
    g = _load(golden_dir, name)
    q, k, v = (np.array(_num(g[x])) for x in ("q", "k", "v"))
    o, lse = oracle.attention_fwd(q, k, v, causal=g["causal"])
    np.testing.assert_allclose(o, np.array(_num(g["O"])), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_num(g["L"])), rtol=0, atol=1e-12)


def test_bwd_golden(golden_dir):
    g = _load(golden_dir, "bwd_two_keys.json")
    q, k, v, do = (np.array(_num(g[x])) for x in ("q", "k", "v", "dO"))
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, do, causal=g["causal"])
    np.testing.assert_allclose(dq, np.array(_num(g["dQ"])), atol=1e-12)
    np.testing.assert_allclose(dk, np.array(_num(g["dK"])), atol=1e-12)
    np.testing.assert_allclose(dv, np.array(_num(g["dV"])), atol=1e-12)


def test_decode_golden(golden_dir):
    g = _load(golden_dir, "decode_table.json")
    o, lse = oracle.paged_decode(np.array(g["q"]), np.array(g["k_cache"]),
                                 np.array(g["v_cache"]), np.array(g["block_table"]),
                                 np.array(g["context_lens"]), block_size=g["block_size"])
    np.testing.assert_allclose(o, np.array(_num(g["O"])), atol=1e-12)
    np.testing.assert_allclose(lse, np.array(_num(g["L"])), atol=1e-12)


def test_e4m3_golden(golden_dir):
    g = _load(golden_dir, "e4m3_rounding.json")
    got = oracle.quantize_e4m3(np.array(g["x"]))
    np.testing.assert_array_equal(got, np.array(g["e4m3"]))


# ------------------------------------------------------------ invariants ---

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    q, k, v = _rand((3, 37, 16), 1)
    rows = np.arange(37)
    _, _, p = oracle.attention_rows(q, rows, k, v, causal)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    if causal:  # nothing above the diagonal
        assert np.all(p[np.triu_indices(37, 1)] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant(causal):
    q, k, _ = _rand((3, 2, 2, 29, 8), 2)
    c = np.linspace(-3, 3, 8)
    v = np.broadcast_to(c, (2, 2, 29, 8))
    o, _ = oracle.attention_fwd(q, k, v, causal=causal)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-12)


def test_key_permutation_invariance():
    q, k, v = _rand((3, 1, 3, 41, 16), 3)
    perm = np.random.default_rng(9).permutation(41)
    o1, l1 = oracle.attention_fwd(q, k, v)
    o2, l2 = oracle.attention_fwd(q, k[..., perm, :], v[..., perm, :])
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_logits(causal):
    """K = 0: every visible key weighs the same, L_i = log(#visible keys)."""
    n, d = 23, 8
    q, v = _rand((2, n, d), 4)
    k = np.zeros((n, d))
    o, lse = oracle.attention_fwd(q, k, v, causal=causal)
    for i in range(n):
        cnt = i + 1 if causal else n
        np.testing.assert_allclose(lse[i], math.log(cnt), atol=1e-12)
        np.testing.assert_allclose(o[i], v[:cnt].mean(axis=0), atol=1e-12)


def test_scale_is_one_over_sqrt_d():
    """Doubling every key equals using scale 2/sqrt(d) (pins where the scale goes)."""
    q, k, v = _rand((3, 17, 32), 5)
    o1, l1 = oracle.attention_fwd(q, 2 * k, v)
    o2, l2 = oracle.attention_fwd(q, k, v, scale=2 / math.sqrt(32))
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_rotation_invariance():
    """(QR)(KR)^T = QK^T for orthogonal R: incoherent processing leaves O, L."""
    q, k, v = _rand((3, 2, 33, 16), 6)
    r = synth.orthogonal_matrix(16, 2003)
    np.testing.assert_allclose(r @ r.T, np.eye(16), atol=1e-12)
    o1, l1 = oracle.attention_fwd(q, k, v)
    o2, l2 = oracle.attention_fwd(q @ r, k @ r, v)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_causal_first_row_and_last_row():
    """Row 0 sees key 0 only; the last row equals the unmasked result."""
    q, k, v = _rand((3, 19, 8), 7)
    oc, lc = oracle.attention_fwd(q, k, v, causal=True)
    on, ln = oracle.attention_fwd(q, k, v, causal=False)
    np.testing.assert_allclose(oc[0], v[0], atol=1e-12)
    np.testing.assert_allclose(lc[0], (q[0] @ k[0]) / math.sqrt(8), atol=1e-12)
    np.testing.assert_allclose(oc[-1], on[-1], atol=1e-12)
    np.testing.assert_allclose(lc[-1], ln[-1], atol=1e-12)
    assert not np.allclose(oc[1:-1], on[1:-1])


# ---------------------------------------- independent implementations ---

def test_tiled_recurrence_matches_page_example():
    """The pages' own tiling demo: N=16, d=8, Br=4, Bc=d, uniform [0,1) inputs
    from seed 456, no scale. The tiled recurrence equals the direct softmax."""
    torch.manual_seed(456)
    n, d = 16, 8
    q = torch.rand((n, d)).double().numpy()
    k = torch.rand((n, d)).double().numpy()
    v = torch.rand((n, d)).double().numpy()
    o_t, l_t = oracle.tiled_online_fwd(q, k, v, br=4, bc=d, scale=1.0)
    o_d, l_d = oracle.attention_fwd(q, k, v, scale=1.0)
    np.testing.assert_allclose(o_t, o_d, atol=1e-12)
    np.testing.assert_allclose(l_t, l_d, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("br,bc", [(1, 1), (4, 8), (16, 16), (7, 13), (64, 32), (200, 200)])
def test_tiled_recurrence_matches_definition(causal, br, bc):
    q, k, v = _rand((3, 131, 16), 11)
    q = q * 3.0  # wide score range so the running max moves a lot
    o_t, l_t = oracle.tiled_online_fwd(q, k, v, br=br, bc=bc, causal=causal)
    o_d, l_d = oracle.attention_fwd(q, k, v, causal=causal)
    np.testing.assert_allclose(o_t, o_d, atol=1e-12)
    np.testing.assert_allclose(l_t, l_d, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_matches_torch_float64(causal):
    """Library routine: torch's scaled_dot_product_attention in float64."""
    q, k, v = _rand((3, 2, 3, 57, 32), 12)
    o, lse = oracle.attention_fwd(q, k, v, causal=causal)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)
    s = (tq @ tk.transpose(-1, -2)) / math.sqrt(32)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(57, 57, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


# ---------------------------------------------------------------- backward ---

@pytest.mark.parametrize("causal", [False, True])
def test_bwd_finite_differences(causal):
    """Central differences of f = sum(O * G), float64, h = 1e-6."""
    n, d = 6, 4
    q, k, v, g = _rand((4, n, d), 13)

    def f(q_, k_, v_):
        o, _ = oracle.attention_fwd(q_, k_, v_, causal=causal)
        return float((o * g).sum())

    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, causal=causal)
    h = 1e-6
    for x, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = [q, k, v]; args_p[which] = xp
            args_m = [q, k, v]; args_m[which] = xm
            num[idx] = (f(*args_p) - f(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_torch_autograd(causal):
    """Library routine: torch autograd through float64 attention."""
    q, k, v, g = _rand((4, 2, 2, 45, 16), 14)
    dq, dk, dv, dd = oracle.attention_bwd(q, k, v, g, causal=causal)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    o.backward(torch.from_numpy(g))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
    # D_i = sum_c dO_ic O_ic equals sum_j P_ij dP_ij
    np.testing.assert_allclose(dd, (g * o.detach().numpy()).sum(-1), atol=1e-11)


def test_bwd_d_identity():
    q, k, v, g = _rand((4, 29, 8), 15)
    o, _ = oracle.attention_fwd(q, k, v, causal=True)
    _, _, p = oracle.attention_rows(q, np.arange(29), k, v, True)
    dp = g @ v.T
    _, _, _, dd = oracle.attention_bwd(q, k, v, g, causal=True)
    np.testing.assert_allclose(dd, (p * dp).sum(axis=1), atol=1e-12)


def test_bwd_row_chunking_is_exact(monkeypatch):
    """Row chunks accumulate dK/dV across chunks: small chunk == one chunk."""
    q, k, v, g = _rand((4, 1, 2, 70, 8), 16)
    ref = oracle.attention_bwd(q, k, v, g, causal=True)
    import oracle.attention as oa
    monkeypatch.setattr(oa, "ROW_CHUNK", 16)
    got = oracle.attention_bwd(q, k, v, g, causal=True)
    for a, b in zip(ref, got):
        np.testing.assert_allclose(a, b, atol=1e-12)


# ----------------------------------------------------- combine / decode ---

@pytest.mark.parametrize("cuts", [[0, 100], [0, 1, 100], [0, 30, 31, 77, 100], list(range(0, 101, 10))])
def test_split_combine_equals_unsplit(cuts):
    q, k, v = _rand((3, 4, 100, 16), 17)
    o_ref, l_ref = oracle.attention_fwd(q[:, :1], k, v)
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.attention_fwd(q[:, :1], k[:, a:b], v[:, a:b])
        parts_o.append(o)
        parts_l.append(l)
    o, l = oracle.combine_partials(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(l, l_ref, atol=1e-12)


def test_combine_ignores_empty_part():
    q, k, v = _rand((3, 2, 50, 8), 18)
    o_ref, l_ref = oracle.attention_fwd(q[:, :1], k, v)
    o, l = oracle.combine_partials(np.stack([o_ref, np.zeros_like(o_ref)]),
                                   np.stack([l_ref, np.full_like(l_ref, -np.inf)]))
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(l, l_ref, atol=1e-12)


def test_decode_equals_forward_on_gathered_sequence():
    """Reduces to the forward definition: a contiguous identity table."""
    hq, hkv, d, bs = 8, 2, 16, 4
    rng = np.random.default_rng(19)
    lens = np.array([1, 4, 5, 37])
    nblk = (lens + bs - 1) // bs
    table = np.zeros((4, nblk.max()), dtype=np.int64)
    start = 0
    for s in range(4):
        table[s, :nblk[s]] = np.arange(start, start + nblk[s])
        start += nblk[s]
    kc = rng.standard_normal((start, hkv, bs, d))
    vc = rng.standard_normal((start, hkv, bs, d))
    q = rng.standard_normal((4, hq, d))
    o, lse = oracle.paged_decode(q, kc, vc, table, lens, block_size=bs)
    for s in range(4):
        blocks = table[s, :nblk[s]]
        for h in range(hq):
            kv = h // (hq // hkv)
            ks = kc[blocks, kv].reshape(-1, d)[:lens[s]]
            vs = vc[blocks, kv].reshape(-1, d)[:lens[s]]
            o_ref, l_ref = oracle.attention_fwd(q[s, h][None], ks, vs)
            np.testing.assert_allclose(o[s, h], o_ref[0], atol=1e-12)
            np.testing.assert_allclose(lse[s, h], l_ref[0], atol=1e-12)


def test_decode_shared_blocks_equal_private_copies():
    """Mapping siblings to one physical block gives the same values as copies."""
    lay = synth.paged_decode_layout(8, 16, 40, 200, seed=5, group=4, share_frac=0.5)
    assert lay["shared_blocks"] > 0
    rng = np.random.default_rng(21)
    P = lay["num_phys"]
    kc = rng.standard_normal((P, 2, 16, 8))
    vc = rng.standard_normal((P, 2, 16, 8))
    q = rng.standard_normal((8, 4, 8))
    o1, l1 = oracle.paged_decode(q, kc, vc, lay["block_table"], lay["context_lens"])
    # private copies: give every logical block its own physical block
    lens = lay["context_lens"]
    nblk = (lens + 15) // 16
    tab2 = np.zeros_like(lay["block_table"])
    kc2, vc2 = [], []
    for s in range(8):
        for b in range(nblk[s]):
            p = lay["block_table"][s, b]
            tab2[s, b] = len(kc2)
            kc2.append(kc[p].copy())
            vc2.append(vc[p].copy())
    o2, l2 = oracle.paged_decode(q, np.stack(kc2), np.stack(vc2), tab2, lens)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ------------------------------------------------------------------ e4m3 ---

def test_e4m3_matches_torch_cast():
    """Library routine: torch.float8_e4m3fn (RNE) on in-range values."""
    rng = np.random.default_rng(22)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 120)])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.quantize_e4m3(x), ref)
    # every representable value maps to itself
    allv = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    allv = allv[np.isfinite(allv)]
    np.testing.assert_array_equal(oracle.quantize_e4m3(allv), allv)


def test_fp8_block_quantize_roundtrip():
    x = _rand((2, 3, 130, 16), 23)[0]
    vals, sc = oracle.fp8_block_quantize(x)
    assert sc.shape == (3, 3)
    # per-block max maps to exactly 448
    for h in range(3):
        for b in range(3):
            blk = vals[h, b * 64:(b + 1) * 64]
            assert np.abs(blk).max() == 448.0
    back = oracle.dequantize_blocks_e4m3(vals, sc)
    # relative error of e4m3 is at most 2^-4 for normal numbers
    big = np.abs(x) > np.repeat(sc, 64, axis=-1)[..., :130, None] * 2 ** -6
    assert np.all(np.abs(back - x)[big] <= np.abs(x)[big] * 2 ** -4 + 1e-15)
    z = np.zeros((1, 64, 4))
    vz, sz = oracle.fp8_block_quantize(z)
    assert sz[0, 0] == 1.0 and np.all(vz == 0)


def test_round_bf16_matches_torch_cast():
    """Library routine: torch's float32 -> bfloat16 cast (RNE)."""
    rng = np.random.default_rng(24)
    x = np.concatenate([rng.standard_normal(50000) * s for s in (1e-30, 1e-3, 1, 7, 1e5)])
    x = x.astype(np.float32).astype(np.float64)           # float32 inputs: one rounding only
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x), ref)
    # worked values: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> 1 (even);
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6 -> 1 + 2^-6 (even)
    np.testing.assert_array_equal(oracle.round_bf16([1 + 2 ** -8, 1 + 3 * 2 ** -8, -3.0, 0.0]),
                                  [1.0, 1 + 2 ** -6, -3.0, 0.0])


# ---------------------------------------------------------------- packed form
def _varlen_case(lens_q, lens_k, H, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], Hkv, d))
    v = rng.standard_normal((cu_k[-1], Hkv, d))
    return q, k, v, cu_q, cu_k


def test_varlen_equal_lengths_match_the_bhnd_forward():
    """Equal lengths, H = Hkv: the packed form is attention_fwd on [B, H, N, d]."""
    B, H, N, d = 3, 2, 37, 8
    q, k, v, cu_q, cu_k = _varlen_case([N] * B, [N] * B, H, H, d, 71)
    for causal in (False, True):
        o, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, causal)
        bhnd = lambda t: t.reshape(B, N, H, d).transpose(0, 2, 1, 3)
        o2, l2 = oracle.attention_fwd(bhnd(q), bhnd(k), bhnd(v), causal)
        np.testing.assert_allclose(bhnd(o), o2, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse.reshape(H, B, N).transpose(1, 0, 2), l2, rtol=0, atol=1e-13)


def test_varlen_brute_force_cross_lengths_gqa_bottom_right():
    """Pure-Python loops over every (sequence, head, query): unequal lengths,
    Hkv < H, bottom-right causal including queries that see no key."""
    lens_q, lens_k = [3, 5, 1, 4], [4, 2, 6, 0]
    H, Hkv, d = 4, 2, 3
    q, k, v, cu_q, cu_k = _varlen_case(lens_q, lens_k, H, Hkv, d, 72)
    for causal in (False, True):
        o, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, causal)
        for b in range(4):
            lq, lk = lens_q[b], lens_k[b]
            for h in range(H):
                for i in range(lq):
                    row = cu_q[b] + i
                    keys = [j for j in range(lk) if not causal or j <= i + lk - lq]
                    if not keys:
                        assert np.all(o[row, h] == 0) and lse[h, row] == -np.inf
                        continue
                    s = [float(q[row, h] @ k[cu_k[b] + j, h // 2]) / math.sqrt(d) for j in keys]
                    mx = max(s)
                    w = [math.exp(x - mx) for x in s]
                    tot = sum(w)
                    exp_o = sum(wi / tot * v[cu_k[b] + j, h // 2] for wi, j in zip(w, keys))
                    np.testing.assert_allclose(o[row, h], exp_o, rtol=1e-12, atol=1e-13)
                    assert abs(lse[h, row] - (mx + math.log(tot))) < 1e-12


def test_varlen_single_query_is_the_decode_rule():
    """Lq = 1, causal: the query sees every key, as the paged decode's newest
    token does (decode definition on an identity block table)."""
    lens_k = [16, 48, 32]
    H, Hkv, d = 8, 2, 16
    q, k, v, cu_q, cu_k = _varlen_case([1, 1, 1], lens_k, H, Hkv, d, 73)
    o, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, causal=True)
    nb = [n // 16 for n in lens_k]
    table = np.zeros((3, max(nb)), dtype=np.int32)
    kc = np.zeros((sum(nb), Hkv, 16, d))
    vc = np.zeros_like(kc)
    p = 0
    for s_ in range(3):
        for j in range(nb[s_]):
            table[s_, j] = p
            rows = slice(cu_k[s_] + 16 * j, cu_k[s_] + 16 * j + 16)
            kc[p] = k[rows].transpose(1, 0, 2)
            vc[p] = v[rows].transpose(1, 0, 2)
            p += 1
    od, ld = oracle.paged_decode(q, kc, vc, table, np.array(lens_k))
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, ld.T, rtol=0, atol=1e-13)


def test_varlen_gqa_equals_repeated_kv_heads():
    lens = [7, 20]
    q, k, v, cu_q, cu_k = _varlen_case(lens, lens, 6, 3, 8, 74)
    o, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, causal=True)
    o2, l2 = oracle.attention_varlen(q, np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1),
                                     cu_q, cu_k, causal=True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, l2)


def test_varlen_against_torch_sdpa():
    """Library routine: torch float64 scaled_dot_product_attention per
    sequence, with an explicit bottom-right mask."""
    lens_q, lens_k = [5, 9], [12, 9]
    q, k, v, cu_q, cu_k = _varlen_case(lens_q, lens_k, 2, 2, 16, 75)
    o, _ = oracle.attention_varlen(q, k, v, cu_q, cu_k, causal=True)
    for b in range(2):
        qs = torch.from_numpy(q[cu_q[b]:cu_q[b + 1]].transpose(1, 0, 2).copy())
        ks = torch.from_numpy(k[cu_k[b]:cu_k[b + 1]].transpose(1, 0, 2).copy())
        vs = torch.from_numpy(v[cu_k[b]:cu_k[b + 1]].transpose(1, 0, 2).copy())
        lq, lk = lens_q[b], lens_k[b]
        mask = torch.from_numpy(np.arange(lk)[None, :] <= np.arange(lq)[:, None] + lk - lq)
        ref = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, attn_mask=mask)
        np.testing.assert_allclose(o[cu_q[b]:cu_q[b + 1]], ref.numpy().transpose(1, 0, 2),
                                   rtol=0, atol=1e-12)


def test_varlen_bwd_equal_lengths_match_bhnd():
    B, H, N, d = 2, 2, 19, 8
    q, k, v, cu_q, cu_k = _varlen_case([N] * B, [N] * B, H, H, d, 76)
    do = np.random.default_rng(77).standard_normal(q.shape)
    bhnd = lambda t: t.reshape(B, N, H, d).transpose(0, 2, 1, 3)
    for causal in (False, True):
        g = oracle.attention_varlen_bwd(q, k, v, do, cu_q, cu_k, causal)
        g2 = oracle.attention_bwd(bhnd(q), bhnd(k), bhnd(v), bhnd(do), causal)
        for a, b_ in zip(g, g2[:3]):
            np.testing.assert_allclose(bhnd(a), b_, rtol=0, atol=1e-13)


def test_varlen_bwd_against_torch_autograd():
    """Library routine: torch float64 autograd through the packed forward with
    unequal lengths, GQA and the bottom-right mask (including rows that see
    no key)."""
    lens_q, lens_k = [6, 3, 9], [4, 8, 9]
    H, Hkv, d = 4, 2, 8
    q, k, v, cu_q, cu_k = _varlen_case(lens_q, lens_k, H, Hkv, d, 78)
    do = np.random.default_rng(79).standard_normal(q.shape)
    tq, tk = [torch.tensor(x, requires_grad=True) for x in (q, k)]
    tv = torch.tensor(v, requires_grad=True)
    outs = []
    for b in range(3):
        lq, lk = lens_q[b], lens_k[b]
        qs = tq[cu_q[b]:cu_q[b + 1]].transpose(0, 1)
        ks = tk[cu_k[b]:cu_k[b + 1]].repeat_interleave(H // Hkv, dim=1).transpose(0, 1)
        vs = tv[cu_k[b]:cu_k[b + 1]].repeat_interleave(H // Hkv, dim=1).transpose(0, 1)
        s = qs @ ks.transpose(1, 2) / math.sqrt(d)
        mask = torch.from_numpy(np.arange(lk)[None, :] <= np.arange(lq)[:, None] + lk - lq)
        s = s.masked_fill(~mask, -torch.inf)
        p = torch.softmax(s, dim=-1).nan_to_num(0.0)       # rows without keys: P = 0
        outs.append((p @ vs).transpose(0, 1))
    o = torch.cat(outs)
    (o * torch.from_numpy(do)).sum().backward()
    g = oracle.attention_varlen_bwd(q, k, v, do, cu_q, cu_k, causal=True)
    for got, ref in zip(g, (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------- paged prefill
def _paged_case(chunks, ctxs, hq, hkv, d, seed, bs=16, share=True):
    rng = np.random.default_rng(seed)
    nb = [-(-c // bs) for c in ctxs]
    n_phys = sum(nb) + 3
    perm = rng.permutation(n_phys)
    table = np.zeros((len(ctxs), max(nb)), dtype=np.int32)
    p = 0
    for s, n in enumerate(nb):
        for j in range(n):
            table[s, j] = perm[p]
            p += 1
    if share and len(ctxs) > 1 and min(nb[:2]) > 1:
        table[1, 0] = table[0, 0]                      # a shared first block
    kc = rng.standard_normal((n_phys, hkv, bs, d))
    vc = rng.standard_normal((n_phys, hkv, bs, d))
    cu_q = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = rng.standard_normal((int(cu_q[-1]), hq, d))
    return q, kc, vc, table, cu_q, np.array(ctxs)


def test_paged_prefill_single_token_chunks_are_the_decode():
    q, kc, vc, tab, cu_q, ctx = _paged_case([1, 1, 1], [40, 16, 77], 8, 2, 16, 90)
    o, lse = oracle.paged_prefill(q, kc, vc, tab, cu_q, ctx)
    od, ld = oracle.paged_decode(q, kc, vc, tab, ctx)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, ld.T, rtol=0, atol=1e-13)


def test_paged_prefill_equals_packed_attention_on_the_gathered_sequence():
    """Contiguous keys gathered by hand (loops over tokens) into the packed
    form; the chunk is the last Lq positions of each context."""
    chunks, ctxs = [5, 20, 3], [40, 20, 70]
    q, kc, vc, tab, cu_q, ctx = _paged_case(chunks, ctxs, 4, 2, 8, 91)
    o, lse = oracle.paged_prefill(q, kc, vc, tab, cu_q, ctx)
    ks, vs = [], []
    for s, n in enumerate(ctxs):
        for t in range(n):
            ks.append(kc[tab[s, t // 16], :, t % 16])
            vs.append(vc[tab[s, t // 16], :, t % 16])
    cu_k = np.concatenate([[0], np.cumsum(ctxs)]).astype(np.int32)
    o2, l2 = oracle.attention_varlen(q, np.stack(ks), np.stack(vs), cu_q, cu_k, causal=True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, l2)


def test_paged_prefill_shared_block_equals_private_copy():
    chunks, ctxs = [7, 9], [35, 50]
    q, kc, vc, tab, cu_q, ctx = _paged_case(chunks, ctxs, 4, 4, 8, 92)
    o, lse = oracle.paged_prefill(q, kc, vc, tab, cu_q, ctx)
    tab2 = tab.copy()
    kc2 = np.concatenate([kc, kc[tab[1, 0]][None]])
    vc2 = np.concatenate([vc, vc[tab[1, 0]][None]])
    tab2[1, 0] = kc.shape[0]                           # sequence 1 gets its own copy
    o2, l2 = oracle.paged_prefill(q, kc2, vc2, tab2, cu_q, ctx)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, l2)


# ------------------------------------------------------------- block sparse
def test_block_sparse_all_ones_is_the_forward():
    rng = np.random.default_rng(95)
    q, k, v = (rng.standard_normal((2, 3, 50, 8)) for _ in range(3))
    for causal in (False, True):
        o, lse = oracle.attention_block_sparse(q, k, v, np.ones((4, 4)), causal, block=16)
        o2, l2 = oracle.attention_fwd(q, k, v, causal)
        np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse, l2, rtol=0, atol=1e-13)


def test_block_sparse_diagonal_mask_is_independent_segments():
    """A block-diagonal mask splits the sequence into independent problems."""
    rng = np.random.default_rng(96)
    q, k, v = (rng.standard_normal((40, 8)) for _ in range(3))
    o, lse = oracle.attention_block_sparse(q, k, v, np.eye(3), False, block=16)
    for a, b in ((0, 16), (16, 32), (32, 40)):
        o2, l2 = oracle.attention_fwd(q[a:b], k[a:b], v[a:b])
        np.testing.assert_allclose(o[a:b], o2, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[a:b], l2, rtol=0, atol=1e-13)


def test_block_sparse_brute_force_with_empty_rows():
    rng = np.random.default_rng(97)
    n, d, blk = 12, 4, 4
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    mask = np.array([[0, 1, 0], [0, 0, 0], [1, 1, 1]])
    for causal in (False, True):
        o, lse = oracle.attention_block_sparse(q, k, v, mask, causal, block=blk)
        for i in range(n):
            keys = [j for j in range(n) if mask[i // blk][j // blk] and (not causal or j <= i)]
            if not keys:
                assert np.all(o[i] == 0) and lse[i] == -np.inf
                continue
            s = [float(q[i] @ k[j]) / math.sqrt(d) for j in keys]
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            np.testing.assert_allclose(o[i], sum(wi / sum(w) * v[j] for wi, j in zip(w, keys)),
                                       rtol=1e-12, atol=1e-13)
            assert abs(lse[i] - (mx + math.log(sum(w)))) < 1e-12


def test_fp8_backward_matches_autograd_through_rotation_and_blocks():
    """attention_fp8_bwd against torch float64 autograd of the FP8 forward's
    function: O = attention((Q R), (K R), V) evaluated at Q = Qh R^T, K = Kh R^T
    (so that Q R = Qh, the dequantised block-scaled codes), with the gradient
    taken with respect to Q, K, V. A sign or transpose slip in the rotation,
    a wrong block scale or a dropped term fails it."""
    import torch

    rng = np.random.default_rng(2024)
    B, H, N, d = 1, 2, 100, 16                       # two 64-row blocks, the second ragged
    R = synth.orthogonal_matrix(d, 77)
    x = {n: rng.standard_normal((B, H, N, d)) * rng.choice([1.0, 8.0], (B, H, N, d), p=[0.95, 0.05])
         for n in ("q", "k", "v", "do")}
    qv, sq = oracle.fp8_block_quantize(x["q"] @ R)
    kv, sk = oracle.fp8_block_quantize(x["k"] @ R)
    vv, sv = oracle.fp8_block_quantize(x["v"])
    assert len(np.unique(sq)) > 2                    # per-block scales really differ
    qh, kh, vh = (oracle.dequantize_blocks_e4m3(a, s) for a, s in ((qv, sq), (kv, sk), (vv, sv)))
    for causal in (False, True):
        o, _ = oracle.attention_fwd(qh, kh, vh, causal=causal)
        dq, dk, dv = oracle.attention_fp8_bwd(qv, sq, kv, sk, vv, sv, R, x["do"], o, causal)
        Rt = torch.from_numpy(R)
        tq = torch.from_numpy(qh @ R.T).requires_grad_(True)
        tk = torch.from_numpy(kh @ R.T).requires_grad_(True)
        tv = torch.from_numpy(vh).requires_grad_(True)
        out = torch.nn.functional.scaled_dot_product_attention(tq @ Rt, tk @ Rt, tv,
                                                               is_causal=causal)
        (out * torch.from_numpy(x["do"])).sum().backward()
        np.testing.assert_allclose(out.detach().numpy(), o, rtol=0, atol=1e-12)
        for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-10)
