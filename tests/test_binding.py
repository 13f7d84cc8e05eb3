"""The Python binding's argument checks, on CPU: every wrapper accepts tensors
of the documented shapes (and passes the right sizes to the C call) and
rejects mis-shaped ones before anything is launched. The C library and the
device check are replaced by fakes; no compute runs."""

import pytest
import torch

import exact_attention_102_b200 as fa

BF, F32, I32, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.startswith("__"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append((name, args))
            return 4096 if name.endswith("workspace_bytes") else 0
        return call


class _Stream:
    cuda_stream = 0


S0 = _Stream()


@pytest.fixture
def lib(monkeypatch):
    f = _FakeLib()
    monkeypatch.setattr(fa, "lib", lambda: f)
    monkeypatch.setattr(fa, "_require_cuda", lambda t, name: None)
    return f


def _t(shape, dtype=BF):
    return torch.zeros(shape, dtype=dtype)


def _launched(lib, name):
    return [args for n, args in lib.calls if n == name]


def _ints(args):
    return [a for a in args if isinstance(a, int)]


def test_device_check_is_real_without_the_fake():
    with pytest.raises(ValueError, match="CUDA"):
        fa._need(_t((2, 2)), "x", BF)


def test_tensors_on_another_device_are_rejected(monkeypatch):
    """Every tensor must be on the current device (the library launches there
    with raw pointers): one tensor on cuda:1 while cuda:0 is current, or a
    stream of cuda:1, is a ValueError before any launch. CPU tensors stand in
    for CUDA ones through a device map."""
    f = _FakeLib()
    monkeypatch.setattr(fa, "lib", lambda: f)
    monkeypatch.setattr(fa, "_current_device", lambda: 0)
    where = {}
    monkeypatch.setattr(fa, "_require_cuda", lambda t, name: fa._check_device(where[id(t)], name))

    def on(dev, t):
        where[id(t)] = torch.device("cuda", dev)
        return t

    q = on(0, _t((1, 2, 64, 64)))
    k, v = on(0, _t(q.shape)), on(1, _t(q.shape))
    with pytest.raises(ValueError, match="cuda:1"):
        fa.fa_fwd(q, k, v, o=on(0, _t(q.shape)), lse=on(0, _t((1, 2, 64), F32)), stream=S0)
    assert f.calls == []
    v0 = on(0, _t(q.shape))
    with pytest.raises(ValueError, match="cuda:1"):
        fa.fa_fwd(q, k, v0, o=on(1, _t(q.shape)), lse=on(0, _t((1, 2, 64), F32)), stream=S0)
    assert f.calls == []

    class _Stream1:
        cuda_stream = 0
        device = torch.device("cuda", 1)

    with pytest.raises(ValueError, match="stream"):
        fa.fa_fwd(q, k, v0, o=on(0, _t(q.shape)), lse=on(0, _t((1, 2, 64), F32)),
                  stream=_Stream1())
    assert f.calls == []
    fa.fa_fwd(q, k, v0, o=on(0, _t(q.shape)), lse=on(0, _t((1, 2, 64), F32)), stream=S0)
    assert len(f.calls) == 1


# ------------------------------------------------------------------ forward
def test_fwd_shapes(lib):
    q = _t((2, 3, 50, 64))
    o, lse = fa.fa_fwd(q, _t(q.shape), _t(q.shape), causal=True, stream=S0)
    assert o.shape == q.shape and lse.shape == (2, 3, 50)
    (args,) = _launched(lib, "fa_fwd")
    assert _ints(args) == [2, 3, 50, 64, 1]
    fa.fa_fwd(q, _t(q.shape), _t(q.shape), o=_t(q.shape), lse=_t((2, 3, 50), F32), stream=S0)
    bad = [dict(k=_t((2, 3, 49, 64))), dict(v=_t((2, 3, 50, 128))),
           dict(o=_t((2, 3, 49, 64))), dict(lse=_t((2, 3, 49), F32)), dict(lse=_t((2, 3, 50)))]
    for kw in bad:
        args = dict(q=q, k=_t(q.shape), v=_t(q.shape))
        args.update(kw)
        n = len(lib.calls)
        with pytest.raises((ValueError, TypeError)):
            fa.fa_fwd(args.pop("q"), args.pop("k"), args.pop("v"), stream=S0, **args)
        assert len(lib.calls) == n                       # nothing launched


def test_fwd_dropout_and_block_sparse_shapes(lib):
    q = _t((1, 2, 300, 128))
    fa.fa_fwd_dropout(q, _t(q.shape), _t(q.shape), 0.1, 7, 3, stream=S0)
    assert _launched(lib, "fa_fwd_dropout")
    with pytest.raises(ValueError):
        fa.fa_fwd_dropout(q, _t(q.shape), _t(q.shape), 0.1, 7, o=_t((1, 2, 299, 128)), stream=S0)
    nb = 3
    fa.fa_fwd_block_sparse(q, _t(q.shape), _t(q.shape), _t((nb, nb), U8), stream=S0)
    fa.fa_fwd_block_sparse(q, _t(q.shape), _t(q.shape), _t((1, 2, nb, nb), U8), stream=S0)
    strides = [a[6] for a in _launched(lib, "fa_fwd_block_sparse")]
    assert strides == [0, nb * nb]
    for m in (_t((nb, nb + 1), U8), _t((2, 2, nb, nb), U8)):
        with pytest.raises(ValueError):
            fa.fa_fwd_block_sparse(q, _t(q.shape), _t(q.shape), m, stream=S0)
    with pytest.raises(ValueError):
        fa.fa_fwd_block_sparse(q, _t(q.shape), _t(q.shape), _t((nb, nb), U8),
                               lse=_t((1, 2, 301), F32), stream=S0)


# ----------------------------------------------------------------- backward
@pytest.mark.parametrize("dropout", [False, True])
def test_bwd_shapes(lib, dropout):
    shape = (1, 2, 70, 128)
    ins = dict(q=_t(shape), k=_t(shape), v=_t(shape), o=_t(shape), lse=_t(shape[:3], F32),
               do=_t(shape))

    def call(**kw):
        a = dict(ins)
        a.update(kw)
        pos = [a.pop(n) for n in ("q", "k", "v", "o", "lse", "do")]
        if dropout:
            return fa.fa_bwd_dropout(*pos, 0.1, 1, stream=S0, **a)
        return fa.fa_bwd(*pos, stream=S0, **a)

    dq, dk, dv = call()
    assert dq.shape == shape and dq.dtype == F32
    assert len(_launched(lib, "fa_bwd_dropout" if dropout else "fa_bwd")) == 1
    for kw in (dict(k=_t((1, 2, 71, 128))), dict(o=_t((1, 2, 70, 64))), dict(do=_t((1, 1, 70, 128))),
               dict(lse=_t((1, 2, 69), F32)), dict(dq=_t(shape[:3] + (64,), F32)),
               dict(dv=_t(shape, BF))):
        with pytest.raises((ValueError, TypeError)):
            call(**kw)
    assert len(_launched(lib, "fa_bwd_dropout" if dropout else "fa_bwd")) == 1


# ------------------------------------------------------------------- varlen
def _cu(lens):
    return torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=I32)


def test_varlen_shapes(lib):
    lens = [5, 9]
    Tq, H, Hkv, d = 14, 4, 2, 64
    q, k, v = _t((Tq, H, d)), _t((Tq, Hkv, d)), _t((Tq, Hkv, d))
    o, lse = fa.fa_fwd_varlen(q, k, v, _cu(lens), _cu(lens), 9, stream=S0)
    assert lse.shape == (H, Tq)
    (args,) = _launched(lib, "fa_fwd_varlen")
    assert _ints(args)[:8] == [2, 9, Tq, Tq, H, Hkv, d, 0]
    with pytest.raises(ValueError):
        fa.fa_fwd_varlen(q, k, v, _cu(lens), _cu([5, 4, 5]), 9, stream=S0)
    with pytest.raises(ValueError):
        fa.fa_fwd_varlen(q, k, v, _cu(lens), _cu(lens), 9, lse=_t((Tq, H), F32), stream=S0)
    with pytest.raises(ValueError):
        fa.fa_fwd_varlen(q, _t((Tq, Hkv, 128)), _t((Tq, Hkv, 128)), _cu(lens), _cu(lens), 9,
                         stream=S0)
    d128 = 128
    q, k = _t((Tq, H, d128)), _t((Tq, Hkv, d128))
    g = fa.fa_bwd_varlen(q, k, _t(k.shape), _t(q.shape), _t((H, Tq), F32), _t(q.shape),
                         _cu(lens), _cu(lens), 9, 9, stream=S0)
    assert [t.shape for t in g] == [q.shape, k.shape, k.shape]
    assert len(_launched(lib, "fa_bwd_varlen")) == 1
    for kw in (dict(dk=_t(q.shape, F32)), dict(dq=_t(k.shape, F32))):
        with pytest.raises(ValueError):
            fa.fa_bwd_varlen(q, k, _t(k.shape), _t(q.shape), _t((H, Tq), F32), _t(q.shape),
                             _cu(lens), _cu(lens), 9, 9, stream=S0, **kw)
    with pytest.raises(ValueError):
        fa.fa_bwd_varlen(q, k, _t(k.shape), _t(q.shape), _t((Tq, H), F32), _t(q.shape),
                         _cu(lens), _cu(lens), 9, 9, stream=S0)


# ----------------------------------------------------- paged cache, pool copy
def test_paged_prefill_and_decode_shapes(lib):
    P, Hkv, bs, d = 40, 2, 16, 128
    kc, vc = _t((P, Hkv, bs, d)), _t((P, Hkv, bs, d))
    chunks, ctx = [3, 5], torch.tensor([20, 40], dtype=I32)
    q = _t((8, 8, d))
    tab = _t((2, 4), I32)
    fa.fa_paged_prefill(q, kc, vc, tab, _cu(chunks), ctx, 5, stream=S0)
    (args,) = _launched(lib, "fa_paged_prefill")
    assert _ints(args) == [P, 4, 2, 5, 8, 8, Hkv, d, bs, 1]
    for t2, c2, v2 in ((_t((3, 4), I32), ctx, vc), (tab, ctx[:1], vc), (tab, ctx, _t((P, Hkv, bs, 64)))):
        with pytest.raises(ValueError):
            fa.fa_paged_prefill(q, kc, v2, t2, _cu(chunks), c2, 5, stream=S0)
    qd = _t((2, 8, d))
    o, lse = fa.paged_attn_decode(qd, kc, vc, tab, ctx, 64, stream=S0)
    assert lse.shape == (2, 8)
    o2, l2 = fa.paged_attn_decode(qd, kc, vc, tab, ctx, 64, want_lse=False, stream=S0)
    assert l2 is None
    assert len(_launched(lib, "paged_attn_decode")) == 2
    for kw in (dict(o=_t((2, 8, 64))), dict(lse=_t((8, 2), F32))):
        with pytest.raises(ValueError):
            fa.paged_attn_decode(qd, kc, vc, tab, ctx, 64, stream=S0, **kw)
    with pytest.raises(ValueError):
        fa.paged_attn_decode(qd, kc, vc, _t((3, 4), I32), ctx, 64, stream=S0)
    fa.paged_attn_decode_noalloc(qd, kc, vc, tab, ctx, 64, _t(qd.shape), _t((2, 8), F32),
                                 stream=S0)
    assert len(_launched(lib, "paged_attn_decode_noalloc")) == 1
    with pytest.raises(ValueError):
        fa.paged_attn_decode_noalloc(qd, kc, vc, tab, ctx, 64, _t((2, 8, 64)), stream=S0)


def test_kv_copy_blocks_shapes(lib):
    kc = _t((10, 2, 16, 128))
    src = torch.tensor([1, 2], dtype=I32)
    fa.kv_copy_blocks(kc, _t(kc.shape), src, torch.tensor([3, 4], dtype=I32), stream=S0)
    (args,) = _launched(lib, "fa_kv_copy_blocks")
    assert _ints(args) == [10, 2, 2 * 16 * 128 * 2]
    with pytest.raises(ValueError):
        fa.kv_copy_blocks(kc, _t(kc.shape), src, torch.tensor([3], dtype=I32), stream=S0)
    with pytest.raises(ValueError):
        fa.kv_copy_blocks(kc, _t((9, 2, 16, 128)), src, src, stream=S0)


# ---------------------------------------------------------------------- FP8
def test_fp8_shapes(lib):
    B, H, N, d = 1, 2, 130, 128
    q = _t((B, H, N, d))
    out = fa.fa_fp8_prepare(q, _t(q.shape), _t(q.shape), _t((d, d), F32), stream=S0)
    assert [t.shape for t in out[3:]] == [(B, H, 3)] * 3
    with pytest.raises(ValueError):
        fa.fa_fp8_prepare(q, _t(q.shape), _t(q.shape), _t((d, 64), F32), stream=S0)
    q8 = _t(q.shape, U8)
    sc = [_t((B, H, 3), F32) for _ in range(3)]
    o, lse = fa.fa_fwd_fp8(q8, _t(q.shape, U8), _t(q.shape, U8), *sc, stream=S0)
    assert o.dtype == BF and lse.shape == (B, H, N)
    with pytest.raises(ValueError):
        fa.fa_fwd_fp8(q8, _t(q.shape, U8), _t(q.shape, U8), sc[0], sc[1], _t((B, H, 2), F32),
                      stream=S0)
    with pytest.raises(ValueError):
        fa.fa_fwd_fp8(q8, _t((B, H, N - 1, d), U8), _t(q.shape, U8), *sc, stream=S0)
