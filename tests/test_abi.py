"""The C-ABI library loads, exports every symbol include/*.h declare, and
rejects bad arguments before touching a GPU (CPU-only; no compute calls)."""

import ctypes
import os
import re
import subprocess

import pytest

import exact_attention_102_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    """Every function the headers under include/ declare."""
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fa_\w+|paged_\w+)\s*\(", src))
    return names


def test_header_declares_binding_exports():
    assert _declared() == set(fa.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = fa.lib()
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert _declared() <= exported
    # nothing else leaks out of the library (hidden visibility)
    assert {s for s in exported if s.startswith(("fa_", "paged_"))} == _declared()


def test_status_strings():
    assert fa.status_str(fa.FA_OK) == "FA_OK"
    assert fa.status_str(fa.FA_ERR_TIMEOUT) == "FA_ERR_TIMEOUT"
    assert fa.status_str(99) == "FA_ERR_UNKNOWN"


def _p(addr):
    return ctypes.c_void_p(addr)


def test_fwd_rejects_bad_arguments_without_gpu():
    L = fa.lib()
    good = 0x10000
    args = [_p(good)] * 5
    # null pointer
    assert L.fa_fwd(_p(0), *args[1:], 1, 1, 128, 64, 0, None) == fa.FA_ERR_INVALID_ARG
    # misaligned pointer
    assert L.fa_fwd(_p(good + 8), *args[1:], 1, 1, 128, 64, 0, None) == fa.FA_ERR_INVALID_ARG
    # non-positive sizes
    for B, H, N in ((0, 1, 1), (1, 0, 1), (1, 1, 0), (-1, 1, 1)):
        assert L.fa_fwd(*args, B, H, N, 64, 0, None) == fa.FA_ERR_INVALID_ARG
    # unsupported head dim
    for d in (32, 96, 256):
        assert L.fa_fwd(*args, 1, 1, 128, d, 0, None) == fa.FA_ERR_UNSUPPORTED


def test_bwd_rejects_bad_workspace_without_gpu():
    L = fa.lib()
    g = _p(0x10000)
    need = L.fa_bwd_workspace_bytes(2, 3, 100, 64)
    assert need >= 2 * (2 * 3 * 128 * 4) + 4 * (2 * 3 * 100 * 64 * 2) and need % 256 == 0
    assert L.fa_bwd(*([g] * 9), _p(0), need, 2, 3, 100, 64, 1, None) == fa.FA_ERR_WORKSPACE
    assert L.fa_bwd(*([g] * 9), g, need - 1, 2, 3, 100, 64, 1, None) == fa.FA_ERR_WORKSPACE
    assert L.fa_bwd(*([g] * 8), _p(0), g, need, 2, 3, 100, 64, 1, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_bwd(*([g] * 9), g, need, 2, 3, 100, 80, 1, None) == fa.FA_ERR_UNSUPPORTED


def test_decode_rejects_bad_arguments_without_gpu():
    L = fa.lib()
    g = _p(0x10000)
    need = L.paged_attn_decode_workspace_bytes(64, 32, 128, 32768)
    assert need > 0 and need % 256 == 0

    def call(Hq=32, Hkv=8, d=128, bs=16, max_ctx=32768, maxb=2048, ws=g, wsb=None, q=g,
             nphys=1000):
        return L.paged_attn_decode(q, g, g, nphys, g, maxb, g, g, g, 64, Hq, Hkv, d, bs, max_ctx,
                                   ws, need if wsb is None else wsb, None)

    assert call(q=_p(0)) == fa.FA_ERR_INVALID_ARG
    assert call(Hq=30) == fa.FA_ERR_INVALID_ARG            # not a multiple of Hkv
    assert call(d=96) == fa.FA_ERR_UNSUPPORTED
    assert call(bs=32) == fa.FA_ERR_UNSUPPORTED
    assert call(Hq=72) == fa.FA_ERR_UNSUPPORTED             # group of 9 (at most 8)
    assert call(maxb=100) == fa.FA_ERR_INVALID_ARG          # table shorter than max_ctx
    assert call(nphys=0) == fa.FA_ERR_INVALID_ARG
    assert call(ws=_p(0)) == fa.FA_ERR_WORKSPACE
    assert call(wsb=need - 1) == fa.FA_ERR_WORKSPACE


def test_fp8_rejects_bad_arguments_without_gpu():
    L = fa.lib()
    g = _p(0x10000)
    assert L.fa_fp8_prepare(*([g] * 10), 1, 1, 128, 96, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_fp8_prepare(*([g] * 9), _p(0), 1, 1, 128, 128, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd_fp8(*([g] * 8), 1, 1, 128, 96, 0, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_fwd_fp8(*([g] * 8), 1, 1, 0, 128, 0, None) == fa.FA_ERR_INVALID_ARG


def test_debug_probe_rejects_bad_limit_without_gpu():
    L = fa.lib()
    assert L.fa_debug_wait_timeout(0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_debug_wait_timeout(2000000, None) == fa.FA_ERR_INVALID_ARG


def test_decode_noalloc_rejects_oversize_without_gpu():
    L = fa.lib()
    g = _p(0x10000)
    # 64 x 32 x 32 splits x 129 floats = 33.8 MB of partials > the 16 MiB scratch
    assert L.paged_attn_decode_noalloc(g, g, g, 1000, g, 2048, g, g, g, 64, 32, 8, 128, 16,
                                       32768, None) == fa.FA_ERR_WORKSPACE
    assert L.paged_attn_decode_noalloc(g, g, g, 1000, g, 2048, g, g, g, 0, 32, 8, 128, 16,
                                       32768, None) == fa.FA_ERR_INVALID_ARG
    # the shared argument checks come before the scratch-size check: an
    # oversize request with an unsupported block size reports the block size
    assert L.paged_attn_decode_noalloc(g, g, g, 1000, g, 2048, g, g, g, 64, 32, 8, 128, 32,
                                       32768, None) == fa.FA_ERR_UNSUPPORTED


def test_fwd_varlen_rejects_bad_arguments_without_a_gpu():
    """Argument checks run before any CUDA call."""
    L = fa.lib()
    p = ctypes.c_void_p(256)            # aligned, never dereferenced
    null = ctypes.c_void_p(0)
    s = ctypes.c_void_p(0)
    call = lambda *a: L.fa_fwd_varlen(*a)
    ok_args = [p, p, p, p, p, p, p, 2, 64, 128, 128, 8, 2, 128, 1, s]
    args = list(ok_args); args[0] = null
    assert call(*args) == fa.FA_ERR_INVALID_ARG            # NULL q
    args = list(ok_args); args[12] = 3
    assert call(*args) == fa.FA_ERR_INVALID_ARG            # H % Hkv != 0
    args = list(ok_args); args[8] = 200
    assert call(*args) == fa.FA_ERR_INVALID_ARG            # max_seqlen_q > total_q
    args = list(ok_args); args[13] = 96
    assert call(*args) == fa.FA_ERR_UNSUPPORTED            # d not in {64, 128}
    args = list(ok_args); args[7] = 0
    assert call(*args) == fa.FA_ERR_INVALID_ARG            # batch < 1


def test_bwd_varlen_rejects_bad_arguments_without_a_gpu():
    L = fa.lib()
    p = ctypes.c_void_p(256)
    s = ctypes.c_void_p(0)
    args = [p] * 10 + [ctypes.c_size_t(1 << 30), p, p, 2, 64, 64, 128, 128, 8, 2, 128, 1, s]
    a = list(args); a[20] = 96                # d not in {64, 128}
    assert L.fa_bwd_varlen(*a) == fa.FA_ERR_UNSUPPORTED
    a = list(args); a[19] = 3                 # H % Hkv != 0
    assert L.fa_bwd_varlen(*a) == fa.FA_ERR_INVALID_ARG
    a = list(args); a[9] = ctypes.c_void_p(0) # no workspace
    assert L.fa_bwd_varlen(*a) == fa.FA_ERR_WORKSPACE
    assert L.fa_bwd_varlen_workspace_bytes(0, 64, 128, 128, 8, 2, 128) == 0


def test_dropout_rejects_bad_probability_and_head_dim_without_gpu():
    L = fa.lib()
    g = _p(0x10000)
    for p in (-0.1, float("nan"), 1.0, 255.6 / 256):
        assert L.fa_fwd_dropout(*([g] * 5), 1, 2, 128, 64, 0, p, 1, 0, None) == fa.FA_ERR_INVALID_ARG
        assert L.fa_bwd_dropout(*([g] * 10), 1 << 30, 1, 2, 128, 128, 0, p, 1, 0,
                                None) == fa.FA_ERR_INVALID_ARG
    # a valid probability still meets the plain argument checks
    assert L.fa_fwd_dropout(_p(0), *([g] * 4), 1, 2, 128, 64, 0, 0.1, 1, 0,
                            None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd_dropout(*([g] * 5), 1, 2, 128, 80, 0, 0.1, 1, 0, None) == fa.FA_ERR_UNSUPPORTED
    need = L.fa_bwd_workspace_bytes(1, 2, 128, 96)
    assert L.fa_bwd_dropout(*([g] * 10), need, 1, 2, 128, 96, 0, 0.1, 1, 0,
                            None) == fa.FA_ERR_UNSUPPORTED          # d not in {64, 128}
    assert L.fa_bwd_dropout(*([g] * 9), g, 0, 1, 2, 128, 128, 0, 0.1, 1, 0,
                            None) == fa.FA_ERR_WORKSPACE
