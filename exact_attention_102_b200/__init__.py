"""Python binding of libfa.so, the B200 (sm_100a) exact-attention C ABI.

Argument marshalling only: each function checks dtypes / shapes / devices,
allocates outputs with torch (device memory is PyTorch's job here), and calls
the C entry point of the same name on the current CUDA stream. Every step of
the computation runs in the library's CUDA kernels. There is no CPU path: a
missing or unloadable library raises.

Functions (see include/fa.h for the contract of each):
    fa_fwd, fa_bwd, fa_bwd_workspace_bytes, paged_attn_decode,
    paged_attn_decode_workspace_bytes, fa_fp8_prepare, fa_fwd_fp8,
    fa_last_device_error, fa_debug_wait_timeout
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_LAUNCH = 3
FA_ERR_TIMEOUT = 4
FA_ERR_WORKSPACE = 5

# the symbols include/fa.h declares
EXPORTS = (
    "fa_status_str", "fa_fwd", "fa_bwd_workspace_bytes", "fa_bwd",
    "paged_attn_decode_workspace_bytes", "paged_attn_decode", "fa_fp8_prepare",
    "fa_fwd_fp8", "fa_last_device_error", "fa_debug_wait_timeout",
    "paged_attn_decode_noalloc", "fa_bwd_time_main_pass", "fa_fwd_varlen",
    "fa_bwd_varlen_workspace_bytes", "fa_bwd_varlen",
    "fa_kv_pool_create", "fa_kv_pool_destroy", "fa_kv_seq_add", "fa_kv_seq_fork", "fa_kv_seq_free",
    "fa_kv_seq_append", "fa_kv_num_free", "fa_kv_refcount", "fa_kv_seq_len", "fa_kv_block_table",
    "fa_kv_copy_blocks", "fa_paged_prefill", "fa_fwd_block_sparse", "fa_fwd_dropout",
    "fa_bwd_dropout", "fa_bwd_fp8",
)


class FAError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfa.so (built in-tree by exact_attention_102_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m exact_attention_102_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, ci, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.fa_status_str.restype = ctypes.c_char_p
    L.fa_status_str.argtypes = [ci]
    L.fa_fwd.restype = ci
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, vp]
    L.fa_bwd_workspace_bytes.restype = sz
    L.fa_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci]
    L.fa_bwd.restype = ci
    L.fa_bwd.argtypes = [vp] * 9 + [vp, sz, ci, ci, ci, ci, ci, vp]
    L.paged_attn_decode_workspace_bytes.restype = sz
    L.paged_attn_decode_workspace_bytes.argtypes = [ci, ci, ci, ci]
    L.paged_attn_decode.restype = ci
    L.paged_attn_decode.argtypes = [vp, vp, vp, ci, vp, ci, vp, vp, vp, ci, ci, ci, ci, ci, ci,
                                    vp, sz, vp]
    L.paged_attn_decode_noalloc.restype = ci
    L.paged_attn_decode_noalloc.argtypes = [vp, vp, vp, ci, vp, ci, vp, vp, vp, ci, ci, ci, ci,
                                            ci, ci, vp]
    L.fa_fp8_prepare.restype = ci
    L.fa_fp8_prepare.argtypes = [vp] * 10 + [ci, ci, ci, ci, vp]
    L.fa_fwd_fp8.restype = ci
    L.fa_fwd_fp8.argtypes = [vp] * 8 + [ci, ci, ci, ci, ci, vp]
    L.fa_bwd_fp8.restype = ci
    L.fa_bwd_fp8.argtypes = [vp] * 14 + [sz] + [ci] * 5 + [vp]
    L.fa_last_device_error.restype = ci
    L.fa_last_device_error.argtypes = [vp]
    L.fa_bwd_time_main_pass.restype = ci
    L.fa_bwd_time_main_pass.argtypes = [vp, vp]
    L.fa_fwd_varlen.restype = ci
    L.fa_fwd_varlen.argtypes = [vp] * 7 + [ci] * 8 + [vp]
    L.fa_bwd_varlen_workspace_bytes.restype = sz
    L.fa_bwd_varlen_workspace_bytes.argtypes = [ci] * 7
    L.fa_bwd_varlen.restype = ci
    L.fa_bwd_varlen.argtypes = [vp] * 10 + [sz, vp, vp] + [ci] * 9 + [vp]
    pi = ctypes.POINTER(ci)
    L.fa_kv_pool_create.restype = ci
    L.fa_kv_pool_create.argtypes = [ci, ci, ci, ci, ctypes.POINTER(vp)]
    L.fa_kv_pool_destroy.restype = None
    L.fa_kv_pool_destroy.argtypes = [vp]
    for name in ("fa_kv_seq_add", "fa_kv_seq_free"):
        getattr(L, name).restype = ci
        getattr(L, name).argtypes = [vp, ci]
    L.fa_kv_seq_fork.restype = ci
    L.fa_kv_seq_fork.argtypes = [vp, ci, ci]
    L.fa_kv_seq_append.restype = ci
    L.fa_kv_seq_append.argtypes = [vp, ci, ci, pi, pi, pi]
    L.fa_kv_num_free.restype = ci
    L.fa_kv_num_free.argtypes = [vp]
    for name in ("fa_kv_refcount", "fa_kv_seq_len"):
        getattr(L, name).restype = ci
        getattr(L, name).argtypes = [vp, ci]
    L.fa_kv_block_table.restype = ci
    L.fa_kv_block_table.argtypes = [vp, pi, ci, pi, ci, pi]
    L.fa_fwd_block_sparse.restype = ci
    L.fa_fwd_block_sparse.argtypes = [vp] * 6 + [ctypes.c_longlong] + [ci] * 5 + [vp]
    L.fa_paged_prefill.restype = ci
    L.fa_paged_prefill.argtypes = [vp, vp, vp, ci, vp, ci, vp, vp, vp, vp] + [ci] * 8 + [vp]
    L.fa_kv_copy_blocks.restype = ci
    L.fa_kv_copy_blocks.argtypes = [vp, vp, ci, vp, vp, ci, ctypes.c_longlong, vp]
    L.fa_debug_wait_timeout.restype = ci
    L.fa_debug_wait_timeout.argtypes = [ctypes.c_uint, vp]
    L.fa_fwd_dropout.argtypes = [vp] * 5 + [ci] * 5 + [ctypes.c_float, ctypes.c_ulonglong,
                                                        ctypes.c_uint, vp]
    L.fa_bwd_dropout.argtypes = [vp] * 10 + [sz] + [ci] * 5 + [ctypes.c_float, ctypes.c_ulonglong,
                                                               ctypes.c_uint, vp]
    _lib = L
    return L


def status_str(status: int) -> str:
    return lib().fa_status_str(int(status)).decode()


def _check(fn, status):
    if status != FA_OK:
        raise FAError(fn, status)


def _current_device():
    return torch.cuda.current_device()


def _stream(stream=None):
    """The cudaStream_t to launch on: the current stream of the current device,
    or `stream`, which must belong to the current device."""
    if stream is None:
        stream = torch.cuda.current_stream()
    dev = getattr(stream, "device", None)
    if isinstance(dev, torch.device) and dev.type == "cuda" and dev.index != _current_device():
        raise ValueError(f"stream belongs to cuda:{dev.index}, but the current device is "
                         f"cuda:{_current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check_device(dev, name):
    """The library launches on the current device and encodes raw pointers, so
    every tensor it touches must live on that device (one tensor elsewhere
    would be read through another GPU's address space)."""
    if dev.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    cur = _current_device()
    if dev.index != cur:
        raise ValueError(f"{name} is on cuda:{dev.index}, but the current device is cuda:{cur}; "
                         "run the call under torch.cuda.device(...) of its tensors")


def _require_cuda(t, name):
    _check_device(t.device, name)


def _need(t, name, dtype, ndim=None, shape=None):
    """Type, dtype, rank, exact shape (when given), contiguity, then device.

    The library receives raw pointers and cannot see sizes, so every tensor it
    reads or writes is checked here against the sizes passed with it."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    _require_cuda(t, name)


def _need_workspace(t):
    if not isinstance(t, torch.Tensor):
        raise TypeError("workspace must be a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _require_cuda(t, "workspace")


def _need_lengths(t, name, n):
    """int32 length / offset array with exactly n entries."""
    _need(t, name, torch.int32, 1, (n,))


def fa_fwd(q, k, v, causal=False, o=None, lse=None, stream=None):
    """O, L = attention forward on bf16 [B, H, N, d] tensors; L is fp32 [B, H, N]."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, shape=q.shape)
    _need(v, "v", torch.bfloat16, shape=q.shape)
    B, H, N, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    _check("fa_fwd", lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                  B, H, N, d, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_fwd_dropout(q, k, v, p_drop, seed, offset=0, causal=False, o=None, lse=None, stream=None):
    """fa_fwd with dropout on P (keep mask from Philox4x32-10 keyed by seed,
    counter word 3 = offset); O = (P o Z) V / keep_prob, L undropped."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, shape=q.shape)
    _need(v, "v", torch.bfloat16, shape=q.shape)
    B, H, N, d = q.shape
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(o, "o", torch.bfloat16, shape=q.shape)
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    _check("fa_fwd_dropout", lib().fa_fwd_dropout(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(bool(causal)),
        float(p_drop), int(seed) & (2**64 - 1), int(offset) & 0xFFFFFFFF, _stream(stream)))
    return o, lse


def fa_bwd_dropout(q, k, v, o, lse, do, p_drop, seed, offset=0, causal=False, dq=None, dk=None,
                   dv=None, workspace=None, stream=None):
    """Gradients of fa_fwd_dropout (same p_drop, seed, offset): fp32 dQ, dK, dV."""
    _need(q, "q", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o), ("do", do)):
        _need(t, n, torch.bfloat16, shape=q.shape)
    B, H, N, d = q.shape
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dv is None else dv
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, n, torch.float32, shape=q.shape)
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8,
                                device=q.device)
    _need_workspace(workspace)
    _check("fa_bwd_dropout", lib().fa_bwd_dropout(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(workspace), workspace.numel() * workspace.element_size(), B, H, N, d,
        int(bool(causal)), float(p_drop), int(seed) & (2**64 - 1), int(offset) & 0xFFFFFFFF,
        _stream(stream)))
    return dq, dk, dv


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal=False, o=None,
                  lse=None, stream=None):
    """O, L for a packed batch: q [Tq, H, d], k / v [Tk, Hkv, d] bf16 (token-major),
    cu_seqlens int32 [batch + 1] on the device; L is fp32 [H, Tq]. Causal is
    aligned to the bottom right (query i of Lq sees keys j <= i + Lk - Lq)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, shape=k.shape)
    if k.shape[2] != q.shape[2]:
        raise ValueError("k and v must be [Tk, Hkv, d] with q's d")
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    if cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q must have batch + 1 >= 2 entries")
    _need_lengths(cu_seqlens_k, "cu_seqlens_k", cu_seqlens_q.numel())
    Tq, H, d = q.shape
    Tk, Hkv, _ = k.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    _need(lse, "lse", torch.float32, shape=(H, Tq))
    _check("fa_fwd_varlen",
           lib().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                               _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, int(max_seqlen_q),
                               Tq, Tk, H, Hkv, d, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_bwd_varlen_workspace_bytes(batch, max_seqlen_q, total_q, total_k, H, Hkv, d):
    return int(lib().fa_bwd_varlen_workspace_bytes(batch, max_seqlen_q, total_q, total_k, H, Hkv,
                                                   d))


def fa_bwd_varlen(q, k, v, o, lse, do, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                  causal=False, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ [Tq, H, d], dK, dV [Tk, Hkv, d] (fp32) of fa_fwd_varlen's attention."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, shape=k.shape)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    _need(do, "do", torch.bfloat16, shape=q.shape)
    if k.shape[2] != q.shape[2]:
        raise ValueError("k and v must be [Tk, Hkv, d] with q's d")
    Tq, H, d = q.shape
    Tk, Hkv, _ = k.shape
    _need(lse, "lse", torch.float32, shape=(H, Tq))
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    if cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q must have batch + 1 >= 2 entries")
    _need_lengths(cu_seqlens_k, "cu_seqlens_k", cu_seqlens_q.numel())
    batch = cu_seqlens_q.numel() - 1
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty(k.shape, dtype=torch.float32, device=q.device) if dv is None else dv
    _need(dq, "dq", torch.float32, shape=q.shape)
    _need(dk, "dk", torch.float32, shape=k.shape)
    _need(dv, "dv", torch.float32, shape=k.shape)
    need = fa_bwd_varlen_workspace_bytes(batch, max_seqlen_q, Tq, Tk, H, Hkv, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace)
    _check("fa_bwd_varlen",
           lib().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                               _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(),
                               _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, int(max_seqlen_q),
                               int(max_seqlen_k), Tq, Tk, H, Hkv, d, int(bool(causal)),
                               _stream(stream)))
    return dq, dk, dv


def fa_fwd_block_sparse(q, k, v, block_mask, causal=False, o=None, lse=None, stream=None):
    """fa_fwd on the (128 x 128) blocks a uint8 mask keeps: block_mask is
    [nb, nb] (shared by all heads) or [B, H, nb, nb], nb = ceil(N / 128)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, shape=q.shape)
    _need(v, "v", torch.bfloat16, shape=q.shape)
    B, H, N, d = q.shape
    nb = (N + 127) // 128
    if not isinstance(block_mask, torch.Tensor):
        raise TypeError("block_mask must be a torch.Tensor")
    if block_mask.shape == (nb, nb):
        stride = 0
    elif block_mask.shape == (B, H, nb, nb):
        stride = nb * nb
    else:
        raise ValueError(f"block_mask must be [{nb}, {nb}] or [B, H, {nb}, {nb}]")
    _need(block_mask, "block_mask", torch.uint8)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    _check("fa_fwd_block_sparse",
           lib().fa_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     _ptr(block_mask), stride, B, H, N, d, int(bool(causal)),
                                     _stream(stream)))
    return o, lse


def fa_paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens_q, context_lens, max_seqlen_q,
                     causal=True, o=None, lse=None, stream=None):
    """O [Tq, Hq, d], L [Hq, Tq] of packed chunks over a paged cache
    ([P, Hkv, 16, d] bf16) through an int32 block table [batch, max_blocks]."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, shape=k_cache.shape)
    if k_cache.shape[3] != q.shape[2]:
        raise ValueError("k_cache and v_cache must be [P, Hkv, block_size, d] with q's d")
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    if cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q must have batch + 1 >= 2 entries")
    batch = cu_seqlens_q.numel() - 1
    _need(block_table, "block_table", torch.int32, 2)
    if block_table.shape[0] != batch:
        raise ValueError(f"block_table must have one row per sequence ({batch})")
    _need_lengths(context_lens, "context_lens", batch)
    Tq, Hq, d = q.shape
    P, Hkv, bs, _ = k_cache.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, Tq), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    _need(lse, "lse", torch.float32, shape=(Hq, Tq))
    _check("fa_paged_prefill",
           lib().fa_paged_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), P, _ptr(block_table),
                                  block_table.shape[1], _ptr(cu_seqlens_q), _ptr(context_lens),
                                  _ptr(o), _ptr(lse), cu_seqlens_q.numel() - 1, int(max_seqlen_q),
                                  Tq, Hq, Hkv, d, bs, int(bool(causal)), _stream(stream)))
    return o, lse


class KVPool:
    """Paged KV-cache block pool (host side, C++ in libfa.so): on-demand
    blocks, forks that share blocks by reference count, copy-on-write."""

    def __init__(self, num_blocks, block_size, max_seqs, max_blocks_per_seq):
        h = ctypes.c_void_p(0)
        _check("fa_kv_pool_create",
               lib().fa_kv_pool_create(num_blocks, block_size, max_seqs, max_blocks_per_seq,
                                       ctypes.byref(h)))
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.max_blocks = max_blocks_per_seq
        self._src, self._dst, self._n = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            lib().fa_kv_pool_destroy(h)
            self._h = None

    def add(self, seq):
        """Returns the fa_status (0 = ok)."""
        return int(lib().fa_kv_seq_add(self._h, seq))

    def fork(self, parent, child):
        return int(lib().fa_kv_seq_fork(self._h, parent, child))

    def free(self, seq):
        return int(lib().fa_kv_seq_free(self._h, seq))

    def append(self, seq, n_tokens):
        """Returns (status, copies): copies lists the (src, dst) block pairs to
        copy on the device before writing the new tokens."""
        st = int(lib().fa_kv_seq_append(self._h, seq, n_tokens, ctypes.byref(self._src),
                                        ctypes.byref(self._dst), ctypes.byref(self._n)))
        copies = [(self._src.value, self._dst.value)] if st == FA_OK and self._n.value else []
        return st, copies

    def num_free(self):
        return int(lib().fa_kv_num_free(self._h))

    def refcount(self, block):
        return int(lib().fa_kv_refcount(self._h, block))

    def seq_len(self, seq):
        return int(lib().fa_kv_seq_len(self._h, seq))

    def block_tables(self, seqs, width=None):
        """(table rows as lists of width entries, lengths) for the sequences."""
        width = self.max_blocks if width is None else width
        n = len(seqs)
        ids = (ctypes.c_int * max(n, 1))(*seqs)
        tab = (ctypes.c_int * max(n * width, 1))()
        lens = (ctypes.c_int * max(n, 1))()
        _check("fa_kv_block_table", lib().fa_kv_block_table(self._h, ids, n, tab, width, lens))
        return [list(tab[i * width:(i + 1) * width]) for i in range(n)], list(lens[:n])


def kv_copy_blocks(k_cache, v_cache, src, dst, stream=None):
    """Copy physical block src[i] -> dst[i] in both paged caches
    ([P][Hkv][block_size][d] bf16); src, dst int32 device tensors."""
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, shape=k_cache.shape)
    _need(src, "src", torch.int32, 1)
    _need(dst, "dst", torch.int32, shape=src.shape)
    block_bytes = k_cache[0].numel() * 2
    _check("fa_kv_copy_blocks",
           lib().fa_kv_copy_blocks(_ptr(k_cache), _ptr(v_cache), k_cache.shape[0], _ptr(src),
                                   _ptr(dst), src.numel(), block_bytes, _stream(stream)))


def fa_bwd_workspace_bytes(B, H, N, d):
    return int(lib().fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd(q, k, v, o, lse, do, causal=False, dq=None, dk=None, dv=None, workspace=None,
           stream=None):
    """dQ, dK, dV (fp32 [B, H, N, d]) of attention, recomputing P from L."""
    _need(q, "q", torch.bfloat16, 4)
    for n, t in (("k", k), ("v", v), ("o", o), ("do", do)):
        _need(t, n, torch.bfloat16, shape=q.shape)
    B, H, N, d = q.shape
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dv is None else dv
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, n, torch.float32, shape=q.shape)
    ws = fa_bwd_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    _need_workspace(workspace)
    _check("fa_bwd", lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  B, H, N, d, int(bool(causal)), _stream(stream)))
    return dq, dk, dv


def paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_ctx):
    return int(lib().paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_ctx))


def _need_decode(q, k_cache, v_cache, block_table, context_lens):
    """Checks shared by the decode calls; returns (S, Hq, d)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, shape=k_cache.shape)
    if k_cache.shape[3] != q.shape[2]:
        raise ValueError("k_cache and v_cache must be [P, Hkv, block_size, d] with q's d")
    S = q.shape[0]
    _need(block_table, "block_table", torch.int32, 2)
    if block_table.shape[0] != S:
        raise ValueError(f"block_table must have one row per sequence ({S})")
    _need_lengths(context_lens, "context_lens", S)
    return tuple(q.shape)


def paged_attn_decode(q, k_cache, v_cache, block_table, context_lens, max_ctx, o=None,
                      lse=None, want_lse=True, workspace=None, stream=None):
    """One-token decode over a paged cache; returns (O bf16 [S, Hq, d], L fp32 [S, Hq] or None)."""
    S, Hq, d = _need_decode(q, k_cache, v_cache, block_table, context_lens)
    Hkv, bs = k_cache.shape[1], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(S, Hq))
    ws = paged_attn_decode_workspace_bytes(S, Hq, d, max_ctx)
    if workspace is None:
        workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=q.device)
    _need_workspace(workspace)
    _check("paged_attn_decode", lib().paged_attn_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), k_cache.shape[0], _ptr(block_table),
        block_table.shape[1],
        _ptr(context_lens), _ptr(o), _ptr(lse), S, Hq, Hkv, d, bs, int(max_ctx),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return o, lse


def paged_attn_decode_noalloc(q, k_cache, v_cache, block_table, context_lens, max_ctx, o,
                              lse=None, stream=None):
    """paged_attn_decode with the library's internal scratch instead of a
    workspace. ``o`` (and ``lse`` if wanted) must be preallocated by the caller:
    this wrapper allocates nothing."""
    S, Hq, d = _need_decode(q, k_cache, v_cache, block_table, context_lens)
    _need(o, "o", torch.bfloat16, shape=q.shape)
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(S, Hq))
    _check("paged_attn_decode_noalloc", lib().paged_attn_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), k_cache.shape[0], _ptr(block_table),
        block_table.shape[1], _ptr(context_lens), _ptr(o), _ptr(lse), S, Hq, k_cache.shape[1], d,
        k_cache.shape[2], int(max_ctx), _stream(stream)))
    return o, lse


def fa_fp8_prepare(q, k, v, R, stream=None):
    """Rotate Q, K by R and quantise Q, K, V to e4m3 with 64-row block scales."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, shape=q.shape)
    _need(v, "v", torch.bfloat16, shape=q.shape)
    B, H, N, d = q.shape
    _need(R, "R", torch.float32, shape=(d, d))
    nb = (N + 63) // 64
    q8, k8, v8 = (torch.empty(q.shape, dtype=torch.uint8, device=q.device) for _ in range(3))
    sq, sk, sv = (torch.empty((B, H, nb), dtype=torch.float32, device=q.device) for _ in range(3))
    _check("fa_fp8_prepare", lib().fa_fp8_prepare(
        _ptr(q), _ptr(k), _ptr(v), _ptr(R), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk),
        _ptr(sv), B, H, N, d, _stream(stream)))
    return q8, k8, v8, sq, sk, sv


def fa_bwd_fp8(q8, k8, v8, sq, sk, sv, R, o, lse, do, causal=False, dq=None, dk=None, dv=None,
               workspace=None, stream=None):
    """Gradients of fa_fwd_fp8 with respect to the unrotated q, k and v (fp32):
    straight through the e4m3 quantisation, back through R (dQ = dQ' R^T)."""
    _need(q8, "q8", torch.uint8, 4)
    _need(k8, "k8", torch.uint8, shape=q8.shape)
    _need(v8, "v8", torch.uint8, shape=q8.shape)
    B, H, N, d = q8.shape
    nb = (N + 63) // 64
    for n, t in (("sq", sq), ("sk", sk), ("sv", sv)):
        _need(t, n, torch.float32, shape=(B, H, nb))
    _need(R, "R", torch.float32, shape=(d, d))
    _need(o, "o", torch.bfloat16, shape=q8.shape)
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    _need(do, "do", torch.bfloat16, shape=q8.shape)
    dq = torch.empty(q8.shape, dtype=torch.float32, device=q8.device) if dq is None else dq
    dk = torch.empty(q8.shape, dtype=torch.float32, device=q8.device) if dk is None else dk
    dv = torch.empty(q8.shape, dtype=torch.float32, device=q8.device) if dv is None else dv
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, n, torch.float32, shape=q8.shape)
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8,
                                device=q8.device)
    _need_workspace(workspace)
    _check("fa_bwd_fp8", lib().fa_bwd_fp8(
        _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(R), _ptr(o), _ptr(lse),
        _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, H, N, d, int(bool(causal)),
        _stream(stream)))
    return dq, dk, dv


def fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=False, o=None, lse=None, stream=None):
    """Attention forward on e4m3 inputs (uint8 storage) with per-block scales."""
    _need(q8, "q8", torch.uint8, 4)
    _need(k8, "k8", torch.uint8, shape=q8.shape)
    _need(v8, "v8", torch.uint8, shape=q8.shape)
    B, H, N, d = q8.shape
    for n, t in (("sq", sq), ("sk", sk), ("sv", sv)):
        _need(t, n, torch.float32, shape=(B, H, (N + 63) // 64))
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    _need(o, "o", torch.bfloat16, shape=(B, H, N, d))
    _need(lse, "lse", torch.float32, shape=(B, H, N))
    _check("fa_fwd_fp8", lib().fa_fwd_fp8(
        _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(o), _ptr(lse),
        B, H, N, d, int(bool(causal)), _stream(stream)))
    return o, lse


def fa_last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(lib().fa_last_device_error(_stream(stream)))


def fa_bwd_time_main_pass(ev_begin, ev_end) -> None:
    """The next fa_bwd call of this thread records the two torch.cuda.Event
    objects around its main pass (profiling)."""
    for ev in (ev_begin, ev_end):
        if not ev.cuda_event:       # torch creates the CUDA event on first record
            ev.record()
    _check("fa_bwd_time_main_pass",
           lib().fa_bwd_time_main_pass(ctypes.c_void_p(ev_begin.cuda_event),
                                       ctypes.c_void_p(ev_end.cuda_event)))


def fa_debug_wait_timeout(timeout_us, stream=None) -> int:
    """Launch the bounded-wait probe; returns the launch status."""
    return int(lib().fa_debug_wait_timeout(int(timeout_us), _stream(stream)))
