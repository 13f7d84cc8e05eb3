"""Softmax trace of the bf16 forward (a profiling tool, not the library).

Builds a separate copy of the library with -DFA_FWD_TRACE into _build/trace_fwd/
(libfa.so itself never carries the trace), runs fa_fwd on the long-sequence
workload (B=1, H=16, N=16384, d=128, causal, seed 1002) and prints, per key
block of CTA 0 (the heaviest pair of query tiles, 127 and 128 key blocks),
how many SM cycles the first softmax warp of each of its two query tiles
spends waiting for S, loading it out of TMEM, on the max and the first 64
keys' exp2 and P (with the O rescale, after which P.V may start on them), on
the other 64 keys, on the row sums and the stores, and arriving; and how far
apart the two tiles run.

Usage: python -m exact_attention_102_b200.trace_fwd   (needs a B200)
"""

from __future__ import annotations

import concurrent.futures
import ctypes
import os
import subprocess
import sys

import numpy as np

from . import build as _b

TRACE_DIR = os.path.join(_b.BUILD, "trace_fwd")
TRACE_LIB = os.path.join(TRACE_DIR, "libfa_trace_fwd.so")


def build_traced() -> str:
    os.makedirs(TRACE_DIR, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(TRACE_DIR, os.path.splitext(src)[0] + ".o")
        cmd = [_b._nvcc(), *_b.ARCH, *_b.FLAGS, "-DFA_FWD_TRACE", "-c",
               os.path.join(_b.CSRC, src), "-o", obj]
        subprocess.run(cmd, check=True)
        return obj

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(_b.SOURCES)) as ex:
        objs = list(ex.map(compile_one, _b.SOURCES))
    subprocess.run([_b._nvcc(), *_b.ARCH, "-shared", "-o", TRACE_LIB, *objs, "-cudart=static"],
                   check=True)
    return TRACE_LIB


def _records(row):
    """Split one trace row into per-block dicts {tag: cycle}; a block starts at tag 1."""
    v = row[row != 0]
    t, g = (v >> 8).astype(np.int64), (v & 0xFF).astype(np.int64)
    out, cur = [], None
    for ti, gi in zip(t, g):
        if gi == 1:
            cur = {}
            out.append(cur)
        if cur is not None:
            cur[int(gi)] = int(ti)
    return out


def _stat(x):
    x = np.asarray(x[2:-2] if len(x) > 8 else x)
    if len(x) == 0:
        return "    -"
    return f"{int(np.median(x)):5d} ({int(np.percentile(x, 10))}-{int(np.percentile(x, 90))})"


def main():
    import torch

    import exact_attention_102_b200 as fa
    import synth

    lib = build_traced()
    fa.LIB_PATH = lib
    fa._lib = None
    torch.cuda.set_device(0)
    B, H, N, d = 1, 16, 16384, 128
    x = synth.attention_inputs(B, H, N, d, 1002, device="cuda", with_dout=False)
    for _ in range(3):
        fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    torch.cuda.synchronize()
    if fa.fa_last_device_error() != fa.FA_OK:
        raise SystemExit("device error")
    buf = np.zeros((2, 4096), dtype=np.uint64)
    fa.lib().fa_fwd_trace_read.argtypes = [ctypes.c_void_p]
    if fa.lib().fa_fwd_trace_read(ctypes.c_void_p(buf.ctypes.data)) != 0:
        raise SystemExit("trace read failed")
    print(f"B={B} H={H} N={N} d={d}, causal; CTA 0, SM cycles per key block, "
          "median (10th-90th percentile):")
    firsts = []
    for t in range(2):
        recs = _records(buf[t])
        firsts.append([r.get(3, 0) for r in recs])

        def span(a, b):
            return [r[b] - r[a] for r in recs if a in r and b in r]

        block = [recs[k + 1][1] - recs[k][1] for k in range(len(recs) - 1)]
        print(f"query tile {t}: {len(recs)} key blocks, O rescaled in "
              f"{sum(1 for r in recs if 9 in r)}")
        print(f"  whole block                            {_stat(block)}")
        print(f"  wait for S                             {_stat(span(1, 2))}")
        print(f"  load S out of TMEM                     {_stat(span(2, 3))}")
        print(f"  max; keys 0-63: exp2, P, O rescale     {_stat(span(3, 4))}")
        print(f"  keys 64-127: exp2, P into TMEM         {_stat(span(4, 5))}")
        print(f"  row sums, wait for the TMEM stores      {_stat(span(5, 6))}")
        print(f"  arrive                                 {_stat(span(6, 7))}")
    n = min(len(firsts[0]), len(firsts[1]))
    off = [firsts[1][k] - firsts[0][k] for k in range(n)]
    print(f"tile 1 behind tile 0 (S loaded), median   {_stat(off)}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
