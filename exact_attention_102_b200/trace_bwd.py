"""Pipeline trace of the backward main pass (a profiling tool, not the library).

Builds a separate copy of the library with -DFA_BWD_TRACE into _build/trace/
(libfa.so itself never carries the trace), runs fa_fwd then fa_bwd on a causal
[B, H, N, d] workload (by default the long-sequence one, B=1, H=16, N=16384,
d=128) and prints, per 128-query step of CTA 0 (a CTA with the most steps,
key block 0), how many SM cycles its
single MMA-issuing thread spends on each product group and each barrier wait,
and what one P / dS warp and one drain warp do meanwhile. A tcgen05.mma is
accepted only as fast as the tensor core drains its queue, so the time to
issue a group of products is, in steady state, the time the tensor core
spends on them.

Usage: python -m exact_attention_102_b200.trace_bwd [--shape B,H,N,d]   (needs a B200;
d = 64 or 128)
"""

from __future__ import annotations

import concurrent.futures
import ctypes
import os
import subprocess
import sys

import numpy as np

from . import build as _b

TRACE_DIR = os.path.join(_b.BUILD, "trace")
TRACE_LIB = os.path.join(TRACE_DIR, "libfa_trace.so")


def build_traced() -> str:
    os.makedirs(TRACE_DIR, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(TRACE_DIR, os.path.splitext(src)[0] + ".o")
        cmd = [_b._nvcc(), *_b.ARCH, *_b.FLAGS, "-DFA_BWD_TRACE", "-c",
               os.path.join(_b.CSRC, src), "-o", obj]
        subprocess.run(cmd, check=True)
        return obj

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(_b.SOURCES)) as ex:
        objs = list(ex.map(compile_one, _b.SOURCES))
    subprocess.run([_b._nvcc(), *_b.ARCH, "-shared", "-o", TRACE_LIB, *objs, "-cudart=static"],
                   check=True)
    return TRACE_LIB


def _records(row):
    """Split one trace row into per-step dicts {tag: cycle}; a step starts at tag 1."""
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
    x = np.asarray(x[20:-20] if len(x) > 60 else x)
    return f"{int(np.median(x)):5d} ({int(np.percentile(x, 10))}-{int(np.percentile(x, 90))})"


def main(argv=None):
    import argparse

    import torch

    import exact_attention_102_b200 as fa
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--shape", default="1,16,16384,128", help="B,H,N,d (d = 64 or 128)")
    B, H, N, d = (int(v) for v in ap.parse_args(argv).shape.split(","))
    if d not in (64, 128):
        raise SystemExit("d must be 64 or 128")
    lib = build_traced()
    fa.LIB_PATH = lib
    fa._lib = None
    torch.cuda.set_device(0)
    x = synth.attention_inputs(B, H, N, d, 1002, device="cuda")
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True)
    for _ in range(3):
        fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=True)
    torch.cuda.synchronize()
    if fa.fa_last_device_error() != fa.FA_OK:
        raise SystemExit("device error")
    buf = np.zeros((3, 8192), dtype=np.uint64)
    if fa.lib().fa_bwd_trace_read(ctypes.c_void_p(buf.ctypes.data)) != 0:
        raise SystemExit("trace read failed")
    mma, pds, drain = (_records(buf[i]) for i in range(3))

    def span(recs, a, b):
        return [r[b] - r[a] for r in recs if a in r and b in r]

    step = [mma[k + 1][1] - mma[k][1] for k in range(len(mma) - 1)]
    print(f"B={B} H={H} N={N} d={d}, causal")
    print(f"steps traced: {len(mma)} (MMA thread), {len(pds)} (P / dS warp), {len(drain)} (drain)")
    print("SM cycles per 128-query step, median (10th-90th percentile):")
    print(f"  step                                       {_stat(step)}")
    if d == 64:
        print(f"  wait dS(i), issue dK(i)                    {_stat(span(mma, 1, 2))}")
        print(f"  issue dP^T(i+1)                            {_stat(span(mma, 3, 4))}")
        print(f"  wait P(i+1), issue dV(i+1)                 {_stat(span(mma, 4, 5))}")
        print(f"  wait stage, issue S^T(i+2)                 {_stat(span(mma, 5, 6))}")
        print(f"  wait for the drain warps to read dQ(i-1)   {_stat(span(mma, 6, 7))}")
        print(f"  issue dQ(i)                                {_stat(span(mma, 7, 8))}")
        print("P / dS warp (warp 4):")
        print(f"  first step: from the loop's start to S(0)  {span(pds, 1, 2)[0] if pds else 0}")
        print(f"  P: load S, exp, store P, arrive            {_stat(span(pds, 2, 3))}")
        print(f"  dS: load dP, dS, stores, arrive            {_stat(span(pds, 4, 6))}")
        return 0
    print(f"  wait dS(i), issue dQ(i)  8 x SS, N = 128   {_stat(span(mma, 1, 2))}")
    print(f"  issue dK(i) second half  4 x SS, N = 128   {_stat(span(mma, 2, 3))}")
    print(f"  wait for the drain warps to read dQ(i)     {_stat(span(mma, 3, 4))}")
    print(f"  dP^T(i+1), wait P(i+1), dV(i+1)            {_stat(span(mma, 4, 5))}")
    print(f"  S^T(i+2), wait dS(i+1) chunks, dK half 1   {_stat(span(mma, 5, 6))}")
    print("P / dS warp (warp 4):")
    print(f"  wait S and L                               {_stat(span(pds, 1, 2))}")
    print(f"  P: load S, exp, store P, arrive            {_stat(span(pds, 2, 3))}")
    print(f"  wait dP and D                              {_stat(span(pds, 3, 4))}")
    print(f"  dS: load dP, dS, stores, arrive            {_stat(span(pds, 4, 6))}")
    print("drain warp (warp 12):")
    print(f"  wait for dQ(i)                             {_stat(span(drain, 1, 2))}")
    print(f"  read dQ out of TMEM, arrive                {_stat(span(drain, 2, 3))}")

if __name__ == "__main__":
    sys.exit(main())
