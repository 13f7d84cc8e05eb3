"""Cycles per tcgen05.mma on this part (a measurement tool, not the library).

Builds csrc/probe/mma_probe.cu into _build/probe/libmmaprobe.so (never into
libfa.so) and prints, for M = 128, K = 16, bf16 operands and fp32
accumulation, the SM cycles one MMA takes when a single thread per CTA (one
CTA per SM) issues them back to back: with the A operand in TMEM (TS) or in
shared memory (SS), for N = 64, 128 and 256. Full tensor rate is
128 x N x 16 multiply-adds per N / 2 cycles (4096 per cycle per SM).

Usage: python -m exact_attention_102_b200.probe_mma   (needs a B200)
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

from . import build as _b

PROBE_DIR = os.path.join(_b.BUILD, "probe")
PROBE_LIB = os.path.join(PROBE_DIR, "libmmaprobe.so")


def build_probe() -> str:
    os.makedirs(PROBE_DIR, exist_ok=True)
    src = os.path.join(_b.CSRC, "probe", "mma_probe.cu")
    subprocess.run([_b._nvcc(), *_b.ARCH, *_b.FLAGS, "-I", _b.CSRC, "-shared", "-o", PROBE_LIB,
                    src, "-cudart=static"], check=True)
    return PROBE_LIB


def measure(lib, ts: int, n: int, iters: int = 2048, ctas: int = 148) -> float:
    out = np.zeros(ctas, dtype=np.uint64)
    rc = lib.mma_probe(ts, n, iters, ctas, out.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise RuntimeError(f"mma_probe returned {rc}")
    return float(np.median(out)) / iters


def main():
    lib = ctypes.CDLL(build_probe())
    lib.mma_probe.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_void_p]
    lib.mma_probe.restype = ctypes.c_int
    print("SM cycles per tcgen05.mma, M = 128, K = 16, bf16 -> fp32, 148 CTAs, median")
    print(f"{'operands':<36}{'N=64':>8}{'N=128':>8}{'N=256':>8}")
    for ts, name in ((1, "A in TMEM, B in shared memory (TS)"), (0, "A and B in shared memory (SS)")):
        row = [measure(lib, ts, n) for n in (64, 128, 256)]
        print(f"{name:<36}" + "".join(f"{c:8.1f}" for c in row))
    print(f"{'full rate (N / 2)':<36}{32.0:8.1f}{64.0:8.1f}{128.0:8.1f}")


if __name__ == "__main__":
    sys.exit(main())
