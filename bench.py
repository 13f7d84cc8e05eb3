"""Benchmark of the exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one forward + backward pass (fa_fwd + fa_bwd through the C ABI) of
the long-sequence workload: B=1, H=16, N=16384, d=128, causal, bf16 inputs
~N(0,1) (synthetic, seeded). The metric is attention fwd+bwd TFLOP/s with the
algorithmic FLOP count 4*B*H*N^2*d (forward) + 10*B*H*N^2*d (backward: five
N x N x d products), halved for the causal mask. Operands (5 bf16 tensors of
67 MB plus 3 fp32 gradients of 134 MB) exceed the 126 MB L2, so no flush is
needed between steps.

Besides the headline, the JSON line carries "parts": the forward and backward
alone, the GPT-2-small-shaped fwd+bwd (B=8, H=12, N=1024, d=64, causal), the
paged decode (64 sequences, 32/8 heads, d=128, contexts U[512, 32768], 16-token
blocks, shuffled table with 4-way prefix sharing) in HBM GB/s, and the FP8
forward (B=4, H=16, N=4096, d=128) when available.

Multi-GPU (torchrun): every rank runs the same per-GPU workload (independent
heads: weak scaling, no collective on the data path); the time is the max over
ranks. --impl reference times the float64 CPU oracle on a bounded sample of
the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD = dict(B=1, H=16, N=16384, d=128, causal=True)
METRIC = "attention fwd+bwd TFLOP/s (bf16)"
# DRAM bytes (read + write) of one d = 128 backward main-pass launch at WORKLOAD,
# from an ncu capture of that launch with the current kernel; None whenever the
# kernel has changed since, until captured again
BWD_MAIN_TRAFFIC = 0.792e9
# the same for one forward launch at WORKLOAD
FWD_TRAFFIC = 0.252e9
# DRAM bytes of one paged-decode launch at the c4 workload (current kernel)
DECODE_TRAFFIC = 4.241e9
# a timed region shorter than this runs at burst clocks: its kernels are held to
# the burst peak; a longer one to the sustained (power-capped) peak
SUSTAINED_REGION_MS = 1000.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def attn_flops(B, H, N, d, causal, bwd=False):
    f = (10.0 if bwd else 4.0) * B * H * N * N * d
    return f / 2 if causal else f


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []          # (arrival time, line)
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            time.sleep(0.3)      # let the sampler start before the region it watches
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        """Keep only samples that arrived inside [t0, t1] (wall clock)."""
        self.window = (t0, t1)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if self.window and not (self.window[0] <= ts <= self.window[1] + 0.03):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# -------------------------------------------------------------- distributed --
def _dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def _barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def _max_over_ranks(x, ws):
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(flops_per_rank, ws, ms_max):
    """Whole-job throughput: every rank did flops_per_rank; the job took the
    slowest rank's time (weak scaling, replicas)."""
    return ws * flops_per_rank / (ms_max / 1e3) / 1e12


def _ev():
    return torch.cuda.Event(enable_timing=True)


# --------------------------------------------------------------- our arm ---
def run_fwd_bwd(fa, B, H, N, d, causal, steps, warmup, ws, seed, sampler_gpu=None, flush_l2=False):
    """Device-resident fwd+bwd steps. Returns timing dict (max over ranks).
    flush_l2 (for problems that fit in L2): a 256 MB buffer is written before
    every step, outside the step's events, and the total is the sum of the
    steps' own spans."""
    x = synth.attention_inputs(B, H, N, d, seed, device="cuda")
    o = torch.empty_like(x["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty((B, H, N, d), dtype=torch.float32, device="cuda") for _ in range(3))
    wsp = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

    def step(evs=None):
        if evs is not None:
            evs[0].record()
        fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal, o=o, lse=lse)
        if evs is not None:
            evs[1].record()
            fa.fa_bwd_time_main_pass(evs[3], evs[4])     # events around the main pass
        fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal, dq=dq, dk=dk, dv=dv,
                  workspace=wsp)
        if evs is not None:
            evs[2].record()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    evs = [[_ev(), _ev(), _ev(), _ev(), _ev()] for _ in range(steps)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if flush_l2 else None
    sampler = ClockSampler(sampler_gpu) if sampler_gpu is not None else None
    if sampler:
        sampler.__enter__()
    _barrier(ws)
    torch.cuda.synchronize()
    start, end = _ev(), _ev()
    t0 = time.time()
    start.record()
    for i in range(steps):
        if flush is not None:
            flush.zero_()                               # outside the step's events
        step(evs[i])
    end.record()
    torch.cuda.synchronize()
    t1 = time.time()
    _barrier(ws)
    if sampler:
        sampler.mark(t0, t1)
        sampler.__exit__()
    assert fa.fa_last_device_error() == fa.FA_OK
    span = (sum(e[0].elapsed_time(e[2]) for e in evs) if flush is not None
            else start.elapsed_time(end))
    total_ms = _max_over_ranks(span, ws)
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    main_ms = float(np.mean([e[3].elapsed_time(e[4]) for e in evs]))
    # launches per step: fa_fwd 1; fa_bwd 4 (amax, fp16 conversion, D/L pre pass, main pass)
    return {"total_ms": total_ms, "fwd_ms": _max_over_ranks(fwd_ms, ws),
            "bwd_ms": _max_over_ranks(bwd_ms, ws), "bwd_main_ms": _max_over_ranks(main_ms, ws),
            "clocks": sampler.summary() if sampler else None, "launches_per_step": 5}


def run_e2e(fa, B, H, N, d, causal, steps, warmup, ws, seed):
    """Same step through the public API from pinned host buffers, as a
    pipeline would run it: every step copies its inputs q, k, v, dO in (H2D),
    runs fa_fwd + fa_bwd, and copies dQ, dK, dV out (D2H), all inside the
    timing; the copies run on streams of their own, so that step i's compute
    overlaps step i+1's H2D and step i-1's D2H (device buffers doubled)."""
    xd = synth.attention_inputs(B, H, N, d, seed, device="cuda")
    host = {n: t.cpu().pin_memory() for n, t in xd.items()}
    dev = [{n: torch.empty_like(t) for n, t in xd.items()} for _ in range(2)]
    del xd
    o = torch.empty_like(dev[0]["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    grads = [[torch.empty((B, H, N, d), dtype=torch.float32, device="cuda") for _ in range(3)]
             for _ in range(2)]
    wsp = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((B, H, N, d), dtype=torch.float32).pin_memory() for _ in range(3)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    computed = [None, None]     # compute of the step that last used buffer b is done
    drained = [None, None]      # D2H of the step that last used buffer b is done

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):              # H2D of step i into buffer b
            if computed[b] is not None:
                s_in.wait_event(computed[b])
            for n in ("q", "k", "v", "do"):
                dev[b][n].copy_(host[n], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
        with torch.cuda.stream(s_cmp):             # fa_fwd + fa_bwd of step i
            s_cmp.wait_event(landed)
            if drained[b] is not None:
                s_cmp.wait_event(drained[b])
            x, g = dev[b], grads[b]
            fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal, o=o, lse=lse)
            fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal, dq=g[0], dk=g[1],
                      dv=g[2], workspace=wsp)
            computed[b] = torch.cuda.Event()
            computed[b].record(s_cmp)
        with torch.cuda.stream(s_out):             # D2H of step i's gradients
            s_out.wait_event(computed[b])
            for hbuf, t in zip(outs, grads[b]):
                hbuf.copy_(t, non_blocking=True)
            drained[b] = torch.cuda.Event()
            drained[b].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    _barrier(ws)
    torch.cuda.synchronize()
    start, end = _ev(), _ev()
    start.record(s_in)                             # before the first H2D
    for st in (s_cmp, s_out):
        st.wait_event(start)
    for i in range(steps):
        step(warmup + i)
    for st in (s_in, s_cmp):                       # end after the last D2H
        s_out.wait_stream(st)
    end.record(s_out)
    torch.cuda.synchronize()
    _barrier(ws)
    ms = _max_over_ranks(start.elapsed_time(end), ws) / steps
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)
    return ms, h2d, d2h


def run_decode(fa, steps, warmup, seed=1004):
    lay = synth.paged_decode_layout(64, 16, 512, 32768, seed)
    q, kc, vc = synth.paged_decode_tensors(64, 32, 8, 128, 16, lay["num_phys"], seed,
                                           device="cuda")
    tab = torch.from_numpy(lay["block_table"]).cuda()
    lens = torch.from_numpy(lay["context_lens"]).cuda()
    o = torch.empty_like(q)
    lse = torch.empty((64, 32), dtype=torch.float32, device="cuda")
    wsp = torch.empty(fa.paged_attn_decode_workspace_bytes(64, 32, 128, 32768), dtype=torch.uint8,
                      device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")   # > L2: flush between calls

    def call():
        fa.paged_attn_decode(q, kc, vc, tab, lens, 32768, o=o, lse=lse, workspace=wsp)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush.zero_()
        a, b = _ev(), _ev()
        a.record()
        call()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    assert fa.fa_last_device_error() == fa.FA_OK
    ms = float(np.mean(ts))
    lens64 = lay["context_lens"].astype(np.int64)
    slab = 16 * 128 * 2                     # one (block, kv head) K or V slab
    logical = int(((lens64 + 15) // 16).sum()) * 8 * slab * 2
    unique = lay["num_phys"] * 8 * slab * 2
    small = 64 * 32 * 128 * 2 * 2 + tab.numel() * 4
    return {"ms": ms, "unique_bytes": unique + small, "logical_bytes": logical + small,
            "shared_fraction": lay["shared_blocks"] / lay["total_blocks"]}


def run_fp8(fa, steps, warmup, seed=1003):
    B, H, N, d = 4, 16, 4096, 128
    x = synth.fp8_inputs(B, H, N, d, seed, device="cuda")
    R = torch.from_numpy(synth.orthogonal_matrix(d, 2003)).float().cuda()
    try:
        q8, k8, v8, sq, sk, sv = fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R)
        o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=False)
    except fa.FAError as e:
        return {"unavailable": str(e)}
    for _ in range(warmup):
        fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=False, o=o, lse=lse)
    torch.cuda.synchronize()
    a, b = _ev(), _ev()
    a.record()
    for _ in range(steps):
        fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=False, o=o, lse=lse)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # the FP8 backward on the same codes (dO ~ N(0, 1), drawn after the inputs)
    g = torch.Generator(device="cuda").manual_seed(seed + 1)
    do = torch.randn((B, H, N, d), generator=g, device="cuda").to(torch.bfloat16)
    grads = [torch.empty((B, H, N, d), device="cuda") for _ in range(3)]
    wsp = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

    def bwd():
        fa.fa_bwd_fp8(q8, k8, v8, sq, sk, sv, R, o, lse, do, causal=False, dq=grads[0],
                      dk=grads[1], dv=grads[2], workspace=wsp)

    nb = max(3, steps // 4)
    for _ in range(warmup):
        bwd()
    torch.cuda.synchronize()
    a.record()
    for _ in range(nb):
        bwd()
    b.record()
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    return {"ms": ms, "flops": attn_flops(B, H, N, d, False), "bwd_ms": a.elapsed_time(b) / nb,
            "bwd_flops": attn_flops(B, H, N, d, False, bwd=True)}


VARLEN = dict(n=16, lo=512, hi=8192, H=16, Hkv=4, d=128, causal=True, seed=1006)


def varlen_flops(lens, H, d, causal):
    """4 d H per visible (query, key) pair; causal with equal lengths sees
    L (L + 1) / 2 pairs per sequence."""
    pairs = sum(L * (L + 1) // 2 if causal else L * L for L in lens)
    return 4.0 * d * H * pairs


def run_fwd_varlen(fa, steps, warmup):
    """Packed causal batch (lengths U[512, 8192], GQA 16 / 4 heads, d = 128)."""
    w = VARLEN
    lens = synth.packed_lengths(w["n"], w["lo"], w["hi"], w["seed"])
    x = synth.packed_inputs(lens, lens, w["H"], w["Hkv"], w["d"], w["seed"], device="cuda")
    cq, ck = torch.from_numpy(x["cu_q"]).cuda(), torch.from_numpy(x["cu_k"]).cuda()
    o, lse = fa.fa_fwd_varlen(x["q"], x["k"], x["v"], cq, ck, max(lens), causal=w["causal"])

    g = torch.randn(x["q"].shape, generator=torch.Generator(device="cuda").manual_seed(w["seed"]),
                    device="cuda").to(torch.bfloat16)
    grads = [torch.empty(t.shape, dtype=torch.float32, device="cuda")
             for t in (x["q"], x["k"], x["k"])]
    wsp = torch.empty(fa.fa_bwd_varlen_workspace_bytes(w["n"], max(lens), x["q"].shape[0],
                                                       x["k"].shape[0], w["H"], w["Hkv"], w["d"]),
                      dtype=torch.uint8, device="cuda")

    def fwd():
        fa.fa_fwd_varlen(x["q"], x["k"], x["v"], cq, ck, max(lens), causal=w["causal"], o=o,
                         lse=lse)

    def bwd():
        fa.fa_bwd_varlen(x["q"], x["k"], x["v"], o, lse, g, cq, ck, max(lens), max(lens),
                         causal=w["causal"], dq=grads[0], dk=grads[1], dv=grads[2], workspace=wsp)

    res = {"flops": varlen_flops(lens, w["H"], w["d"], w["causal"]), "tokens": int(sum(lens))}
    for name, op in (("ms", fwd), ("bwd_ms", bwd)):
        for _ in range(warmup):
            op()
        torch.cuda.synchronize()
        a, b = _ev(), _ev()
        a.record()
        for _ in range(steps):
            op()
        b.record()
        torch.cuda.synchronize()
        assert fa.fa_last_device_error() == fa.FA_OK
        res[name] = a.elapsed_time(b) / steps
    return res


PREFILL = dict(n=16, chunk=512, lo=1024, hi=16384, Hq=32, Hkv=8, d=128, seed=1007)


def run_paged_prefill(fa, steps, warmup):
    """Chunks of 512 new tokens for 16 sequences whose caches hold U[1024, 16384]
    tokens (chunk included) in shuffled 16-token blocks; causal (bottom right)."""
    w = PREFILL
    rng = np.random.default_rng(w["seed"])
    ctxs = rng.integers(w["lo"], w["hi"] + 1, w["n"]).astype(np.int32)
    nb = [-(-int(c) // 16) for c in ctxs]
    perm = rng.permutation(sum(nb)).astype(np.int32)
    table = np.zeros((w["n"], max(nb)), dtype=np.int32)
    p = 0
    for s_, n in enumerate(nb):
        table[s_, :n] = perm[p:p + n]
        p += n
    g = torch.Generator(device="cuda").manual_seed(w["seed"])
    kc = torch.randn((sum(nb), w["Hkv"], 16, w["d"]), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn_like(kc)
    q = torch.randn((w["n"] * w["chunk"], w["Hq"], w["d"]), generator=g,
                    device="cuda").to(torch.bfloat16)
    cu_q = torch.arange(0, w["n"] * w["chunk"] + 1, w["chunk"], dtype=torch.int32, device="cuda")
    tab = torch.from_numpy(table).cuda()
    ctx = torch.from_numpy(ctxs).cuda()
    o, lse = fa.fa_paged_prefill(q, kc, vc, tab, cu_q, ctx, w["chunk"])
    for _ in range(warmup):
        fa.fa_paged_prefill(q, kc, vc, tab, cu_q, ctx, w["chunk"], o=o, lse=lse)
    torch.cuda.synchronize()
    a, b = _ev(), _ev()
    a.record()
    for _ in range(steps):
        fa.fa_paged_prefill(q, kc, vc, tab, cu_q, ctx, w["chunk"], o=o, lse=lse)
    b.record()
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    ms = a.elapsed_time(b) / steps
    L = w["chunk"]
    pairs = sum(L * (int(c) - L) + L * (L + 1) // 2 for c in ctxs)
    flops = 4.0 * w["d"] * w["Hq"] * pairs
    return {"ms": ms, "TFLOP/s": flops / (ms / 1e3) / 1e12, "tokens": int(w["n"] * L)}


SPARSE = dict(B=1, H=16, N=16384, d=128, density=0.25, causal=True, seed=1008)


def run_block_sparse(fa, steps, warmup):
    """Long-sequence causal forward with a random 128 x 128 block mask of
    density 0.25 shared by the heads (diagonal blocks kept)."""
    w = SPARSE
    nb = w["N"] // 128
    m = (np.random.default_rng(w["seed"]).random((nb, nb)) < w["density"]).astype(np.uint8)
    np.fill_diagonal(m, 1)
    x = synth.attention_inputs(w["B"], w["H"], w["N"], w["d"], w["seed"], device="cuda",
                               with_dout=False)
    mt = torch.from_numpy(m).cuda()
    o, lse = fa.fa_fwd_block_sparse(x["q"], x["k"], x["v"], mt, causal=w["causal"])
    for _ in range(warmup):
        fa.fa_fwd_block_sparse(x["q"], x["k"], x["v"], mt, causal=w["causal"], o=o, lse=lse)
    torch.cuda.synchronize()
    a, b = _ev(), _ev()
    a.record()
    for _ in range(steps):
        fa.fa_fwd_block_sparse(x["q"], x["k"], x["v"], mt, causal=w["causal"], o=o, lse=lse)
    b.record()
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    ms = a.elapsed_time(b) / steps
    # kept (query, key) pairs: full kept blocks below the diagonal, half of the diagonal ones
    kept = sum(int(m[i, j]) for i in range(nb) for j in range(i)) * 128 * 128 + nb * 128 * 129 // 2
    flops = 4.0 * w["B"] * w["H"] * w["d"] * kept
    return {"ms": ms, "TFLOP/s": flops / (ms / 1e3) / 1e12,
            "kept_fraction": kept / (w["N"] * (w["N"] + 1) / 2)}


DROPOUT = dict(B=1, H=16, N=16384, d=128, causal=True, p=0.1, seed=1009)


def run_dropout(fa, steps, warmup):
    """The long-sequence causal workload with dropout p = 0.1 on P: forward
    and backward timed separately (same FLOP count as without dropout)."""
    w = DROPOUT
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    x = synth.attention_inputs(B, H, N, d, w["seed"], device="cuda")
    o, lse = fa.fa_fwd_dropout(x["q"], x["k"], x["v"], w["p"], w["seed"], 0, causal=w["causal"])
    g = [torch.empty((B, H, N, d), device="cuda") for _ in range(3)]
    wsp = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

    def fwd(off):
        fa.fa_fwd_dropout(x["q"], x["k"], x["v"], w["p"], w["seed"], off, causal=w["causal"],
                          o=o, lse=lse)

    def bwd(off):
        fa.fa_bwd_dropout(x["q"], x["k"], x["v"], o, lse, x["do"], w["p"], w["seed"], off,
                          causal=w["causal"], dq=g[0], dk=g[1], dv=g[2], workspace=wsp)

    out = {}
    for name, op in (("fwd", fwd), ("bwd", bwd)):
        for i in range(warmup):
            op(i)
        torch.cuda.synchronize()
        a, b = _ev(), _ev()
        a.record()
        for i in range(steps):
            op(i)
        b.record()
        torch.cuda.synchronize()
        assert fa.fa_last_device_error() == fa.FA_OK
        out[name + "_ms"] = a.elapsed_time(b) / steps
    out["fwd_TFLOP/s"] = attn_flops(B, H, N, d, w["causal"]) / (out["fwd_ms"] / 1e3) / 1e12
    out["bwd_TFLOP/s"] = attn_flops(B, H, N, d, w["causal"], bwd=True) / (out["bwd_ms"] / 1e3) / 1e12
    return out


def run_kv_pool(fa, steps):
    """Block pool on a decoding schedule: 64 sequences = 16 prompts of 500
    tokens forked 4 ways, then `steps` rounds of one token per sequence
    (on-demand blocks; the shared partial last block of each prompt is copied
    on write by 3 of its 4 sequences in the first round); host time per append. Then the device copy of 4096 blocks of
    32 KiB per cache (K and V) in GB/s (read + write)."""
    pool = fa.KVPool(65536, 16, 64, 1100)
    t0 = time.perf_counter()
    for p in range(16):
        pool.add(4 * p)
        pool.append(4 * p, 500)
        for c in range(1, 4):
            pool.fork(4 * p, 4 * p + c)
    n_app, n_cow = 0, 0
    for _ in range(steps):
        for s in range(64):
            st, copies = pool.append(s, 1)
            n_app += 1
            n_cow += len(copies)
    host_s = time.perf_counter() - t0
    kc = torch.zeros((8192, 8, 16, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    src = torch.arange(0, 4096, dtype=torch.int32, device="cuda")
    dst = torch.arange(4096, 8192, dtype=torch.int32, device="cuda")
    for _ in range(3):
        fa.kv_copy_blocks(kc, vc, src, dst)
    torch.cuda.synchronize()
    a, b = _ev(), _ev()
    a.record()
    for _ in range(10):
        fa.kv_copy_blocks(kc, vc, src, dst)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / 10
    moved = 2 * 2 * 4096 * kc[0].numel() * 2          # K and V, read + write
    return {"appends": n_app, "copy_on_write": n_cow, "us_per_append": 1e6 * host_s / n_app,
            "copy_ms": ms, "copy_GB/s": moved / (ms / 1e3) / 1e9}


# ---------------------------------------------------------- CPU baseline ---
def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else _cores()
    except Exception:
        return _cores()


def oracle_sample(N, seed=1002):
    """The float64 oracle (as it stands) on one head of the long-sequence
    workload truncated to N positions: forward + backward. Returns (s, flops)."""
    import oracle
    x = synth.attention_inputs(1, 1, N, 128, seed, device="cpu")
    q, k, v, do = (synth.to_f64(x[n])[0, 0] for n in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    o, lse = oracle.attention_fwd(q, k, v, causal=True)
    oracle.attention_bwd(q, k, v, do, causal=True, o=o)
    dt = time.perf_counter() - t0
    return dt, attn_flops(1, 1, N, 128, True) + attn_flops(1, 1, N, 128, True, bwd=True)


def cpu_baseline(N=16384):
    dt, fl = oracle_sample(N)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"float64 oracle fwd+bwd of 1 of 16 heads (B=1, N={N}, d=128, causal), "
                      f"{dt:.1f} s on the host"}


def run_reference(args, ws, rank):
    """--impl reference: the oracle on the host cores, same metric and config."""
    if rank != 0:
        return
    N = 4096
    for _ in range(args.warmup):
        oracle_sample(N)
    t = []
    fl = 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample(N)
        t.append(dt)
    ms = 1e3 * float(np.mean(t))
    val = fl / (ms / 1e3) / 1e12
    cores = _blas_threads()
    sample = (f"each step: float64 oracle fwd+bwd of one head of the workload truncated to "
              f"N={N} (B=1, d=128, causal)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": _config(),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def _config():
    w = WORKLOAD
    return {"workload": f"long-sequence attention fwd+bwd: B={w['B']} H={w['H']} N={w['N']} "
                        f"d={w['d']} causal bf16",
            "global_batch": w["B"], "seq_len": w["N"], "heads": w["H"], "head_dim": w["d"],
            "causal": w["causal"], "parallelism": "replicas (independent heads per GPU)",
            "operands": "fwd bf16 x bf16 -> fp32; bwd fp16 x fp16 -> fp32 (each input tensor "
                        "times a power of two from its largest magnitude, then fp16: exact for "
                        "every element within 2^30 of that magnitude; P and dS rounded to fp16)",
            "l2": "operands larger than L2 (335 MB bf16 + 403 MB fp32), no flush"}


def run_case(fa, case, shape, causal, steps, warmup):
    """One operation at one size, for profilers: warmup + steps launches."""
    if case == "dropout":                 # the fixed dropout workload (shape unused)
        print(json.dumps(run_dropout(fa, steps, warmup)))
        return
    if case == "block_sparse":            # the fixed block-sparse workload (shape unused)
        print(json.dumps(run_block_sparse(fa, steps, warmup)))
        return
    if case == "paged_prefill":           # the fixed prefill workload (shape unused)
        print(json.dumps(run_paged_prefill(fa, steps, warmup)))
        return
    if case == "kv_pool":                 # the fixed pool schedule (shape unused)
        print(json.dumps(run_kv_pool(fa, steps)))
        return
    if case == "fwd_varlen":              # the fixed packed workload (shape unused)
        res = run_fwd_varlen(fa, steps, warmup)
        print(json.dumps({"case": case, "ms": res["ms"],
                          "TFLOP/s": res["flops"] / (res["ms"] / 1e3) / 1e12,
                          "bwd_ms": res["bwd_ms"],
                          "bwd_TFLOP/s": 2.5 * res["flops"] / (res["bwd_ms"] / 1e3) / 1e12}))
        return
    B, H, N, d = shape
    x = synth.attention_inputs(B, H, N, d, 1002, device="cuda", with_dout=case == "bwd")
    if case == "fwd":
        o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)

        def op():
            fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal, o=o, lse=lse)
    elif case == "bwd":
        o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=causal)
        g = [torch.empty((B, H, N, d), device="cuda") for _ in range(3)]
        wsp = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

        def op():
            fa.fa_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal, dq=g[0], dk=g[1],
                      dv=g[2], workspace=wsp)
    elif case == "fp8":
        R = torch.from_numpy(synth.orthogonal_matrix(d, 2003)).float().cuda()
        q8, k8, v8, sq, sk, sv = fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R)
        o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)

        def op():
            fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal, o=o, lse=lse)
    elif case == "fp8_bwd":
        x = synth.fp8_inputs(B, H, N, d, 1003, device="cuda")
        R = torch.from_numpy(synth.orthogonal_matrix(d, 2003)).float().cuda()
        q8, k8, v8, sq, sk, sv = fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R)
        o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)
        g = torch.Generator(device="cuda").manual_seed(1004)
        do = torch.randn((B, H, N, d), generator=g, device="cuda").to(torch.bfloat16)
        grads = [torch.empty((B, H, N, d), device="cuda") for _ in range(3)]
        wsp = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")

        def op():
            fa.fa_bwd_fp8(q8, k8, v8, sq, sk, sv, R, o, lse, do, causal=causal, dq=grads[0],
                          dk=grads[1], dv=grads[2], workspace=wsp)
    elif case == "decode":
        S = B          # sequences; contexts U[512, N]
        lay = synth.paged_decode_layout(S, 16, 512, N, 1004)
        q, kc, vc = synth.paged_decode_tensors(S, 32, 8, 128, 16, lay["num_phys"], 1004,
                                               device="cuda")
        tab = torch.from_numpy(lay["block_table"]).cuda()
        lens = torch.from_numpy(lay["context_lens"]).cuda()

        def op():
            fa.paged_attn_decode(q, kc, vc, tab, lens, N)
    else:
        raise SystemExit(f"unknown case {case}")
    for _ in range(warmup):
        op()
    torch.cuda.synchronize()
    a, b = _ev(), _ev()
    a.record()
    for _ in range(steps):
        op()
    b.record()
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    print(json.dumps({"case": case, "shape": shape, "causal": causal,
                      "ms": a.elapsed_time(b) / max(steps, 1)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=120)   # ~0.5 s timed: several clock samples
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-parts", action="store_true", help="headline only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default="headline",
                    help="headline (default) or one op for profilers: fwd, bwd, fp8, fp8_bwd, "
                         "decode")
    ap.add_argument("--shape", default="1,16,16384,128",
                    help="B,H,N,d for --case (decode: sequences,_,max context,_)")
    ap.add_argument("--causal", type=int, default=1)
    args = ap.parse_args()
    if args.case != "headline":
        import exact_attention_102_b200 as fa
        torch.cuda.set_device(0)
        run_case(fa, args.case, [int(v) for v in args.shape.split(",")], bool(args.causal),
                 args.steps, args.warmup)
        return
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, ws, rank)
        return

    import exact_attention_102_b200 as fa
    ws, rank, local = _dist_init()
    peaks = _peaks()
    w = WORKLOAD
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if "CUDA_VISIBLE_DEVICES" in os.environ else local
    r = run_fwd_bwd(fa, w["B"], w["H"], w["N"], w["d"], w["causal"], args.steps, args.warmup, ws,
                    seed=1002, sampler_gpu=gpu_index)
    f_fwd = attn_flops(w["B"], w["H"], w["N"], w["d"], w["causal"])
    f_bwd = attn_flops(w["B"], w["H"], w["N"], w["d"], w["causal"], bwd=True)
    ms = r["total_ms"] / args.steps
    value = whole_job_value(f_fwd + f_bwd, ws, ms)
    e2e_ms, h2d, d2h = run_e2e(fa, w["B"], w["H"], w["N"], w["d"], w["causal"],
                               max(3, args.steps // 4), 2, ws, seed=1002)
    e2e_val = ws * (f_fwd + f_bwd) / (e2e_ms / 1e3) / 1e12

    peak_t = peaks["bf16_tflops"]
    peak_s = peaks.get("bf16_tflops_sustained") or peak_t
    # a sub-second timed region runs at burst clocks (the burst peak applies);
    # a seconds-long one settles under the power cap (the sustained peak)
    sustained = r["total_ms"] >= SUSTAINED_REGION_MS
    peak = peak_s if sustained else peak_t
    peak_src = (f"{'measured' if peaks['source'] == 'measured' else 'fallback'} bf16 "
                + ("sustained (cuBLAS, seconds-long loop)" if sustained else "burst (cuBLAS)")
                + f": timed region {r['total_ms']:.0f} ms")
    bwd_t = f_bwd / (r["bwd_ms"] / 1e3) / 1e12
    fwd_t = f_fwd / (r["fwd_ms"] / 1e3) / 1e12
    main_t = f_bwd / (r["bwd_main_ms"] / 1e3) / 1e12
    if r["bwd_main_ms"] >= r["fwd_ms"]:
        kern, ach = "bwd_ts_kernel<128> (fa_bwd main pass)", main_t
        traffic = BWD_MAIN_TRAFFIC
    else:
        kern, ach, traffic = "fwd_kernel (fa_fwd)", fwd_t, FWD_TRAFFIC
    roof = {"bound": "tensor", "kernel": kern, "achieved": ach, "peak": peak,
            "unit": "TFLOP/s", "frac": ach / peak, "peak_source": peak_src,
            "traffic": traffic,
            "forward": {"kernel": "fwd_kernel (fa_fwd)", "achieved": fwd_t, "frac": fwd_t / peak,
                        "traffic": FWD_TRAFFIC},
            "backward_whole": {"achieved": bwd_t, "frac": bwd_t / peak}}
    clk = r["clocks"]
    if clk and clk.get("sm_mhz") and clk.get("sm_max_mhz"):
        # step time scaled to the maximum SM clock (time x median MHz / max MHz)
        clk["ms_per_step_at_max_clock"] = ms * clk["sm_mhz"] / clk["sm_max_mhz"]

    parts = {}
    if not args.no_parts:
        parts["fwd"] = {"ms": r["fwd_ms"], "TFLOP/s": fwd_t, "frac_of_bf16_peak": fwd_t / peak_t}
        parts["bwd"] = {"ms": r["bwd_ms"], "TFLOP/s": bwd_t, "frac_of_bf16_peak": bwd_t / peak_t,
                        "main_pass_ms": r["bwd_main_ms"], "main_pass_TFLOP/s": main_t}
        c1 = run_fwd_bwd(fa, 8, 12, 1024, 64, True, args.steps, args.warmup, 1, seed=1001,
                         flush_l2=True)
        f1 = attn_flops(8, 12, 1024, 64, True) + attn_flops(8, 12, 1024, 64, True, bwd=True)
        parts["gpt2_small_fwd_bwd"] = {
            "ms": c1["total_ms"] / args.steps,
            "TFLOP/s": f1 / (c1["total_ms"] / args.steps / 1e3) / 1e12,
            "fwd_ms": c1["fwd_ms"], "bwd_ms": c1["bwd_ms"],
            "l2": "256 MB written before every step, outside its timing"}
        dec = run_decode(fa, args.steps, args.warmup)
        gbs = dec["unique_bytes"] / (dec["ms"] / 1e3) / 1e9
        parts["paged_decode"] = {
            "ms": dec["ms"], "GB/s_unique": gbs,
            "GB/s_logical": dec["logical_bytes"] / (dec["ms"] / 1e3) / 1e9,
            "shared_block_fraction": dec["shared_fraction"],
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": DECODE_TRAFFIC}}
        vl = run_fwd_varlen(fa, args.steps, args.warmup)
        parts["fwd_varlen"] = {
            "workload": f"packed causal batch: {VARLEN['n']} sequences, lengths "
                        f"U[{VARLEN['lo']}, {VARLEN['hi']}] (seed {VARLEN['seed']}), "
                        f"H={VARLEN['H']} on Hkv={VARLEN['Hkv']}, d={VARLEN['d']}",
            "ms": vl["ms"], "tokens": vl["tokens"],
            "TFLOP/s": vl["flops"] / (vl["ms"] / 1e3) / 1e12,
            "bwd_ms": vl["bwd_ms"], "bwd_TFLOP/s": 2.5 * vl["flops"] / (vl["bwd_ms"] / 1e3) / 1e12}
        pp = run_paged_prefill(fa, args.steps, args.warmup)
        parts["paged_prefill"] = dict(pp, workload=(
            f"{PREFILL['n']} chunks of {PREFILL['chunk']} tokens over paged caches of "
            f"U[{PREFILL['lo']}, {PREFILL['hi']}] tokens, Hq={PREFILL['Hq']} on "
            f"Hkv={PREFILL['Hkv']}, d={PREFILL['d']}, causal"))
        bs = run_block_sparse(fa, args.steps, args.warmup)
        parts["block_sparse_fwd"] = dict(bs, workload=(
            f"causal B={SPARSE['B']} H={SPARSE['H']} N={SPARSE['N']} d={SPARSE['d']}, "
            f"random 128 x 128 block mask, density {SPARSE['density']} + diagonal"))
        dr = run_dropout(fa, max(3, args.steps // 4), args.warmup)
        parts["dropout"] = dict(dr, workload=(
            f"causal B={DROPOUT['B']} H={DROPOUT['H']} N={DROPOUT['N']} d={DROPOUT['d']}, "
            f"dropout p={DROPOUT['p']} on P (Philox4x32-10 keep mask)"))
        kvp = run_kv_pool(fa, 64)
        parts["kv_pool"] = dict(kvp, roofline={
            "bound": "hbm", "achieved": kvp["copy_GB/s"], "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": kvp["copy_GB/s"] / peaks["hbm_gbs"]})
        f8 = run_fp8(fa, args.steps, args.warmup)
        if "ms" in f8:
            t8 = f8["flops"] / (f8["ms"] / 1e3) / 1e12
            p8 = 2.0 * peak_t
            parts["fp8_fwd"] = {"ms": f8["ms"], "TFLOP/s": t8, "roofline": {
                "bound": "tensor", "achieved": t8, "peak": p8, "unit": "TFLOP/s", "frac": t8 / p8,
                "peak_source": f"{peaks['source']} bf16 burst x 2 (nominal fp8/bf16 ratio)"}}
            tb = f8["bwd_flops"] / (f8["bwd_ms"] / 1e3) / 1e12
            parts["fp8_bwd"] = {
                "ms": f8["bwd_ms"], "TFLOP/s": tb, "workload": "backward of the FP8 forward on its "
                "codes (fp16 products, block scales in fp32, rotation back)",
                "roofline": {"bound": "tensor", "achieved": tb, "peak": peak_t, "unit": "TFLOP/s",
                             "frac": tb / peak_t,
                             "peak_source": f"{peaks['source']} bf16 burst (fp16 products)"}}
        else:
            parts["fp8_fwd"] = f8

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:   # the host baseline: N = 1 only
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": _config(),
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "copies": "own streams: step i's H2D and D2H overlap steps i-1 and i+1"},
            "gpu_launches": r["launches_per_step"] * args.steps,
            "clocks": clk, "parts": parts,
        }
        print(json.dumps(line))
    if ws > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
