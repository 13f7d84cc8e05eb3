"""FP8 path: fa_fp8_prepare (rotation by an orthogonal R, per-64-row e4m3
block quantisation) and fa_fwd_fp8, through the C ABI.

The FP8 result is compared with the bf16 forward oracle on the original
(unrotated, unquantised) inputs: (QR)(KR)^T = QK^T, so quantisation is the
only difference, and the FP8 tolerance (5e-2) applies. The prepare step is
pinned separately against the oracle's own e4m3 block quantiser applied to
Q R computed in float64."""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import FP8_TOL, assert_bf16_close, assert_lse_close, f64

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_attention_102_b200")


def _e4m3_to_f64(t):
    return t.view(torch.float8_e4m3fn).to("cpu", torch.float64).numpy()


def _prepare(B, H, N, seed):
    x = synth.fp8_inputs(B, H, N, 128, seed, device="cuda")
    r64 = synth.orthogonal_matrix(128, 2003)
    R = torch.from_numpy(r64).float().cuda()
    out = fa.fa_fp8_prepare(x["q"], x["k"], x["v"], R)
    torch.cuda.synchronize()
    return x, r64, out


def test_prepare_matches_oracle_quantiser():
    B, H, N = 1, 3, 300
    x, r64, (q8, k8, v8, sq, sk, sv) = _prepare(B, H, N, 31)
    # R as the kernel sees it (fp32), applied in float64 by the test
    r32 = r64.astype(np.float32).astype(np.float64)
    for name, t8, sc, rot in (("q", q8, sq, True), ("k", k8, sk, True), ("v", v8, sv, False)):
        src = f64(x[name])
        if rot:
            src = src @ r32
        vals, scales = oracle.fp8_block_quantize(src)
        np.testing.assert_allclose(f64(sc), scales, rtol=1e-5)
        got = _e4m3_to_f64(t8)
        # rotation rounding (fp32 on the GPU) may move a value across an e4m3
        # rounding boundary: allow rare one-step differences, nothing else
        diff = got != vals
        assert diff.mean() < 2e-3, f"{name}: {diff.mean():.2e} of codes differ"
        step = np.abs(vals) * 2.0 ** -3 + 2.0 ** -9
        assert np.all(np.abs(got - vals)[diff] <= step[diff] * 1.01)


def test_fp8_config_sampled_rows():
    """B=4, H=16, N=4096, d=128, no mask, seed 1003: 0.1% outliers x50, R from
    seed 2003; sampled rows of 8 heads vs the bf16 oracle on original inputs."""
    B, H, N = 4, 16, 4096
    x, _, (q8, k8, v8, sq, sk, sv) = _prepare(B, H, N, 1003)
    o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=False)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 1, N - 1], rng.choice(N, 200, replace=False)]))
    for b, h in ((0, 0), (0, 7), (1, 3), (1, 15), (2, 9), (3, 0), (3, 8), (3, 15)):
        q = f64(x["q"][b, h, rows])
        o_ref, l_ref, _ = oracle.attention_rows(q, rows, f64(x["k"][b, h]), f64(x["v"][b, h]), False)
        assert_bf16_close(f64(o[b, h, rows]), o_ref, FP8_TOL, f"O b{b} h{h}")
        assert_lse_close(f64(lse[b, h, rows]), l_ref, rtol=FP8_TOL)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 257, 640])
def test_fp8_ragged_shapes(N, causal):
    B, H = 1, 2
    x, _, (q8, k8, v8, sq, sk, sv) = _prepare(B, H, N, 40 + N)
    o, lse = fa.fa_fwd_fp8(q8, k8, v8, sq, sk, sv, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_last_device_error() == fa.FA_OK
    o_ref, l_ref = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), causal=causal)
    assert_bf16_close(f64(o), o_ref, FP8_TOL, "O")
    assert_lse_close(f64(lse), l_ref, rtol=FP8_TOL)
