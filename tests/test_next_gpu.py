"""GPU parity of the ops beyond the block pass: the gated residual fused with the
Cache-DiT residual-change statistics.  Called through the C ABI, compared with the fp64
oracle on the same seeded inputs.

Tolerance of the sums: each thread adds at most U*E = 32 |differences| of one row in
fp32 (relative error <= 32 * 2^-24 ~ 2e-6) before widening to fp64, and r = gate*y is
formed in fp32 (per-element error <= 2^-24 |r| <= 2^-24 (|r - c| + |c|)).  So the
reference sum is checked to 1e-5 relative, and the difference sum to 1e-5 of the
sample's total mass sum|r - c| + sum|c| -- the scale of the change ratio that the
reuse decision reads."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from dit_block_b200 import sol, workloads
from parity_util import assert_close, to_f64, to_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dit_block_b200 import build
    build.build()
    sol.lib()


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def check_sums(got, want):
    got = np.asarray(got.cpu() if hasattr(got, "cpu") else got, np.float64).reshape(-1, 2)
    want = np.asarray(want, np.float64).reshape(-1, 2)
    mass = want[:, 0] + want[:, 1]
    assert np.all(np.abs(got[:, 0] - want[:, 0]) <= 1e-5 * mass + 1e-12), (got, want)
    assert np.all(np.abs(got[:, 1] - want[:, 1]) <= 1e-5 * want[:, 1] + 1e-12), (got, want)


def randn(shape, dtype, seed, std=1.0, mean=0.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std + mean).to(dtype).to(DEV)


@pytest.mark.parametrize("dtype", [torch.float32, BF])
@pytest.mark.parametrize("n,d,B,S", [(1, 8, 1, 1), (37, 256, 3, 2), (301, 5120, 2, 2), (129, 1000, 5, 1),
                                     (2049, 64, 4, 1)])
@pytest.mark.parametrize("refresh", [True, False])
def test_cache_diff(orc, dtype, n, d, B, S, refresh):
    if dtype == torch.float32 and d % 4:
        pytest.skip("width")
    tps = max(1, (n + B - 1) // B)
    x = randn((n, d), dtype, 1)
    y = randn((n, d), dtype, 2)
    cache = randn((n, d), dtype, 3, std=0.1)
    gate = randn((B * S, d), dtype, 4, std=0.1)
    g = torch.Generator().manual_seed(5)
    sid = torch.randint(0, S, (n,), generator=g, dtype=torch.uint8).to(DEV)
    cache0 = cache.clone()
    out = torch.empty_like(x)
    sums = torch.full((B, 2), 123.0, dtype=torch.float64, device=DEV)  # cleared by the call
    sol.gated_residual_cache_diff(out, x, y, gate, cache, sums, refresh=refresh, stream_id=sid,
                                  n_streams=S, tokens_per_sample=tps)
    torch.cuda.synchronize()
    want_o, want_r, want_s = orc.gated_residual_cache_diff(
        to_oracle(x), to_oracle(y), to_oracle(gate), to_oracle(cache0), n_samples=B,
        stream_id=to_oracle(sid), n_streams=S, tokens_per_sample=tps)
    assert_close(to_f64(out), want_o, dtype, "out")
    check_sums(sums, want_s)
    if refresh:
        assert_close(to_f64(cache), want_r, dtype, "refreshed cache")
    else:
        assert torch.equal(cache, cache0)
    # the output is exactly the plain gated residual's
    o2 = torch.empty_like(x)
    sol.gated_residual(o2, x, y, gate, stream_id=sid, n_streams=S, tokens_per_sample=tps)
    torch.cuda.synchronize()
    assert torch.equal(out, o2)


def test_cache_diff_second_step_against_refreshed_cache(orc):
    """Step 1 refreshes an empty cache with r = gate*y rounded to the tensor dtype; step 2
    on the same inputs sees only that rounding as change (zero for fp32, whose products
    of the inputs are exact)."""
    n, d = 500, 5120
    for dtype in (BF, torch.float32):
        x, y = randn((n, d), dtype, 1), randn((n, d), dtype, 2)
        gate = randn((1, d), dtype, 3, std=0.1)
        cache = torch.zeros_like(x)
        out = torch.empty_like(x)
        sums = torch.empty((1, 2), dtype=torch.float64, device=DEV)
        sol.gated_residual_cache_diff(out, x, y, gate, cache, sums, refresh=True)
        first = sums.clone()
        sol.gated_residual_cache_diff(out, x, y, gate, cache, sums, refresh=True)
        torch.cuda.synchronize()
        X, Y, G = to_oracle(x), to_oracle(y), to_oracle(gate)
        _, r1, s1 = orc.gated_residual_cache_diff(X, Y, G, to_oracle(torch.zeros_like(x)))
        c1 = to_oracle(torch.from_numpy(r1).to(dtype))  # the stored cache: r rounded (torch, RNE)
        _, _, s2 = orc.gated_residual_cache_diff(X, Y, G, c1)
        check_sums(first, s1)
        check_sums(sums, s2)
        if dtype == torch.float32:
            assert sums[0, 0].item() == 0.0


def test_cache_diff_rejects_too_few_sample_sums():
    x = randn((10, 64), BF, 1)
    sums = torch.zeros((2, 2), dtype=torch.float64, device=DEV)
    with pytest.raises(sol.SolError) as e:
        sol.gated_residual_cache_diff(torch.empty_like(x), x, x.clone(), None, x.clone(), sums,
                                      tokens_per_sample=3)  # 10 tokens span 4 samples
    assert e.value.status == sol.ERR_INVALID_ARGUMENT
    torch.cuda.synchronize()
    assert torch.all(sums == 0)


def test_cache_diff_full_workload(orc):
    """fullres_10s: the sums over all 245,952 tokens against the oracle, evaluated in row
    chunks; out and the refreshed cache on sampled rows."""
    w = workloads.WORKLOADS["fullres_10s"]
    n, d = w.n_tokens, w.d
    x = workloads.activation(w, "x", n, d, DEV)
    y = workloads.activation(w, "y_mlp", n, d, DEV)
    cache = workloads.activation(w, "y_attn", n, d, DEV)  # a stand-in previous residual
    gate = workloads.modulation(w, "gate_mlp", DEV)
    cache0 = cache.clone()
    out = torch.empty_like(x)
    sums = torch.empty((1, 2), dtype=torch.float64, device=DEV)
    sol.gated_residual_cache_diff(out, x, y, gate, cache, sums, refresh=True,
                                  tokens_per_sample=w.tokens_per_sample)
    torch.cuda.synchronize()
    G = to_oracle(gate)
    tot = np.zeros(2)
    step = 16384
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        _, _, s = orc.gated_residual_cache_diff(to_oracle(x[r0:r1]), to_oracle(y[r0:r1]), G,
                                                to_oracle(cache0[r0:r1]), n_samples=1)
        tot += s[0]
    check_sums(sums, tot)
    rows = torch.tensor([0, 1, 12345, 200000, n - 1], device=DEV)
    R = rows.cpu().numpy()
    wo, wr, _ = orc.gated_residual_cache_diff(to_oracle(x[rows]), to_oracle(y[rows]), G,
                                              to_oracle(cache0[rows]), n_samples=1,
                                              tokens_per_sample=w.tokens_per_sample, rows=R)
    assert_close(to_f64(out[rows]), wo, BF, "full out")
    assert_close(to_f64(cache[rows]), wr, BF, "full refreshed cache")
