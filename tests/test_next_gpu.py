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


# --------------------------------------------------------- SubBlock pooled epilogue

POOL_CASES = [  # dtype, head_dim, dims, n_heads, grid, samples, audio tokens per sample, block
    (BF, 128, (32, 48, 48), 40, (3, 4, 6), 2, 0, 64),
    (BF, 128, (32, 48, 48), 3, (2, 5, 7), 1, 0, 16),     # ragged last block (70 = 16*4 + 6)
    (BF, 64, (16, 24, 24), 5, (4, 3, 3), 3, 0, 8),
    (BF, 128, (32, 48, 48), 40, (2, 3, 4), 2, 5, 64),    # packed video+audio, explicit positions
    (torch.float32, 128, (32, 48, 48), 2, (2, 4, 4), 1, 0, 64),
    (torch.float32, 32, (8, 12, 12), 7, (3, 3, 3), 2, 0, 5),
    (BF, 128, (32, 48, 48), 8, (3, 3, 5), 2, 3, 7),      # staged kernel, 1 vector a thread, odd blocks
    (BF, 128, (32, 48, 48), 48, (2, 2, 3), 1, 0, 5),     # staged kernel at its widest (6 vectors a thread)
    (BF, 128, (32, 48, 48), 2, (2, 3, 3), 2, 1, 64),     # 2 heads: one warp busy; 19-token blocks
    (BF, 128, (32, 48, 48), 6, (1, 3, 3), 2, 0, 4),      # blocks of 4, 4 and 1 token (fewer than the ring)
]


@pytest.mark.parametrize("dtype,head_dim,dims,Hh,grid,B,audio,block", POOL_CASES)
def test_epilogue_pool(orc, dtype, head_dim, dims, Hh, grid, B, audio, block):
    w = workloads.Workload("p", 13, dtype, B, grid, audio, 64, Hh, head_dim, 64, rope_dims=dims)
    pos, _ = workloads.token_layout(w)
    n, tps, hd = w.n_tokens, w.tokens_per_sample, Hh * head_dim
    qkv = randn((n, 3 * hd), dtype, 21, std=1.5)
    wq = randn((head_dim,), dtype, 22, std=0.02, mean=1.0)
    wk = randn((head_dim,), dtype, 23, std=0.02, mean=1.0)
    rope = sol.Rope3D(dims, 10000.0, w.max_pos)
    P = None if pos is None else pos.to(DEV)
    nb = sol.subblock_count(n, tps, block)
    pq = torch.full((nb, hd), 99.0, dtype=dtype, device=DEV)
    pk = torch.full((nb, hd), 99.0, dtype=dtype, device=DEV)
    common = dict(n_heads=Hh, head_dim=head_dim, wq=wq, wk=wk, pos=P, grid=grid, tokens_per_sample=tps)
    got = qkv.clone()
    sol.dit_epilogue_pool(got, pq, pk, rope, block_tokens=block, **common)
    ref = qkv.clone()
    sol.dit_epilogue(ref, rope, **common)
    torch.cuda.synchronize()
    assert torch.equal(got, ref), "the fused pooling changed the epilogue's results"
    want = orc.dit_epilogue(to_oracle(qkv), to_oracle(wq), to_oracle(wk), n_heads=Hh, head_dim=head_dim,
                            pos=None if pos is None else pos.numpy(), grid=grid, tokens_per_sample=tps,
                            dims=dims)
    wpq = orc.block_mean(want[:, :hd], tokens_per_sample=tps, block=block)
    wpk = orc.block_mean(want[:, hd:], tokens_per_sample=tps, block=block)
    assert wpq.shape[0] == nb
    assert_close(to_f64(pq), wpq, dtype, "pooled q")
    assert_close(to_f64(pk), wpk, dtype, "pooled k")
    rope.close()


def test_epilogue_pool_full_workload(orc):
    """fullres_10s in the bench's launch configuration: in-place results equal the plain
    epilogue's bit for bit; pooled rows of sampled blocks match the oracle's means."""
    w = workloads.WORKLOADS["fullres_10s"]
    n, tps, hd, blk = w.n_tokens, w.tokens_per_sample, w.hd, 64
    qkv = workloads.activation(w, "qkv", n, 3 * w.hd, DEV)
    wq = workloads.norm_weight(w, "wq", DEV)
    wk = workloads.norm_weight(w, "wk", DEV)
    rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
    nb = sol.subblock_count(n, tps, blk)
    assert nb == 3843
    pq = torch.empty((nb, hd), dtype=BF, device=DEV)
    pk = torch.empty((nb, hd), dtype=BF, device=DEV)
    common = dict(n_heads=w.n_heads, head_dim=w.head_dim, wq=wq, wk=wk, grid=w.grid, tokens_per_sample=tps)
    picks = [0, 1, 1000, nb - 1]
    rows = np.concatenate([np.arange(b * blk, (b + 1) * blk) for b in picks])
    R = torch.from_numpy(rows).to(DEV)
    qkv_rows = to_oracle(qkv.index_select(0, R))
    ref = qkv.clone()
    sol.dit_epilogue(ref, rope, **common)
    sol.dit_epilogue_pool(qkv, pq, pk, rope, block_tokens=blk, **common)
    torch.cuda.synchronize()
    assert torch.equal(qkv, ref)
    del ref
    want = orc.dit_epilogue(qkv_rows, to_oracle(wq), to_oracle(wk), n_heads=w.n_heads, head_dim=w.head_dim,
                            grid=w.grid, tokens_per_sample=tps, dims=w.rope_dims, rows=rows)
    for i, b in enumerate(picks):
        seg = want[i * blk:(i + 1) * blk]
        assert_close(to_f64(pq[b:b + 1]), seg[:, :hd].mean(axis=0, keepdims=True), BF, f"pooled q {b}")
        assert_close(to_f64(pk[b:b + 1]), seg[:, hd:].mean(axis=0, keepdims=True), BF, f"pooled k {b}")
    rope.close()


# ------------------------------------------------- convention variants and output layouts

EX_CASES = [  # dtype, head_dim, dims, n_heads, grid, samples
    (BF, 128, (32, 48, 48), 40, (3, 4, 5), 2),
    (BF, 64, (16, 16, 32), 5, (4, 3, 3), 3),
    (torch.float32, 128, (32, 48, 48), 3, (2, 4, 4), 1),
    (torch.float32, 32, (8, 8, 16), 7, (3, 3, 3), 2),
    (BF, 128, (32, 48, 48), 8, (2, 3, 5), 3),   # 8 heads: rotate-half across heads on the register kernel
    (BF, 128, (32, 48, 48), 48, (2, 3, 4), 2),  # CTA-per-token kernel at its widest (6 slots a thread)
    (BF, 128, (32, 48, 48), 2, (3, 3, 3), 1),   # CTA-per-token kernel, one slot, 2 of 8 warps busy
    (BF, 128, (16, 48, 64), 6, (2, 3, 5), 2),   # another split: rotate-half chunk edges move
]


@pytest.mark.parametrize("dtype,head_dim,dims,Hh,grid,B", EX_CASES)
@pytest.mark.parametrize("span", [sol.NORM_PER_HEAD, sol.NORM_ACROSS_HEADS])
@pytest.mark.parametrize("pairing", [sol.ROPE_INTERLEAVED, sol.ROPE_HALF])
def test_qk_ex_conventions_and_layouts(orc, dtype, head_dim, dims, Hh, grid, B, span, pairing):
    T, H, W = grid
    tps = T * H * W
    n, hd = B * tps, Hh * head_dim
    qkv = randn((n, 3 * hd), dtype, 31, std=1.5)
    wlen = hd if span == sol.NORM_ACROSS_HEADS else head_dim
    wq = randn((wlen,), dtype, 32, std=0.02, mean=1.0)
    wk = randn((wlen,), dtype, 33, std=0.02, mean=1.0)
    rope = sol.Rope3D(dims, 10000.0, (T + 1, H + 2, W))
    q, k = qkv[:, :hd], qkv[:, hd:2 * hd]
    common = dict(n_heads=Hh, head_dim=head_dim, wq=wq, wk=wk, grid=grid, tokens_per_sample=tps,
                  norm_span=span, pairing=pairing)
    # token-major, out of place
    qo, ko = torch.empty((n, hd), dtype=dtype, device=DEV), torch.empty((n, hd), dtype=dtype, device=DEV)
    sol.qk_rmsnorm_rope3d_ex(qo, ko, q, k, rope, **common)
    # head-major [B, Hh, N, D] for attention
    qh = torch.empty((B, Hh, tps, head_dim), dtype=dtype, device=DEV)
    kh = torch.empty_like(qh)
    sol.qk_rmsnorm_rope3d_ex(qh, kh, q, k, rope, out_strides=(head_dim, tps * head_dim, Hh * tps * head_dim),
                             **common)
    # token-major in place on the packed row
    inplace = qkv.clone()
    sol.qk_rmsnorm_rope3d_ex(inplace[:, :hd], inplace[:, hd:2 * hd], inplace[:, :hd], inplace[:, hd:2 * hd],
                             rope, **common)
    torch.cuda.synchronize()
    wq_o, wk_o = orc.qk_rmsnorm_rope3d_ex(to_oracle(q.contiguous()), to_oracle(k.contiguous()), to_oracle(wq),
                                          to_oracle(wk), n_heads=Hh, head_dim=head_dim, grid=grid,
                                          tokens_per_sample=tps, dims=dims, norm_span=span, pairing=pairing)
    assert_close(to_f64(qo), wq_o, dtype, "q")
    assert_close(to_f64(ko), wk_o, dtype, "k")
    assert torch.equal(qh.permute(0, 2, 1, 3).reshape(n, hd), qo)
    assert torch.equal(kh.permute(0, 2, 1, 3).reshape(n, hd), ko)
    assert torch.equal(inplace[:, :hd], qo) and torch.equal(inplace[:, hd:2 * hd], ko)
    assert torch.equal(inplace[:, 2 * hd:], qkv[:, 2 * hd:])
    if span == sol.NORM_PER_HEAD and pairing == sol.ROPE_INTERLEAVED:
        q2, k2 = torch.empty_like(qo), torch.empty_like(ko)
        sol.qk_rmsnorm_rope3d(q2, k2, q, k, rope, n_heads=Hh, head_dim=head_dim, wq=wq, wk=wk, grid=grid,
                              tokens_per_sample=tps)
        torch.cuda.synchronize()
        assert torch.equal(q2, qo) and torch.equal(k2, ko)
    rope.close()


@pytest.mark.parametrize("span", [sol.NORM_PER_HEAD, sol.NORM_ACROSS_HEADS])
@pytest.mark.parametrize("pairing", [sol.ROPE_INTERLEAVED, sol.ROPE_HALF])
def test_qk_ex_explicit_positions_packed_and_clamped(orc, span, pairing):
    """Explicit packed video+audio positions through the staged kernel (bf16, 128-dim heads,
    an even head count), token-major and head-major; positions past the table clamp."""
    w = workloads.Workload("t", 7, BF, 2, (2, 3, 4), 5, 64, 4, 128, 64)
    pos, sid = workloads.token_layout(w)
    n, hd = pos.shape[0], w.hd
    q, k = randn((n, hd), BF, 41, std=1.5), randn((n, hd), BF, 42, std=1.5)
    wlen = hd if span == sol.NORM_ACROSS_HEADS else 128
    wq, wk = randn((wlen,), BF, 43, std=0.02, mean=1.0), randn((wlen,), BF, 44, std=0.02, mean=1.0)
    rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
    P = pos.to(DEV)
    common = dict(n_heads=w.n_heads, head_dim=128, wq=wq, wk=wk, norm_span=span, pairing=pairing)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    sol.qk_rmsnorm_rope3d_ex(qo, ko, q, k, rope, pos=P, **common)
    # one sample of n tokens, head-major [1, heads, n, 128]
    qh = torch.empty((1, w.n_heads, n, 128), dtype=BF, device=DEV)
    kh = torch.empty_like(qh)
    sol.qk_rmsnorm_rope3d_ex(qh, kh, q, k, rope, pos=P, out_strides=(128, n * 128, w.n_heads * n * 128), **common)
    torch.cuda.synchronize()
    want_q, want_k = orc.qk_rmsnorm_rope3d_ex(to_oracle(q), to_oracle(k), to_oracle(wq), to_oracle(wk),
                                              n_heads=w.n_heads, head_dim=128, pos=pos.numpy(),
                                              dims=w.rope_dims, theta=w.theta, norm_span=span, pairing=pairing)
    assert_close(to_f64(qo), want_q, BF, "q")
    assert_close(to_f64(ko), want_k, BF, "k")
    assert torch.equal(qh[0].permute(1, 0, 2).reshape(n, hd), qo)
    assert torch.equal(kh[0].permute(1, 0, 2).reshape(n, hd), ko)
    big = P.clone()
    big[:, 0] += 1000
    big[:3, 1] = -4
    clamped = torch.minimum(big, torch.tensor(w.max_pos, device=DEV, dtype=torch.int32) - 1).clamp_min(0)
    a, b = torch.empty_like(q), torch.empty_like(q)
    sol.qk_rmsnorm_rope3d_ex(a, b, q, k, rope, pos=big.contiguous(), **common)
    c, d = torch.empty_like(q), torch.empty_like(q)
    sol.qk_rmsnorm_rope3d_ex(c, d, q, k, rope, pos=clamped.contiguous(), **common)
    torch.cuda.synchronize()
    assert torch.equal(a, c) and torch.equal(b, d)
    rope.close()


def test_qk_ex_rejects_bad_layouts():
    rope = sol.Rope3D((32, 48, 48), 10000.0, (4, 4, 4))
    q = randn((8, 128), BF, 1)
    with pytest.raises(sol.SolError) as e:  # rotate-half needs chunks that are multiples of 16
        r2 = sol.Rope3D((40, 40, 48), 10000.0, (4, 4, 4))
        try:
            sol.qk_rmsnorm_rope3d_ex(torch.empty_like(q), torch.empty_like(q), q, q.clone(), r2, n_heads=1,
                                     head_dim=128, grid=(2, 2, 2), tokens_per_sample=8, pairing=sol.ROPE_HALF)
        finally:
            r2.close()
    assert e.value.status == sol.ERR_UNSUPPORTED
    with pytest.raises(sol.SolError) as e:  # an output overlapping the inputs in another layout
        sol.qk_rmsnorm_rope3d_ex(q, torch.empty_like(q), q, q.clone(), rope, n_heads=1, head_dim=128,
                                 grid=(2, 2, 2), tokens_per_sample=8, out_strides=(256, 128, 0))
    assert e.value.status == sol.ERR_INVALID_ARGUMENT
    rope.close()
