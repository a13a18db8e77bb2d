"""GPU parity of the linear-layer calls (sol_linear*, sol_adaln_*) against the fp64 oracle.

Bar.  The tensor cores read bf16 operands and accumulate in fp32, so each product
y_j = sum_k h_k W_jk carries an error bounded by 2^-8 * S_j with S_j = sum_k |h_k W_jk|
(the oracle's linear_magnitude): at most 2^-9 relative from rounding the operand h to
bf16 (zero for a plain bf16 input) plus at most K * 2^-24 <= 2^-10 relative from fp32
accumulation for K <= 16384.  That bound is propagated through the fused operator
(below, per test) and the usual bf16 store bar max(2 ulp, 1e-3) is added on top.
Sizes span several 128 x 256 tiles, a ragged last tile of rows, several tiles per CTA
(both TMEM accumulators) and the full-size layer shapes at a few hundred tokens.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

from dit_block_b200 import sol, workloads as wl
from parity_util import to_oracle, tolerance

pytestmark = pytest.mark.gpu

ACC = 2.0 ** -8  # operand rounding + fp32 accumulation, relative to S = sum |h_k W_jk|

SMALL = dataclasses.replace(wl.WORKLOADS["tiny"], name="linear_small", index=10, dtype=torch.bfloat16,
                            grid=(3, 11, 13), d=512, n_heads=2, head_dim=128, inner=384,
                            rope_dims=(32, 48, 48), outlier_frac=1e-3)
PACKED = dataclasses.replace(SMALL, name="linear_packed", index=11, batch=2, grid=(2, 7, 9),
                             audio_per_sample=20, outlier_frac=0.0)
FULL = wl.WORKLOADS["fullres_10s"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    sol.lib()
    sol.device_errors(clear=True)
    yield
    assert sol.device_errors() == 0


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def check(got: torch.Tensor, want: np.ndarray, bound: np.ndarray, what: str):
    """|g - o| <= bound + max(2 ulp_bf16(o), 1e-3) elementwise."""
    g = f64(got)
    assert g.shape == want.shape, (g.shape, want.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - want)
    tol = bound + tolerance(want, torch.bfloat16)
    bad = err > tol
    if bad.any():
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} out of tolerance; worst at {i}: "
                             f"gpu {g[i]!r} oracle {want[i]!r} err {err[i]:.3e} tol {tol[i]:.3e}")


def sel_kwargs(w):
    pos, sid = wl.token_layout(w)
    kw = dict(n_streams=w.n_streams, tokens_per_sample=w.tokens_per_sample if w.batch > 1 else 0)
    return pos, sid, kw


# ------------------------------------------------------------------------------ tests

@pytest.mark.parametrize("m", [1, 128, 421])
def test_linear_plain(oracle_mod, m):
    w = SMALL
    a = wl.activation(w, "attn", m, w.d, "cuda")
    W = wl.linear_weight(w, "w_o", 768, w.d, "cuda")
    out = torch.full((m, 768), float("nan"), dtype=torch.bfloat16, device="cuda")
    sol.linear(out, a, W)
    torch.cuda.synchronize()
    A, Wh = to_oracle(a), to_oracle(W)
    check(out, oracle_mod.linear(A, Wh), ACC * oracle_mod.linear_magnitude(A, Wh), f"linear m={m}")


def test_linear_many_tiles_per_cta(oracle_mod):
    # 128 m-blocks x 4 n-blocks = 512 tiles: every CTA cycles both accumulators twice
    w = SMALL
    m, k, n = 16384 - 77, 256, 1024
    a = wl.activation(w, "attn", m, k, "cuda")
    W = wl.linear_weight(w, "w_o", n, k, "cuda")
    out = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    sol.linear(out, a, W)
    torch.cuda.synchronize()
    A, Wh = to_oracle(a), to_oracle(W)
    check(out, oracle_mod.linear(A, Wh), ACC * oracle_mod.linear_magnitude(A, Wh), "linear 512 tiles")


def test_linear_strided_rows(oracle_mod):
    # every operand a column slice of a wider buffer (row strides above the row width)
    w = SMALL
    m = 300
    abuf = wl.activation(w, "attn", m, w.d + 64, "cuda")
    Wbuf = wl.linear_weight(w, "w_o", 512, w.d + 128, "cuda")
    obuf = torch.zeros((m, 512 + 256), dtype=torch.bfloat16, device="cuda")
    a, W, out = abuf[:, 64:], Wbuf[:, :w.d], obuf[:, 256:]
    sol.linear(out, a, W)
    torch.cuda.synchronize()
    A, Wh = to_oracle(a), to_oracle(W)
    check(out, oracle_mod.linear(A, Wh), ACC * oracle_mod.linear_magnitude(A, Wh), "linear strided")
    assert torch.all(obuf[:, :256] == 0), "wrote outside the output columns"


@pytest.mark.parametrize("w", [SMALL, PACKED], ids=lambda w: w.name)
@pytest.mark.parametrize("alias", [False, True])
def test_linear_gated_residual(oracle_mod, w, alias):
    m = w.n_tokens
    _, sid, kw = sel_kwargs(w)
    sid = None if sid is None else sid.cuda()
    x = wl.activation(w, "x", m, w.d, "cuda")
    a = wl.activation(w, "attn", m, w.d, "cuda")
    W = wl.linear_weight(w, "w_o", w.d, w.d, "cuda")
    gate = wl.modulation(w, "gate_msa", "cuda")
    X, A, Wh, G = to_oracle(x), to_oracle(a), to_oracle(W), to_oracle(gate)
    out = x if alias else torch.empty_like(x)
    sol.linear_gated_residual(out, x, a, W, gate, stream_id=sid, **kw)
    torch.cuda.synchronize()
    want = oracle_mod.linear_gated_residual(X, A, Wh, G, stream_id=to_oracle(sid), **kw)
    # the product error scaled by |gate|, bounded by the largest gate of each column
    gmax = np.abs(oracle_mod.to_f64(G)).max(axis=0)
    bound = ACC * gmax[None, :] * oracle_mod.linear_magnitude(A, Wh)
    check(out, want, bound, f"linear_gated_residual {w.name} alias={alias}")


def test_linear_gated_residual_null_gate_is_identity():
    w = SMALL
    m = 200
    x = wl.activation(w, "x", m, w.d, "cuda")
    a = wl.activation(w, "attn", m, w.d, "cuda")
    W = wl.linear_weight(w, "w_o", w.d, w.d, "cuda")
    out = torch.empty_like(x)
    sol.linear_gated_residual(out, x, a, W, None)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), x.view(torch.int16)) or torch.equal(out, x)


@pytest.mark.parametrize("m", [421, 128])
def test_linear_swiglu(oracle_mod, m):
    w = SMALL
    a = wl.activation(w, "x", m, w.d, "cuda")
    W = wl.linear_weight(w, "w_up", 2 * w.inner, w.d, "cuda")
    out = torch.empty((m, w.inner), dtype=torch.bfloat16, device="cuda")
    sol.linear_swiglu(out, a, W)
    torch.cuda.synchronize()
    A, Wh = to_oracle(a), to_oracle(W)
    want = oracle_mod.linear_swiglu(A, Wh, w.inner)
    u = oracle_mod.linear(A, Wh)
    S = oracle_mod.linear_magnitude(A, Wh)
    ga, up = u[:, :w.inner], u[:, w.inner:]
    ea, eb = ACC * S[:, :w.inner], ACC * S[:, w.inner:]
    silu = ga / (1 + np.exp(-ga))
    # |silu'| <= 1.1: d(silu(a) b) <= 1.1 ea (|b| + eb) + |silu(a)| eb
    bound = 1.1 * ea * (np.abs(up) + eb) + np.abs(silu) * eb
    check(out, want, bound, f"linear_swiglu m={m}")


def modulation_rows(n, stream_id, n_streams, tokens_per_sample):
    """Modulation row of each token (the selection rule of sol_modsel)."""
    tok = np.arange(n)
    sample = tok // tokens_per_sample if tokens_per_sample > 0 else np.zeros(n, np.int64)
    sid = np.zeros(n, np.int64) if stream_id is None else np.minimum(stream_id.astype(np.int64), n_streams - 1)
    return sample * n_streams + sid


def adaln_projection_bound(oracle_mod, x, W, shift, scale, h, rows_r, eps):
    """Error bound of AdaLN(x) . W^T as the library computes it, for either strategy:
    * operand transform: h rounded to bf16 (2^-9 |h|) plus fp32 accumulation -> ACC * S;
    * weight fold: V = bf16(W (1 + scale_r)) rounded (2^-9 |(x - mean) rstd g W| <= 2^-9
      (|h| + |shift|) |W|), plus fp32 accumulation of x . V^T and of c_r = sum_k V, both
      multiplied by rstd (K 2^-23 rstd (|x| |g| + |mean| |g|) . |W|^T).
    Returns the larger of the two, elementwise."""
    X = oracle_mod.to_f64(x)
    Wf = np.abs(oracle_mod.to_f64(W))
    n, K = X.shape
    mu = X.mean(1)
    rs = 1.0 / np.sqrt(((X - mu[:, None]) ** 2).mean(1) + eps)
    G = np.abs(1.0 + oracle_mod.to_f64(scale)[rows_r]) if scale is not None else np.ones_like(X)
    Sh = np.abs(oracle_mod.to_f64(shift)[rows_r]) if shift is not None else np.zeros_like(X)
    S = np.abs(h) @ Wf.T
    fold = 2.0 ** -9 * ((np.abs(h) + Sh) @ Wf.T)
    fold += K * 2.0 ** -23 * rs[:, None] * (((np.abs(X) + np.abs(mu)[:, None]) * G) @ Wf.T)
    return np.maximum(ACC * S, fold)


def adaln_inputs(w, m):
    pos, sid, kw = sel_kwargs(w)
    x = wl.activation(w, "x", m, w.d, "cuda")
    shift = wl.modulation(w, "shift_msa", "cuda")
    scale = wl.modulation(w, "scale_msa", "cuda")
    sid = None if sid is None else sid[:m].cuda()
    pos = None if pos is None else pos[:m].cuda()
    return x, shift, scale, sid, pos, kw


@pytest.mark.parametrize("w", [SMALL, PACKED], ids=lambda w: w.name)
def test_adaln_linear(oracle_mod, w):
    m = w.n_tokens
    x, shift, scale, sid, _, kw = adaln_inputs(w, m)
    W = wl.linear_weight(w, "w_qkv", 768, w.d, "cuda")
    out = torch.empty((m, 768), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 768, w.d, **kw)
    sol.adaln_linear(out, x, W, shift, scale, workspace=ws, eps=w.eps, stream_id=sid, **kw)
    torch.cuda.synchronize()
    y, h = oracle_mod.adaln_linear(to_oracle(x), to_oracle(W), to_oracle(shift), to_oracle(scale), eps=w.eps,
                                   stream_id=to_oracle(sid), **kw)
    rr = modulation_rows(m, to_oracle(sid), w.n_streams, kw["tokens_per_sample"])
    bound = adaln_projection_bound(oracle_mod, to_oracle(x), to_oracle(W), to_oracle(shift), to_oracle(scale), h,
                                   rr, w.eps)
    check(out, y, bound, f"adaln_linear {w.name}")
    # with the weights folded, the workspace starts with each row's mean and 1/sqrt(var + eps)
    sol.adaln_linear(out, x, W, shift, scale, workspace=ws, strategy="fold", eps=w.eps, stream_id=sid, **kw)
    torch.cuda.synchronize()
    check(out, y, bound, f"adaln_linear {w.name}, weights folded")
    xf = f64(x)
    mu = xf.mean(1)
    rs = 1 / np.sqrt(((xf - mu[:, None]) ** 2).mean(1) + w.eps)
    st = ws[:8 * m].view(torch.float32).view(m, 2).cpu().double().numpy()
    np.testing.assert_allclose(st[:, 0], mu, rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(st[:, 1], rs, rtol=1e-4)


def qk_bound(pre, E, wq, wk, n_heads, eps):
    """Error bound of q|k after RMSNorm + RoPE given the bound E on the projection:
    with e_j <= E_j on a head vector v, r' = sqrt(mean v'^2 + eps) moves by at most
    rms(E), so each normalised element moves by at most |w_j| E_j / r' + |v_j w_j| rms(E) /
    (r r'), and a rotation of a pair moves an element by at most sqrt(2) times the larger
    move of the pair."""
    n = pre.shape[0]
    hd = pre.shape[1] // 2
    v = pre.reshape(n, 2 * n_heads, 128)
    E = E.reshape(n, 2 * n_heads, 128)
    w = np.concatenate([np.broadcast_to(wq, (n_heads, 128)), np.broadcast_to(wk, (n_heads, 128))])[None]
    r = np.sqrt((v ** 2).mean(-1, keepdims=True) + eps)
    rms_e = np.sqrt((E ** 2).mean(-1, keepdims=True))
    r1 = np.maximum(r - rms_e, 1e-30)
    d = np.abs(w) * E / r1 + np.abs(v * w) * rms_e / (r * r1)
    pm = np.maximum(d[..., 0::2], d[..., 1::2])
    return (np.sqrt(2.0) * np.repeat(pm, 2, axis=-1)).reshape(n, 2 * hd)


@pytest.mark.parametrize("w", [SMALL, PACKED], ids=lambda w: w.name)
def test_adaln_qkv_rope(oracle_mod, w):
    m = w.n_tokens
    x, shift, scale, sid, pos, kw = adaln_inputs(w, m)
    hd = w.hd
    W = wl.linear_weight(w, "w_qkv", 3 * hd, w.d, "cuda")
    wq, wk = wl.norm_weight(w, "wq", "cuda"), wl.norm_weight(w, "wk", "cuda")
    qkv = torch.empty((m, 3 * hd), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 3 * hd, w.d, **kw)
    grid = w.grid
    with sol.Rope3D(w.rope_dims, w.theta, w.max_pos) as rope:
        sol.adaln_qkv_rope(qkv, x, W, rope, shift, scale, workspace=ws, n_heads=w.n_heads, wq=wq, wk=wk,
                           pos=pos, grid=grid, eps=w.eps, stream_id=sid, **kw)
        torch.cuda.synchronize()
    Wh = to_oracle(W)
    want, pre, h = oracle_mod.adaln_qkv_rope(
        to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), to_oracle(wq), to_oracle(wk), n_heads=w.n_heads,
        head_dim=128, pos=to_oracle(pos), grid=grid, tokens_per_sample=kw["tokens_per_sample"],
        dims=w.rope_dims, theta=w.theta, eps=w.eps, stream_id=to_oracle(sid), n_streams=w.n_streams)
    rr = modulation_rows(m, to_oracle(sid), w.n_streams, kw["tokens_per_sample"])
    E = adaln_projection_bound(oracle_mod, to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), h, rr, w.eps)
    bq = qk_bound(pre[:, :2 * hd], E[:, :2 * hd], f64(wq), f64(wk), w.n_heads, w.eps)
    check(qkv[:, :2 * hd], want[:, :2 * hd], bq, f"adaln_qkv_rope q|k {w.name}")
    check(qkv[:, 2 * hd:], want[:, 2 * hd:], E[:, 2 * hd:], f"adaln_qkv_rope v {w.name}")


# ----------------------------------------------------- the block's layer shapes (d 5120)

FULL_M = 200  # a ragged tile of rows at full width


def test_full_shape_output_projection_gated(oracle_mod):
    w = FULL
    x = wl.activation(w, "x", FULL_M, w.d, "cuda")
    a = wl.activation(w, "attn", FULL_M, w.d, "cuda")
    W = wl.linear_weight(w, "w_o", w.d, w.d, "cuda")
    gate = wl.modulation(w, "gate_msa", "cuda")
    out = torch.empty_like(x)
    sol.linear_gated_residual(out, x, a, W, gate)
    torch.cuda.synchronize()
    A, Wh, G = to_oracle(a), to_oracle(W), to_oracle(gate)
    want = oracle_mod.linear_gated_residual(to_oracle(x), A, Wh, G)
    bound = ACC * np.abs(oracle_mod.to_f64(G))[0][None, :] * oracle_mod.linear_magnitude(A, Wh)
    check(out, want, bound, "O projection + gated residual, d 5120")


def test_full_shape_up_projection_swiglu(oracle_mod):
    w = FULL
    a = wl.activation(w, "x", FULL_M, w.d, "cuda")
    W = wl.linear_weight(w, "w_up", 2 * w.inner, w.d, "cuda")
    out = torch.empty((FULL_M, w.inner), dtype=torch.bfloat16, device="cuda")
    sol.linear_swiglu(out, a, W)
    torch.cuda.synchronize()
    A, Wh = to_oracle(a), to_oracle(W)
    u = oracle_mod.linear(A, Wh)
    S = oracle_mod.linear_magnitude(A, Wh)
    want = oracle_mod.swiglu(np.ascontiguousarray(u), w.inner)
    ga, up = u[:, :w.inner], u[:, w.inner:]
    ea, eb = ACC * S[:, :w.inner], ACC * S[:, w.inner:]
    bound = 1.1 * ea * (np.abs(up) + eb) + np.abs(ga / (1 + np.exp(-ga))) * eb
    check(out, want, bound, "up projection + SwiGLU, 5120 -> 2 x 13824")


def test_full_shape_down_projection_gated(oracle_mod):
    w = FULL
    x = wl.activation(w, "x", FULL_M, w.d, "cuda")
    a = wl.activation(w, "act", FULL_M, w.inner, "cuda")
    W = wl.linear_weight(w, "w_down", w.d, w.inner, "cuda")
    gate = wl.modulation(w, "gate_mlp", "cuda")
    out = torch.empty_like(x)
    sol.linear_gated_residual(out, x, a, W, gate)
    torch.cuda.synchronize()
    A, Wh, G = to_oracle(a), to_oracle(W), to_oracle(gate)
    want = oracle_mod.linear_gated_residual(to_oracle(x), A, Wh, G)
    bound = ACC * np.abs(oracle_mod.to_f64(G))[0][None, :] * oracle_mod.linear_magnitude(A, Wh)
    check(out, want, bound, "down projection + gated residual, 13824 -> 5120")


def test_full_shape_adaln_qkv_rope(oracle_mod):
    w = FULL
    m = FULL_M
    x = wl.activation(w, "x", m, w.d, "cuda")
    shift = wl.modulation(w, "shift_msa", "cuda")
    scale = wl.modulation(w, "scale_msa", "cuda")
    W = wl.linear_weight(w, "w_qkv", 3 * w.hd, w.d, "cuda")
    wq, wk = wl.norm_weight(w, "wq", "cuda"), wl.norm_weight(w, "wk", "cuda")
    qkv = torch.empty((m, 3 * w.hd), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 3 * w.hd, w.d)
    with sol.Rope3D(w.rope_dims, w.theta, w.max_pos) as rope:
        sol.adaln_qkv_rope(qkv, x, W, rope, shift, scale, workspace=ws, n_heads=w.n_heads, wq=wq, wk=wk,
                           grid=w.grid, eps=w.eps)
        torch.cuda.synchronize()
    Wh = to_oracle(W)
    want, pre, h = oracle_mod.adaln_qkv_rope(
        to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), to_oracle(wq), to_oracle(wk), n_heads=w.n_heads,
        head_dim=128, grid=w.grid, dims=w.rope_dims, theta=w.theta, eps=w.eps)
    hd = w.hd
    E = adaln_projection_bound(oracle_mod, to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), h,
                               np.zeros(m, np.int64), w.eps)
    bq = qk_bound(pre[:, :2 * hd], E[:, :2 * hd], f64(wq), f64(wk), w.n_heads, w.eps)
    check(qkv[:, :2 * hd], want[:, :2 * hd], bq, "AdaLN -> QKV -> QK norm + RoPE, q|k")
    check(qkv[:, 2 * hd:], want[:, 2 * hd:], E[:, 2 * hd:], "AdaLN -> QKV, v")


# ------------------------------------------- the other shapes and strategies of the kernel

@pytest.mark.parametrize("rows", [None, 128, 77], ids=lambda r: "pair" if r is None else f"single{r}")
@pytest.mark.parametrize("strategy", ["stage", "fold", "transform"])
def test_alternative_shapes_and_strategies(oracle_mod, strategy, rows):
    """Each AdaLN strategy (h staged through the workspace, weights folded, operand
    transformed; the caller's choice) and both tile shapes (CTA pairs above 128 rows, one
    CTA per tile at 128 rows or fewer) compute the same results under the same bounds."""
    w = PACKED
    m = w.n_tokens if rows is None else rows
    env = f"{strategy}, {m} rows"
    x, shift, scale, sid, pos, kw = adaln_inputs(w, m)
    hd = w.hd
    W = wl.linear_weight(w, "w_qkv", 3 * hd, w.d, "cuda")
    wq, wk = wl.norm_weight(w, "wq", "cuda"), wl.norm_weight(w, "wk", "cuda")
    qkv = torch.empty((m, 3 * hd), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 3 * hd, w.d, **kw)
    with sol.Rope3D(w.rope_dims, w.theta, w.max_pos) as rope:
        sol.adaln_qkv_rope(qkv, x, W, rope, shift, scale, workspace=ws, n_heads=w.n_heads, wq=wq, wk=wk,
                           pos=pos, grid=w.grid, strategy=strategy, eps=w.eps, stream_id=sid, **kw)
        torch.cuda.synchronize()
    Wh = to_oracle(W)
    want, pre, h = oracle_mod.adaln_qkv_rope(
        to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), to_oracle(wq), to_oracle(wk), n_heads=w.n_heads,
        head_dim=128, pos=to_oracle(pos), grid=w.grid, tokens_per_sample=kw["tokens_per_sample"],
        dims=w.rope_dims, theta=w.theta, eps=w.eps, stream_id=to_oracle(sid), n_streams=w.n_streams)
    rr = modulation_rows(m, to_oracle(sid), w.n_streams, kw["tokens_per_sample"])
    E = adaln_projection_bound(oracle_mod, to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), h, rr, w.eps)
    bq = qk_bound(pre[:, :2 * hd], E[:, :2 * hd], f64(wq), f64(wk), w.n_heads, w.eps)
    check(qkv[:, :2 * hd], want[:, :2 * hd], bq, f"adaln_qkv_rope q|k {env}")
    check(qkv[:, 2 * hd:], want[:, 2 * hd:], E[:, 2 * hd:], f"adaln_qkv_rope v {env}")
    # the epilogues without AdaLN in the same shape
    a = wl.activation(w, "attn", m, w.d, "cuda")
    Wup = wl.linear_weight(w, "w_up", 2 * w.inner, w.d, "cuda")
    out = torch.empty((m, w.inner), dtype=torch.bfloat16, device="cuda")
    sol.linear_swiglu(out, a, Wup)
    torch.cuda.synchronize()
    A, Wu = to_oracle(a), to_oracle(Wup)
    u = oracle_mod.linear(A, Wu)
    S = oracle_mod.linear_magnitude(A, Wu)
    ga, up = u[:, :w.inner], u[:, w.inner:]
    ea, eb = ACC * S[:, :w.inner], ACC * S[:, w.inner:]
    bound = 1.1 * ea * (np.abs(up) + eb) + np.abs(ga / (1 + np.exp(-ga))) * eb
    check(out, oracle_mod.swiglu(np.ascontiguousarray(u), w.inner), bound, f"linear_swiglu {env}")
    gate = wl.modulation(w, "gate_msa", "cuda")
    Wo = wl.linear_weight(w, "w_o", w.d, w.d, "cuda")
    xo = torch.empty_like(x)
    sol.linear_gated_residual(xo, x, a, Wo, gate, stream_id=sid, **kw)
    torch.cuda.synchronize()
    Wo_h, G = to_oracle(Wo), to_oracle(gate)
    want_g = oracle_mod.linear_gated_residual(to_oracle(x), A, Wo_h, G, stream_id=to_oracle(sid), **kw)
    gmax = np.abs(oracle_mod.to_f64(G)).max(axis=0)
    check(xo, want_g, ACC * gmax[None, :] * oracle_mod.linear_magnitude(A, Wo_h), f"linear_gated_residual {env}")
    # AdaLN into the up projection with SwiGLU, same shape and strategy
    ws2 = sol.adaln_workspace(m, 2 * w.inner, w.d, **kw)
    sol.adaln_linear_swiglu(out, x, Wup, shift, scale, workspace=ws2, strategy=strategy, eps=w.eps, stream_id=sid,
                            **kw)
    torch.cuda.synchronize()
    want, u2, h2 = oracle_mod.adaln_linear_swiglu(to_oracle(x), Wu, to_oracle(shift), to_oracle(scale), w.inner,
                                                  eps=w.eps, stream_id=to_oracle(sid), **kw)
    E2 = adaln_projection_bound(oracle_mod, to_oracle(x), Wu, to_oracle(shift), to_oracle(scale), h2, rr, w.eps)
    ga, up = u2[:, :w.inner], u2[:, w.inner:]
    ea, eb = E2[:, :w.inner], E2[:, w.inner:]
    bound = 1.1 * ea * (np.abs(up) + eb) + np.abs(ga / (1 + np.exp(-ga))) * eb
    check(out, want, bound, f"adaln_linear_swiglu {env}")


# ------------------------------------ the size bench.py times (--linear-tokens), sampled rows

BENCH_M = 32768


def sample_rows(m, n=48, seed=7):
    rng = np.random.default_rng(seed)
    rows = np.concatenate([[0, 1, 127, 128, 255, 256, m - 1], rng.choice(m, n - 7, replace=False)])
    return np.unique(rows)


@pytest.mark.parametrize("strategy", ["stage", "fold"])
def test_bench_size_adaln_qkv_rope_sampled(oracle_mod, strategy):
    w = FULL
    m = BENCH_M
    x = wl.activation(w, "x", m, w.d, "cuda")
    shift, scale = wl.modulation(w, "shift_msa", "cuda"), wl.modulation(w, "scale_msa", "cuda")
    W = wl.linear_weight(w, "w_qkv", 3 * w.hd, w.d, "cuda")
    wq, wk = wl.norm_weight(w, "wq", "cuda"), wl.norm_weight(w, "wk", "cuda")
    qkv = torch.empty((m, 3 * w.hd), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 3 * w.hd, w.d)
    with sol.Rope3D(w.rope_dims, w.theta, w.max_pos) as rope:
        sol.adaln_qkv_rope(qkv, x, W, rope, shift, scale, workspace=ws, n_heads=w.n_heads, wq=wq, wk=wk,
                           grid=w.grid, strategy=strategy, eps=w.eps)
        torch.cuda.synchronize()
    rows = sample_rows(m)
    xs = to_oracle(x[torch.from_numpy(rows).cuda()])
    Wh = to_oracle(W)
    want, pre, h = oracle_mod.adaln_qkv_rope(
        xs, Wh, to_oracle(shift), to_oracle(scale), to_oracle(wq), to_oracle(wk), n_heads=w.n_heads, head_dim=128,
        grid=w.grid, dims=w.rope_dims, theta=w.theta, eps=w.eps, rows=rows)
    hd = w.hd
    E = adaln_projection_bound(oracle_mod, xs, Wh, to_oracle(shift), to_oracle(scale), h,
                               np.zeros(len(rows), np.int64), w.eps)
    got = qkv[torch.from_numpy(rows).cuda()]
    bq = qk_bound(pre[:, :2 * hd], E[:, :2 * hd], f64(wq), f64(wk), w.n_heads, w.eps)
    check(got[:, :2 * hd], want[:, :2 * hd], bq, "AdaLN -> QKV -> QK norm + RoPE at 32,768 tokens, q|k")
    check(got[:, 2 * hd:], want[:, 2 * hd:], E[:, 2 * hd:], "AdaLN -> QKV at 32,768 tokens, v")


def test_bench_size_mlp_sampled(oracle_mod):
    w = FULL
    m = BENCH_M
    x = wl.activation(w, "x", m, w.d, "cuda")
    act = wl.activation(w, "act", m, w.inner, "cuda")
    Wup = wl.linear_weight(w, "w_up", 2 * w.inner, w.d, "cuda")
    Wdn = wl.linear_weight(w, "w_down", w.d, w.inner, "cuda")
    gate = wl.modulation(w, "gate_mlp", "cuda")
    up = torch.empty((m, w.inner), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    sol.linear_swiglu(up, x, Wup)
    sol.linear_gated_residual(out, x, act, Wdn, gate)
    torch.cuda.synchronize()
    rows = sample_rows(m, seed=11)
    ri = torch.from_numpy(rows).cuda()
    xs, As = to_oracle(x[ri]), to_oracle(act[ri])
    Wu, Wd, G = to_oracle(Wup), to_oracle(Wdn), to_oracle(gate)
    u = oracle_mod.linear(xs, Wu)
    S = oracle_mod.linear_magnitude(xs, Wu)
    ga, b_ = u[:, :w.inner], u[:, w.inner:]
    ea, eb = ACC * S[:, :w.inner], ACC * S[:, w.inner:]
    bound = 1.1 * ea * (np.abs(b_) + eb) + np.abs(ga / (1 + np.exp(-ga))) * eb
    check(up[ri], oracle_mod.swiglu(np.ascontiguousarray(u), w.inner), bound, "up + SwiGLU at 32,768 tokens")
    want = oracle_mod.linear_gated_residual(xs, As, Wd, G)
    bound = ACC * np.abs(oracle_mod.to_f64(G))[0][None, :] * oracle_mod.linear_magnitude(As, Wd)
    check(out[ri], want, bound, "down + gated residual at 32,768 tokens")


@pytest.mark.parametrize("w", [SMALL, PACKED], ids=lambda w: w.name)
def test_adaln_linear_swiglu(oracle_mod, w):
    m = w.n_tokens
    x, shift, scale, sid, _, kw = adaln_inputs(w, m)
    W = wl.linear_weight(w, "w_up", 2 * w.inner, w.d, "cuda")
    out = torch.empty((m, w.inner), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 2 * w.inner, w.d, **kw)
    sol.adaln_linear_swiglu(out, x, W, shift, scale, workspace=ws, eps=w.eps, stream_id=sid, **kw)
    torch.cuda.synchronize()
    Wh = to_oracle(W)
    want, u, h = oracle_mod.adaln_linear_swiglu(to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), w.inner,
                                                eps=w.eps, stream_id=to_oracle(sid), **kw)
    rr = modulation_rows(m, to_oracle(sid), w.n_streams, kw["tokens_per_sample"])
    E = adaln_projection_bound(oracle_mod, to_oracle(x), Wh, to_oracle(shift), to_oracle(scale), h, rr, w.eps)
    ga, up = u[:, :w.inner], u[:, w.inner:]
    ea, eb = E[:, :w.inner], E[:, w.inner:]
    bound = 1.1 * ea * (np.abs(up) + eb) + np.abs(ga / (1 + np.exp(-ga))) * eb
    check(out, want, bound, f"adaln_linear_swiglu {w.name}")


@pytest.mark.parametrize("strategy", ["stage", "fold"])
def test_bench_size_adaln_linear_swiglu_sampled(oracle_mod, strategy):
    """AdaLN -> up projection + SwiGLU at the size bench.py times, both AdaLN strategies,
    checked on sampled rows (the first and last tiles included)."""
    w = FULL
    m = BENCH_M
    x = wl.activation(w, "x", m, w.d, "cuda")
    shift, scale = wl.modulation(w, "shift_mlp", "cuda"), wl.modulation(w, "scale_mlp", "cuda")
    W = wl.linear_weight(w, "w_up", 2 * w.inner, w.d, "cuda")
    out = torch.empty((m, w.inner), dtype=torch.bfloat16, device="cuda")
    ws = sol.adaln_workspace(m, 2 * w.inner, w.d)
    sol.adaln_linear_swiglu(out, x, W, shift, scale, workspace=ws, strategy=strategy, eps=w.eps)
    torch.cuda.synchronize()
    rows = sample_rows(m, seed=13)
    ri = torch.from_numpy(rows).cuda()
    xs, Wh = to_oracle(x[ri]), to_oracle(W)
    want, u, h = oracle_mod.adaln_linear_swiglu(xs, Wh, to_oracle(shift), to_oracle(scale), w.inner, eps=w.eps,
                                                rows=rows)
    E = adaln_projection_bound(oracle_mod, xs, Wh, to_oracle(shift), to_oracle(scale), h,
                               np.zeros(len(rows), np.int64), w.eps)
    ga, up = u[:, :w.inner], u[:, w.inner:]
    ea, eb = E[:, :w.inner], E[:, w.inner:]
    bound = 1.1 * ea * (np.abs(up) + eb) + np.abs(ga / (1 + np.exp(-ga))) * eb
    check(out[ri], want, bound, f"AdaLN -> up + SwiGLU at 32,768 tokens ({strategy})")
