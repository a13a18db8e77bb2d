"""Pins for the oracle's linear-layer compositions (AdaLN -> QKV projection -> QK norm +
RoPE, SwiGLU on the up projection, gated residual on the output / down projection).

Each composition reuses per-token oracle functions pinned in test_oracle_pins.py; what
is new is the orientation of the product y = a . W^T, the split of the up projection
into its gated and multiplying halves, and the wiring of each step.  Permutation weights
catch a transposed W (a non-involutive permutation P gives a[:, pi] for W = P and
a[:, pi^-1] for W = P^T), the hand-worked examples catch a swapped half, and linearity
catches a dropped or doubled term.  CPU only.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

from conftest import read_golden

RNG = np.random.default_rng(4321)


def perm_matrix(pi: np.ndarray) -> np.ndarray:
    """W with W[j, pi[j]] = 1, so that a . W^T = a[:, pi]."""
    n = len(pi)
    w = np.zeros((n, n), np.float64)
    w[np.arange(n), pi] = 1.0
    return w


def cyclic(n: int, shift: int) -> np.ndarray:
    return (np.arange(n) + shift) % n


def test_linear_golden(oracle_mod):
    g = read_golden("linear_2x3.txt")
    a = np.array([g["a0"], g["a1"]], np.float64)
    w = np.array([g["w0"], g["w1"]], np.float64)
    y = oracle_mod.linear(a, w)
    np.testing.assert_array_equal(y, np.array([g["y0"], g["y1"]]))


def test_linear_orientation_by_permutation(oracle_mod):
    a = RNG.standard_normal((5, 7))
    pi = cyclic(7, 3)  # a 7-cycle: not its own inverse
    y = oracle_mod.linear(a, perm_matrix(pi))
    np.testing.assert_array_equal(y, a[:, pi])
    assert not np.array_equal(y, a[:, np.argsort(pi)])


def test_linear_is_torch_linear_and_widens_bf16_exactly(oracle_mod):
    a32 = RNG.standard_normal((6, 16)).astype(np.float32)
    w32 = RNG.standard_normal((9, 16)).astype(np.float32)
    ta = torch.from_numpy(a32).to(torch.bfloat16)
    tw = torch.from_numpy(w32).to(torch.bfloat16)
    a_bits = ta.view(torch.int16).numpy().view(np.uint16)
    w_bits = tw.view(torch.int16).numpy().view(np.uint16)
    ref = F.linear(ta.double(), tw.double()).numpy()
    np.testing.assert_allclose(oracle_mod.linear(a_bits, w_bits), ref, rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(oracle_mod.to_f64(a_bits), ta.double().numpy())


def test_linear_magnitude_bounds_the_product(oracle_mod):
    a = RNG.standard_normal((4, 32))
    w = RNG.standard_normal((6, 32))
    m = oracle_mod.linear_magnitude(a, w)
    assert np.all(m >= np.abs(oracle_mod.linear(a, w)) - 1e-12)
    # equal when every term is non-negative
    np.testing.assert_allclose(oracle_mod.linear_magnitude(np.abs(a), np.abs(w)),
                               oracle_mod.linear(np.abs(a), np.abs(w)), rtol=1e-14)


def test_linear_swiglu_golden(oracle_mod):
    g = read_golden("linear_swiglu_k2.txt")
    a = np.array([g["a"]], np.float64)
    w = np.array([g["w0"], g["w1"], g["w2"], g["w3"]], np.float64)
    out = oracle_mod.linear_swiglu(a, w, 2)
    np.testing.assert_allclose(out[0], g["out"], rtol=1e-15, atol=0)


def test_linear_swiglu_halves_by_permutation(oracle_mod):
    k, inner = 12, 6
    a = RNG.standard_normal((5, k))
    p1, p2 = cyclic(k, 5)[:inner], cyclic(k, 1)[inner:]
    w = np.concatenate([perm_matrix(cyclic(k, 5))[:inner], perm_matrix(cyclic(k, 1))[inner:]])
    out = oracle_mod.linear_swiglu(a, w, inner)
    ta = torch.from_numpy(a)
    ref = (F.silu(ta[:, p1]) * ta[:, p2]).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-14, atol=1e-15)
    swapped = (F.silu(ta[:, p2]) * ta[:, p1]).numpy()
    assert np.abs(out - swapped).max() > 1e-3


def test_linear_gated_residual_special_gates_and_rows(oracle_mod):
    n, k = 6, 8
    x = RNG.standard_normal((n, k))
    a = RNG.standard_normal((n, k))
    pi = cyclic(k, 3)
    w = perm_matrix(pi)
    zero = np.zeros((1, k))
    np.testing.assert_array_equal(oracle_mod.linear_gated_residual(x, a, w, zero), x)
    one = np.ones((1, k))
    np.testing.assert_allclose(oracle_mod.linear_gated_residual(x, a, w, one), x + a[:, pi],
                               rtol=1e-15, atol=1e-15)
    # two samples of three tokens: each uses its own gate row
    gate = RNG.standard_normal((2, k))
    out = oracle_mod.linear_gated_residual(x, a, w, gate, tokens_per_sample=3)
    y = a[:, pi]
    ref = np.concatenate([x[:3] + gate[0] * y[:3], x[3:] + gate[1] * y[3:]])
    np.testing.assert_allclose(out, ref, rtol=1e-15, atol=1e-15)


def test_linear_gated_residual_linear_in_weights(oracle_mod):
    n, k, m = 5, 16, 8
    x = RNG.standard_normal((n, m))
    a = RNG.standard_normal((n, k))
    w1, w2 = RNG.standard_normal((m, k)), RNG.standard_normal((m, k))
    gate = RNG.standard_normal((1, m))
    f = lambda w: oracle_mod.linear_gated_residual(x, a, w, gate) - x
    np.testing.assert_allclose(f(w1 + w2), f(w1) + f(w2), rtol=1e-12, atol=1e-12)


def test_adaln_linear_by_permutation_is_layer_norm_modulated(oracle_mod):
    n, d = 7, 16
    x = RNG.standard_normal((n, d)) * 3 + 1
    shift = RNG.standard_normal((1, d)) * 0.1
    scale = RNG.standard_normal((1, d)) * 0.1
    pi = cyclic(d, 5)
    y, h = oracle_mod.adaln_linear(x, perm_matrix(pi), shift, scale, eps=1e-6)
    tx = torch.from_numpy(x)
    ref_h = (F.layer_norm(tx, (d,), eps=1e-6) * (1 + torch.from_numpy(scale))
             + torch.from_numpy(shift)).numpy()
    np.testing.assert_allclose(h, ref_h, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(y, h[:, pi])


def test_adaln_linear_rows_select_modulation(oracle_mod):
    n, d, m = 6, 8, 4
    x = RNG.standard_normal((n, d))
    w = RNG.standard_normal((m, d))
    shift = RNG.standard_normal((4, d)) * 0.1
    scale = RNG.standard_normal((4, d)) * 0.1
    sid = np.array([0, 1, 0, 1, 1, 0], np.uint8)
    full, _ = oracle_mod.adaln_linear(x, w, shift, scale, stream_id=sid, n_streams=2,
                                      tokens_per_sample=3)
    rows = np.array([4, 1])
    part, _ = oracle_mod.adaln_linear(np.ascontiguousarray(x[rows]), w, shift, scale,
                                      stream_id=sid, n_streams=2, tokens_per_sample=3, rows=rows)
    np.testing.assert_array_equal(part, full[rows])
    # token 4 is sample 1, stream 1 -> row 3 of each modulation tensor
    tx = torch.from_numpy(x[4:5])
    h4 = (F.layer_norm(tx, (d,), eps=1e-6) * (1 + torch.from_numpy(scale[3])) +
          torch.from_numpy(shift[3])).numpy()
    np.testing.assert_allclose(part[0], (h4 @ w.T)[0], rtol=1e-12, atol=1e-12)


def test_adaln_qkv_rope_wiring(oracle_mod):
    n_heads, head_dim = 2, 16
    hd = n_heads * head_dim
    d = 3 * hd
    n = 5
    x = RNG.standard_normal((n, d))
    shift = RNG.standard_normal((1, d)) * 0.1
    scale = RNG.standard_normal((1, d)) * 0.1
    wq = 1 + RNG.standard_normal(head_dim) * 0.02
    wk = 1 + RNG.standard_normal(head_dim) * 0.02
    pi = cyclic(d, 7)
    w = perm_matrix(pi)
    pos = RNG.integers(0, 5, size=(n, 3)).astype(np.int32)
    kw = dict(n_heads=n_heads, head_dim=head_dim, pos=pos, dims=(4, 6, 6), eps=1e-6)
    out, pre, h = oracle_mod.adaln_qkv_rope(x, w, shift, scale, wq, wk, **kw)
    np.testing.assert_array_equal(pre, h[:, pi])
    qk = oracle_mod.dit_epilogue(np.ascontiguousarray(h[:, pi]), wq, wk, **kw)
    np.testing.assert_array_equal(out[:, :2 * hd], qk)
    np.testing.assert_array_equal(out[:, 2 * hd:], h[:, pi][:, 2 * hd:])
    # q and k come out with the RMS of their weights (norm then a rotation)
    qh = out[:, :hd].reshape(n, n_heads, head_dim)
    rms_q = np.sqrt((qh ** 2).mean(-1))
    pre_q = pre[:, :hd].reshape(n, n_heads, head_dim)
    expect = np.sqrt(((pre_q * wq) ** 2).mean(-1) / ((pre_q ** 2).mean(-1) + 1e-6))
    np.testing.assert_allclose(rms_q, expect, rtol=1e-12)


def test_adaln_linear_swiglu_by_permutation(oracle_mod):
    n, d, inner = 6, 16, 8
    x = RNG.standard_normal((n, d)) * 2 - 0.5
    shift = RNG.standard_normal((1, d)) * 0.1
    scale = RNG.standard_normal((1, d)) * 0.1
    p1, p2 = cyclic(d, 3)[:inner], cyclic(d, 11)[inner:]
    w = np.concatenate([perm_matrix(cyclic(d, 3))[:inner], perm_matrix(cyclic(d, 11))[inner:]])
    out, u, h = oracle_mod.adaln_linear_swiglu(x, w, shift, scale, inner, eps=1e-6)
    th = torch.from_numpy(h)
    np.testing.assert_allclose(out, (F.silu(th[:, p1]) * th[:, p2]).numpy(), rtol=1e-13, atol=1e-14)
    np.testing.assert_array_equal(u, np.concatenate([h[:, p1], h[:, p2]], axis=1))
    ref_h = (F.layer_norm(torch.from_numpy(x), (d,), eps=1e-6) * (1 + torch.from_numpy(scale))
             + torch.from_numpy(shift)).numpy()
    np.testing.assert_allclose(h, ref_h, rtol=1e-12, atol=1e-13)
