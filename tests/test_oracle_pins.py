"""Pins for the fp64 oracle: library special cases, invariants, closed forms and brute force.

Each test pins the oracle to something other than itself, so that a plausible slip in
oracle.c (a dropped term, a wrong sign or index, a swapped operand, the wrong half or
the wrong frequency) fails at least one of them.  CPU only.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from conftest import read_golden

RNG = np.random.default_rng(1234)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 with torch (round to nearest even) and return the bits."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


# ----------------------------------------------------------------------------- AdaLN


def test_adaln_golden(oracle_mod):
    g = read_golden("adaln_d4.txt")
    x = np.array([g["x"], g["x2"]], np.float64)
    shift = np.array([g["shift"], g["shift2"]], np.float64)
    scale = np.array([g["scale"], g["scale2"]], np.float64)
    # one modulation row per sample: two samples of one token each
    h = oracle_mod.adaln_modulate(x, shift, scale, eps=g["eps"][0], tokens_per_sample=1)
    np.testing.assert_array_equal(h[0], g["h"])
    h = oracle_mod.adaln_modulate(x, shift, scale, eps=g["eps2"][0], tokens_per_sample=1)
    np.testing.assert_array_equal(h[1], g["h2"])


@pytest.mark.parametrize("d", [4, 256, 5120])
def test_adaln_zero_modulation_is_layer_norm(oracle_mod, d):
    x = RNG.standard_normal((7, d)) * 3 + 1.5
    h = oracle_mod.adaln_modulate(x, None, None, eps=1e-6)
    ref = F.layer_norm(torch.from_numpy(x), (d,), eps=1e-6).numpy()
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_adaln_is_affine_layer_norm_with_one_plus_scale(oracle_mod):
    d = 384
    x = RNG.standard_normal((5, d))
    shift = RNG.standard_normal((1, d)) * 0.1
    scale = RNG.standard_normal((1, d)) * 0.1
    h = oracle_mod.adaln_modulate(x, shift, scale, eps=1e-6)
    ref = F.layer_norm(torch.from_numpy(x), (d,), weight=torch.from_numpy(1.0 + scale[0]),
                       bias=torch.from_numpy(shift[0]), eps=1e-6).numpy()
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_adaln_moments_and_invariances(oracle_mod):
    d, eps = 512, 1e-6
    x = RNG.standard_normal((6, d)) * np.array([[0.01], [0.1], [1], [10], [50], [1e3]])
    h = oracle_mod.adaln_modulate(x, None, None, eps=eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(h.mean(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(h.var(axis=1), var / (var + eps), rtol=1e-10)
    # translation invariance LN(x + c) = LN(x); modulation is added after the norm
    shift = RNG.standard_normal((1, d)) * 0.1
    scale = RNG.standard_normal((1, d)) * 0.1
    h1 = oracle_mod.adaln_modulate(x, shift, scale, eps=eps)
    h2 = oracle_mod.adaln_modulate(x + 17.25, shift, scale, eps=eps)
    np.testing.assert_allclose(h1, h2, rtol=1e-9, atol=1e-9)
    # shift enters additively, scale as a (1 + scale) factor on the normalised row
    h0 = oracle_mod.adaln_modulate(x, None, scale, eps=eps)
    np.testing.assert_allclose(h1 - h0, np.broadcast_to(shift, h1.shape), atol=1e-12)
    hn = oracle_mod.adaln_modulate(x, None, None, eps=eps)
    np.testing.assert_allclose(h0, hn * (1 + scale), rtol=1e-12, atol=1e-12)


def test_adaln_outlier_row_two_pass(oracle_mod):
    # a row with +-50 outliers and a huge common offset: one-pass E[x^2]-E[x]^2 in fp64
    # would lose digits; the two-pass definition must still match torch's layer_norm.
    d = 5120
    x = RNG.standard_normal((3, d))
    x[:, ::997] = 50.0
    x[1] += 1e6
    h = oracle_mod.adaln_modulate(x, None, None, eps=1e-6)
    ref = F.layer_norm(torch.from_numpy(x), (d,), eps=1e-6).numpy()
    np.testing.assert_allclose(h, ref, rtol=1e-9, atol=1e-9)


def test_modulation_selection_by_sample_and_stream(oracle_mod):
    """The batched call equals independent calls on each (sample, stream) piece with its
    own single modulation row: rows are laid out sample-major, stream-minor."""
    d, B, S, tps = 64, 3, 2, 5
    n = B * tps
    x = RNG.standard_normal((n, d))
    y = RNG.standard_normal((n, d))
    shift = RNG.standard_normal((B * S, d))
    scale = RNG.standard_normal((B * S, d))
    gate = RNG.standard_normal((B * S, d))
    sid = RNG.integers(0, S, size=n).astype(np.uint8)
    h = oracle_mod.adaln_modulate(x, shift, scale, stream_id=sid, n_streams=S, tokens_per_sample=tps)
    o = oracle_mod.gated_residual(x, y, gate, stream_id=sid, n_streams=S, tokens_per_sample=tps)
    for b in range(B):
        for s in range(S):
            rows = [i for i in range(b * tps, (b + 1) * tps) if sid[i] == s]
            if not rows:
                continue
            r = b * S + s
            hp = oracle_mod.adaln_modulate(np.ascontiguousarray(x[rows]), shift[r:r + 1],
                                           scale[r:r + 1])
            op = oracle_mod.gated_residual(np.ascontiguousarray(x[rows]),
                                           np.ascontiguousarray(y[rows]), gate[r:r + 1])
            np.testing.assert_array_equal(h[rows], hp)
            np.testing.assert_array_equal(o[rows], op)


def test_adaln_bf16_and_f32_inputs_widen_exactly(oracle_mod):
    d = 256
    x32 = (RNG.standard_normal((4, d)) * 2).astype(np.float32)
    xb = bf16_bits(x32)
    h_b = oracle_mod.adaln_modulate(xb, None, None)
    h_ref = oracle_mod.adaln_modulate(bits_to_f64(xb), None, None)
    np.testing.assert_array_equal(h_b, h_ref)
    h_f = oracle_mod.adaln_modulate(x32, None, None)
    h_ref = oracle_mod.adaln_modulate(x32.astype(np.float64), None, None)
    np.testing.assert_array_equal(h_f, h_ref)


# ---------------------------------------------------------------------- gated residual


def test_gated_residual_golden(oracle_mod):
    g = read_golden("gated_residual_d2.txt")
    x = np.array([g["x"]]); y = np.array([g["y"]]); gate = np.array([g["gate"]])
    o = oracle_mod.gated_residual(x, y, gate)
    np.testing.assert_array_equal(o[0], g["o"])


def test_gated_residual_special_gates(oracle_mod):
    d = 5120
    x = bf16_bits(RNG.standard_normal((3, d)).astype(np.float32))
    y = bf16_bits(RNG.standard_normal((3, d)).astype(np.float32))
    zero = bf16_bits(np.zeros((1, d), np.float32))
    one = bf16_bits(np.ones((1, d), np.float32))
    np.testing.assert_array_equal(oracle_mod.gated_residual(x, y, zero), bits_to_f64(x))
    np.testing.assert_array_equal(oracle_mod.gated_residual(x, y, None), bits_to_f64(x))
    # bf16 + bf16 is exact in fp64
    np.testing.assert_array_equal(oracle_mod.gated_residual(x, y, one), bits_to_f64(x) + bits_to_f64(y))


def test_gated_residual_linear_in_gate(oracle_mod):
    d = 300
    x = RNG.standard_normal((4, d)); y = RNG.standard_normal((4, d))
    g1 = RNG.standard_normal((1, d)); g2 = RNG.standard_normal((1, d))
    o1 = oracle_mod.gated_residual(x, y, g1)
    o2 = oracle_mod.gated_residual(x, y, g2)
    o12 = oracle_mod.gated_residual(x, y, g1 + g2)
    np.testing.assert_allclose(o1 + o2 - x, o12, rtol=1e-12, atol=1e-12)
    # y enters through the gate only: swapping the roles of x and y changes the result
    assert not np.allclose(oracle_mod.gated_residual(y, x, g1), o1)


# ----------------------------------------------------------------------------- SwiGLU


def test_silu_closed_forms(oracle_mod):
    g = read_golden("silu_closed_forms.txt")
    for c, k, ratio in g[None]:
        a = float(c) * math.log(float(k))
        o = oracle_mod.swiglu_ab(np.array([[a]]), np.array([[1.0]]))[0, 0]
        assert abs(o / a - float(ratio)) < 1e-15
    assert oracle_mod.swiglu_ab(np.zeros((1, 4)), np.ones((1, 4))).tolist() == [[0.0] * 4]


def test_swiglu_is_torch_silu_times_second_half(oracle_mod):
    n, inner = 6, 512
    a = RNG.standard_normal((n, inner)) * 4
    b = RNG.standard_normal((n, inner))
    u = np.ascontiguousarray(np.concatenate([a, b], axis=1))
    o = oracle_mod.swiglu(u)
    ref = (F.silu(torch.from_numpy(a)) * torch.from_numpy(b)).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-13, atol=1e-15)
    # the first half is the gated one: with b = 1 the result is silu(a), not a*silu(1)
    u1 = np.ascontiguousarray(np.concatenate([a, np.ones_like(a)], axis=1))
    np.testing.assert_allclose(oracle_mod.swiglu(u1), F.silu(torch.from_numpy(a)).numpy(),
                               rtol=1e-13, atol=1e-15)


def test_silu_odd_part_and_limits(oracle_mod):
    a = RNG.standard_normal((3, 200)) * 6
    one = np.ones_like(a)
    sp = oracle_mod.swiglu_ab(a, one)
    sm = oracle_mod.swiglu_ab(np.ascontiguousarray(-a), one)
    np.testing.assert_allclose(sp - sm, a, rtol=1e-13, atol=1e-13)  # silu(x) - silu(-x) = x
    big = np.array([[40.0, 80.0, -40.0, -80.0, -800.0]])
    o = oracle_mod.swiglu_ab(big, np.ones_like(big))[0]
    assert abs(o[0] - 40.0) < 1e-12 and abs(o[1] - 80.0) < 1e-12
    assert 0 >= o[2] > -1e-15 and 0 >= o[3] > -1e-30 and o[4] == 0.0


# ------------------------------------------------------------------ QK RMSNorm + RoPE


def _qk(oracle_mod, v, w=None, pos=None, eps=1e-6, n_heads=1, head_dim=128, dims=(32, 48, 48)):
    qo, _ = oracle_mod.qk_rmsnorm_rope3d(v, None, w, None, n_heads=n_heads, head_dim=head_dim,
                                        pos=pos, dims=dims, eps=eps)
    return qo


def test_rmsnorm_at_origin_is_torch_rms_norm(oracle_mod):
    n, Hh, Dh = 5, 3, 128
    v = RNG.standard_normal((n, Hh * Dh)) * 2.5
    w = 1 + 0.02 * RNG.standard_normal(Dh)
    pos = np.zeros((n, 3), np.int32)
    out = _qk(oracle_mod, v, w, pos, n_heads=Hh)
    ref = F.rms_norm(torch.from_numpy(v).view(n, Hh, Dh), (Dh,), weight=torch.from_numpy(w),
                     eps=1e-6).reshape(n, Hh * Dh).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_rmsnorm_unit_rms_and_scale_invariance(oracle_mod):
    v = RNG.standard_normal((4, 128)) * np.array([[0.05], [1.0], [20.0], [300.0]])
    pos = np.array([[3, 7, 11]] * 4, np.int32)
    out = _qk(oracle_mod, v, None, pos, eps=1e-6)
    ms = (v * v).mean(axis=1)
    np.testing.assert_allclose(np.sqrt((out * out).mean(axis=1)), np.sqrt(ms / (ms + 1e-6)),
                               rtol=1e-12)
    out0 = _qk(oracle_mod, v, None, pos, eps=0.0)
    out1 = _qk(oracle_mod, v * 7.5, None, pos, eps=0.0)
    np.testing.assert_allclose(out0, out1, rtol=1e-12, atol=1e-12)


def test_rope_golden_angles(oracle_mod):
    """One nonzero input pair: the output is the same pair turned by the angle worked by
    hand; every other element stays zero."""
    g = read_golden("rope3d_angles.txt")
    axis_of = {"t": 0, "h": 1, "w": 2}
    for axis, off, D, j, p, angle in g[None]:
        off, D, j, p, angle = int(off), int(D), int(j), int(p), float(angle)
        v = np.zeros((1, 128))
        v[0, off + 2 * j] = 1.0
        pos = np.zeros((1, 3), np.int32)
        pos[0, axis_of[axis]] = p
        out = _qk(oracle_mod, v, None, pos, eps=0.0)[0]
        r = math.sqrt(128.0)  # RMS of a one-hot 128-vector is 1/sqrt(128)
        assert abs(out[off + 2 * j] - r * math.cos(angle)) < 1e-12
        assert abs(out[off + 2 * j + 1] - r * math.sin(angle)) < 1e-12
        rest = np.delete(out, [off + 2 * j, off + 2 * j + 1])
        assert np.all(rest == 0.0)


def test_rope_axis_chunks(oracle_mod):
    """A move along one axis touches exactly that axis' chunk: t = dims [0,32),
    h = [32,80), w = [80,128)."""
    v = RNG.standard_normal((1, 128))
    base = _qk(oracle_mod, v, None, np.zeros((1, 3), np.int32))[0]
    for ax, (lo, hi) in enumerate([(0, 32), (32, 80), (80, 128)]):
        pos = np.zeros((1, 3), np.int32)
        pos[0, ax] = 5
        out = _qk(oracle_mod, v, None, pos)[0]
        changed = np.nonzero(out != base)[0]
        assert changed.min() >= lo and changed.max() < hi and len(changed) == hi - lo


def test_rope_preserves_pair_norms_and_inverts(oracle_mod):
    v = RNG.standard_normal((6, 128))
    pos = RNG.integers(0, 90, size=(6, 3)).astype(np.int32)
    out = _qk(oracle_mod, v, None, pos, eps=0.0)
    base = _qk(oracle_mod, v, None, np.zeros_like(pos), eps=0.0)
    np.testing.assert_allclose(np.hypot(out[:, 0::2], out[:, 1::2]),
                               np.hypot(base[:, 0::2], base[:, 1::2]), rtol=1e-13)
    # R(-p) R(p) = I; the second RMSNorm acts on a unit-RMS vector and changes nothing
    back = _qk(oracle_mod, out, None, -pos, eps=0.0)
    np.testing.assert_allclose(back, base, rtol=1e-12, atol=1e-12)


def test_rope_relative_positions(oracle_mod):
    """<R(m) q, R(n) k> depends only on m - n along each axis."""
    q = RNG.standard_normal((1, 128)); k = RNG.standard_normal((1, 128))
    m = np.array([[4, 9, 2]], np.int32); nn = np.array([[1, 3, 30]], np.int32)
    ref = (_qk(oracle_mod, q, None, m, eps=0.0) @ _qk(oracle_mod, k, None, nn, eps=0.0).T).item()
    for c in ([0, 0, 7], [11, 0, 0], [0, 13, 0], [5, 6, 40]):
        c = np.array([c], np.int32)
        got = (_qk(oracle_mod, q, None, m + c, eps=0.0) @ _qk(oracle_mod, k, None, nn + c, eps=0.0).T).item()
        assert abs(got - ref) < 1e-11
    # and it does change with the offset
    got = (_qk(oracle_mod, q, None, m + np.array([[1, 0, 0]], np.int32), eps=0.0)
           @ _qk(oracle_mod, k, None, nn, eps=0.0).T).item()
    assert abs(got - ref) > 1e-6


def _rotation_matrix(p, dims=(32, 48, 48), theta=10000.0):
    """Explicit block-diagonal rotation of one head vector, built entry by entry."""
    D = sum(dims)
    R = np.zeros((D, D))
    off = 0
    for c, Dc in enumerate(dims):
        for j in range(Dc // 2):
            phi = p[c] * theta ** (-2.0 * j / Dc)
            a, b = off + 2 * j, off + 2 * j + 1
            R[a, a] = math.cos(phi); R[a, b] = -math.sin(phi)
            R[b, a] = math.sin(phi); R[b, b] = math.cos(phi)
        off += Dc
    return R


def test_rope_brute_force_tiny_grid(oracle_mod):
    """On the 2x4x4 grid with implicit positions, every token equals the explicit
    rotation matrix times the torch-RMS-normalised head vector."""
    T, H, W, Hh, Dh = 2, 4, 4, 2, 128
    n = T * H * W
    v = RNG.standard_normal((n, Hh * Dh))
    w = 1 + 0.02 * RNG.standard_normal(Dh)
    out, _ = oracle_mod.qk_rmsnorm_rope3d(v, None, w, None, n_heads=Hh, head_dim=Dh,
                                         grid=(T, H, W), tokens_per_sample=n)
    vn = F.rms_norm(torch.from_numpy(v).view(n, Hh, Dh), (Dh,), weight=torch.from_numpy(w),
                    eps=1e-6).numpy()
    idx = 0
    for t in range(T):
        for h in range(H):
            for ww in range(W):
                R = _rotation_matrix((t, h, ww))
                for hh in range(Hh):
                    np.testing.assert_allclose(out[idx, hh * Dh:(hh + 1) * Dh], R @ vn[idx, hh],
                                               rtol=1e-12, atol=1e-12)
                idx += 1


def test_rope_complex_form_packed_positions(oracle_mod):
    """Explicit positions of a packed video+audio layout (from the workload generator)
    against the complex-number form z' = z * exp(i*phi); audio tokens leave the h and w
    chunks untouched."""
    from dit_block_b200 import workloads
    w = workloads.Workload("t", 9, torch.float32, 2, (2, 3, 2), 4, 64, 1, 128, 64)
    pos, sid = workloads.token_layout(w)
    pos = pos.numpy()
    n = pos.shape[0]
    v = RNG.standard_normal((n, 128))
    out = _qk(oracle_mod, v, None, pos, eps=0.0)
    vn = v / np.sqrt((v * v).mean(axis=1, keepdims=True))
    freqs = np.concatenate([10000.0 ** (-2.0 * np.arange(Dc // 2) / Dc) for Dc in (32, 48, 48)])
    axis = np.repeat([0, 1, 2], [16, 24, 24])
    phi = pos[:, axis] * freqs[None, :]
    z = (vn[:, 0::2] + 1j * vn[:, 1::2]) * np.exp(1j * phi)
    np.testing.assert_allclose(out[:, 0::2], z.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[:, 1::2], z.imag, rtol=1e-12, atol=1e-12)
    audio = sid.numpy() == 1
    np.testing.assert_allclose(out[audio][:, 32:], vn[audio][:, 32:], rtol=1e-13, atol=1e-13)


def test_implicit_grid_positions_match_explicit_meshgrid(oracle_mod):
    """pos == NULL derives (t, h, w) of each sample's row-major grid; compare with positions
    laid out by torch.meshgrid for a 2-sample batch."""
    T, H, W = 3, 2, 5
    tpsamp = T * H * W
    tt, hh, ww = torch.meshgrid(torch.arange(T), torch.arange(H), torch.arange(W), indexing="ij")
    one = torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], 1)
    pos = torch.cat([one, one]).to(torch.int32).numpy()
    v = RNG.standard_normal((2 * tpsamp, 2 * 128))
    a, _ = oracle_mod.qk_rmsnorm_rope3d(v, None, n_heads=2, head_dim=128, grid=(T, H, W),
                                       tokens_per_sample=tpsamp)
    b, _ = oracle_mod.qk_rmsnorm_rope3d(v, None, n_heads=2, head_dim=128, pos=pos)
    np.testing.assert_array_equal(a, b)


def test_q_and_k_use_their_own_weights(oracle_mod):
    v = RNG.standard_normal((3, 256))
    wq = 1 + 0.02 * RNG.standard_normal(128); wk = 1 + 0.02 * RNG.standard_normal(128)
    pos = np.array([[1, 2, 3]] * 3, np.int32)
    qo, ko = oracle_mod.qk_rmsnorm_rope3d(v, v, wq, wk, n_heads=2, head_dim=128, pos=pos)
    np.testing.assert_array_equal(qo, _qk(oracle_mod, v, wq, pos, n_heads=2))
    np.testing.assert_array_equal(ko, _qk(oracle_mod, v, wk, pos, n_heads=2))
    assert not np.array_equal(qo, ko)


# ------------------------------------------------------------------ fused prologue / epilogue


def test_prologue_is_composition(oracle_mod):
    d = 256
    x = bf16_bits(RNG.standard_normal((6, d)).astype(np.float32))
    y = bf16_bits(RNG.standard_normal((6, d)).astype(np.float32))
    gate, shift, scale = (bf16_bits((0.1 * RNG.standard_normal((1, d))).astype(np.float32))
                          for _ in range(3))
    xo, h = oracle_mod.dit_prologue(x, y, gate, shift, scale)
    x_ref = oracle_mod.gated_residual(x, y, gate)
    np.testing.assert_array_equal(xo, x_ref)
    # AdaLN of the unrounded fp64 residual sum
    np.testing.assert_array_equal(h, oracle_mod.adaln_modulate(x_ref, shift, scale))
    xo2, h2 = oracle_mod.dit_prologue(x, None, gate, shift, scale)
    assert xo2 is None
    np.testing.assert_array_equal(h2, oracle_mod.adaln_modulate(x, shift, scale))


def test_epilogue_is_q_and_k_slices(oracle_mod):
    Hh, Dh, n = 2, 128, 9
    qkv = RNG.standard_normal((n, 3 * Hh * Dh))
    wq = 1 + 0.02 * RNG.standard_normal(Dh); wk = 1 + 0.02 * RNG.standard_normal(Dh)
    out = oracle_mod.dit_epilogue(qkv, wq, wk, n_heads=Hh, head_dim=Dh, grid=(1, 3, 3),
                                  tokens_per_sample=n)
    hd = Hh * Dh
    q = np.ascontiguousarray(qkv[:, :hd]); k = np.ascontiguousarray(qkv[:, hd:2 * hd])
    qo, ko = oracle_mod.qk_rmsnorm_rope3d(q, k, wq, wk, n_heads=Hh, head_dim=Dh, grid=(1, 3, 3),
                                         tokens_per_sample=n)
    np.testing.assert_array_equal(out[:, :hd], qo)
    np.testing.assert_array_equal(out[:, hd:], ko)


def test_bad_split_rejected(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.qk_rmsnorm_rope3d(np.zeros((1, 128)), None, n_heads=1, head_dim=128,
                                     pos=np.zeros((1, 3), np.int32), dims=(32, 48, 47))


def test_row_subsets_equal_rows_of_the_full_sequence(oracle_mod):
    """Evaluating a subset of rows with their global token indices gives exactly those
    rows of the full evaluation (modulation row, stream id and implicit position all
    follow the global index)."""
    B, T, H, W, d, Hh, Dh = 2, 2, 3, 4, 64, 2, 128
    tps = T * H * W
    n = B * tps
    x = RNG.standard_normal((n, d)); y = RNG.standard_normal((n, d))
    S = 2
    mods = [RNG.standard_normal((B * S, d)) for _ in range(3)]
    sid = RNG.integers(0, S, size=n).astype(np.uint8)
    qkv = RNG.standard_normal((n, 3 * Hh * Dh))
    rows = np.array([0, 5, tps - 1, tps, tps + 7, n - 1])
    kw = dict(stream_id=sid, n_streams=S, tokens_per_sample=tps)
    full = oracle_mod.dit_prologue(x, y, *mods, **kw)
    sub = oracle_mod.dit_prologue(np.ascontiguousarray(x[rows]), np.ascontiguousarray(y[rows]),
                                  *mods, rows=rows, **kw)
    np.testing.assert_array_equal(sub[0], full[0][rows])
    np.testing.assert_array_equal(sub[1], full[1][rows])
    ek = dict(n_heads=Hh, head_dim=Dh, grid=(T, H, W), tokens_per_sample=tps)
    e_full = oracle_mod.dit_epilogue(qkv, **ek)
    e_sub = oracle_mod.dit_epilogue(np.ascontiguousarray(qkv[rows]), rows=rows, **ek)
    np.testing.assert_array_equal(e_sub, e_full[rows])


# ------------------------------------------------------- Cache-DiT residual change


def test_cache_diff_golden(oracle_mod):
    g = read_golden("cache_diff_d2.txt")
    x = np.array(g["x"]).reshape(2, 2); y = np.array(g["y"]).reshape(2, 2)
    gate = np.array(g["gate"]).reshape(2, 2); cache = np.array(g["cache"]).reshape(2, 2)
    out, r, sums = oracle_mod.gated_residual_cache_diff(x, y, gate, cache, n_samples=2,
                                                        tokens_per_sample=1)
    np.testing.assert_array_equal(out.reshape(-1), g["out"])
    np.testing.assert_array_equal(sums.reshape(-1), g["sums"])
    np.testing.assert_array_equal(r, gate * y)


def test_cache_diff_invariants(oracle_mod):
    d, B, tps = 96, 3, 7
    n = B * tps
    x = RNG.standard_normal((n, d)); y = RNG.standard_normal((n, d))
    gate = RNG.standard_normal((B, d)) * 0.1
    # the output is the plain gated residual
    out, r, sums = oracle_mod.gated_residual_cache_diff(x, y, gate, np.zeros((n, d)), n_samples=B,
                                                        tokens_per_sample=tps)
    np.testing.assert_array_equal(out, oracle_mod.gated_residual(x, y, gate, tokens_per_sample=tps))
    # an all-zero cache: no reference mass, the change is the residual's own L1 mass
    np.testing.assert_array_equal(sums[:, 1], 0.0)
    for b in range(B):
        np.testing.assert_allclose(sums[b, 0], np.abs(r[b * tps:(b + 1) * tps]).sum(), rtol=1e-13)
    # comparing against its own refreshed cache: no change
    _, r2, sums2 = oracle_mod.gated_residual_cache_diff(x, y, gate, r, n_samples=B, tokens_per_sample=tps)
    np.testing.assert_array_equal(sums2[:, 0], 0.0)
    np.testing.assert_allclose(sums2[:, 1], sums[:, 0], rtol=1e-13)
    # scaling y and the cache together scales both sums (the ratio is scale free)
    c = RNG.standard_normal((n, d)) * 0.1
    _, _, s1 = oracle_mod.gated_residual_cache_diff(x, y, gate, c, n_samples=B, tokens_per_sample=tps)
    _, _, s2 = oracle_mod.gated_residual_cache_diff(x, 4 * y, gate, 4 * c, n_samples=B, tokens_per_sample=tps)
    np.testing.assert_allclose(s2, 4 * s1, rtol=1e-12)
    # samples are independent: sample b's sums depend only on its rows
    c2 = c.copy(); c2[tps:2 * tps] += 1.0
    _, _, s3 = oracle_mod.gated_residual_cache_diff(x, y, gate, c2, n_samples=B, tokens_per_sample=tps)
    np.testing.assert_array_equal(s3[[0, 2]], s1[[0, 2]])
    assert not np.allclose(s3[1], s1[1])


def test_cache_diff_packed_streams_share_one_decision(oracle_mod):
    """Video and audio tokens of a sample use their own gates but add into one sum."""
    d, B, S, tps = 32, 2, 2, 9
    n = B * tps
    x = RNG.standard_normal((n, d)); y = RNG.standard_normal((n, d)); c = RNG.standard_normal((n, d))
    gate = RNG.standard_normal((B * S, d))
    sid = np.array(([0] * 6 + [1] * 3) * B, np.uint8)
    _, r, sums = oracle_mod.gated_residual_cache_diff(x, y, gate, c, n_samples=B, stream_id=sid,
                                                      n_streams=S, tokens_per_sample=tps)
    for b in range(B):
        blk = slice(b * tps, (b + 1) * tps)
        np.testing.assert_allclose(sums[b, 0], np.abs(r[blk] - c[blk]).sum(), rtol=1e-13)
        np.testing.assert_allclose(sums[b, 1], np.abs(c[blk]).sum(), rtol=1e-13)
    # the audio rows of sample 1 took gate row 3
    np.testing.assert_allclose(r[tps + 6], gate[3] * y[tps + 6], rtol=0, atol=0)


# ------------------------------------------------------------- SubBlock block means


def test_block_mean_layout_and_ragged_tail(oracle_mod):
    """A 130-token sample in 64-token blocks gives blocks of 64, 64 and 2 tokens; the
    next sample starts a new block.  Rows are filled with their token index, so each
    block mean is the mean of a run of integers (closed form (first + last) / 2)."""
    tps, B, blk = 130, 2, 64
    n = B * tps
    v = np.repeat(np.arange(n, dtype=np.float64)[:, None], 3, axis=1)
    p = oracle_mod.block_mean(v, tokens_per_sample=tps, block=blk)
    assert p.shape == (6, 3)
    starts_ends = [(0, 63), (64, 127), (128, 129), (130, 193), (194, 257), (258, 259)]
    for row, (a, b) in enumerate(starts_ends):
        np.testing.assert_array_equal(p[row], (a + b) / 2.0)


def test_block_mean_constant_blocks_and_linearity(oracle_mod):
    n, w = 200, 16
    base = RNG.standard_normal((4, w))
    v = np.repeat(base, [64, 64, 64, 8], axis=0)
    p = oracle_mod.block_mean(v, block=64)
    np.testing.assert_allclose(p, base, rtol=1e-14)
    a = RNG.standard_normal((n, w)); b = RNG.standard_normal((n, w))
    np.testing.assert_allclose(oracle_mod.block_mean(2 * a - b, block=64),
                               2 * oracle_mod.block_mean(a, block=64) - oracle_mod.block_mean(b, block=64),
                               rtol=1e-13, atol=1e-14)


# ------------------------------------------------- convention variants (norm span, pairing)


def _qkx(oracle_mod, v, w=None, pos=None, eps=1e-6, n_heads=1, head_dim=128, **kw):
    qo, _ = oracle_mod.qk_rmsnorm_rope3d_ex(v, None, w, None, n_heads=n_heads, head_dim=head_dim, pos=pos,
                                            eps=eps, **kw)
    return qo


def test_ex_defaults_equal_the_base_oracle(oracle_mod):
    v = RNG.standard_normal((5, 3 * 128)); w = 1 + 0.02 * RNG.standard_normal(128)
    pos = RNG.integers(0, 40, size=(5, 3)).astype(np.int32)
    np.testing.assert_array_equal(_qkx(oracle_mod, v, w, pos, n_heads=3), _qk(oracle_mod, v, w, pos, n_heads=3))


def test_rope_half_golden_angles(oracle_mod):
    g = read_golden("rope3d_half_angles.txt")
    axis_of = {"t": 0, "h": 1, "w": 2}
    for axis, off, D, j, p, angle in g[None]:
        off, D, j, p, angle = int(off), int(D), int(j), int(p), float(angle)
        v = np.zeros((1, 128)); v[0, off + j] = 1.0
        pos = np.zeros((1, 3), np.int32); pos[0, axis_of[axis]] = p
        out = _qkx(oracle_mod, v, None, pos, eps=0.0, pairing=oracle_mod.ROPE_HALF)[0]
        r = math.sqrt(128.0)
        assert abs(out[off + j] - r * math.cos(angle)) < 1e-12
        assert abs(out[off + j + D // 2] - r * math.sin(angle)) < 1e-12
        assert np.all(np.delete(out, [off + j, off + j + D // 2]) == 0.0)


def _half_to_interleaved_perm(dims=(32, 48, 48)):
    """Index map: interleaved position 2j (2j+1) of a chunk holds rotate-half element j (j+D/2)."""
    perm = []
    off = 0
    for D in dims:
        for j in range(D // 2):
            perm += [off + j, off + j + D // 2]
        off += D
    return np.array(perm)


def test_rope_half_is_interleaved_in_permuted_coordinates(oracle_mod):
    """rotate-half(x) = P^T interleaved(P x), P the permutation pairing (j, j + D/2) as (2j, 2j+1)."""
    perm = _half_to_interleaved_perm()
    v = RNG.standard_normal((7, 128))
    pos = RNG.integers(0, 60, size=(7, 3)).astype(np.int32)
    half = _qkx(oracle_mod, v, None, pos, eps=0.0, pairing=oracle_mod.ROPE_HALF)
    inter = _qkx(oracle_mod, np.ascontiguousarray(v[:, perm]), None, pos, eps=0.0)
    back = np.empty_like(inter); back[:, perm] = inter
    np.testing.assert_allclose(half, back, rtol=1e-13, atol=1e-13)


def test_rope_half_relative_positions(oracle_mod):
    q = RNG.standard_normal((1, 128)); k = RNG.standard_normal((1, 128))
    m = np.array([[4, 9, 2]], np.int32); nn = np.array([[1, 3, 30]], np.int32)
    f = lambda v, p: _qkx(oracle_mod, v, None, p, eps=0.0, pairing=oracle_mod.ROPE_HALF)
    ref = (f(q, m) @ f(k, nn).T).item()
    for c in ([0, 0, 7], [11, 0, 0], [5, 6, 40]):
        c = np.array([c], np.int32)
        assert abs((f(q, m + c) @ f(k, nn + c).T).item() - ref) < 1e-11


def test_norm_across_heads_is_torch_rms_norm_over_the_row(oracle_mod):
    n, Hh, Dh = 4, 3, 128
    v = RNG.standard_normal((n, Hh * Dh)) * np.array([[0.5], [1], [3], [20]])
    w = 1 + 0.02 * RNG.standard_normal(Hh * Dh)
    out = _qkx(oracle_mod, v, w, np.zeros((n, 3), np.int32), n_heads=Hh,
               norm_span=oracle_mod.NORM_ACROSS_HEADS)
    ref = F.rms_norm(torch.from_numpy(v), (Hh * Dh,), weight=torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    # and it differs from the per-head span when heads have different scales
    v2 = v.copy(); v2[:, :Dh] *= 10
    a = _qkx(oracle_mod, v2, None, np.zeros((n, 3), np.int32), n_heads=Hh, norm_span=oracle_mod.NORM_ACROSS_HEADS)
    b = _qkx(oracle_mod, v2, None, np.zeros((n, 3), np.int32), n_heads=Hh)
    assert not np.allclose(a, b)
