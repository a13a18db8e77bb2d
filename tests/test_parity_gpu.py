"""GPU parity: every libsol op, called through the C ABI, against the fp64 oracle on the
same seeded inputs.  Small shapes are compared element by element in full; the full
workloads (31k-252k tokens) are run in the launch configuration the benchmark times
and compared on sampled rows.  Edge cases: empty inputs, ragged widths and row counts,
strided rows with guard bands, in-place calls, multi-sample / multi-stream modulation,
explicit packed positions, clamped ids and positions, and the widest supported rows.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from dit_block_b200 import block, sol, workloads
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
    yield
    torch.cuda.synchronize()


@pytest.fixture(scope="module")
def orc():
    import oracle
    oracle.build()
    return oracle


def randn(shape, dtype, seed, std=1.0, mean=0.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std + mean).to(dtype).to(DEV)


# --------------------------------------------------------------------------- small cases

SHAPES = [  # (n_tokens, d): several rows per CTA wave, ragged widths, a single row
    (1, 8), (37, 256), (301, 5120), (67, 5128), (129, 1000), (5, 16384), (2049, 64),
    (19, 6144), (23, 1024)]  # the widest register-resident rows; the narrowest 4-warp prologue


@pytest.mark.parametrize("dtype", [torch.float32, BF])
@pytest.mark.parametrize("n,d", SHAPES)
def test_adaln_and_gated_residual(orc, dtype, n, d):
    if dtype == torch.float32 and d % 4:
        pytest.skip("width")
    B, S = 3, 2
    tps = max(1, (n + B - 1) // B)
    x = randn((n, d), dtype, 1, std=2.0, mean=0.5)
    y = randn((n, d), dtype, 2)
    shift, scale, gate = (randn((B * S, d), dtype, 10 + i, std=0.1) for i in range(3))
    g = torch.Generator().manual_seed(3)
    sid = torch.randint(0, S, (n,), generator=g, dtype=torch.uint8).to(DEV)
    kw = dict(stream_id=sid, n_streams=S, tokens_per_sample=tps)
    okw = dict(stream_id=to_oracle(sid), n_streams=S, tokens_per_sample=tps)

    h = torch.empty_like(x)
    sol.adaln_modulate(h, x, shift, scale, eps=1e-6, **kw)
    o = torch.empty_like(x)
    sol.gated_residual(o, x, y, gate, **kw)
    xo, h2 = torch.empty_like(x), torch.empty_like(x)
    sol.dit_prologue(xo, h2, x, y, gate, shift, scale, eps=1e-6, **kw)
    h3 = torch.empty_like(x)
    sol.dit_prologue(None, h3, x, None, gate, shift, scale, eps=1e-6, **kw)
    torch.cuda.synchronize()

    X, Y = to_oracle(x), to_oracle(y)
    Sh, Sc, G = to_oracle(shift), to_oracle(scale), to_oracle(gate)
    assert_close(to_f64(h), orc.adaln_modulate(X, Sh, Sc, **okw), dtype, "adaln")
    assert_close(to_f64(o), orc.gated_residual(X, Y, G, **okw), dtype, "gated residual")
    xw, hw = orc.dit_prologue(X, Y, G, Sh, Sc, **okw)
    assert_close(to_f64(xo), xw, dtype, "prologue x'")
    assert_close(to_f64(h2), hw, dtype, "prologue h")
    assert_close(to_f64(h3), orc.adaln_modulate(X, Sh, Sc, **okw), dtype, "prologue without residual")


@pytest.mark.parametrize("dtype", [torch.float32, BF])
@pytest.mark.parametrize("n,inner", [(1, 8), (33, 512), (97, 13824), (300, 1000), (4099, 24)])
def test_swiglu(orc, dtype, n, inner):
    if dtype == torch.float32 and inner % 4:
        pytest.skip("width")
    u = randn((n, 2 * inner), dtype, 5, std=3.0)
    out = torch.empty((n, inner), dtype=dtype, device=DEV)
    sol.swiglu(out, u, inner=inner)
    torch.cuda.synchronize()
    assert_close(to_f64(out), orc.swiglu(to_oracle(u), inner), dtype, "swiglu")


def test_swiglu_extremes(orc):
    """Large positive / negative pre-activations (exp overflow region) stay exact to tol."""
    vals = torch.tensor([0.0, -0.0, 1.0, -1.0, 20.0, -20.0, 88.0, -88.0, 90.0, -90.0, 1e4, -1e4,
                         3e38, -3e38, 1e-30, -1e-30], dtype=torch.float32)
    a = vals.repeat(8).view(8, 16)
    b = torch.ones_like(a) * 0.5
    for dtype in (torch.float32, BF):
        A, Bt = a.to(dtype).to(DEV), b.to(dtype).to(DEV)
        out = torch.empty_like(A)
        sol.swiglu_ab(out, A, Bt)
        torch.cuda.synchronize()
        assert_close(to_f64(out), orc.swiglu_ab(to_oracle(A), to_oracle(Bt)), dtype, "swiglu extremes")


QK_CASES = [  # dtype, head_dim, dims, n_heads, grid (T,H,W), samples
    (BF, 128, (32, 48, 48), 40, (3, 4, 5), 2),
    (BF, 128, (30, 50, 48), 3, (2, 5, 7), 1),     # chunk edges inside a lane's slice
    (BF, 64, (16, 24, 24), 5, (4, 3, 3), 3),
    (BF, 256, (64, 96, 96), 2, (2, 2, 9), 1),
    (torch.float32, 128, (32, 48, 48), 2, (2, 4, 4), 1),
    (torch.float32, 64, (16, 24, 24), 3, (5, 2, 3), 2),
    (torch.float32, 32, (8, 12, 12), 7, (3, 3, 3), 1),
    (BF, 128, (32, 48, 48), 48, (2, 3, 4), 2),   # CTA-per-token kernel at its widest (6 vectors a thread)
    (BF, 128, (32, 48, 48), 2, (3, 3, 3), 1),    # CTA-per-token kernel, 2 of its 8 warps busy
    (BF, 128, (32, 48, 48), 6, (2, 3, 5), 2),    # 6 of 8 warps busy
    (BF, 128, (16, 56, 56), 24, (3, 2, 2), 1),   # 3 vectors a thread, another split
]


@pytest.mark.parametrize("dtype,head_dim,dims,Hh,grid,B", QK_CASES)
def test_qk_rmsnorm_rope3d_and_epilogue(orc, dtype, head_dim, dims, Hh, grid, B):
    T, H, W = grid
    tps = T * H * W
    n = B * tps
    hd = Hh * head_dim
    qkv = randn((n, 3 * hd), dtype, 7, std=1.5)
    wq = randn((head_dim,), dtype, 8, std=0.02, mean=1.0)
    wk = randn((head_dim,), dtype, 9, std=0.02, mean=1.0)
    rope = sol.Rope3D(dims, 10000.0, (T + 3, H + 1, W + 2))
    q, k = qkv[:, :hd], qkv[:, hd:2 * hd]
    qo = torch.empty((n, hd), dtype=dtype, device=DEV)
    ko = torch.empty((n, hd), dtype=dtype, device=DEV)
    common = dict(n_heads=Hh, head_dim=head_dim, grid=grid, tokens_per_sample=tps, eps=1e-6)
    sol.qk_rmsnorm_rope3d(qo, ko, q, k, rope, wq=wq, wk=wk, **common)
    epi = qkv.clone()
    sol.dit_epilogue(epi, rope, wq=wq, wk=wk, **common)
    torch.cuda.synchronize()
    QKV = to_oracle(qkv)
    ocommon = dict(n_heads=Hh, head_dim=head_dim, grid=grid, tokens_per_sample=tps, dims=dims,
                   eps=1e-6)
    want = orc.dit_epilogue(QKV, to_oracle(wq), to_oracle(wk), **ocommon)
    assert_close(to_f64(qo), want[:, :hd], dtype, "q")
    assert_close(to_f64(ko), want[:, hd:], dtype, "k")
    assert_close(to_f64(epi[:, :2 * hd]), want, dtype, "epilogue q,k")
    assert torch.equal(epi[:, 2 * hd:], qkv[:, 2 * hd:]), "epilogue touched v"
    # the separate-output call and the in-place epilogue agree bit for bit
    assert torch.equal(epi[:, :hd], qo) and torch.equal(epi[:, hd:2 * hd], ko)
    rope.close()


def test_qk_separate_strided_tensors_and_guard_bands(orc):
    """q and k in separate tensors with different row strides, written out of place into
    outputs with other strides: every row matches the oracle and nothing between or around
    the output rows is written."""
    n, Hh = 101, 40
    hd = Hh * 128
    qb, q = _guarded(n, hd, hd + 64, BF)
    kb, k = _guarded(n, hd, hd + 128, BF)
    q.copy_(randn((n, hd), BF, 31, std=1.5))
    k.copy_(randn((n, hd), BF, 32, std=1.5))
    qob, qo = _guarded(n, hd, hd + 256, BF)
    kob, ko = _guarded(n, hd, hd + 8, BF)
    wq = randn((128,), BF, 33, std=0.02, mean=1.0)
    wk = randn((128,), BF, 34, std=0.02, mean=1.0)
    grid = (3, 5, 7)
    with sol.Rope3D((32, 48, 48), 10000.0, (4, 5, 7)) as rope:
        sol.qk_rmsnorm_rope3d(qo, ko, q, k, rope, n_heads=Hh, head_dim=128, wq=wq, wk=wk, grid=grid,
                              tokens_per_sample=0)
        torch.cuda.synchronize()
    want_q, want_k = orc.qk_rmsnorm_rope3d(to_oracle(q.contiguous()), to_oracle(k.contiguous()), to_oracle(wq),
                                          to_oracle(wk), n_heads=Hh, head_dim=128, grid=grid)
    assert_close(to_f64(qo.contiguous()), want_q, BF, "strided q")
    assert_close(to_f64(ko.contiguous()), want_k, BF, "strided k")
    assert _guards_intact(qob, n, hd, hd + 256) and _guards_intact(kob, n, hd, hd + 8)
    assert _guards_intact(qb, n, hd, hd + 64) and _guards_intact(kb, n, hd, hd + 128)


def test_qk_explicit_positions_packed_and_clamped(orc):
    """Packed video+audio positions passed explicitly; positions past the table clamp."""
    w = workloads.Workload("t", 7, BF, 2, (2, 3, 4), 5, 64, 3, 128, 64)
    pos, sid = workloads.token_layout(w)
    n = pos.shape[0]
    hd = w.hd
    q = randn((n, hd), BF, 11)
    k = randn((n, hd), BF, 12)
    rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
    qo, ko = torch.empty_like(q), torch.empty_like(k)
    P = pos.to(DEV)
    sol.qk_rmsnorm_rope3d(qo, ko, q, k, rope, n_heads=w.n_heads, head_dim=128, pos=P)
    torch.cuda.synchronize()
    want_q, want_k = orc.qk_rmsnorm_rope3d(to_oracle(q), to_oracle(k), n_heads=w.n_heads,
                                          head_dim=128, pos=pos.numpy())
    assert_close(to_f64(qo), want_q, BF, "packed q")
    assert_close(to_f64(ko), want_k, BF, "packed k")
    # out-of-range positions clamp to the last table row / to 0
    big = P.clone()
    big[:, 0] += 1000
    big[:3, 1] = -4
    clamped = torch.minimum(big, torch.tensor(w.max_pos, device=DEV, dtype=torch.int32) - 1).clamp_min(0)
    a, b = torch.empty_like(q), torch.empty_like(q)
    sol.qk_rmsnorm_rope3d(a, b, q, k, rope, n_heads=w.n_heads, head_dim=128, pos=big.contiguous())
    c, dd = torch.empty_like(q), torch.empty_like(q)
    sol.qk_rmsnorm_rope3d(c, dd, q, k, rope, n_heads=w.n_heads, head_dim=128, pos=clamped.contiguous())
    torch.cuda.synchronize()
    assert torch.equal(a, c) and torch.equal(b, dd)
    rope.close()


# ------------------------------------------------------------------------- edge cases

def test_zero_tokens_is_a_no_op():
    x = randn((4, 64), BF, 1)
    out = torch.full_like(x, 7.0)
    sol.gated_residual(out[:0], x[:0], x[:0], None)
    sol.adaln_modulate(out[:0], x[:0])
    sol.swiglu(out[:0, :32], x[:0], inner=32)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_gate_zero_is_identity_bitwise():
    x = randn((513, 5120), BF, 1, std=3.0)
    y = randn((513, 5120), BF, 2, std=1e3)
    out = torch.empty_like(x)
    sol.gated_residual(out, x, y, torch.zeros((1, 5120), dtype=BF, device=DEV))
    o2 = torch.empty_like(x)
    sol.gated_residual(o2, x, y, None)
    torch.cuda.synchronize()
    assert torch.equal(out, x) and torch.equal(o2, x)  # == treats -0 and +0 alike


def test_in_place_equals_out_of_place():
    n, d = 777, 5120
    x = randn((n, d), BF, 1)
    y = randn((n, d), BF, 2)
    gate, shift, scale = (randn((1, d), BF, 20 + i, std=0.1) for i in range(3))
    h = torch.empty_like(x)
    sol.adaln_modulate(h, x, shift, scale)
    xi = x.clone()
    sol.adaln_modulate(xi, xi, shift, scale)
    o = torch.empty_like(x)
    sol.gated_residual(o, x, y, gate)
    xg = x.clone()
    sol.gated_residual(xg, xg, y, gate)
    xo, hh = torch.empty_like(x), torch.empty_like(x)
    sol.dit_prologue(xo, hh, x, y, gate, shift, scale)
    xp, hp = x.clone(), torch.empty_like(x)
    sol.dit_prologue(xp, hp, xp, y, gate, shift, scale)
    torch.cuda.synchronize()
    assert torch.equal(h, xi) and torch.equal(o, xg) and torch.equal(xo, xp) and torch.equal(hh, hp)


def _guarded(rows, cols, ld, dtype, pad_rows=3, sentinel=-12345.0):
    """A [rows, cols] view with row stride ld inside a buffer with sentinel rows before
    and after it and sentinel columns past cols."""
    buf = torch.full(((rows + 2 * pad_rows) * ld,), sentinel, dtype=dtype, device=DEV)
    view = buf[pad_rows * ld:(pad_rows + rows) * ld].view(rows, ld)[:, :cols]
    return buf, view


def _guards_intact(buf, rows, cols, ld, pad_rows=3, sentinel=-12345.0):
    full = buf.view(rows + 2 * pad_rows, ld)
    ok = torch.all(full[:pad_rows] == sentinel) and torch.all(full[pad_rows + rows:] == sentinel)
    if cols < ld:
        ok = ok and torch.all(full[pad_rows:pad_rows + rows, cols:] == sentinel)
    return bool(ok)


@pytest.mark.parametrize("dtype", [torch.float32, BF])
def test_strided_rows_and_guard_bands(orc, dtype):
    n, d, ld = 203, 2056, 2056 + 24
    inner = 1032
    xb, x = _guarded(n, d, ld, dtype)
    x.copy_(randn((n, d), dtype, 1))
    yb, y = _guarded(n, d, ld, dtype)
    y.copy_(randn((n, d), dtype, 2))
    gate, shift, scale = (randn((2, d), dtype, 30 + i, std=0.1) for i in range(3))
    kw = dict(tokens_per_sample=102)  # rows 0..101 -> sample 0, 102..202 -> sample 1
    hb, h = _guarded(n, d, ld, dtype)
    ob, o = _guarded(n, d, ld, dtype)
    xob, xo = _guarded(n, d, ld, dtype)
    h2b, h2 = _guarded(n, d, ld, dtype)
    sol.adaln_modulate(h, x, shift, scale, **kw)
    sol.gated_residual(o, x, y, gate, **kw)
    sol.dit_prologue(xo, h2, x, y, gate, shift, scale, **kw)
    ub, u = _guarded(n, 2 * inner + 40, 2 * inner + 48, dtype)
    u.copy_(randn((n, 2 * inner + 40), dtype, 4))
    sb, s = _guarded(n, inner, inner + 16, dtype)
    sol.swiglu(s, u, inner=inner)
    torch.cuda.synchronize()
    for buf, cols, l in ((hb, d, ld), (ob, d, ld), (xob, d, ld), (h2b, d, ld), (sb, inner, inner + 16)):
        assert _guards_intact(buf, n, cols, l), "a kernel wrote outside its rows"
    X, Y = to_oracle(x), to_oracle(y)
    M = [to_oracle(t) for t in (shift, scale, gate)]
    assert_close(to_f64(h), orc.adaln_modulate(X, M[0], M[1], **kw), dtype, "strided adaln")
    assert_close(to_f64(o), orc.gated_residual(X, Y, M[2], **kw), dtype, "strided gated")
    xw, hw = orc.dit_prologue(X, Y, M[2], M[0], M[1], **kw)
    assert_close(to_f64(xo), xw, dtype, "strided prologue x'")
    assert_close(to_f64(h2), hw, dtype, "strided prologue h")
    assert_close(to_f64(s), orc.swiglu(np.ascontiguousarray(to_oracle(u)[:, :2 * inner]), inner),
                 dtype, "strided swiglu")


def test_stream_ids_past_n_streams_clamp():
    n, d = 64, 256
    x = randn((n, d), BF, 1)
    shift = randn((2, d), BF, 2)
    sid = torch.full((n,), 9, dtype=torch.uint8, device=DEV)
    last = torch.ones_like(sid)
    a, b = torch.empty_like(x), torch.empty_like(x)
    sol.adaln_modulate(a, x, shift, None, stream_id=sid, n_streams=2)
    sol.adaln_modulate(b, x, shift, None, stream_id=last, n_streams=2)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_errors_raise_without_launch():
    x = randn((8, 64), BF, 1)
    with pytest.raises(sol.SolError) as e:
        sol.adaln_modulate(x[:, 1:], x)  # misaligned output
    assert e.value.status == sol.ERR_MISALIGNED
    with pytest.raises(sol.SolError):
        sol.gated_residual(x, x, x)  # out aliases y


# --------------------------------------------------------------- full-size workloads

def _sample_rows(w: workloads.Workload, k: int = 40) -> np.ndarray:
    n = w.n_tokens
    g = np.random.default_rng(w.index)
    rows = {0, 1, n - 1, n - 2}
    for b in range(w.batch):
        s0 = b * w.tokens_per_sample
        rows |= {s0, s0 + w.video_per_sample - 1, s0 + w.tokens_per_sample - 1}
        if w.audio_per_sample:
            rows |= {s0 + w.video_per_sample, s0 + w.video_per_sample + 1}
    rows |= set(g.integers(0, n, size=k).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < n), dtype=np.int64)


@pytest.mark.parametrize("name", ["tiny", "lowres", "fullres_5s", "fullres_10s", "packed_av"])
def test_block_step_full_workload(orc, name):
    """The five launches of one block pass at the workload's full size, checked against the
    oracle on sampled rows (all rows for the tiny workload)."""
    w = workloads.WORKLOADS[name]
    torch.cuda.empty_cache()
    bufs = block.BlockBuffers.allocate(w, DEV)
    i = bufs.inp
    rows = np.arange(w.n_tokens) if w.n_tokens <= 64 else _sample_rows(w)
    R = torch.from_numpy(rows).to(DEV)
    pick = lambda t: to_oracle(t.index_select(0, R))
    qkv0 = pick(i["qkv"])  # before the in-place epilogue
    bufs.step()
    torch.cuda.synchronize()
    X, YA, YM, U = pick(i["x"]), pick(i["y_attn"]), pick(i["y_mlp"]), pick(i["u"])
    mods = {k: to_oracle(i[k]) for k in ("shift_msa", "scale_msa", "gate_msa", "shift_mlp",
                                         "scale_mlp", "gate_mlp")}
    sid = to_oracle(i["stream_id"])
    pos = None if i["pos"] is None else i["pos"].cpu().numpy()
    sel = dict(stream_id=sid, n_streams=w.n_streams, tokens_per_sample=w.tokens_per_sample,
               rows=rows)
    dt = w.dtype
    assert_close(to_f64(bufs.h1.index_select(0, R)),
                 orc.adaln_modulate(X, mods["shift_msa"], mods["scale_msa"], eps=w.eps, **sel), dt,
                 f"{name} adaln")
    want = orc.dit_epilogue(qkv0, to_oracle(i["wq"]), to_oracle(i["wk"]), n_heads=w.n_heads,
                            head_dim=w.head_dim, pos=pos, grid=w.grid,
                            tokens_per_sample=w.tokens_per_sample, dims=w.rope_dims,
                            theta=w.theta, eps=w.eps, rows=rows)
    assert_close(to_f64(i["qkv"].index_select(0, R)[:, :2 * w.hd]), want, dt, f"{name} epilogue")
    xw, hw = orc.dit_prologue(X, YA, mods["gate_msa"], mods["shift_mlp"], mods["scale_mlp"],
                              eps=w.eps, **sel)
    assert_close(to_f64(bufs.x1.index_select(0, R)), xw, dt, f"{name} prologue x'")
    assert_close(to_f64(bufs.h2.index_select(0, R)), hw, dt, f"{name} prologue h")
    assert_close(to_f64(bufs.act.index_select(0, R)), orc.swiglu(U, w.inner), dt, f"{name} swiglu")
    # The pass feeds the GPU's x' into the gated residual; the oracle takes no input from
    # the GPU, so the same launch (same shapes, same launch configuration) is checked on
    # the generated residual stream x instead, and the pass's own output is checked for
    # determinism against a repeat of its launch.
    x2b = torch.empty_like(bufs.x2)
    sol.gated_residual(x2b, i["x"], i["y_mlp"], i["gate_mlp"], **bufs.sel())
    x2c = torch.empty_like(bufs.x2)
    sol.gated_residual(x2c, bufs.x1, i["y_mlp"], i["gate_mlp"], **bufs.sel())
    torch.cuda.synchronize()
    assert_close(to_f64(x2b.index_select(0, R)),
                 orc.gated_residual(X, YM, mods["gate_mlp"], **sel), dt, f"{name} gated residual")
    assert torch.equal(x2c, bufs.x2)
    del x2b, x2c
    bufs.close()
    del bufs
    torch.cuda.empty_cache()


def test_adjacent_buffers_are_not_overlaps(orc):
    """An output that starts right where the input's last row ends is legal."""
    n, inner = 9, 64
    buf = torch.empty(n * 2 * inner + n * inner, dtype=BF, device=DEV)
    u = buf[:n * 2 * inner].view(n, 2 * inner)
    u.copy_(randn((n, 2 * inner), BF, 3))
    out = buf[n * 2 * inner:].view(n, inner)
    sol.swiglu(out, u, inner=inner)
    x = buf[:n * 2 * inner].view(n, 2 * inner)[:, :inner]  # strided rows, ld = 2*inner
    o2 = torch.empty((n, inner), dtype=BF, device=DEV)
    sol.gated_residual(o2, x, out, None)
    torch.cuda.synchronize()
    assert_close(to_f64(out), orc.swiglu(to_oracle(u), inner), BF, "adjacent swiglu")
    assert torch.equal(o2, x)


@pytest.mark.parametrize("d", [1024, 5120])
@pytest.mark.parametrize("ld_h_extra,ld_x_extra", [(0, 0), (64, 64), (0, 64), (128, 0)])
def test_adaln_row_strides_select_kernels(orc, d, ld_h_extra, ld_x_extra):
    """bf16 AdaLN at widths the four-warp row kernel takes: equal row strides of h and x
    run it, different strides the one-warp kernel; both match the oracle and leave the
    padding between rows untouched."""
    n = 77
    ld_h, ld_x = d + ld_h_extra, d + ld_x_extra
    xb, x = _guarded(n, d, ld_x, BF)
    x.copy_(randn((n, d), BF, 91, std=2.0, mean=0.5))
    hb, h = _guarded(n, d, ld_h, BF)
    shift, scale = (randn((2, d), BF, 92 + i, std=0.1) for i in range(2))
    kw = dict(tokens_per_sample=40)  # rows 0..39 -> sample 0, 40..76 -> sample 1
    sol.adaln_modulate(h, x, shift, scale, eps=1e-6, **kw)
    torch.cuda.synchronize()
    want = orc.adaln_modulate(to_oracle(x.contiguous()), to_oracle(shift), to_oracle(scale), **kw)
    assert_close(to_f64(h.contiguous()), want, BF, f"adaln d={d} ld_h={ld_h} ld_x={ld_x}")
    assert _guards_intact(hb, n, d, ld_h)
