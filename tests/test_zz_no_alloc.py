"""The allocation-free QK RMSNorm + 3D RoPE entry point, called through the C ABI.

sol_qk_rmsnorm_rope3d_noalloc serves callers that cannot allocate device memory while
they run (engines whose pool already holds the GPU's memory, plugin execute callbacks):
it keeps its cos/sin table in a fixed array inside the library instead of a handle made
by cudaMalloc.  Its output must match the regular entry point's within the parity
tolerance, on consecutive calls that rebuild the shared table for different shapes, and
the fp64 oracle's (bf16 and fp32, positions outside the table clamped).

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import pytest
import torch

from dit_block_b200 import sol, workloads
from parity_util import assert_close, to_oracle, tolerance, to_f64

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


def _randn(shape, dtype, seed, std=1.0, mean=0.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std + mean).to(dtype).to(DEV)


def _close(got, want, dtype, what):
    g, w = to_f64(got), to_f64(want)
    bad = abs(g - w) > tolerance(w, dtype)
    assert not bad.any(), f"{what}: {int(bad.sum())} elements differ beyond tolerance"


def _case_grid():
    """Video-only grid, implicit positions, 40 heads of 128, two samples."""
    grid, Hh, B = (5, 6, 7), 40, 2
    n = B * grid[0] * grid[1] * grid[2]
    qkv = _randn((n, 3 * Hh * 128), BF, 1, std=1.5)
    return dict(dtype=BF, qkv=qkv, Hh=Hh, head_dim=128, dims=(32, 48, 48), theta=10000.0,
                max_pos=(9, 6, 8), pos=None, grid=grid, tps=grid[0] * grid[1] * grid[2])


def _case_packed():
    """Packed video + audio with explicit positions and a different split and theta."""
    w = workloads.Workload("t", 8, BF, 2, (3, 4, 5), 37, 64, 6, 128, 64)
    pos, _ = workloads.token_layout(w)
    n = pos.shape[0]
    qkv = _randn((n, 3 * w.hd), BF, 2)
    return dict(dtype=BF, qkv=qkv, Hh=w.n_heads, head_dim=128, dims=(16, 56, 56), theta=500.0,
                max_pos=w.max_pos, pos=pos.to(DEV), grid=(0, 0, 0), tps=0)


def _run_both(c):
    Hh, hd = c["Hh"], c["Hh"] * c["head_dim"]
    qkv = c["qkv"]
    q, k = qkv[:, :hd], qkv[:, hd:2 * hd]
    wq = _randn((c["head_dim"],), c["dtype"], 3, std=0.02, mean=1.0)
    wk = _randn((c["head_dim"],), c["dtype"], 4, std=0.02, mean=1.0)
    common = dict(n_heads=Hh, head_dim=c["head_dim"], wq=wq, wk=wk, pos=c["pos"], grid=c["grid"],
                  tokens_per_sample=c["tps"])
    ref_q, ref_k = torch.empty_like(q), torch.empty_like(k)
    with sol.Rope3D(c["dims"], c["theta"], c["max_pos"]) as rope:
        sol.qk_rmsnorm_rope3d(ref_q, ref_k, q, k, rope, **common)
        torch.cuda.synchronize()
    got_q, got_k = torch.full_like(q, 7.0), torch.full_like(k, 7.0)
    sol.qk_rmsnorm_rope3d_noalloc(got_q, got_k, q, k, dims=c["dims"], theta=c["theta"],
                                  max_pos=c["max_pos"], **common)
    torch.cuda.synchronize()
    return (got_q, got_k), (ref_q, ref_k)


def test_noalloc_matches_regular_entry_point_on_consecutive_calls():
    for name, case in (("grid", _case_grid()), ("packed", _case_packed()), ("grid again", _case_grid())):
        (gq, gk), (rq, rk) = _run_both(case)
        _close(gq, rq, case["dtype"], f"{name} q")
        _close(gk, rk, case["dtype"], f"{name} k")


def test_noalloc_in_place_on_packed_qkv():
    c = _case_grid()
    hd = c["Hh"] * c["head_dim"]
    ref = c["qkv"].clone()
    with sol.Rope3D(c["dims"], c["theta"], c["max_pos"]) as rope:
        sol.dit_epilogue(ref, rope, n_heads=c["Hh"], head_dim=128, grid=c["grid"],
                         tokens_per_sample=c["tps"])
    got = c["qkv"].clone()
    q, k = got[:, :hd], got[:, hd:2 * hd]
    sol.qk_rmsnorm_rope3d_noalloc(q, k, q, k, n_heads=c["Hh"], head_dim=128, max_pos=c["max_pos"],
                                  grid=c["grid"], tokens_per_sample=c["tps"])
    torch.cuda.synchronize()
    _close(got, ref, BF, "in-place qkv")


def test_noalloc_rejects_tables_beyond_its_array():
    q = torch.zeros((4, 128), dtype=BF, device=DEV)
    o = torch.empty_like(q)
    # dims (32, 48, 48) over (3000, 8, 8): 3000*16 + 8*24 + 8*24 = 48,384 entries fit ...
    sol.qk_rmsnorm_rope3d_noalloc(o, o.clone(), q, q.clone(), n_heads=1, head_dim=128,
                                  max_pos=(3000, 8, 8), pos=torch.zeros((4, 3), dtype=torch.int32, device=DEV))
    # ... (5000, 8, 8) needs 80,384 > 65,536
    with pytest.raises(sol.SolError) as e:
        sol.qk_rmsnorm_rope3d_noalloc(o, o.clone(), q, q.clone(), n_heads=1, head_dim=128,
                                      max_pos=(5000, 8, 8),
                                      pos=torch.zeros((4, 3), dtype=torch.int32, device=DEV))
    assert e.value.status == sol.ERR_UNSUPPORTED
    assert "65536" in str(e.value)
    torch.cuda.synchronize()


def _oracle_qk(oracle_mod, c, q, k, wq, wk, pos):
    return oracle_mod.qk_rmsnorm_rope3d(
        to_oracle(q), to_oracle(k), to_oracle(wq), to_oracle(wk), n_heads=c["Hh"], head_dim=c["head_dim"],
        pos=pos, grid=c["grid"], tokens_per_sample=c["tps"], dims=c["dims"], theta=c["theta"])


def test_noalloc_matches_oracle_with_clamped_positions(oracle_mod):
    """The (16, 56, 56) split at theta 500 straight against the fp64 oracle, with explicit
    positions, some of them outside the table (the library clamps them into it; the oracle
    gets the clamped positions)."""
    c = _case_packed()
    hd = c["Hh"] * c["head_dim"]
    q, k = c["qkv"][:, :hd], c["qkv"][:, hd:2 * hd]
    pos = c["pos"].clone()
    n = pos.shape[0]
    mx = torch.tensor(c["max_pos"], dtype=torch.int32, device=DEV)
    pos[0] = mx + 5          # beyond the table on every axis
    pos[n // 2] = -3         # below it
    pos[n - 1, 0] = mx[0]    # exactly one past the last row
    wq = _randn((128,), BF, 3, std=0.02, mean=1.0)
    wk = _randn((128,), BF, 4, std=0.02, mean=1.0)
    gq, gk = torch.empty_like(q), torch.empty_like(k)
    sol.qk_rmsnorm_rope3d_noalloc(gq, gk, q, k, n_heads=c["Hh"], head_dim=128, wq=wq, wk=wk, pos=pos,
                                  dims=c["dims"], theta=c["theta"], max_pos=c["max_pos"])
    torch.cuda.synchronize()
    clamped = torch.minimum(torch.clamp(pos, min=0), mx - 1)
    oq, ok = _oracle_qk(oracle_mod, c, q, k, wq, wk, to_oracle(clamped))
    assert_close(to_f64(gq), oq, BF, "noalloc q vs oracle")
    assert_close(to_f64(gk), ok, BF, "noalloc k vs oracle")
    # the regular entry point clamps the same way
    rq, rk = torch.empty_like(q), torch.empty_like(k)
    with sol.Rope3D(c["dims"], c["theta"], c["max_pos"]) as rope:
        sol.qk_rmsnorm_rope3d(rq, rk, q, k, rope, n_heads=c["Hh"], head_dim=128, wq=wq, wk=wk, pos=pos)
        torch.cuda.synchronize()
    _close(gq, rq, BF, "clamped q vs regular")
    _close(gk, rk, BF, "clamped k vs regular")


def test_noalloc_f32_matches_oracle_and_regular(oracle_mod):
    """fp32 path (tight 1e-5 bound): 2 heads of 128 on the 2 x 4 x 4 grid."""
    grid = (2, 4, 4)
    n = 32
    qkv = _randn((n, 3 * 256), torch.float32, 5)
    c = dict(Hh=2, head_dim=128, dims=(32, 48, 48), theta=10000.0, grid=grid, tps=0)
    q, k = qkv[:, :256], qkv[:, 256:512]
    wq = _randn((128,), torch.float32, 6, std=0.02, mean=1.0)
    wk = _randn((128,), torch.float32, 7, std=0.02, mean=1.0)
    for call in range(2):  # two calls in a row, the second over the table the first built
        gq, gk = torch.full_like(q, 7.0), torch.full_like(k, 7.0)
        sol.qk_rmsnorm_rope3d_noalloc(gq, gk, q, k, n_heads=2, head_dim=128, wq=wq, wk=wk, grid=grid,
                                      max_pos=grid, dims=c["dims"], theta=c["theta"])
        torch.cuda.synchronize()
        oq, ok = _oracle_qk(oracle_mod, c, q, k, wq, wk, None)
        assert_close(to_f64(gq), oq, torch.float32, f"f32 noalloc q vs oracle, call {call}")
        assert_close(to_f64(gk), ok, torch.float32, f"f32 noalloc k vs oracle, call {call}")
        rq, rk = torch.empty_like(q), torch.empty_like(k)
        with sol.Rope3D(c["dims"], c["theta"], grid) as rope:
            sol.qk_rmsnorm_rope3d(rq, rk, q, k, rope, n_heads=2, head_dim=128, wq=wq, wk=wk, grid=grid)
            torch.cuda.synchronize()
        _close(gq, rq, torch.float32, f"f32 q vs regular, call {call}")
        _close(gk, rk, torch.float32, f"f32 k vs regular, call {call}")
