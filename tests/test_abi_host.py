"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/sol.h declares, and rejects bad arguments before any CUDA call.

The pointers passed here are fake addresses; every call below fails validation on the
host, so none of them reaches the CUDA runtime or the device."""
from __future__ import annotations

import ctypes

import pytest

from dit_block_b200 import build, sol


@pytest.fixture(scope="module")
def L():
    build.build()
    return sol.lib()


FAKE = 1 << 20  # 16-byte aligned fake address (never dereferenced)
SEL = sol.ModSel(None, 1, 0)


def last(L):
    return L.sol_last_error().decode()


def test_exports_every_declared_symbol(L):
    names = sol.header_functions()
    assert len(names) == 27
    for n in names:
        assert hasattr(L, n), f"libsol.so does not export {n}"
        assert n in sol.SIGNATURES, f"binding has no signature for {n}"


def test_status_strings_and_version(L):
    assert L.sol_abi_version() == 2
    assert L.sol_status_string(0) == b"ok"
    for s in range(1, 5):
        assert L.sol_status_string(s) and L.sol_status_string(s) != b"ok"
    assert L.sol_status_string(99) == b"unknown status"


@pytest.mark.parametrize("dt", [sol.F32, sol.BF16])
def test_adaln_validation(L, dt):
    bad_d = 7
    assert L.sol_adaln_modulate(FAKE, 8, FAKE, 8, None, None, 0, SEL, 4, bad_d, 1e-6, dt, None) \
        in (sol.ERR_INVALID_ARGUMENT, sol.ERR_UNSUPPORTED)
    assert L.sol_adaln_modulate(None, 8, FAKE, 8, None, None, 0, SEL, 4, 8, 1e-6, dt, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert "h is NULL" in last(L)
    assert L.sol_adaln_modulate(FAKE + 4, 8, FAKE, 8, None, None, 0, SEL, 4, 8, 1e-6, dt, None) \
        == sol.ERR_MISALIGNED
    assert L.sol_adaln_modulate(FAKE, 6, FAKE, 8, None, None, 0, SEL, 4, 8, 1e-6, dt, None) \
        == sol.ERR_INVALID_ARGUMENT  # ld below width
    assert L.sol_adaln_modulate(FAKE, 8, FAKE, 8, None, None, 0, SEL, -1, 8, 1e-6, dt, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_modulate(FAKE, 8, FAKE, 8, None, None, 0, SEL, 4, 8, -1.0, dt, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_modulate(FAKE, 8, FAKE, 8, None, None, 0, SEL, 4, 8, float("nan"), dt, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_modulate(FAKE, 1 << 20, FAKE, 1 << 20, None, None, 0, SEL, 4, 1 << 20, 1e-6,
                                dt, None) == sol.ERR_UNSUPPORTED  # wider than one CTA row holds
    assert "wider" in last(L)


def test_leading_dimension_must_keep_rows_16_byte_aligned(L):
    # bf16 rows of ld 12 elements are 24 bytes apart: rejected; f32 ld 12 is 48 bytes: fine
    assert L.sol_gated_residual(FAKE, 12, FAKE, 16, FAKE, 16, None, 0, SEL, 2, 8, sol.BF16, None) \
        == sol.ERR_MISALIGNED
    assert "multiple of 8" in last(L)


def test_overlap_rules(L):
    # h partially overlapping x is rejected; h == x is allowed (passes validation; with
    # n_tokens = 0 nothing is launched)
    n, d = 4, 64
    assert L.sol_adaln_modulate(FAKE + 128, d, FAKE, d, None, None, 0, SEL, n, d, 1e-6, sol.BF16, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_modulate(FAKE, d, FAKE, d, None, None, 0, SEL, 0, d, 1e-6, sol.BF16, None) == sol.OK
    # prologue: h may not alias x
    assert L.sol_dit_prologue(FAKE, FAKE, FAKE, None, None, None, None, d, 0, SEL, n, d, 1e-6,
                              sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    # swiglu output may not overlap its inputs
    assert L.sol_swiglu(FAKE, 64, FAKE, FAKE + 64, 128, 4, 32, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT


def test_modsel_validation(L):
    bad = sol.ModSel(None, 0, 0)
    assert L.sol_gated_residual(FAKE, 8, FAKE + 4096, 8, FAKE + 8192, 8, None, 0, bad, 2, 8, sol.BF16,
                                None) == sol.ERR_INVALID_ARGUMENT
    bad = sol.ModSel(None, 1, -5)
    assert L.sol_gated_residual(FAKE, 8, FAKE + 4096, 8, FAKE + 8192, 8, None, 0, bad, 2, 8, sol.BF16,
                                None) == sol.ERR_INVALID_ARGUMENT


def test_dtype_and_required_tensors(L):
    assert L.sol_swiglu(FAKE, 8, FAKE + 4096, FAKE + 8192, 8, 2, 8, 7, None) == sol.ERR_UNSUPPORTED
    assert L.sol_swiglu(FAKE, 8, None, FAKE + 8192, 8, 2, 8, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_gated_residual(FAKE, 8, FAKE + 4096, 8, None, 8, None, 0, SEL, 2, 8, sol.BF16, None) \
        == sol.ERR_INVALID_ARGUMENT
    # prologue with a residual needs x_out
    assert L.sol_dit_prologue(None, FAKE, FAKE + 4096, FAKE + 8192, None, None, None, 8, 0, SEL, 2, 8,
                              1e-6, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT


def test_rope_create_validation(L):
    h = ctypes.c_void_p()
    assert L.sol_rope3d_create(ctypes.byref(h), 32, 47, 48, 1e4, 8, 8, 8) == sol.ERR_INVALID_ARGUMENT
    assert h.value is None
    assert L.sol_rope3d_create(ctypes.byref(h), 32, 48, 48, 1.0, 8, 8, 8) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_rope3d_create(ctypes.byref(h), 32, 48, 48, 1e4, 0, 8, 8) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_rope3d_create(None, 32, 48, 48, 1e4, 8, 8, 8) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_rope3d_destroy(None) == sol.OK


def test_qk_validation_without_tables(L):
    assert L.sol_qk_rmsnorm_rope3d(FAKE, FAKE, 256, 256, FAKE, FAKE, 256, 256, None, None, None, 2, 4, 4,
                                   32, None, 32, 2, 128, 1e-6, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert "rope is NULL" in last(L)
    assert L.sol_dit_epilogue(FAKE, 768, None, None, None, 2, 4, 4, 32, None, 32, 2, 128, 1e-6,
                              sol.BF16, None) == sol.ERR_INVALID_ARGUMENT


def test_binding_raises_with_reason():
    with pytest.raises(sol.SolError) as e:
        sol._check(sol.lib().sol_swiglu(None, 8, None, None, 8, 1, 8, sol.BF16, None), "sol_swiglu")
    assert e.value.status == sol.ERR_INVALID_ARGUMENT
    assert "NULL" in str(e.value)


def test_subblock_count(L):
    assert L.sol_subblock_count(245952, 245952, 64) == 3843
    assert L.sol_subblock_count(2 * 130, 130, 64) == 6     # 64 + 64 + 2 per sample
    assert L.sol_subblock_count(100, 0, 64) == 2
    assert L.sol_subblock_count(0, 0, 64) == 0
    assert L.sol_subblock_count(10, 0, 0) == 0


def test_linear_validation(L):
    n, k, d = 300, 512, 768
    # bf16 only
    assert L.sol_linear(FAKE, d, FAKE, k, FAKE, k, n, d, k, sol.F32, None) == sol.ERR_UNSUPPORTED
    assert "bf16" in last(L)
    # k a multiple of 64, output width a multiple of 256
    assert L.sol_linear(FAKE, d, FAKE, 520, FAKE, 520, n, d, 520, sol.BF16, None) == sol.ERR_UNSUPPORTED
    assert L.sol_linear(FAKE, 640, FAKE, k, FAKE, k, n, 640, k, sol.BF16, None) == sol.ERR_UNSUPPORTED
    assert L.sol_linear(FAKE, d, FAKE, k, FAKE, k, 1 << 31, d, k, sol.BF16, None) == sol.ERR_UNSUPPORTED
    assert L.sol_linear(FAKE, d, FAKE, k, FAKE, k, -1, d, k, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_linear(FAKE, d, FAKE, k, None, k, n, d, k, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_linear(FAKE, d, FAKE + 8, k, FAKE, k, n, d, k, sol.BF16, None) == sol.ERR_MISALIGNED
    # out overlapping a
    assert L.sol_linear(FAKE + 64, d, FAKE, k, FAKE << 4, k, n, d, k, sol.BF16, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert "overlaps" in last(L)
    # n_tokens == 0: valid, nothing launched
    assert L.sol_linear(None, d, None, k, FAKE, k, 0, d, k, sol.BF16, None) == sol.OK


def test_linear_epilogue_variants_validation(L):
    n, k, d = 300, 512, 768
    x, a, w, out = FAKE, FAKE << 2, FAKE << 3, FAKE << 4
    # gated residual: out may be x itself but not partially overlap it
    assert L.sol_linear_gated_residual(x + 64, d, x, d, a, k, w, k, None, 0, SEL, n, d, k, sol.BF16, None) \
        == sol.ERR_INVALID_ARGUMENT
    assert L.sol_linear_gated_residual(out, d, x, d, a, k, w, k, None, 0, sol.ModSel(None, 0, 0), n, d, k,
                                       sol.BF16, None) == sol.ERR_INVALID_ARGUMENT  # n_streams 0
    assert L.sol_linear_gated_residual(out, d, x, d, a, k, w, k, None, 0, SEL, n, 640, k, sol.BF16, None) \
        == sol.ERR_UNSUPPORTED
    # SwiGLU: W has 2*inner rows, inner a multiple of 128
    assert L.sol_linear_swiglu(out, 192, a, k, w, k, n, 192, k, sol.BF16, None) == sol.ERR_UNSUPPORTED
    assert L.sol_linear_swiglu(out, 256, a, k, w, k, n, 256, k, sol.F32, None) == sol.ERR_UNSUPPORTED
    # AdaLN variants need a workspace of sol_adaln_workspace_bytes
    need = L.sol_adaln_workspace_bytes(n, d, k, SEL)
    assert need >= n * 8 + d * k * 2
    # the shared region holds the larger of the folded weights and the staged h
    tall = 100_000  # more tokens than output columns: h (n * k) outgrows the folded weights (d * k)
    assert L.sol_adaln_workspace_bytes(tall, d, k, SEL) >= tall * 8 + tall * k * 2
    assert L.sol_adaln_workspace_bytes(tall, d, k, SEL) < tall * 8 + tall * k * 2 + d * k * 2
    ws = FAKE << 6
    assert L.sol_adaln_linear(out, d, x, k, None, None, 0, SEL, w, k, None, need, 0, n, d, k, 1e-6, sol.BF16,
                              None) == sol.ERR_INVALID_ARGUMENT
    assert "workspace" in last(L)
    assert L.sol_adaln_linear(out, d, x, k, None, None, 0, SEL, w, k, ws, need - 1, 0, n, d, k, 1e-6, sol.BF16,
                              None) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_linear(out, d, x, k, None, None, 0, SEL, w, k, ws + 16, need, 0, n, d, k, 1e-6, sol.BF16,
                              None) == sol.ERR_MISALIGNED
    assert L.sol_adaln_linear(out, d, x, k, None, None, 0, SEL, w, k, ws, need, 0, n, d, k, float("inf"),
                              sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    # workspace overlapping x
    assert L.sol_adaln_linear(out, d, x, k, None, None, 0, SEL, w, k, x + 1024, need, 0, n, d, k, 1e-6,
                              sol.BF16, None) in (sol.ERR_INVALID_ARGUMENT, sol.ERR_MISALIGNED)
    # at most 32 modulation rows: 33 samples of 10 tokens
    many = sol.ModSel(None, 1, 10)
    assert L.sol_adaln_workspace_bytes(330, d, k, many) == 0
    assert L.sol_adaln_linear(out, d, x, k, None, None, 0, many, w, k, ws, need, 0, 330, d, k, 1e-6, sol.BF16,
                              None) == sol.ERR_UNSUPPORTED
    # the QKV call is built for head_dim 128 and an even head count
    assert L.sol_adaln_qkv_rope(out, 768, x, k, None, None, 0, SEL, w, k, ws, need, 0, None, None, None,
                                2, 4, 4, None, n, 4, 64, k, 1e-6, sol.BF16, None) == sol.ERR_UNSUPPORTED
    assert L.sol_adaln_qkv_rope(out, 1152, x, k, None, None, 0, SEL, w, k, ws, need, 0, None, None, None,
                                2, 4, 4, None, n, 3, 128, k, 1e-6, sol.BF16, None) == sol.ERR_UNSUPPORTED
    assert L.sol_adaln_qkv_rope(out, 768, x, k, None, None, 0, SEL, w, k, ws, need, 0, None, None, None,
                                2, 4, 4, None, n, 2, 128, k, 1e-6, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert "rope is NULL" in last(L)
    # the AdaLN strategy is an argument: only the three sol_adaln_strategy values pass
    for bad in (-1, 3):
        assert L.sol_adaln_linear(out, d, x, k, None, None, 0, SEL, w, k, ws, need, bad, n, d, k, 1e-6,
                                  sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
        assert "strategy" in last(L)


def test_adaln_linear_swiglu_validation(L):
    n, k, inner = 300, 512, 384
    x, w, out = FAKE, FAKE << 3, FAKE << 4
    need = L.sol_adaln_workspace_bytes(n, 2 * inner, k, SEL)
    ws = FAKE << 6
    assert L.sol_adaln_linear_swiglu(out, inner, x, k, None, None, 0, SEL, w, k, ws, need, 0, n, inner, k, 1e-6,
                                     sol.F32, None) == sol.ERR_UNSUPPORTED
    assert L.sol_adaln_linear_swiglu(out, 192, x, k, None, None, 0, SEL, w, k, ws, need, 0, n, 192, k, 1e-6,
                                     sol.BF16, None) == sol.ERR_UNSUPPORTED  # inner not a multiple of 128
    assert L.sol_adaln_linear_swiglu(out, inner, x, k, None, None, 0, SEL, w, k, None, need, 0, n, inner, k, 1e-6,
                                     sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_linear_swiglu(out, inner, x, k, None, None, 0, SEL, w, k, ws, need - 256, 0, n, inner, k,
                                     1e-6, sol.BF16, None) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_adaln_linear_swiglu(None, inner, None, k, None, None, 0, SEL, w, k, None, 0, 0, 0, inner, k, 1e-6,
                                     sol.BF16, None) == sol.OK


def test_block_host_validation(L):
    """sol_dit_block_host checks its description, streams and workspace before it enqueues
    anything (no GPU needed for these refusals)."""
    import ctypes
    d = sol.BlockHostDesc()
    d.x = d.qkv = d.y_attn = d.u = d.y_mlp = FAKE
    d.rope = FAKE << 2
    d.grid_T, d.grid_H, d.grid_W = 2, 4, 4
    d.n_tokens, d.tokens_per_sample, d.n_streams = 32, 0, 1
    d.d, d.n_heads, d.head_dim, d.inner, d.eps, d.dt = 256, 2, 128, 512, 1e-6, sol.F32
    ref = ctypes.byref(d)
    need = L.sol_dit_block_host_workspace_bytes(ref, 16, 2)
    # constants (6 modulation rows, wq, wk) + 2 slots of 16 rows: x, qkv, y_attn, u, y_mlp,
    # h1, x1, h2, act, x2 (fp32), positions and stream ids, each region 256-byte aligned
    slot = 16 * 4 * (256 * 7 + 768 + 1024 + 512) + 256 + 256
    assert need >= 6 * 256 * 4 + 2 * 128 * 4 + 2 * slot
    assert L.sol_dit_block_host_workspace_bytes(ref, 0, 2) == 0
    assert L.sol_dit_block_host_workspace_bytes(None, 16, 2) == 0
    ws, s1, s2, s3 = FAKE << 8, 1, 2, 3
    assert L.sol_dit_block_host(None, ws, need, 16, 2, s1, s2, s3) == sol.ERR_INVALID_ARGUMENT
    assert L.sol_dit_block_host(ref, ws, need, 16, 2, s1, s1, s3) == sol.ERR_INVALID_ARGUMENT
    assert "distinct" in last(L)
    assert L.sol_dit_block_host(ref, ws, need - 1, 16, 2, s1, s2, s3) == sol.ERR_INVALID_ARGUMENT
    assert "workspace" in last(L)
    assert L.sol_dit_block_host(ref, ws + 16, need, 16, 2, s1, s2, s3) == sol.ERR_MISALIGNED
    assert L.sol_dit_block_host(ref, ws, need, 16, 0, s1, s2, s3) == sol.ERR_INVALID_ARGUMENT
    d.y_mlp = None
    assert L.sol_dit_block_host(ref, ws, need, 16, 2, s1, s2, s3) == sol.ERR_INVALID_ARGUMENT
    assert "required" in last(L)
    d.y_mlp = FAKE
    d.grid_W = 3  # 2 x 4 x 3 = 24 cells for 32 tokens of implicit positions
    assert L.sol_dit_block_host(ref, ws, need, 16, 2, s1, s2, s3) == sol.ERR_INVALID_ARGUMENT
    d.grid_W = 4
    d.d = 250  # not a multiple of 4 fp32 elements
    assert L.sol_dit_block_host(ref, ws, need, 16, 2, s1, s2, s3) == sol.ERR_MISALIGNED
    d.d, d.dt = 256, 7
    assert L.sol_dit_block_host(ref, ws, need, 16, 2, s1, s2, s3) == sol.ERR_UNSUPPORTED
    d.dt, d.rope = sol.F32, None
    assert L.sol_dit_block_host(ref, ws, need, 16, 2, s1, s2, s3) == sol.ERR_INVALID_ARGUMENT
    assert "rope" in last(L)
    d.rope, d.n_tokens = FAKE << 2, 0
    assert L.sol_dit_block_host(ref, None, 0, 16, 2, s1, s2, s3) == sol.OK


def test_selftest_validation(L):
    for bad in (0, -3, 1001):
        assert L.sol_selftest_wait_timeout(bad, None) == sol.ERR_INVALID_ARGUMENT
        assert "polls" in last(L)
