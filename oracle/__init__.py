"""fp64 CPU oracle for the fused DiT per-token operators (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline and
reference arm may import this package.  The product library (``dit_block_b200``)
never imports it and shares no code with it.

The per-token arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module marshals numpy arrays into it, and composes it with fp64 numpy matmuls for the
linear-layer fusions at its end.  Inputs are numpy arrays of ``float32``,
``float64`` or ``uint16`` (the raw bits of bf16 values); every output is ``float64``.
Each function names the operator it computes; the definitions and the page passages
they follow are in the header of ``oracle.c``.

Parity status: every function is pinned: the per-token operators by
``tests/test_oracle_pins.py``, the linear-layer compositions at the end of this module
by ``tests/test_oracle_linear_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP, no fast-math) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        I = ctypes.c_int
        lib.oracle_num_threads.restype = I
        lib.oracle_adaln_modulate.argtypes = [P, I64, P, I64, I, P, P, I64, I, P, I32, I64, P, I64, I64, D]
        lib.oracle_adaln_modulate.restype = None
        lib.oracle_gated_residual.argtypes = [P, I64, P, I64, P, I64, I, P, I64, I, P, I32, I64, P, I64, I64]
        lib.oracle_gated_residual.restype = None
        lib.oracle_gated_residual_cache_diff.argtypes = [P, P, P, I64, P, I64, P, I64, I, P, I64, I,
                                                         P, I64, I, P, I32, I64, P, I64, I64]
        lib.oracle_gated_residual_cache_diff.restype = None
        lib.oracle_qk_rmsnorm_rope3d_ex.argtypes = [P, P, P, P, I64, I64, I, P, P, I, P, I32, I32, I32,
                                                    I64, I32, I32, I32, D, P, I64, I32, I32, D, I, I]
        lib.oracle_qk_rmsnorm_rope3d_ex.restype = I
        lib.oracle_block_mean.argtypes = [P, P, I64, I64, I64, I64]
        lib.oracle_block_mean.restype = I64
        lib.oracle_swiglu.argtypes = [P, I64, P, P, I64, I, I64, I64]
        lib.oracle_swiglu.restype = None
        lib.oracle_qk_rmsnorm_rope3d.argtypes = [P, P, I64, I64, P, P, I64, I64, I, P, P, I, P,
                                                 I32, I32, I32, I64, I32, I32, I32, D, P, I64, I32,
                                                 I32, D]
        lib.oracle_qk_rmsnorm_rope3d.restype = I
        lib.oracle_dit_prologue.argtypes = [P, P, P, P, I, P, P, P, I64, I64, I, P, I32, I64, P, I64, I64, D]
        lib.oracle_dit_prologue.restype = None
        lib.oracle_dit_epilogue.argtypes = [P, P, I64, I, P, P, I, P, I32, I32, I32, I64,
                                            I32, I32, I32, D, P, I64, I32, I32, D]
        lib.oracle_dit_epilogue.restype = I
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().oracle_num_threads())


def _code(a: np.ndarray | None) -> int:
    if a is None:
        return F32
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float64:
        return F64
    raise TypeError(f"oracle inputs are float32, float64 or uint16 (bf16 bits), got {a.dtype}")


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags.c_contiguous, "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _rows(rows, n):
    """Global token index of each row passed (None: rows are tokens 0..n-1)."""
    if rows is None:
        return None
    r = np.ascontiguousarray(rows, dtype=np.int64)
    assert r.shape == (n,), "rows must hold one global token index per row"
    return r


def _ld(a: np.ndarray) -> int:
    return a.shape[-1] if a.ndim > 1 else a.shape[0]


def _mod_args(mod: np.ndarray | None, stream_id, n_streams, tokens_per_sample):
    ld_mod = _ld(mod) if mod is not None else 0
    sid = None
    if stream_id is not None:
        sid = np.ascontiguousarray(stream_id, dtype=np.uint8)
    return ld_mod, sid, int(n_streams), int(tokens_per_sample)


def adaln_modulate(x, shift=None, scale=None, *, eps=1e-6, stream_id=None, n_streams=1,
                   tokens_per_sample=0, rows=None, n_tokens=None, d=None):
    """h = LN(x) * (1 + scale[r]) + shift[r] per token row of x ([N, ld_x], first d columns).

    rows: optional global token index of each row of x (stream_id is then indexed by it)."""
    n = x.shape[0] if n_tokens is None else n_tokens
    d = x.shape[1] if d is None else d
    mod = shift if shift is not None else scale
    ld_mod, sid, S, tps = _mod_args(mod, stream_id, n_streams, tokens_per_sample)
    rw = _rows(rows, n)
    out = np.empty((n, d), np.float64)
    _load().oracle_adaln_modulate(out.ctypes.data, d, _ptr(x), _ld(x), _code(x), _ptr(shift),
                                  _ptr(scale), ld_mod, _code(mod), _ptr(sid), S, tps, _ptr(rw), n,
                                  d, float(eps))
    return out


def gated_residual(x, y, gate=None, *, stream_id=None, n_streams=1, tokens_per_sample=0,
                   rows=None, n_tokens=None, d=None):
    """o = x + gate[r] * y per token row."""
    assert x.dtype == y.dtype
    n = x.shape[0] if n_tokens is None else n_tokens
    d = x.shape[1] if d is None else d
    ld_mod, sid, S, tps = _mod_args(gate, stream_id, n_streams, tokens_per_sample)
    rw = _rows(rows, n)
    out = np.empty((n, d), np.float64)
    _load().oracle_gated_residual(out.ctypes.data, d, _ptr(x), _ld(x), _ptr(y), _ld(y), _code(x),
                                  _ptr(gate), ld_mod, _code(gate), _ptr(sid), S, tps, _ptr(rw),
                                  n, d)
    return out


def gated_residual_cache_diff(x, y, gate, cache, *, n_samples=1, stream_id=None, n_streams=1,
                              tokens_per_sample=0, rows=None):
    """Gated residual plus Cache-DiT residual-change sums.  Returns (out, r, sums) with
    out = x + gate*y, r = gate*y (the refreshed cache) and sums [n_samples, 2] =
    (sum |r - cache|, sum |cache|) per sample."""
    assert x.dtype == y.dtype
    n, d = x.shape
    ld_mod, sid, S, tps = _mod_args(gate, stream_id, n_streams, tokens_per_sample)
    rw = _rows(rows, n)
    out = np.empty((n, d), np.float64)
    r = np.empty((n, d), np.float64)
    sums = np.empty((n_samples, 2), np.float64)
    _load().oracle_gated_residual_cache_diff(out.ctypes.data, r.ctypes.data, sums.ctypes.data,
                                             int(n_samples), _ptr(x), _ld(x), _ptr(y), _ld(y),
                                             _code(x), _ptr(gate), ld_mod, _code(gate), _ptr(cache),
                                             _ld(cache), _code(cache), _ptr(sid), S, tps, _ptr(rw),
                                             n, d)
    return out, r, sums


def swiglu(u, inner=None, *, n_tokens=None):
    """o[:, j] = silu(u[:, j]) * u[:, inner + j] for the packed up-projection u [N, 2*inner]."""
    n = u.shape[0] if n_tokens is None else n_tokens
    inner = u.shape[1] // 2 if inner is None else inner
    out = np.empty((n, inner), np.float64)
    esz = u.dtype.itemsize
    _load().oracle_swiglu(out.ctypes.data, inner, _ptr(u), u.ctypes.data + inner * esz,
                          _ld(u), _code(u), n, inner)
    return out


def swiglu_ab(a, b):
    """o = silu(a) * b for two separate [N, inner] tensors of one dtype."""
    assert a.shape == b.shape and a.dtype == b.dtype
    n, inner = a.shape
    out = np.empty((n, inner), np.float64)
    _load().oracle_swiglu(out.ctypes.data, inner, _ptr(a), _ptr(b), inner, _code(a), n, inner)
    return out


def _pos_ptr(pos):
    if pos is None:
        return None, None
    p = np.ascontiguousarray(pos, dtype=np.int32)
    assert p.ndim == 2 and p.shape[1] == 3
    return p, p.ctypes.data


def qk_rmsnorm_rope3d(q, k, wq=None, wk=None, *, n_heads, head_dim, pos=None, grid=(0, 0, 0),
                      tokens_per_sample=0, dims=(32, 48, 48), theta=10000.0, eps=1e-6,
                      rows=None):
    """QK RMSNorm then 3D RoPE on each head vector of q [N, ld_q] and k [N, ld_k].

    Either q or k may be None.  Returns (q_out, k_out) as [N, n_heads*head_dim] float64."""
    src = q if q is not None else k
    n = src.shape[0]
    hd = n_heads * head_dim
    qo = np.empty((n, hd), np.float64) if q is not None else None
    ko = np.empty((n, hd), np.float64) if k is not None else None
    w = wq if wq is not None else wk
    pos_arr, pos_p = _pos_ptr(pos)
    rw = _rows(rows, n)
    rc = _load().oracle_qk_rmsnorm_rope3d(
        _ptr(qo), _ptr(ko), hd, hd, _ptr(q), _ptr(k), _ld(q) if q is not None else 0,
        _ld(k) if k is not None else 0, _code(src), _ptr(wq), _ptr(wk), _code(w), pos_p,
        int(grid[0]), int(grid[1]), int(grid[2]), int(tokens_per_sample), int(dims[0]),
        int(dims[1]), int(dims[2]), float(theta), _ptr(rw), n, int(n_heads), int(head_dim),
        float(eps))
    if rc != 0:
        raise ValueError("RoPE split does not fit head_dim (dims must be even and sum to it)")
    return qo, ko


def dit_prologue(x, y=None, gate=None, shift=None, scale=None, *, eps=1e-6, stream_id=None,
                 n_streams=1, tokens_per_sample=0, rows=None):
    """Fused prologue: x' = x + gate*y (when y is given), h = AdaLN(x').  Returns (x', h);
    x' is None when y is None."""
    n, d = x.shape
    mod = next((m for m in (gate, shift, scale) if m is not None), None)
    ld_mod, sid, S, tps = _mod_args(mod, stream_id, n_streams, tokens_per_sample)
    xo = np.empty((n, d), np.float64) if y is not None else None
    h = np.empty((n, d), np.float64)
    rw = _rows(rows, n)
    _load().oracle_dit_prologue(_ptr(xo), h.ctypes.data, _ptr(x), _ptr(y), _code(x), _ptr(gate),
                                _ptr(shift), _ptr(scale), d, ld_mod, _code(mod), _ptr(sid), S, tps,
                                _ptr(rw), n, d, float(eps))
    return xo, h


def dit_epilogue(qkv, wq=None, wk=None, *, n_heads, head_dim, pos=None, grid=(0, 0, 0),
                 tokens_per_sample=0, dims=(32, 48, 48), theta=10000.0, eps=1e-6, rows=None):
    """Fused QKV epilogue on packed rows [q | k | v]: returns [N, 2*n_heads*head_dim] with the
    normed+rotated q then k."""
    n = qkv.shape[0]
    hd = n_heads * head_dim
    out = np.empty((n, 2 * hd), np.float64)
    w = wq if wq is not None else wk
    pos_arr, pos_p = _pos_ptr(pos)
    rw = _rows(rows, n)
    rc = _load().oracle_dit_epilogue(
        out.ctypes.data, _ptr(qkv), _ld(qkv), _code(qkv), _ptr(wq), _ptr(wk), _code(w), pos_p,
        int(grid[0]), int(grid[1]), int(grid[2]), int(tokens_per_sample), int(dims[0]),
        int(dims[1]), int(dims[2]), float(theta), _ptr(rw), n, int(n_heads), int(head_dim),
        float(eps))
    if rc != 0:
        raise ValueError("RoPE split does not fit head_dim (dims must be even and sum to it)")
    return out


def block_mean(v, *, tokens_per_sample=0, block=64):
    """Means of `block`-token blocks of the fp64 rows v [N, width]; blocks restart at every
    sample boundary.  Returns [n_blocks, width]."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    n, width = v.shape
    tps = tokens_per_sample if tokens_per_sample > 0 else n
    per_sample = -(-tps // block)
    n_blocks = -(-n // tps) * per_sample if n else 0
    out = np.full((n_blocks, width), np.nan)
    got = _load().oracle_block_mean(out.ctypes.data, v.ctypes.data, n, width, int(tokens_per_sample),
                                    int(block))
    return out[:got]


NORM_PER_HEAD, NORM_ACROSS_HEADS = 0, 1
ROPE_INTERLEAVED, ROPE_HALF = 0, 1


def qk_rmsnorm_rope3d_ex(q, k, wq=None, wk=None, *, n_heads, head_dim, pos=None, grid=(0, 0, 0),
                         tokens_per_sample=0, dims=(32, 48, 48), theta=10000.0, eps=1e-6, rows=None,
                         norm_span=NORM_PER_HEAD, pairing=ROPE_INTERLEAVED):
    """QK RMSNorm + 3D RoPE with a choice of norm span (per head, or across all heads with
    weights [n_heads*head_dim]) and rotary pairing (interleaved, or rotate-half).  Returns
    token-major (q_out, k_out) float64 arrays."""
    src = q if q is not None else k
    n = src.shape[0]
    hd = n_heads * head_dim
    qo = np.empty((n, hd), np.float64) if q is not None else None
    ko = np.empty((n, hd), np.float64) if k is not None else None
    w = wq if wq is not None else wk
    pos_arr, pos_p = _pos_ptr(pos)
    rw = _rows(rows, n)
    rc = _load().oracle_qk_rmsnorm_rope3d_ex(
        _ptr(qo), _ptr(ko), _ptr(q), _ptr(k), _ld(q) if q is not None else 0, _ld(k) if k is not None else 0,
        _code(src), _ptr(wq), _ptr(wk), _code(w), pos_p, int(grid[0]), int(grid[1]), int(grid[2]),
        int(tokens_per_sample), int(dims[0]), int(dims[1]), int(dims[2]), float(theta), _ptr(rw), n,
        int(n_heads), int(head_dim), float(eps), int(norm_span), int(pairing))
    if rc != 0:
        raise ValueError("RoPE split does not fit head_dim (dims must be even and sum to it)")
    return qo, ko


# ---------------------------------------------------------------------------------------
# The per-token operators fused into the block's linear layers.
#
# [STM-RES] (section "Resultado principal") credits the fused kernels with cutting
# memory traffic, intermediate tensors and launches without changing the math.  The
# per-token operators sit between the DiT block's linear layers: AdaLN feeds the QKV
# projection, QK RMSNorm + 3D RoPE follows it, the gated residual follows the output
# projection and the MLP down projection, and SwiGLU follows the MLP up projection.
# Each function below is the composition, in fp64 with no intermediate rounding, of
# a linear layer y = a . W^T (W stored [out_features, in_features], the usual linear-
# layer layout; no bias) with the oracle operator on its input or output side.  The
# product a . W^T is one numpy fp64 matmul (a library primitive used as one step).
# ---------------------------------------------------------------------------------------

def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of float32 / float64 / uint16 (bf16 bits) to float64."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype in (np.float32, np.float64):
        return a.astype(np.float64)
    raise TypeError(f"oracle inputs are float32, float64 or uint16 (bf16 bits), got {a.dtype}")


def linear(a, w):
    """y = a . W^T: a [N, K], W [out, K] -> [N, out] float64."""
    a64, w64 = to_f64(a), to_f64(w)
    assert a64.shape[1] == w64.shape[1], "a and W must share the inner dimension"
    return a64 @ w64.T


def linear_magnitude(a, w):
    """|a| . |W|^T: the sum of |a_k W_jk| behind each output of linear(a, W) (an error-
    bound helper: rounding the operands or the partial sums moves y by at most a small
    multiple of this)."""
    return np.abs(to_f64(a)) @ np.abs(to_f64(w)).T


def linear_gated_residual(x, a, w, gate=None, *, stream_id=None, n_streams=1,
                          tokens_per_sample=0, rows=None):
    """out = x + gate[r] * (a . W^T): the gated residual on the output projection (or the
    MLP down projection)."""
    y = np.ascontiguousarray(linear(a, w))
    return gated_residual(to_f64(x), y, gate, stream_id=stream_id, n_streams=n_streams,
                          tokens_per_sample=tokens_per_sample, rows=rows)


def linear_swiglu(a, w, inner=None):
    """out = silu(a . W1^T) * (a . W2^T) with W = [W1; W2] ([2*inner, K]): SwiGLU on the MLP
    up projection, whose first `inner` outputs are the gated half."""
    u = np.ascontiguousarray(linear(a, w))
    return swiglu(u, inner)


def adaln_linear(x, w, shift=None, scale=None, *, eps=1e-6, stream_id=None, n_streams=1,
                 tokens_per_sample=0, rows=None):
    """y = AdaLN(x) . W^T, AdaLN(x) = LN(x) * (1 + scale[r]) + shift[r].  Returns (y, h) with
    h = AdaLN(x) in float64 (the exact operand of the product)."""
    h = adaln_modulate(x, shift, scale, eps=eps, stream_id=stream_id, n_streams=n_streams,
                       tokens_per_sample=tokens_per_sample, rows=rows)
    return linear(h, w), h


def adaln_qkv_rope(x, w, shift=None, scale=None, wq=None, wk=None, *, n_heads, head_dim,
                   pos=None, grid=(0, 0, 0), tokens_per_sample=0, dims=(32, 48, 48),
                   theta=10000.0, eps=1e-6, stream_id=None, n_streams=1, rows=None):
    """The attention input of a block: qkv = AdaLN(x) . W^T ([N, 3*n_heads*head_dim], q | k | v),
    then QK RMSNorm + 3D RoPE on q and k (v as projected).  Returns (qkv_out, qkv_pre, h):
    the result, the projection before the norm, and the AdaLN output."""
    y, h = adaln_linear(x, w, shift, scale, eps=eps, stream_id=stream_id, n_streams=n_streams,
                        tokens_per_sample=tokens_per_sample, rows=rows)
    hd = n_heads * head_dim
    assert y.shape[1] == 3 * hd, "W must have 3 * n_heads * head_dim rows"
    y = np.ascontiguousarray(y)
    qk = dit_epilogue(y, wq, wk, n_heads=n_heads, head_dim=head_dim, pos=pos, grid=grid,
                      tokens_per_sample=tokens_per_sample, dims=dims, theta=theta, eps=eps,
                      rows=rows)
    out = y.copy()
    out[:, :2 * hd] = qk
    return out, y, h


def adaln_linear_swiglu(x, w, shift=None, scale=None, inner=None, *, eps=1e-6, stream_id=None, n_streams=1,
                        tokens_per_sample=0, rows=None):
    """The MLP input of a block: u = AdaLN(x) . W^T with W = [W1; W2] ([2*inner, d]), then
    SwiGLU silu(u[:, :inner]) * u[:, inner:].  Returns (out, u, h)."""
    u, h = adaln_linear(x, w, shift, scale, eps=eps, stream_id=stream_id, n_streams=n_streams,
                        tokens_per_sample=tokens_per_sample, rows=rows)
    u = np.ascontiguousarray(u)
    return swiglu(u, inner), u, h
