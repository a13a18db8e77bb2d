"""ctypes binding of libsol (include/sol.h), same names without the ``sol_`` prefix.

Argument marshalling only: every op runs in the CUDA kernels of ``libsol.so``.  Tensors
are torch CUDA tensors, 2-D with unit column stride; their row stride is passed as the
leading dimension.  Ops run on torch's current CUDA stream unless ``stream`` is given
(a ``torch.cuda.Stream`` or a raw ``cudaStream_t`` integer).  A non-OK status raises
:class:`SolError` with the library's one-line reason.  If ``libsol.so`` is missing the
first call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsol.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "sol.h")

OK, ERR_INVALID_ARGUMENT, ERR_MISALIGNED, ERR_UNSUPPORTED, ERR_CUDA = range(5)
F32, BF16 = 0, 1


class SolError(RuntimeError):
    def __init__(self, status: int, func: str, detail: str):
        super().__init__(f"{func}: status {status}: {detail}")
        self.status = status


class ModSel(ctypes.Structure):
    _fields_ = [("stream_id", ctypes.c_void_p), ("n_streams", ctypes.c_int32),
                ("tokens_per_sample", ctypes.c_int64)]


_P, _I64, _I32, _F, _D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double


class QkDesc(ctypes.Structure):
    """sol_qk_desc (include/sol.h)."""
    _fields_ = [("q_out", _P), ("k_out", _P), ("out_token_stride", _I64), ("out_head_stride", _I64),
                ("out_sample_stride", _I64), ("q", _P), ("k", _P), ("ld_q", _I64), ("ld_k", _I64),
                ("wq", _P), ("wk", _P), ("pos", _P), ("grid_T", _I32), ("grid_H", _I32), ("grid_W", _I32),
                ("tokens_per_sample", _I64), ("rope", _P), ("n_tokens", _I64), ("n_heads", _I32),
                ("head_dim", _I32), ("eps", _F), ("norm_span", _I32), ("rope_pairing", _I32),
                ("dt", ctypes.c_int)]


class BlockHostDesc(ctypes.Structure):
    """sol_block_host_desc (include/sol.h)."""
    _fields_ = [("x", _P), ("qkv", _P), ("y_attn", _P), ("u", _P), ("y_mlp", _P), ("pos", _P),
                ("stream_id", _P), ("h1", _P), ("qk", _P), ("x1", _P), ("h2", _P), ("act", _P), ("x2", _P),
                ("shift_msa", _P), ("scale_msa", _P), ("gate_msa", _P), ("shift_mlp", _P), ("scale_mlp", _P),
                ("gate_mlp", _P), ("wq", _P), ("wk", _P), ("rope", _P), ("grid_T", _I32), ("grid_H", _I32),
                ("grid_W", _I32), ("n_tokens", _I64), ("tokens_per_sample", _I64), ("n_streams", _I32),
                ("d", _I64), ("n_heads", _I32), ("head_dim", _I32), ("inner", _I64), ("eps", _F),
                ("dt", ctypes.c_int)]


NORM_PER_HEAD, NORM_ACROSS_HEADS = 0, 1
ADALN_STAGE, ADALN_FOLD, ADALN_TRANSFORM = 0, 1, 2
_STRATEGIES = {"stage": ADALN_STAGE, "fold": ADALN_FOLD, "transform": ADALN_TRANSFORM}
ROPE_INTERLEAVED, ROPE_HALF = 0, 1
_E = ctypes.c_int  # enums

# argument types per exported function, in header order
SIGNATURES = {
    "sol_status_string": ([_E], ctypes.c_char_p),
    "sol_last_error": ([], ctypes.c_char_p),
    "sol_abi_version": ([], _I32),
    "sol_device_errors": ([ctypes.POINTER(ctypes.c_uint32), _I32], _E),
    "sol_selftest_wait_timeout": ([_I32, _P], _E),
    "sol_adaln_modulate": ([_P, _I64, _P, _I64, _P, _P, _I64, ModSel, _I64, _I64, _F, _E, _P], _E),
    "sol_gated_residual": ([_P, _I64, _P, _I64, _P, _I64, _P, _I64, ModSel, _I64, _I64, _E, _P], _E),
    "sol_gated_residual_cache_diff": ([_P, _I64, _P, _I64, _P, _I64, _P, _I64, ModSel, _P, _I64, _I32,
                                       _P, _I64, _I64, _I64, _E, _P], _E),
    "sol_swiglu": ([_P, _I64, _P, _P, _I64, _I64, _I64, _E, _P], _E),
    "sol_rope3d_create": ([ctypes.POINTER(_P), _I32, _I32, _I32, _D, _I32, _I32, _I32], _E),
    "sol_rope3d_destroy": ([_P], _E),
    "sol_qk_rmsnorm_rope3d": ([_P, _P, _I64, _I64, _P, _P, _I64, _I64, _P, _P, _P, _I32, _I32,
                               _I32, _I64, _P, _I64, _I32, _I32, _F, _E, _P], _E),
    "sol_dit_prologue": ([_P, _P, _P, _P, _P, _P, _P, _I64, _I64, ModSel, _I64, _I64, _F, _E, _P], _E),
    "sol_dit_epilogue": ([_P, _I64, _P, _P, _P, _I32, _I32, _I32, _I64, _P, _I64, _I32, _I32, _F,
                          _E, _P], _E),
    "sol_subblock_count": ([_I64, _I64, _I32], _I64),
    "sol_qk_rmsnorm_rope3d_ex": ([ctypes.POINTER(QkDesc), _P], _E),
    "sol_dit_epilogue_pool": ([_P, _I64, _P, _P, _P, _I32, _I32, _I32, _I64, _P, _I64, _I32, _I32, _F,
                               _P, _P, _I64, _I32, _E, _P], _E),
    "sol_qk_rmsnorm_rope3d_noalloc": ([_P, _P, _I64, _I64, _P, _P, _I64, _I64, _P, _P, _P, _I32, _I32,
                                       _I32, _I64, _I32, _I32, _I32, _D, _I32, _I32, _I32, _I64,
                                       _I32, _I32, _F, _E, _P], _E),
    "sol_dit_block_host_workspace_bytes": ([ctypes.POINTER(BlockHostDesc), _I64, _I32], ctypes.c_size_t),
    "sol_dit_block_host": ([ctypes.POINTER(BlockHostDesc), _P, ctypes.c_size_t, _I64, _I32, _P, _P, _P], _E),
    "sol_linear": ([_P, _I64, _P, _I64, _P, _I64, _I64, _I64, _I64, _E, _P], _E),
    "sol_linear_gated_residual": ([_P, _I64, _P, _I64, _P, _I64, _P, _I64, _P, _I64, ModSel, _I64, _I64,
                                   _I64, _E, _P], _E),
    "sol_linear_swiglu": ([_P, _I64, _P, _I64, _P, _I64, _I64, _I64, _I64, _E, _P], _E),
    "sol_adaln_workspace_bytes": ([_I64, _I64, _I64, ModSel], ctypes.c_size_t),
    "sol_adaln_linear": ([_P, _I64, _P, _I64, _P, _P, _I64, ModSel, _P, _I64, _P, ctypes.c_size_t, _I32, _I64,
                          _I64, _I64, _F, _E, _P], _E),
    "sol_adaln_linear_swiglu": ([_P, _I64, _P, _I64, _P, _P, _I64, ModSel, _P, _I64, _P, ctypes.c_size_t, _I32,
                                 _I64, _I64, _I64, _F, _E, _P], _E),
    "sol_adaln_qkv_rope": ([_P, _I64, _P, _I64, _P, _P, _I64, ModSel, _P, _I64, _P, ctypes.c_size_t, _I32, _P,
                            _P, _P, _I32, _I32, _I32, _P, _I64, _I32, _I32, _I64, _F, _E, _P], _E),
}

_lib = None


def header_functions() -> list[str]:
    """Names of every function include/sol.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"\b(sol_[a-z0-9_]+)\s*\(", text)


def lib() -> ctypes.CDLL:
    """The loaded libsol.so with argument types set (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libsol.so is not built at {LIB_PATH}; run "
                              "`python -m dit_block_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status: int, func: str):
    if status != OK:
        raise SolError(status, func, lib().sol_last_error().decode())


def status_string(status: int) -> str:
    return lib().sol_status_string(status).decode()


def abi_version() -> int:
    return int(lib().sol_abi_version())


def device_errors(clear: bool = False) -> int:
    """Error flags libsol kernels raised on the current device (0 in normal operation)."""
    f = ctypes.c_uint32(0)
    _check(lib().sol_device_errors(ctypes.byref(f), int(clear)), "sol_device_errors")
    return int(f.value)


def selftest_wait_timeout(polls: int = 8, stream=None):
    """Run the bounded-wait failure path on purpose (sol_selftest_wait_timeout): afterwards
    device_errors() reports bit 2 until cleared."""
    _check(lib().sol_selftest_wait_timeout(int(polls), _stream(stream)), "sol_selftest_wait_timeout")


# ------------------------------------------------------------------------- marshalling

def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"libsol takes float32 or bfloat16 tensors, got {t.dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _ld(t: torch.Tensor | None) -> int:
    if t is None:
        return 0
    if t.dim() == 1:
        return t.shape[0]
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("tensors must be 2-D with unit column stride")
    return t.stride(0)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _sel(stream_id: torch.Tensor | None, n_streams: int, tokens_per_sample: int) -> ModSel:
    if stream_id is not None and stream_id.dtype != torch.uint8:
        raise TypeError("stream_id must be uint8")
    return ModSel(_ptr(stream_id), int(n_streams), int(tokens_per_sample))


def _mod_ld(*mods) -> int:
    for m in mods:
        if m is not None:
            return _ld(m)
    return 0


# ----------------------------------------------------------------------------- the ops

def adaln_modulate(h, x, shift=None, scale=None, *, eps=1e-6, stream_id=None, n_streams=1,
                   tokens_per_sample=0, d=None, stream=None):
    """h = LN(x) * (1 + scale[r]) + shift[r]  (sol_adaln_modulate)."""
    n = x.shape[0]
    d = x.shape[1] if d is None else d
    _check(lib().sol_adaln_modulate(_ptr(h), _ld(h), _ptr(x), _ld(x), _ptr(shift), _ptr(scale),
                                    _mod_ld(shift, scale), _sel(stream_id, n_streams, tokens_per_sample),
                                    n, d, eps, _dtype(x), _stream(stream)), "sol_adaln_modulate")
    return h


def gated_residual(out, x, y, gate=None, *, stream_id=None, n_streams=1, tokens_per_sample=0,
                   d=None, stream=None):
    """out = x + gate[r] * y  (sol_gated_residual)."""
    n = x.shape[0]
    d = x.shape[1] if d is None else d
    _check(lib().sol_gated_residual(_ptr(out), _ld(out), _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(gate),
                                    _mod_ld(gate), _sel(stream_id, n_streams, tokens_per_sample), n, d,
                                    _dtype(x), _stream(stream)), "sol_gated_residual")
    return out


def gated_residual_cache_diff(out, x, y, gate, cache, sums, *, refresh=True, stream_id=None,
                              n_streams=1, tokens_per_sample=0, d=None, stream=None):
    """out = x + gate[r]*y and, per sample, sums[s] = (sum |gate*y - cache|, sum |cache|);
    with refresh the cache becomes gate*y (sol_gated_residual_cache_diff).  sums is a
    float64 device tensor [n_samples, 2]."""
    if sums.dtype != torch.float64 or not sums.is_contiguous():
        raise TypeError("sums must be a contiguous float64 tensor [n_samples, 2]")
    n = x.shape[0]
    d = x.shape[1] if d is None else d
    _check(lib().sol_gated_residual_cache_diff(
        _ptr(out), _ld(out), _ptr(x), _ld(x), _ptr(y), _ld(y), _ptr(gate), _mod_ld(gate),
        _sel(stream_id, n_streams, tokens_per_sample), _ptr(cache), _ld(cache), int(bool(refresh)),
        _ptr(sums), sums.numel() // 2, n, d, _dtype(x), _stream(stream)), "sol_gated_residual_cache_diff")
    return out


def swiglu(out, u, *, inner=None, stream=None):
    """out = silu(u[:, :inner]) * u[:, inner:2*inner] for the packed up-projection u."""
    inner = u.shape[1] // 2 if inner is None else inner
    b = u.data_ptr() + inner * u.element_size()
    _check(lib().sol_swiglu(_ptr(out), _ld(out), u.data_ptr(), b, _ld(u), u.shape[0], inner,
                            _dtype(u), _stream(stream)), "sol_swiglu")
    return out


def swiglu_ab(out, a, b, *, stream=None):
    """out = silu(a) * b for two tensors with the same leading dimension."""
    if _ld(a) != _ld(b):
        raise ValueError("a and b must share a leading dimension")
    _check(lib().sol_swiglu(_ptr(out), _ld(out), _ptr(a), _ptr(b), _ld(a), a.shape[0], a.shape[1],
                            _dtype(a), _stream(stream)), "sol_swiglu")
    return out


class Rope3D:
    """Library-owned 3D RoPE cos/sin tables on the current device (sol_rope3d_create)."""

    def __init__(self, dims=(32, 48, 48), theta=10000.0, max_pos=(64, 64, 128)):
        h = ctypes.c_void_p()
        _check(lib().sol_rope3d_create(ctypes.byref(h), int(dims[0]), int(dims[1]), int(dims[2]),
                                       float(theta), int(max_pos[0]), int(max_pos[1]),
                                       int(max_pos[2])), "sol_rope3d_create")
        self.handle = h.value
        self.dims = tuple(dims)
        self.theta = theta
        self.max_pos = tuple(max_pos)

    def close(self):
        if self.handle:
            _check(lib().sol_rope3d_destroy(self.handle), "sol_rope3d_destroy")
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def qk_rmsnorm_rope3d(q_out, k_out, q, k, rope: Rope3D, *, n_heads, head_dim, wq=None, wk=None,
                      pos=None, grid=(0, 0, 0), tokens_per_sample=0, eps=1e-6, stream=None):
    """QK RMSNorm then 3D RoPE on every head vector of q and k (sol_qk_rmsnorm_rope3d)."""
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous()):
        raise TypeError("pos must be a contiguous int32 [N, 3] tensor")
    _check(lib().sol_qk_rmsnorm_rope3d(
        _ptr(q_out), _ptr(k_out), _ld(q_out), _ld(k_out), _ptr(q), _ptr(k), _ld(q), _ld(k),
        _ptr(wq), _ptr(wk), _ptr(pos), int(grid[0]), int(grid[1]), int(grid[2]),
        int(tokens_per_sample), rope.handle, q.shape[0], int(n_heads), int(head_dim), eps,
        _dtype(q), _stream(stream)), "sol_qk_rmsnorm_rope3d")


def dit_prologue(x_out, h, x, y=None, gate=None, shift=None, scale=None, *, eps=1e-6,
                 stream_id=None, n_streams=1, tokens_per_sample=0, stream=None):
    """x' = x + gate*y (if y), h = AdaLN(x') in one pass (sol_dit_prologue)."""
    ld = _ld(x)
    _check(lib().sol_dit_prologue(_ptr(x_out), _ptr(h), _ptr(x), _ptr(y), _ptr(gate), _ptr(shift),
                                  _ptr(scale), ld, _mod_ld(gate, shift, scale),
                                  _sel(stream_id, n_streams, tokens_per_sample), x.shape[0],
                                  x.shape[1], eps, _dtype(x), _stream(stream)), "sol_dit_prologue")


def dit_epilogue(qkv, rope: Rope3D, *, n_heads, head_dim, wq=None, wk=None, pos=None,
                 grid=(0, 0, 0), tokens_per_sample=0, eps=1e-6, stream=None):
    """QK RMSNorm + 3D RoPE on the q and k parts of packed [q | k | v] rows, in place."""
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous()):
        raise TypeError("pos must be a contiguous int32 [N, 3] tensor")
    _check(lib().sol_dit_epilogue(_ptr(qkv), _ld(qkv), _ptr(wq), _ptr(wk), _ptr(pos), int(grid[0]),
                                  int(grid[1]), int(grid[2]), int(tokens_per_sample), rope.handle,
                                  qkv.shape[0], int(n_heads), int(head_dim), eps, _dtype(qkv),
                                  _stream(stream)), "sol_dit_epilogue")


NOALLOC_MAX_ROPE_ENTRIES = 65536


def qk_rmsnorm_rope3d_noalloc(q_out, k_out, q, k, *, n_heads, head_dim, dims=(32, 48, 48),
                              theta=10000.0, max_pos, wq=None, wk=None, pos=None, grid=(0, 0, 0),
                              tokens_per_sample=0, eps=1e-6, stream=None):
    """sol_qk_rmsnorm_rope3d without a sol_rope3d handle: for callers that cannot allocate
    device memory.  The cos/sin table for (dims, theta, max_pos) is rebuilt by every call
    in a fixed library array (at most NOALLOC_MAX_ROPE_ENTRIES pairs); calls that overlap
    on the GPU race on it."""
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous()):
        raise TypeError("pos must be a contiguous int32 [N, 3] tensor")
    _check(lib().sol_qk_rmsnorm_rope3d_noalloc(
        _ptr(q_out), _ptr(k_out), _ld(q_out), _ld(k_out), _ptr(q), _ptr(k), _ld(q), _ld(k),
        _ptr(wq), _ptr(wk), _ptr(pos), int(grid[0]), int(grid[1]), int(grid[2]),
        int(tokens_per_sample), int(dims[0]), int(dims[1]), int(dims[2]), float(theta),
        int(max_pos[0]), int(max_pos[1]), int(max_pos[2]), q.shape[0], int(n_heads),
        int(head_dim), eps, _dtype(q), _stream(stream)), "sol_qk_rmsnorm_rope3d_noalloc")


BLOCK_HOST_IN = ("x", "qkv", "y_attn", "u", "y_mlp")
BLOCK_HOST_OUT = ("h1", "qk", "x1", "h2", "act", "x2")
BLOCK_HOST_MOD = ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp")


def block_host_desc(inputs: dict, outputs: dict, mods: dict, rope: Rope3D, *, n_heads: int, head_dim: int,
                    inner: int, wq=None, wk=None, pos=None, stream_id=None, grid=(0, 0, 0), tokens_per_sample=0,
                    n_streams=1, eps=1e-6) -> BlockHostDesc:
    """sol_block_host_desc over HOST tensors (pinned for overlapped copies): inputs
    BLOCK_HOST_IN, outputs BLOCK_HOST_OUT (missing or None: not copied back), modulation rows
    BLOCK_HOST_MOD (missing or None: zero), wq / wk, pos [N, 3] int32, stream_id [N] uint8."""
    x = inputs["x"]
    for t in list(inputs.values()) + [v for v in outputs.values() if v is not None]:
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("sol_dit_block_host takes contiguous host tensors")
    if pos is not None and (pos.dtype != torch.int32 or pos.is_cuda):
        raise TypeError("pos must be a host int32 [N, 3] tensor")
    if stream_id is not None and (stream_id.dtype != torch.uint8 or stream_id.is_cuda):
        raise TypeError("stream_id must be a host uint8 tensor")
    g = lambda k, dct: _ptr(dct.get(k))
    return BlockHostDesc(
        *(g(k, inputs) for k in BLOCK_HOST_IN), _ptr(pos), _ptr(stream_id), *(g(k, outputs) for k in BLOCK_HOST_OUT),
        *(g(k, mods) for k in BLOCK_HOST_MOD), _ptr(wq), _ptr(wk), rope.handle, int(grid[0]), int(grid[1]),
        int(grid[2]), x.shape[0], int(tokens_per_sample), int(n_streams), x.shape[1], int(n_heads), int(head_dim),
        int(inner), float(eps), _dtype(x))


def dit_block_host_workspace_bytes(desc: BlockHostDesc, chunk_tokens: int, n_slots: int) -> int:
    return int(lib().sol_dit_block_host_workspace_bytes(ctypes.byref(desc), int(chunk_tokens), int(n_slots)))


def dit_block_host(desc: BlockHostDesc, workspace: torch.Tensor, *, chunk_tokens: int, n_slots: int, s_in, s_comp,
                   s_out):
    """One block pass over host tensors (sol_dit_block_host): enqueued on s_comp with the
    copies on s_in / s_out; the host outputs are filled once s_comp reaches the end."""
    _check(lib().sol_dit_block_host(ctypes.byref(desc), _ptr(workspace), workspace.numel(), int(chunk_tokens),
                                    int(n_slots), _stream(s_in), _stream(s_comp), _stream(s_out)),
           "sol_dit_block_host")


def subblock_count(n_tokens: int, tokens_per_sample: int = 0, block_tokens: int = 64) -> int:
    """Blocks of block_tokens tokens in the sequence (blocks restart at each sample)."""
    return int(lib().sol_subblock_count(int(n_tokens), int(tokens_per_sample), int(block_tokens)))


def dit_epilogue_pool(qkv, pooled_q, pooled_k, rope: Rope3D, *, n_heads, head_dim, wq=None, wk=None,
                      pos=None, grid=(0, 0, 0), tokens_per_sample=0, block_tokens=64, eps=1e-6,
                      stream=None):
    """sol_dit_epilogue plus per-block means of the normalised, rotated q and k."""
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous()):
        raise TypeError("pos must be a contiguous int32 [N, 3] tensor")
    if _ld(pooled_q) != _ld(pooled_k):
        raise ValueError("pooled_q and pooled_k must share a leading dimension")
    _check(lib().sol_dit_epilogue_pool(
        _ptr(qkv), _ld(qkv), _ptr(wq), _ptr(wk), _ptr(pos), int(grid[0]), int(grid[1]), int(grid[2]),
        int(tokens_per_sample), rope.handle, qkv.shape[0], int(n_heads), int(head_dim), eps,
        _ptr(pooled_q), _ptr(pooled_k), _ld(pooled_q), int(block_tokens), _dtype(qkv), _stream(stream)),
        "sol_dit_epilogue_pool")


def qk_rmsnorm_rope3d_ex(q_out, k_out, q, k, rope: Rope3D, *, n_heads, head_dim, wq=None, wk=None, pos=None,
                         grid=(0, 0, 0), tokens_per_sample=0, eps=1e-6, norm_span=NORM_PER_HEAD,
                         pairing=ROPE_INTERLEAVED, out_strides=None, stream=None):
    """sol_qk_rmsnorm_rope3d_ex.  out_strides = (token, head, sample) element strides of
    q_out and k_out (default: token-major rows like q_out's).  q_out / k_out are passed as
    base pointers (tensors of any shape)."""
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous()):
        raise TypeError("pos must be a contiguous int32 [N, 3] tensor")
    n = q.shape[0]
    if out_strides is None:
        ld = _ld(q_out)
        tps = tokens_per_sample if tokens_per_sample > 0 else n
        out_strides = (ld, head_dim, tps * ld)
    d = QkDesc(_ptr(q_out), _ptr(k_out), int(out_strides[0]), int(out_strides[1]), int(out_strides[2]),
               _ptr(q), _ptr(k), _ld(q), _ld(k), _ptr(wq), _ptr(wk), _ptr(pos), int(grid[0]), int(grid[1]),
               int(grid[2]), int(tokens_per_sample), rope.handle, n, int(n_heads), int(head_dim), float(eps),
               int(norm_span), int(pairing), _dtype(q))
    _check(lib().sol_qk_rmsnorm_rope3d_ex(ctypes.byref(d), _stream(stream)), "sol_qk_rmsnorm_rope3d_ex")


# ------------------------------------------------------- linear layers with fused operators

def linear(out, a, w, *, stream=None):
    """out = a . W^T on the tensor cores (sol_linear); W is [n_out, k]."""
    _check(lib().sol_linear(_ptr(out), _ld(out), _ptr(a), _ld(a), _ptr(w), _ld(w), a.shape[0], w.shape[0],
                            a.shape[1], _dtype(a), _stream(stream)), "sol_linear")
    return out


def linear_gated_residual(out, x, a, w, gate=None, *, stream_id=None, n_streams=1, tokens_per_sample=0,
                          stream=None):
    """out = x + gate[r] * (a . W^T)  (sol_linear_gated_residual); out may be x."""
    _check(lib().sol_linear_gated_residual(
        _ptr(out), _ld(out), _ptr(x), _ld(x), _ptr(a), _ld(a), _ptr(w), _ld(w), _ptr(gate), _mod_ld(gate),
        _sel(stream_id, n_streams, tokens_per_sample), a.shape[0], w.shape[0], a.shape[1], _dtype(a),
        _stream(stream)), "sol_linear_gated_residual")
    return out


def linear_swiglu(out, a, w, *, stream=None):
    """out = silu(a . W1^T) * (a . W2^T) with W = [W1; W2] of [2*inner, k]  (sol_linear_swiglu)."""
    _check(lib().sol_linear_swiglu(_ptr(out), _ld(out), _ptr(a), _ld(a), _ptr(w), _ld(w), a.shape[0],
                                   w.shape[0] // 2, a.shape[1], _dtype(a), _stream(stream)),
           "sol_linear_swiglu")
    return out


def adaln_workspace_bytes(n_tokens: int, n_out: int, d: int, *, n_streams=1, tokens_per_sample=0) -> int:
    """Bytes of workspace the sol_adaln_* calls need (sol_adaln_workspace_bytes)."""
    return int(lib().sol_adaln_workspace_bytes(int(n_tokens), int(n_out), int(d),
                                               ModSel(None, int(n_streams), int(tokens_per_sample))))


def adaln_workspace(n_tokens: int, n_out: int, d: int, *, n_streams=1, tokens_per_sample=0,
                    device=None) -> torch.Tensor:
    """A workspace for the sol_adaln_* calls (uint8 device tensor; torch allocations are
    256-byte aligned)."""
    nb = adaln_workspace_bytes(n_tokens, n_out, d, n_streams=n_streams, tokens_per_sample=tokens_per_sample)
    if nb == 0:
        raise ValueError("no workspace size for these arguments (more than 32 modulation rows?)")
    return torch.empty((nb,), dtype=torch.uint8, device=device or "cuda")


def _strategy(strategy) -> int:
    """A sol_adaln_strategy from its name ("stage", "fold", "transform") or its value."""
    return _STRATEGIES[strategy] if isinstance(strategy, str) else int(strategy)


def adaln_linear(out, x, w, shift=None, scale=None, *, workspace, strategy="stage", eps=1e-6, stream_id=None,
                 n_streams=1, tokens_per_sample=0, stream=None):
    """out = AdaLN(x) . W^T  (sol_adaln_linear; `strategy` stages h through the workspace,
    folds the modulation into the weights or transforms the operand: sol_adaln_strategy)."""
    _check(lib().sol_adaln_linear(
        _ptr(out), _ld(out), _ptr(x), _ld(x), _ptr(shift), _ptr(scale), _mod_ld(shift, scale),
        _sel(stream_id, n_streams, tokens_per_sample), _ptr(w), _ld(w), _ptr(workspace), workspace.numel(),
        _strategy(strategy), x.shape[0], w.shape[0], x.shape[1], eps, _dtype(x), _stream(stream)),
        "sol_adaln_linear")
    return out


def adaln_linear_swiglu(out, x, w, shift=None, scale=None, *, workspace, strategy="stage", eps=1e-6,
                        stream_id=None, n_streams=1, tokens_per_sample=0, stream=None):
    """out = silu(h . W1^T) * (h . W2^T), h = AdaLN(x), W = [W1; W2]  (sol_adaln_linear_swiglu)."""
    _check(lib().sol_adaln_linear_swiglu(
        _ptr(out), _ld(out), _ptr(x), _ld(x), _ptr(shift), _ptr(scale), _mod_ld(shift, scale),
        _sel(stream_id, n_streams, tokens_per_sample), _ptr(w), _ld(w), _ptr(workspace), workspace.numel(),
        _strategy(strategy), x.shape[0], w.shape[0] // 2, x.shape[1], eps, _dtype(x), _stream(stream)),
        "sol_adaln_linear_swiglu")
    return out


def adaln_qkv_rope(qkv, x, w, rope: Rope3D, shift=None, scale=None, *, workspace, n_heads, head_dim=128,
                   wq=None, wk=None, pos=None, grid=(0, 0, 0), strategy="stage", eps=1e-6, stream_id=None,
                   n_streams=1, tokens_per_sample=0, stream=None):
    """qkv = AdaLN(x) . W^T, then QK RMSNorm + 3D RoPE on q and k  (sol_adaln_qkv_rope)."""
    _check(lib().sol_adaln_qkv_rope(
        _ptr(qkv), _ld(qkv), _ptr(x), _ld(x), _ptr(shift), _ptr(scale), _mod_ld(shift, scale),
        _sel(stream_id, n_streams, tokens_per_sample), _ptr(w), _ld(w), _ptr(workspace), workspace.numel(),
        _strategy(strategy), _ptr(wq), _ptr(wk),
        _ptr(pos), int(grid[0]), int(grid[1]), int(grid[2]), rope.handle, x.shape[0], n_heads, head_dim,
        x.shape[1], eps, _dtype(x), _stream(stream)), "sol_adaln_qkv_rope")
    return qkv
