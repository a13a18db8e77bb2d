"""Seeded synthetic inputs shaped like the DiT-block workloads (no operator arithmetic).

This module only draws random tensors and lays out token structure (grids, packed
video+audio positions, stream ids).  It computes none of the operators, so both the
CUDA path and the fp64 oracle can be fed from it.

Workloads (all tokens are rows; d = hidden width, Hh x Dh heads, I = SwiGLU width):

* ``tiny``        fp32, 1 sample, latent grid 2x4x4 (32 tokens), d=256, 2x128 heads, I=512.
* ``lowres``      bf16, grid 31x24x42 (31,248 tokens): 672x384 px, 121 frames,
                  /16 spatial and /4 temporal latent compression.
* ``fullres_5s``  bf16, grid 31x48x84 (124,992 tokens): 1344x768 px, 24 FPS, 5 s.
* ``fullres_10s`` bf16, grid 61x48x84 (245,952 tokens): 1344x768 px, 24 FPS, 10 s,
                  with 0.1% of every activation element replaced by +-50.
* ``packed_av``   bf16, 2 samples, each 124,992 video tokens (31x48x84) followed by
                  1,252 audio tokens at positions (p, 0, 0); stream 0 = video, 1 = audio.

The bf16 workloads use d=5120, 40x128 heads, I=13,824.  Distributions: activations
(x, y, u, q/k/v) ~ N(0, 1); shift, scale, gate ~ N(0, 0.1^2); RMSNorm weights
~ 1 + N(0, 0.02^2).  RoPE: theta = 10000, head-dim split (t, h, w) = (32, 48, 48);
eps = 1e-6.  Tensor ``tid`` of workload ``k`` is drawn from a generator seeded with
``1000 * k + tid``; draws are fp32 and then rounded to the workload dtype.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    dtype: torch.dtype
    batch: int
    grid: tuple[int, int, int]     # (T, H, W) latent grid of the video tokens of one sample
    audio_per_sample: int          # audio tokens appended after the video tokens
    d: int
    n_heads: int
    head_dim: int
    inner: int                     # SwiGLU output width (input width is 2*inner)
    outlier_frac: float = 0.0
    outlier_mag: float = 50.0
    rope_dims: tuple[int, int, int] = (32, 48, 48)
    theta: float = 10000.0
    eps: float = 1e-6

    @property
    def video_per_sample(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def tokens_per_sample(self) -> int:
        return self.video_per_sample + self.audio_per_sample

    @property
    def n_tokens(self) -> int:
        return self.batch * self.tokens_per_sample

    @property
    def n_streams(self) -> int:
        return 2 if self.audio_per_sample else 1

    @property
    def packed(self) -> bool:
        return self.audio_per_sample > 0

    @property
    def hd(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def max_pos(self) -> tuple[int, int, int]:
        """Table extents needed per axis (audio positions run along t)."""
        T, H, W = self.grid
        return (max(T, self.audio_per_sample), H, W)


BF16 = torch.bfloat16
WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 0, torch.float32, 1, (2, 4, 4), 0, 256, 2, 128, 512),
        Workload("lowres", 1, BF16, 1, (31, 24, 42), 0, 5120, 40, 128, 13824),
        Workload("fullres_5s", 2, BF16, 1, (31, 48, 84), 0, 5120, 40, 128, 13824),
        Workload("fullres_10s", 3, BF16, 1, (61, 48, 84), 0, 5120, 40, 128, 13824,
                 outlier_frac=1e-3),
        Workload("packed_av", 4, BF16, 2, (31, 48, 84), 1252, 5120, 40, 128, 13824),
    ]
}

# tensor ids (seed = 1000 * workload.index + id)
TID = {"x": 1, "y_attn": 2, "y_mlp": 3, "u": 4, "qkv": 5,
       "shift_msa": 10, "scale_msa": 11, "gate_msa": 12,
       "shift_mlp": 13, "scale_mlp": 14, "gate_mlp": 15, "wq": 20, "wk": 21,
       # linear-layer weights and the activations that feed them
       "w_qkv": 30, "w_o": 31, "w_up": 32, "w_down": 33, "attn": 34, "act": 35}

_CHUNK_ELEMS = 1 << 26  # draw at most 64M fp32 values at a time (bounded temporaries)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def fill_normal_(out: torch.Tensor, seed: int, mean: float = 0.0, std: float = 1.0,
                 outlier_frac: float = 0.0, outlier_mag: float = 50.0) -> torch.Tensor:
    """Fill a 2-D tensor (rows may be strided) with seeded N(mean, std^2) draws, row chunk
    by row chunk; optionally replace a seeded fraction of elements by +-outlier_mag."""
    assert out.dim() == 2
    g = _gen(out.device, seed)
    rows, cols = out.shape
    step = max(1, _CHUNK_ELEMS // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        v = torch.randn((r1 - r0, cols), generator=g, device=out.device, dtype=torch.float32)
        if std != 1.0:
            v.mul_(std)
        if mean != 0.0:
            v.add_(mean)
        if outlier_frac > 0.0:
            hit = torch.rand((r1 - r0, cols), generator=g, device=out.device) < outlier_frac
            sign = torch.rand((r1 - r0, cols), generator=g, device=out.device) < 0.5
            mag = torch.where(sign, torch.full_like(v, outlier_mag), torch.full_like(v, -outlier_mag))
            v = torch.where(hit, mag, v)
        out[r0:r1].copy_(v)
        del v
    return out


def activation(w: Workload, name: str, rows: int, cols: int, device="cpu",
               dtype: torch.dtype | None = None) -> torch.Tensor:
    t = torch.empty((rows, cols), dtype=dtype or w.dtype, device=device)
    return fill_normal_(t, 1000 * w.index + TID[name], 0.0, 1.0, w.outlier_frac, w.outlier_mag)


def modulation(w: Workload, name: str, device="cpu") -> torch.Tensor:
    """One row of length d per (sample, stream): [batch * n_streams, d]."""
    t = torch.empty((w.batch * w.n_streams, w.d), dtype=w.dtype, device=device)
    return fill_normal_(t, 1000 * w.index + TID[name], 0.0, 0.1)


def norm_weight(w: Workload, name: str, device="cpu") -> torch.Tensor:
    t = torch.empty((1, w.head_dim), dtype=w.dtype, device=device)
    return fill_normal_(t, 1000 * w.index + TID[name], 1.0, 0.02).view(w.head_dim)


def linear_weight(w: Workload, name: str, out_features: int, in_features: int, device="cpu") -> torch.Tensor:
    """Linear-layer weight [out_features, in_features] ~ N(0, 1/in_features), so a product
    with unit-variance activations has unit variance."""
    t = torch.empty((out_features, in_features), dtype=w.dtype, device=device)
    return fill_normal_(t, 1000 * w.index + TID[name], 0.0, in_features ** -0.5)


def token_layout(w: Workload):
    """(pos, stream_id) for the workload.

    Video-only workloads return (None, None): positions follow the row-major (t, h, w)
    grid of each sample implicitly.  The packed workload returns explicit int32
    positions [N, 3] and uint8 stream ids [N]: per sample, the video tokens in (t, h, w)
    row-major order with stream 0, then the audio tokens at (p, 0, 0) with stream 1."""
    if not w.packed:
        return None, None
    T, H, W = w.grid
    tt, hh, ww = torch.meshgrid(torch.arange(T), torch.arange(H), torch.arange(W), indexing="ij")
    video = torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], dim=1)
    audio = torch.zeros((w.audio_per_sample, 3), dtype=torch.int64)
    audio[:, 0] = torch.arange(w.audio_per_sample)
    one = torch.cat([video, audio], dim=0)
    pos = one.repeat(w.batch, 1).to(torch.int32).contiguous()
    sid_one = torch.cat([torch.zeros(w.video_per_sample, dtype=torch.uint8),
                         torch.ones(w.audio_per_sample, dtype=torch.uint8)])
    sid = sid_one.repeat(w.batch).contiguous()
    return pos, sid


def block_inputs(w: Workload, device="cpu", n_tokens: int | None = None) -> dict:
    """Every input of one DiT-block pass over the workload, on ``device``.

    x: residual stream [N, d]; qkv: QKV-projection output [N, 3*Hh*Dh]; y_attn: attention
    output projection [N, d]; u: up-projection output [N, 2*I]; y_mlp: down-projection
    output [N, d]; six modulation rows (shift/scale/gate for the attention and MLP
    halves); wq, wk: RMSNorm weights [Dh]; pos / stream_id as in token_layout()."""
    n = w.n_tokens if n_tokens is None else n_tokens
    pos, sid = token_layout(w)
    out = {
        "x": activation(w, "x", n, w.d, device),
        "qkv": activation(w, "qkv", n, 3 * w.hd, device),
        "y_attn": activation(w, "y_attn", n, w.d, device),
        "u": activation(w, "u", n, 2 * w.inner, device),
        "y_mlp": activation(w, "y_mlp", n, w.d, device),
        "wq": norm_weight(w, "wq", device),
        "wk": norm_weight(w, "wk", device),
        "pos": None if pos is None else pos[:n].to(device),
        "stream_id": None if sid is None else sid[:n].to(device),
    }
    for k in ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp"):
        out[k] = modulation(w, k, device)
    return out
