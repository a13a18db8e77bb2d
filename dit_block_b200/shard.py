"""Token-sharded split of one workload over ranks (one process per GPU, no exchange).

Every operator of the block pass works on one token row at a time, and 3D RoPE reads the
token's global (t, h, w) position, so a contiguous range of tokens per rank needs no
collective on the data path: a rank carries the positions and stream ids of its range and
the modulation rows (a few KB, replicated) of the samples its range touches.  The
packed video+audio stack of the pages (stamatios.com, "SGLang acelera video do
MiniMax-H3...", section "Resultado principal": video and audio tokens run through one
packed DiT stack) is split the same way: a range may start or end inside a sample, or
span a sample boundary.

A rank's range is cut at sample boundaries into pieces.  Each piece is one call per
operator with that sample's modulation rows (tokens_per_sample = 0: the piece is one
sample), the stream ids of its tokens and, unless the piece starts at its sample's
first token of a video-only workload, explicit positions.
"""
from __future__ import annotations

import dataclasses

import torch

from . import sol
from .block import OPS
from .workloads import Workload, activation, modulation, norm_weight

MOD_NAMES = ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp")


def token_ranges(n_tokens: int, world: int) -> list[tuple[int, int]]:
    """Contiguous [t0, t1) per rank, covering every token exactly once; sizes differ by at
    most one token (the first n_tokens % world ranks take one more)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    base, extra = divmod(int(n_tokens), int(world))
    out, t = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((t, t + n))
        t += n
    return out


@dataclasses.dataclass(frozen=True)
class Piece:
    start: int    # global index of its first token
    length: int
    sample: int   # the one sample it lies in
    offset: int   # index of its first token inside the rank's range


def pieces(w: Workload, t0: int, t1: int) -> list[Piece]:
    """[t0, t1) cut at sample boundaries."""
    tps = w.tokens_per_sample
    out, t = [], t0
    while t < t1:
        b = t // tps
        end = min(t1, (b + 1) * tps)
        out.append(Piece(t, end - t, b, t - t0))
        t = end
    return out


def positions(w: Workload, t0: int, t1: int) -> torch.Tensor:
    """Global (t, h, w) positions of tokens [t0, t1) as int32 [t1 - t0, 3]: per sample the
    video tokens in row-major (t, h, w) order, then the audio tokens at (p, 0, 0)."""
    T, H, W = w.grid
    n = torch.arange(t0, t1, dtype=torch.int64)
    local = n % w.tokens_per_sample
    video = local < w.video_per_sample
    pos = torch.zeros((t1 - t0, 3), dtype=torch.int64)
    pos[:, 0] = torch.where(video, local // (H * W), local - w.video_per_sample)
    pos[:, 1] = torch.where(video, (local // W) % H, torch.zeros_like(local))
    pos[:, 2] = torch.where(video, local % W, torch.zeros_like(local))
    return pos.to(torch.int32).contiguous()


def stream_ids(w: Workload, t0: int, t1: int) -> torch.Tensor | None:
    """Stream id (0 video, 1 audio) of tokens [t0, t1), or None for a video-only workload."""
    if not w.packed:
        return None
    local = torch.arange(t0, t1, dtype=torch.int64) % w.tokens_per_sample
    return (local >= w.video_per_sample).to(torch.uint8).contiguous()


def needs_explicit_positions(w: Workload, p: Piece) -> bool:
    """The implicit grid of the kernels counts tokens from the call's first one, so only a
    video-only piece that starts at its sample's first token can use it."""
    return w.packed or p.start != p.sample * w.tokens_per_sample


@dataclasses.dataclass(frozen=True)
class PieceCall:
    rows: slice           # the piece's rows inside the rank's tensors
    mod_rows: slice       # its sample's rows of every modulation tensor
    explicit_pos: bool    # pass the piece's positions (else the implicit grid)


def piece_call(w: Workload, p: Piece) -> PieceCall:
    """What one call per operator over piece p is given: its rows, its sample's
    modulation rows (with tokens_per_sample 0 and n_streams rows per sample) and whether
    it needs explicit positions."""
    S = w.n_streams
    return PieceCall(slice(p.offset, p.offset + p.length), slice(p.sample * S, (p.sample + 1) * S),
                     needs_explicit_positions(w, p))


def shard_inputs(w: Workload, t0: int, t1: int, device="cpu") -> dict:
    """Inputs of one rank's range: activations for its t1 - t0 rows (drawn from the
    workload's seeded generators; their values do not affect the split), the replicated
    modulation rows and RMSNorm weights, and the global positions / stream ids of its
    tokens."""
    n = t1 - t0
    inp = {
        "x": activation(w, "x", n, w.d, device),
        "qkv": activation(w, "qkv", n, 3 * w.hd, device),
        "y_attn": activation(w, "y_attn", n, w.d, device),
        "u": activation(w, "u", n, 2 * w.inner, device),
        "y_mlp": activation(w, "y_mlp", n, w.d, device),
        "wq": norm_weight(w, "wq", device),
        "wk": norm_weight(w, "wk", device),
        "pos": positions(w, t0, t1).to(device),
        "stream_id": None,
    }
    sid = stream_ids(w, t0, t1)
    if sid is not None:
        inp["stream_id"] = sid.to(device)
    for k in MOD_NAMES:
        inp[k] = modulation(w, k, device)
    return inp


class ShardBuffers:
    """One rank's part of the block pass: the same five launches as
    ``block.BlockBuffers``, issued once per piece of the rank's token range."""

    def __init__(self, w: Workload, t0: int, t1: int, device="cuda", inputs: dict | None = None):
        self.w, self.t0, self.t1 = w, int(t0), int(t1)
        self.inp = shard_inputs(w, t0, t1, device) if inputs is None else inputs
        n = self.t1 - self.t0
        e = lambda cols: torch.empty((n, cols), dtype=w.dtype, device=device)
        self.h1, self.x1, self.h2, self.act, self.x2 = e(w.d), e(w.d), e(w.d), e(w.inner), e(w.d)
        self.pieces = pieces(w, self.t0, self.t1)
        self.rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)

    @property
    def n_tokens(self) -> int:
        return self.t1 - self.t0

    def _piece_args(self, p: Piece):
        w, i = self.w, self.inp
        c = piece_call(w, p)
        sl = c.rows
        sid = i["stream_id"]
        sel = dict(stream_id=None if sid is None else sid[sl], n_streams=w.n_streams, tokens_per_sample=0)
        mod = {k: i[k][c.mod_rows] for k in MOD_NAMES}
        pos = i["pos"][sl] if c.explicit_pos else None
        return sl, sel, mod, pos

    def launch(self, op: str, stream=None):
        """Issue one of the five launches of the pass: SwiGLU once over the range, the
        others once per piece (they select modulation rows or positions per sample)."""
        w, i = self.w, self.inp
        if op == "swiglu":
            sol.swiglu(self.act, i["u"], inner=w.inner, stream=stream)
            return
        for p in self.pieces:
            sl, sel, m, pos = self._piece_args(p)
            if op == "adaln_modulate":
                sol.adaln_modulate(self.h1[sl], i["x"][sl], m["shift_msa"], m["scale_msa"], eps=w.eps,
                                   stream=stream, **sel)
            elif op == "dit_epilogue":
                sol.dit_epilogue(i["qkv"][sl], self.rope, n_heads=w.n_heads, head_dim=w.head_dim, wq=i["wq"],
                                 wk=i["wk"], pos=pos, grid=w.grid, tokens_per_sample=0, eps=w.eps,
                                 stream=stream)
            elif op == "dit_prologue":
                sol.dit_prologue(self.x1[sl], self.h2[sl], i["x"][sl], i["y_attn"][sl], m["gate_msa"],
                                 m["shift_mlp"], m["scale_mlp"], eps=w.eps, stream=stream, **sel)
            elif op == "gated_residual":
                sol.gated_residual(self.x2[sl], self.x1[sl], i["y_mlp"][sl], m["gate_mlp"], stream=stream,
                                   **sel)
            else:
                raise KeyError(op)

    def step(self, stream=None):
        for op in OPS:
            self.launch(op, stream)

    def close(self):
        self.rope.close()
