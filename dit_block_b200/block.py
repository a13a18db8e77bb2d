"""One pass of the per-token hot path of a DiT block, as five libsol launches.

In a DiT block the per-token operators sit between the GEMMs and attention:

    h1  = AdaLN(x; shift_msa, scale_msa)                 -> QKV GEMM      (sol_adaln_modulate)
    q,k = RMSNorm + 3D RoPE on the QKV output, in place   -> attention     (sol_dit_epilogue)
    x1  = x + gate_msa * y_attn;  h2 = AdaLN(x1; mlp mod)  -> up GEMM       (sol_dit_prologue)
    act = silu(u[:, :I]) * u[:, I:]                         -> down GEMM     (sol_swiglu)
    x2  = x1 + gate_mlp * y_mlp                             -> next block    (sol_gated_residual)

The GEMMs and attention are outside this library; their outputs (qkv, y_attn, u, y_mlp)
are inputs here.  ``BlockBuffers`` holds every input and output of one pass on one
device; ``step`` issues the five launches on one stream.
"""
from __future__ import annotations

import dataclasses

import torch

from . import sol
from .workloads import Workload, block_inputs

OPS = ("adaln_modulate", "dit_epilogue", "dit_prologue", "swiglu", "gated_residual")


def bytes_per_token(w: Workload) -> dict:
    """Algorithmic HBM bytes per token of each launch: every element each op must read
    or write, counted once (modulation rows, weights, tables, positions and stream ids
    are shared by all tokens and left out; they are < 0.1% at the bf16 sizes)."""
    e = torch.empty((), dtype=w.dtype).element_size()
    d, hd, inner = w.d, w.hd, w.inner
    return {
        "adaln_modulate": 2 * d * e,                 # read x, write h1
        "dit_epilogue": 4 * hd * e,                  # read q, k; write q, k
        "dit_prologue": 4 * d * e,                   # read x, y; write x', h
        "swiglu": 3 * inner * e,                     # read a, b; write out
        "gated_residual": 3 * d * e,                 # read x, y; write out
    }


@dataclasses.dataclass
class BlockBuffers:
    w: Workload
    inp: dict
    h1: torch.Tensor
    x1: torch.Tensor
    h2: torch.Tensor
    act: torch.Tensor
    x2: torch.Tensor
    rope: sol.Rope3D

    @classmethod
    def allocate(cls, w: Workload, device="cuda", n_tokens: int | None = None, inputs=None):
        inp = block_inputs(w, device, n_tokens) if inputs is None else inputs
        n = inp["x"].shape[0]
        empty = lambda cols: torch.empty((n, cols), dtype=w.dtype, device=device)
        rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
        return cls(w, inp, empty(w.d), empty(w.d), empty(w.d), empty(w.inner), empty(w.d), rope)

    @property
    def n_tokens(self) -> int:
        return self.inp["x"].shape[0]

    def sel(self) -> dict:
        w = self.w
        return dict(stream_id=self.inp["stream_id"], n_streams=w.n_streams,
                    tokens_per_sample=w.tokens_per_sample)

    def launch(self, op: str, stream=None):
        """Issue one of the five launches of the pass."""
        w, i = self.w, self.inp
        if op == "adaln_modulate":
            sol.adaln_modulate(self.h1, i["x"], i["shift_msa"], i["scale_msa"], eps=w.eps,
                               stream=stream, **self.sel())
        elif op == "dit_epilogue":
            sol.dit_epilogue(i["qkv"], self.rope, n_heads=w.n_heads, head_dim=w.head_dim,
                             wq=i["wq"], wk=i["wk"], pos=i["pos"], grid=w.grid,
                             tokens_per_sample=w.tokens_per_sample, eps=w.eps, stream=stream)
        elif op == "dit_prologue":
            sol.dit_prologue(self.x1, self.h2, i["x"], i["y_attn"], i["gate_msa"], i["shift_mlp"],
                             i["scale_mlp"], eps=w.eps, stream=stream, **self.sel())
        elif op == "swiglu":
            sol.swiglu(self.act, i["u"], inner=w.inner, stream=stream)
        elif op == "gated_residual":
            sol.gated_residual(self.x2, self.x1, i["y_mlp"], i["gate_mlp"], stream=stream,
                               **self.sel())
        else:
            raise KeyError(op)

    def step(self, stream=None):
        for op in OPS:
            self.launch(op, stream)

    def capture(self, steps: int = 1) -> torch.cuda.CUDAGraph:
        """Record `steps` passes into a CUDA graph; ``graph.replay()`` then issues them as
        one launch instead of five kernel launches per pass, which matters at small token
        counts.  One eager pass runs first, outside the capture, so that every kernel's
        one-time attribute and occupancy setup is done (the op modifies q and k in place,
        so that pass counts like any other).  The graph reads and writes these buffers: it
        stays valid while they live, and their contents may change between replays."""
        dev = self.inp["x"].device
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self.step()
        torch.cuda.current_stream(dev).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps):
                self.step()
        return g

    def close(self):
        self.rope.close()
