"""The block hot path over host-resident tensors, through the C ABI's host-buffer call.

``HostBlockPipeline.run`` takes one block pass whose inputs and outputs live in pinned
host memory and hands it to ``sol_dit_block_host`` (include/sol.h), which cuts the token
sequence into chunks (a chunk never straddles two samples) and runs each chunk through
three CUDA streams:

    copy-in  (H2D: x, qkv, y_attn, u, y_mlp of the chunk; positions and stream ids)
    compute  (the five libsol launches of ``block.BlockBuffers.step`` on the chunk)
    copy-out (D2H: h1, q|k, x1, h2, act, x2 of the chunk -- those the caller asked for)

with ``n_slots`` device buffers of a caller-owned workspace rotating between them, so that
while chunk i computes, chunk i+1 is uploaded and chunk i-1 downloaded.  A PCIe-bound pass
then takes about max(H2D, D2H) instead of their sum plus the compute.  The library issues
every copy and launch; this class only owns the workspace and the streams.
"""
from __future__ import annotations

import torch

from . import sol
from .workloads import Workload, token_layout

IN_NAMES = sol.BLOCK_HOST_IN
OUT_NAMES = sol.BLOCK_HOST_OUT
MOD_NAMES = sol.BLOCK_HOST_MOD


def host_buffers(w: Workload, n_tokens: int | None = None, pin: bool = True):
    """Empty pinned host tensors for one pass: (inputs, outputs, modulation)."""
    n = w.n_tokens if n_tokens is None else n_tokens
    e = lambda cols: torch.empty((n, cols), dtype=w.dtype, pin_memory=pin)
    inputs = {"x": e(w.d), "qkv": e(3 * w.hd), "y_attn": e(w.d), "u": e(2 * w.inner), "y_mlp": e(w.d)}
    outputs = {"h1": e(w.d), "qk": e(2 * w.hd), "x1": e(w.d), "h2": e(w.d), "act": e(w.inner),
               "x2": e(w.d)}
    mods = {k: torch.empty((w.batch * w.n_streams, w.d), dtype=w.dtype, pin_memory=pin) for k in MOD_NAMES}
    return inputs, outputs, mods


class HostBlockPipeline:
    def __init__(self, w: Workload, device="cuda", chunk_tokens: int = 8192, n_slots: int = 3):
        self.w = w
        self.dev = torch.device(device)
        self.chunk = int(chunk_tokens)
        self.n_slots = int(n_slots)
        self.rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
        self.wq = torch.ones((w.head_dim,), dtype=w.dtype, pin_memory=True)
        self.wk = torch.ones((w.head_dim,), dtype=w.dtype, pin_memory=True)
        pos, sid = token_layout(w)  # explicit for packed video+audio, None for a video-only grid
        self.pos = None if pos is None else pos.pin_memory()
        self.sid = None if sid is None else sid.pin_memory()
        self.ws = None
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_comp = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)

    def chunks(self, n_tokens: int):
        """(start, length, sample) of every chunk the library cuts (a chunk never crosses a
        sample): the same rule as sol_dit_block_host, for callers that plan around it."""
        tps = self.w.tokens_per_sample
        out = []
        for b0 in range(0, n_tokens, tps):
            b1 = min(n_tokens, b0 + tps)
            for c0 in range(b0, b1, self.chunk):
                out.append((c0, min(self.chunk, b1 - c0), b0 // tps))
        return out

    def set_weights(self, wq: torch.Tensor, wk: torch.Tensor):
        """RMSNorm weights for q and k (copied by the library at every pass)."""
        self.wq.copy_(wq)
        self.wk.copy_(wk)

    def bytes_per_pass(self, n_tokens: int, outputs=OUT_NAMES) -> tuple[int, int]:
        """(H2D, D2H) bytes one run() moves for n_tokens tokens, copying back `outputs`."""
        w = self.w
        e = torch.empty((), dtype=w.dtype).element_size()
        h2d = n_tokens * (w.d + 3 * w.hd + w.d + 2 * w.inner + w.d) * e
        h2d += len(MOD_NAMES) * w.batch * w.n_streams * w.d * e + 2 * w.head_dim * e
        if self.pos is not None:
            h2d += n_tokens * (3 * 4 + 1)  # positions and stream ids
        width = {"h1": w.d, "qk": 2 * w.hd, "x1": w.d, "h2": w.d, "act": w.inner, "x2": w.d}
        d2h = n_tokens * sum(width[k] for k in outputs) * e
        return h2d, d2h

    def desc(self, host_in: dict, host_out: dict, host_mod: dict) -> sol.BlockHostDesc:
        w = self.w
        n = host_in["x"].shape[0]
        pos = None if self.pos is None else self.pos[:n]
        sid = None if self.sid is None else self.sid[:n]
        return sol.block_host_desc(host_in, host_out, host_mod, self.rope, n_heads=w.n_heads, head_dim=w.head_dim,
                                   inner=w.inner, wq=self.wq, wk=self.wk, pos=pos, stream_id=sid, grid=w.grid,
                                   tokens_per_sample=w.tokens_per_sample, n_streams=w.n_streams, eps=w.eps)

    def run(self, host_in: dict, host_out: dict, host_mod: dict):
        """Enqueue one pass over pinned host tensors (outputs missing from host_out, or None,
        stay on the device); returns the event that marks its end (wait on it, or
        synchronise, before reading host_out)."""
        d = self.desc(host_in, host_out, host_mod)
        need = sol.dit_block_host_workspace_bytes(d, self.chunk, self.n_slots)
        if need == 0:
            raise ValueError("sol_dit_block_host_workspace_bytes refused these sizes")
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.empty((need,), dtype=torch.uint8, device=self.dev)
        cur = torch.cuda.current_stream(self.dev)
        self.s_comp.wait_stream(cur)  # start after the caller's prior work
        sol.dit_block_host(d, self.ws, chunk_tokens=self.chunk, n_slots=self.n_slots, s_in=self.s_in,
                           s_comp=self.s_comp, s_out=self.s_out)
        done = torch.cuda.Event()
        done.record(self.s_comp)
        cur.wait_event(done)
        # the workspace stays in use until the pass ends on s_comp
        self.ws.record_stream(self.s_comp)
        return done

    def close(self):
        self.rope.close()
