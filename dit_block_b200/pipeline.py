"""The block hot path over host-resident tensors, with copies overlapped with compute.

``HostBlockPipeline.run`` takes one block pass whose inputs and outputs live in pinned
host memory.  It cuts the token sequence into chunks (a chunk never straddles two
samples) and runs each chunk through three CUDA streams:

    copy-in  (H2D: x, qkv, y_attn, u, y_mlp of the chunk)
    compute  (the five libsol launches of ``block.BlockBuffers.step`` on the chunk)
    copy-out (D2H: h1, q|k, x1, h2, act, x2 of the chunk)

with ``n_slots`` device buffers rotating between them, so that while chunk i computes,
chunk i+1 is uploaded and chunk i-1 downloaded.  A PCIe-bound pass then takes about
max(H2D, D2H) instead of their sum plus the compute.

Positions and stream ids are passed explicitly per chunk (slices of one sample's
layout, uploaded once), and each chunk gets its own sample's modulation rows, so the
results equal those of one call over the whole sequence.
"""
from __future__ import annotations

import torch

from . import sol
from .workloads import Workload

IN_NAMES = ("x", "qkv", "y_attn", "u", "y_mlp")
OUT_NAMES = ("h1", "qk", "x1", "h2", "act", "x2")
MOD_NAMES = ("shift_msa", "scale_msa", "gate_msa", "shift_mlp", "scale_mlp", "gate_mlp")


def sample_layout(w: Workload):
    """(pos [tokens_per_sample, 3] int32, stream_id [tokens_per_sample] uint8) of one sample:
    video tokens in (t, h, w) row-major order (stream 0), then audio tokens at (p, 0, 0)
    (stream 1)."""
    T, H, W = w.grid
    tt, hh, ww = torch.meshgrid(torch.arange(T), torch.arange(H), torch.arange(W), indexing="ij")
    video = torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], dim=1)
    audio = torch.zeros((w.audio_per_sample, 3), dtype=torch.int64)
    audio[:, 0] = torch.arange(w.audio_per_sample)
    pos = torch.cat([video, audio]).to(torch.int32).contiguous()
    sid = torch.cat([torch.zeros(w.video_per_sample, dtype=torch.uint8),
                     torch.ones(w.audio_per_sample, dtype=torch.uint8)]).contiguous()
    return pos, sid


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
        e = lambda cols: torch.empty((self.n_slots, self.chunk, cols), dtype=w.dtype, device=self.dev)
        self.din = {"x": e(w.d), "qkv": e(3 * w.hd), "y_attn": e(w.d), "u": e(2 * w.inner),
                    "y_mlp": e(w.d)}
        self.dout = {"h1": e(w.d), "x1": e(w.d), "h2": e(w.d), "act": e(w.inner), "x2": e(w.d)}
        self.dmod = {k: torch.empty((w.batch * w.n_streams, w.d), dtype=w.dtype, device=self.dev)
                     for k in MOD_NAMES}
        self.wq = torch.empty((w.head_dim,), dtype=w.dtype, device=self.dev)
        self.wk = torch.empty((w.head_dim,), dtype=w.dtype, device=self.dev)
        pos, sid = sample_layout(w)
        self.pos = pos.to(self.dev)
        self.sid = sid.to(self.dev)
        self.rope = sol.Rope3D(w.rope_dims, w.theta, w.max_pos)
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_comp = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)

    def chunks(self, n_tokens: int):
        """(start, length, sample) of every chunk; a chunk never crosses a sample."""
        tps = self.w.tokens_per_sample
        out = []
        for b0 in range(0, n_tokens, tps):
            b1 = min(n_tokens, b0 + tps)
            for c0 in range(b0, b1, self.chunk):
                out.append((c0, min(self.chunk, b1 - c0), b0 // tps))
        return out

    def set_weights(self, wq: torch.Tensor, wk: torch.Tensor):
        self.wq.copy_(wq)
        self.wk.copy_(wk)

    def bytes_per_pass(self, n_tokens: int) -> tuple[int, int]:
        """(H2D, D2H) bytes one run() moves for n_tokens tokens."""
        w = self.w
        e = torch.empty((), dtype=w.dtype).element_size()
        h2d = n_tokens * (w.d + 3 * w.hd + w.d + 2 * w.inner + w.d) * e
        h2d += len(MOD_NAMES) * w.batch * w.n_streams * w.d * e
        d2h = n_tokens * (w.d + 2 * w.hd + w.d + w.d + w.inner + w.d) * e
        return h2d, d2h

    def _compute(self, slot: int, c0: int, L: int, b: int):
        w, i, o = self.w, self.din, self.dout
        S = w.n_streams
        m = {k: v[b * S:(b + 1) * S] for k, v in self.dmod.items()}
        local = c0 - b * w.tokens_per_sample
        sel = dict(stream_id=self.sid[local:local + L] if w.packed else None, n_streams=S,
                   tokens_per_sample=0)
        pos = self.pos[local:local + L]
        st = self.s_comp
        x, qkv, ya, u, ym = (i[k][slot, :L] for k in IN_NAMES)
        h1, x1, h2, act, x2 = (o[k][slot, :L] for k in ("h1", "x1", "h2", "act", "x2"))
        sol.adaln_modulate(h1, x, m["shift_msa"], m["scale_msa"], eps=w.eps, stream=st, **sel)
        sol.dit_epilogue(qkv, self.rope, n_heads=w.n_heads, head_dim=w.head_dim, wq=self.wq, wk=self.wk,
                         pos=pos, eps=w.eps, stream=st)
        sol.dit_prologue(x1, h2, x, ya, m["gate_msa"], m["shift_mlp"], m["scale_mlp"], eps=w.eps,
                         stream=st, **sel)
        sol.swiglu(act, u, inner=w.inner, stream=st)
        sol.gated_residual(x2, x1, ym, m["gate_mlp"], stream=st, **sel)

    def run(self, host_in: dict, host_out: dict, host_mod: dict):
        """Enqueue one pass over pinned host tensors; returns the event that marks its end
        on the copy-out stream (wait on it, or synchronise, before reading host_out)."""
        w = self.w
        n = host_in["x"].shape[0]
        hd = w.hd
        cur = torch.cuda.current_stream(self.dev)
        # modulation rows (tiny) first; every stream starts after the caller's prior work
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_stream(cur)
        with torch.cuda.stream(self.s_in):
            for k in MOD_NAMES:
                self.dmod[k].copy_(host_mod[k], non_blocking=True)
        mods_in = torch.cuda.Event()
        mods_in.record(self.s_in)
        self.s_comp.wait_event(mods_in)
        in_done, comp_done, out_done = {}, {}, {}
        for j, (c0, L, b) in enumerate(self.chunks(n)):
            slot = j % self.n_slots
            # upload: the slot's previous chunk must be computed and downloaded (its q|k
            # are downloaded from the input slot itself)
            if j >= self.n_slots:
                self.s_in.wait_event(out_done[j - self.n_slots])
            with torch.cuda.stream(self.s_in):
                for k in IN_NAMES:
                    self.din[k][slot, :L].copy_(host_in[k][c0:c0 + L], non_blocking=True)
            in_done[j] = torch.cuda.Event()
            in_done[j].record(self.s_in)
            # compute: inputs present, and the slot's previous outputs downloaded
            self.s_comp.wait_event(in_done[j])
            if j >= self.n_slots:
                self.s_comp.wait_event(out_done[j - self.n_slots])
            self._compute(slot, c0, L, b)
            comp_done[j] = torch.cuda.Event()
            comp_done[j].record(self.s_comp)
            # download
            self.s_out.wait_event(comp_done[j])
            with torch.cuda.stream(self.s_out):
                o = self.dout
                host_out["h1"][c0:c0 + L].copy_(o["h1"][slot, :L], non_blocking=True)
                host_out["qk"][c0:c0 + L].copy_(self.din["qkv"][slot, :L, :2 * hd], non_blocking=True)
                for k in ("x1", "h2", "act", "x2"):
                    host_out[k][c0:c0 + L].copy_(o[k][slot, :L], non_blocking=True)
            out_done[j] = torch.cuda.Event()
            out_done[j].record(self.s_out)
        done = torch.cuda.Event()
        done.record(self.s_out)
        cur.wait_event(done)
        return done

    def close(self):
        self.rope.close()
