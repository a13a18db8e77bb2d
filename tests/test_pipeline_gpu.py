"""The host-buffer pass (sol_dit_block_host through pipeline.HostBlockPipeline: chunked,
three streams, every copy issued by the library) gives bit-identical results to one pass
of the five launches over the whole sequence, on a video-only grid (positions generated
per chunk from the implicit grid) and on a packed video+audio batch (explicit positions and
stream ids) whose chunks stop at sample boundaries; outputs left out stay on the device."""
from __future__ import annotations

import pytest
import torch

from dit_block_b200 import block, pipeline, sol, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dit_block_b200 import build
    build.build()


CASES = [
    workloads.Workload("grid", 11, torch.bfloat16, 1, (5, 6, 7), 0, 512, 4, 128, 768),
    workloads.Workload("packed", 12, torch.bfloat16, 3, (3, 4, 5), 23, 256, 2, 128, 512),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("chunk", [16, 50, 4096])
def test_pipeline_matches_single_pass(w, chunk):
    bufs = block.BlockBuffers.allocate(w, "cuda")
    i = bufs.inp
    qkv0 = i["qkv"].clone()
    bufs.step()
    torch.cuda.synchronize()
    n = bufs.n_tokens
    host_in, host_out, host_mod = pipeline.host_buffers(w, n)
    for k in pipeline.IN_NAMES:
        host_in[k].copy_(qkv0 if k == "qkv" else i[k])
    for k in pipeline.MOD_NAMES:
        host_mod[k].copy_(i[k])
    pipe = pipeline.HostBlockPipeline(w, "cuda", chunk_tokens=chunk, n_slots=3)
    pipe.set_weights(i["wq"], i["wk"])
    for _ in range(2):  # twice: slots are reused across passes
        pipe.run(host_in, host_out, host_mod)
    torch.cuda.synchronize()
    assert torch.equal(host_out["h1"], bufs.h1.cpu())
    assert torch.equal(host_out["qk"], i["qkv"][:, :2 * w.hd].cpu())
    assert torch.equal(host_out["x1"], bufs.x1.cpu())
    assert torch.equal(host_out["h2"], bufs.h2.cpu())
    assert torch.equal(host_out["act"], bufs.act.cpu())
    assert torch.equal(host_out["x2"], bufs.x2.cpu())
    h2d, d2h = pipe.bytes_per_pass(n)
    layout = 0 if pipe.pos is None else pipe.pos.numel() * 4 + pipe.sid.numel()
    assert h2d == sum(t.numel() * t.element_size() for t in host_in.values()) + \
        sum(t.numel() * t.element_size() for t in host_mod.values()) + \
        pipe.wq.numel() * pipe.wq.element_size() * 2 + layout
    assert d2h == sum(t.numel() * t.element_size() for t in host_out.values())
    # only x2 back: the other outputs are not copied (their host buffers keep a sentinel)
    only = {"x2": torch.full_like(host_out["x2"], 7.0)}
    sentinel = {k: torch.full_like(v, 7.0) for k, v in host_out.items() if k != "x2"}
    pipe.run(host_in, {**only, **{k: None for k in sentinel}}, host_mod)
    torch.cuda.synchronize()
    assert torch.equal(only["x2"], bufs.x2.cpu())
    assert pipe.bytes_per_pass(n, outputs=("x2",))[1] == only["x2"].numel() * only["x2"].element_size()
    assert all(torch.all(v == 7.0) for v in sentinel.values())
    pipe.close()
    bufs.close()


def test_host_pass_validation():
    w = CASES[0]
    n = 40
    host_in, host_out, host_mod = pipeline.host_buffers(w, n)
    pipe = pipeline.HostBlockPipeline(w, "cuda", chunk_tokens=16, n_slots=2)
    d = pipe.desc(host_in, host_out, host_mod)
    need = sol.dit_block_host_workspace_bytes(d, 16, 2)
    assert need > 0
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with pytest.raises(sol.SolError) as e:
        sol.dit_block_host(d, ws, chunk_tokens=16, n_slots=2, s_in=s1, s_comp=s1, s_out=s2)
    assert "distinct" in str(e.value)
    with pytest.raises(sol.SolError) as e:
        sol.dit_block_host(d, ws[:need - 256], chunk_tokens=16, n_slots=2, s_in=s1, s_comp=s2,
                           s_out=torch.cuda.Stream())
    assert "workspace" in str(e.value)
    bad = pipe.desc(host_in, host_out, host_mod)
    bad.head_dim = 96  # the epilogue's own check rejects it before anything is enqueued
    with pytest.raises(sol.SolError):
        sol.dit_block_host(bad, ws, chunk_tokens=16, n_slots=2, s_in=s1, s_comp=s2, s_out=torch.cuda.Stream())
    torch.cuda.synchronize()
    pipe.close()


def test_chunks_never_cross_samples():
    w = CASES[1]
    pipe = pipeline.HostBlockPipeline.__new__(pipeline.HostBlockPipeline)
    pipe.w, pipe.chunk = w, 17
    ch = pipe.chunks(w.n_tokens)
    assert sum(L for _, L, _ in ch) == w.n_tokens
    for c0, L, b in ch:
        assert c0 // w.tokens_per_sample == b == (c0 + L - 1) // w.tokens_per_sample


@pytest.mark.parametrize("w", CASES[:2], ids=lambda w: w.name)
def test_graph_replay_equals_eager_passes(w):
    """BlockBuffers.capture: a captured pass replayed is bit-identical to the same passes
    issued eagerly (capture runs one eager pass first, so both sides run two)."""
    n = min(w.n_tokens, 3000)
    eager = block.BlockBuffers.allocate(w, "cuda", n_tokens=n)
    graph = block.BlockBuffers.allocate(w, "cuda", inputs={k: v.clone() if torch.is_tensor(v) else v
                                                           for k, v in eager.inp.items()})
    eager.step()
    eager.step()
    g = graph.capture(steps=1)
    g.replay()
    torch.cuda.synchronize()
    for name in ("h1", "x1", "h2", "act", "x2"):
        assert torch.equal(getattr(eager, name), getattr(graph, name)), name
    assert torch.equal(eager.inp["qkv"], graph.inp["qkv"])
    del g
    eager.close()
    graph.close()
