"""The token-sharded pass (dit_block_b200.shard.ShardBuffers) on the GPU: the ranks'
ranges, run one after another on one device (each rank's launches are independent; no
rank waits on another), reproduce the single-rank pass (block.BlockBuffers) bit for bit
-- every operator is a per-token function of its row, its sample's modulation rows and
its global position, whichever call the row is in."""
from __future__ import annotations

import dataclasses

import pytest
import torch

from dit_block_b200 import block, shard, sol, workloads as wl

pytestmark = pytest.mark.gpu

BASE = dataclasses.replace(wl.WORKLOADS["lowres"], d=1024, n_heads=8, inner=1024)
PACKED = dataclasses.replace(BASE, name="shard_gpu_packed", index=42, batch=3, grid=(4, 6, 7), audio_per_sample=13)
VIDEO = dataclasses.replace(BASE, name="shard_gpu_video", index=43, batch=1, grid=(5, 8, 9), outlier_frac=1e-3)


def _same(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


@pytest.mark.parametrize("w", [PACKED, VIDEO], ids=lambda w: w.name)
@pytest.mark.parametrize("world", [2, 3, 5])
def test_shards_reproduce_the_single_rank_pass(w, world):
    sol.lib()
    inp = wl.block_inputs(w, "cuda")
    qkv0 = inp["qkv"].clone()
    full = block.BlockBuffers.allocate(w, "cuda", inputs={**inp, "qkv": qkv0.clone()})
    full.step()
    torch.cuda.synchronize()
    hd = w.hd
    n = w.n_tokens
    for t0, t1 in shard.token_ranges(n, world):
        mine = {k: inp[k][t0:t1].clone() for k in ("x", "y_attn", "u", "y_mlp")}
        mine["qkv"] = qkv0[t0:t1].clone()
        mine.update({k: inp[k] for k in ("wq", "wk", *shard.MOD_NAMES)})
        mine["pos"] = shard.positions(w, t0, t1).cuda()
        sid = shard.stream_ids(w, t0, t1)
        mine["stream_id"] = None if sid is None else sid.cuda()
        part = shard.ShardBuffers(w, t0, t1, "cuda", inputs=mine)
        part.step()
        torch.cuda.synchronize()
        for name in ("h1", "x1", "h2", "act", "x2"):
            assert _same(getattr(part, name), getattr(full, name)[t0:t1]), f"{name}[{t0}:{t1}] of {world} ranks"
        assert _same(part.inp["qkv"][:, :2 * hd], full.inp["qkv"][t0:t1, :2 * hd]), f"q|k[{t0}:{t1}]"
        assert _same(part.inp["qkv"][:, 2 * hd:], qkv0[t0:t1, 2 * hd:]), "v must be untouched"
        part.close()
    full.close()
    assert sol.device_errors() == 0
