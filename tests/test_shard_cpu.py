"""The token-sharded split (dit_block_b200.shard) on CPU: the ranges, the pieces cut at
sample boundaries, the global positions and stream ids, and -- over two and four gloo ranks --
the fp64 oracle run on each rank's pieces reproducing the single-rank oracle over the
whole sequence bit for bit.  The split needs no collective on the data path; the test
gathers the ranks' results only to compare them."""
from __future__ import annotations

import dataclasses
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from dit_block_b200 import shard, workloads as wl  # noqa: E402

# small shapes of the two layouts: packed video+audio (3 samples, so that a two-way split
# falls inside a sample) and video only (one sample, split inside it)
PACKED = dataclasses.replace(wl.WORKLOADS["tiny"], name="shard_packed", index=40, batch=3, grid=(2, 3, 4),
                             audio_per_sample=5)
VIDEO = dataclasses.replace(wl.WORKLOADS["tiny"], name="shard_video", index=41, grid=(3, 4, 5))


def test_ranges_cover_every_token_once():
    for n in (0, 1, 7, 29, 252488):
        for world in (1, 2, 3, 8):
            r = shard.token_ranges(n, world)
            assert len(r) == world and r[0][0] == 0 and r[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [t1 - t0 for t0, t1 in r]
            assert max(sizes) - min(sizes) <= 1


def test_pieces_cut_at_sample_boundaries():
    w = PACKED
    tps = w.tokens_per_sample  # 29
    ps = shard.pieces(w, 20, 70)
    assert [(p.start, p.length, p.sample, p.offset) for p in ps] == [
        (20, 9, 0, 0), (29, 29, 1, 9), (58, 12, 2, 38)]
    assert sum(p.length for p in ps) == 50
    for p in ps:
        assert p.start // tps == p.sample == (p.start + p.length - 1) // tps
    assert shard.pieces(w, 29, 58) == [shard.Piece(29, 29, 1, 0)]
    assert shard.pieces(w, 5, 5) == []


def test_positions_and_stream_ids_match_the_layout():
    pos, sid = wl.token_layout(PACKED)
    n = PACKED.n_tokens
    for t0, t1 in ((0, n), (3, 40), (57, 60)):
        assert torch.equal(shard.positions(PACKED, t0, t1), pos[t0:t1])
        assert torch.equal(shard.stream_ids(PACKED, t0, t1), sid[t0:t1])
    # video only: the row-major grid of each sample
    T, H, W = VIDEO.grid
    tt, hh, ww = torch.meshgrid(torch.arange(T), torch.arange(H), torch.arange(W), indexing="ij")
    grid = torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], 1).to(torch.int32)
    assert torch.equal(shard.positions(VIDEO, 0, VIDEO.n_tokens), grid)
    assert shard.stream_ids(VIDEO, 0, 10) is None


def test_explicit_positions_only_where_the_implicit_grid_cannot_serve():
    assert not shard.needs_explicit_positions(VIDEO, shard.Piece(0, 10, 0, 0))
    assert shard.needs_explicit_positions(VIDEO, shard.Piece(7, 10, 0, 0))
    assert shard.needs_explicit_positions(PACKED, shard.Piece(0, 29, 0, 0))


def _bits(t):
    c = t.contiguous()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16).copy()
    return c.numpy().copy()


def _oracle_pass(o, w, a, pos, sid, n_streams, tps, rows=slice(None)):
    """The five operators of the pass on the oracle over a[rows]; sid / pos already sliced."""
    sel = dict(stream_id=sid, n_streams=n_streams, tokens_per_sample=tps)
    x, qkv, ya, u, ym = (np.ascontiguousarray(a[k][rows]) for k in ("x", "qkv", "y_attn", "u", "y_mlp"))
    grid = w.grid
    out = {
        "h1": o.adaln_modulate(x, a["shift_msa"], a["scale_msa"], eps=w.eps, **sel),
        "qk": o.dit_epilogue(qkv, a["wq"], a["wk"], n_heads=w.n_heads, head_dim=w.head_dim, pos=pos, grid=grid,
                             tokens_per_sample=tps, dims=w.rope_dims, theta=w.theta, eps=w.eps),
        "act": o.swiglu(u, w.inner),
        "x2": o.gated_residual(x, ym, a["gate_mlp"], **sel),
    }
    out["x1"], out["h2"] = o.dit_prologue(x, ya, a["gate_msa"], a["shift_mlp"], a["scale_mlp"], eps=w.eps, **sel)
    return out


def _shard_oracle(o, w, a, t0, t1):
    """One rank's part, piece by piece, with the arguments shard.ShardBuffers gives each
    call (shard.piece_call): the sample's modulation rows, tokens_per_sample 0, and the
    stream ids and positions of the rank's range sliced to the piece."""
    sid_r = shard.stream_ids(w, t0, t1)
    pos_r = shard.positions(w, t0, t1).numpy()
    mine = {k: v[t0:t1] for k, v in a.items() if k in ("x", "qkv", "y_attn", "u", "y_mlp")}
    parts = []
    for p in shard.pieces(w, t0, t1):
        c = shard.piece_call(w, p)
        mod = {k: a[k][c.mod_rows] for k in shard.MOD_NAMES}
        sid = None if sid_r is None else sid_r[c.rows].numpy()
        pos = pos_r[c.rows] if c.explicit_pos else None
        parts.append(_oracle_pass(o, w, {**a, **mine, **mod}, pos, sid, w.n_streams, 0, c.rows))
    if not parts:
        return {}
    return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}


def _inputs(w):
    inp = wl.block_inputs(w, "cpu")
    return {k: _bits(v) for k, v in inp.items() if isinstance(v, torch.Tensor) and k not in ("pos", "stream_id")}


def _worker(rank, world, port, q):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    res = {}
    for w in (PACKED, VIDEO):
        a = _inputs(w)
        t0, t1 = shard.token_ranges(w.n_tokens, world)[rank]
        mine = _shard_oracle(oracle, w, a, t0, t1)
        gathered = [None] * world
        dist.all_gather_object(gathered, ((t0, t1), mine))
        res[w.name] = gathered
    q.put((rank, res))
    dist.destroy_process_group()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("world", [2, 4])
def test_ranks_reproduce_the_single_rank_oracle(world):
    """Two ranks cut both layouts inside a sample; four ranks also give one rank the end of
    one sample and the start of the next."""
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = [q.get(timeout=300) for _ in ps]
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for w in (PACKED, VIDEO):
        a = _inputs(w)
        pos, sid = wl.token_layout(w)
        whole = _oracle_pass(oracle, w, a, None if pos is None else pos.numpy(),
                             None if sid is None else sid.numpy(), w.n_streams,
                             w.tokens_per_sample if w.batch > 1 else 0)
        for rank, got in res:
            gathered = got[w.name]
            covered = np.zeros(w.n_tokens, np.int64)
            for (t0, t1), part in gathered:
                covered[t0:t1] += 1
                for k, v in part.items():
                    assert np.array_equal(v, whole[k][t0:t1]), f"{w.name} rank {rank}: {k}[{t0}:{t1}]"
            assert np.all(covered == 1), f"{w.name}: tokens not covered exactly once"
        # the first cut falls inside a sample for both layouts
        assert shard.token_ranges(w.n_tokens, world)[0][1] % w.tokens_per_sample != 0
    if world == 4:  # a rank whose range spans a sample boundary
        assert any(len(shard.pieces(PACKED, t0, t1)) > 1 for t0, t1 in shard.token_ranges(PACKED.n_tokens, 4))
