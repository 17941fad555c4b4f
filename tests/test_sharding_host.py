"""KV-group sharding host logic on CPU (gloo ranks, world sizes 2 and 4).

Each rank holds KV groups [r G / W, (r + 1) G / W): its K/V slice, its query
heads and indexer tensors.  A stand-in for the library computes, per local
head h, a value that depends on the head's query row, its group's K/V and
indexer weight, so a wrong slice or a misplaced head after the all-gather of
the outputs shows up.  The gathered output must equal the same stand-in run on
the full, unsharded tensors.
"""
import dataclasses
import datetime
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed=0, S=2, N=5, L=40, G=4, Hg=3, D=6, H=2, Di=4):
    import torch
    g = torch.Generator().manual_seed(seed)
    t = lambda *shape: torch.randn(*shape, generator=g)  # noqa: E731
    return dict(q=t(S, N, G * Hg, D), idx_q=t(S, N, G, H, Di), idx_w=t(S, N, G, H), kp=t(S, L, Di), c=t(S, L, Di),
                k=t(S, L, G, D), v=t(S, L, G, D))


class _StandIn:
    """The library's role on a rank: caches sized for its groups, and a
    forward whose output for local head h mixes the head's query, its group's
    K and V rows at the query position and its group's first indexer weight."""

    def __init__(self, p, S, L, D, Di):
        import torch
        G = p.num_kv_groups
        self.p = p
        self.kp = torch.zeros(S, L, Di)
        self.c = torch.zeros(S, L, Di)
        self.k = torch.zeros(S, L, G, D)
        self.v = torch.zeros(S, L, G, D)

    def forward(self, q_pos0, q, idx_q, idx_w, sel, sel_count, out, **kw):
        Hg = self.p.heads_per_group
        pos = q_pos0
        for h in range(q.shape[2]):
            g = h // Hg
            out[:, :, h] = q[:, :, h] * (1 + idx_w[:, :, g, :1]) + self.k[:, pos, g][:, None] - self.v[:, pos, g][:, None] \
                + idx_q[:, :, g, 0, :1] + self.kp[:, pos, :1][:, None]
        sel.fill_(0)
        sel_count.fill_(0)


def _expected(x, G, Hg, q_pos0=3):
    import torch
    out = torch.empty_like(x["q"])
    pos = q_pos0
    for h in range(G * Hg):
        g = h // Hg
        out[:, :, h] = x["q"][:, :, h] * (1 + x["idx_w"][:, :, g, :1]) + x["k"][:, pos, g][:, None] \
            - x["v"][:, pos, g][:, None] + x["idx_q"][:, :, g, 0, :1] + x["kp"][:, pos, :1][:, None]
    return out


def _rank_main(rank, world, port, out_q):
    import torch
    import torch.distributed as dist

    from sparse_long_context_sgqa_b200 import sharding as Sh
    from sparse_long_context_sgqa_b200.binding import Params

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = _inputs()
        S, L, G, D = x["k"].shape
        Di = x["kp"].shape[-1]
        p = Params(num_kv_groups=G, heads_per_group=3, head_dim=D, idx_heads=2, idx_dim=Di, topk=4)
        layer = Sh.GroupShardedSGQA(p, world, rank, lambda lp: _StandIn(lp, S, L, D, Di))
        layer.load_cache(x["kp"], x["c"], x["k"], x["v"])
        assert layer.local_params.num_kv_groups == G // world
        full = layer.forward(3, x["q"], x["idx_q"], x["idx_w"])
        local = layer.forward(3, x["q"], x["idx_q"], x["idx_w"], gather=False)
        out_q.put((rank, full, local, (layer.g0, layer.g1)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_group_sharded_forward_gathers_every_head_in_place(world):
    import torch
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out_q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = _inputs()
    G, Hg = 4, 3
    want = _expected(x, G, Hg)
    for rank, full, local, (g0, g1) in sorted(res, key=lambda r: r[0]):
        assert (g0, g1) == (rank * G // world, (rank + 1) * G // world)
        assert torch.allclose(full, want), rank
        assert torch.allclose(local, want[:, :, g0 * Hg:g1 * Hg]), rank


def test_group_range_rejects_uneven_splits():
    from sparse_long_context_sgqa_b200 import sharding as Sh
    assert Sh.group_range(4, 4, 3) == (3, 4)
    with pytest.raises(ValueError):
        Sh.group_range(4, 3, 0)
