"""Seeded synthetic inputs for the Sparse GQA hot path.

This module holds only input generation: random draws, the pre-boundary
transforms that the model applies before the sparse core (RMS/Layer
normalisation and rotary embedding), and the planted structure described
below.  It holds none of the method's own arithmetic (merge, score, selection,
attention).  The tests, the oracle checks and the benchmark all draw their
inputs from here.

Workloads (shapes follow the page "Step-5-Preview: Sparse Reads Are Not a
Compressed KV Cache", section "Two paths leave the same hidden state": Q
[N, 64, 192], K/V [N, 4, 192]; indexer with a 64-dim proxy space and a 32-dim
rotary span; block 8, top-512 blocks):

* ``tiny``        N=256, one KV group (16 heads), 4 indexer heads, top-8,
                  plain fp32 N(0,1) draws, seed 0.
* ``prefill8k``   N=8192 single chunk, seed 1.
* ``prefill128k`` N=131072 in 8192-query chunks, seed 2.
* ``decode``      16 sequences x 262144 cached tokens, one query each, seed 3.
* ``prefill1m``   N=1048576 in 8192-query chunks, seed 4 (B=8, top-512);
  ``prefill1m_b1`` the same with B=1, top-2048 tokens.
* ``prefill128k_indep`` the 128K workload with independent queries (no shared
  segment direction): a stress case for the 8-query grouping, whose adjacent
  queries then overlap only through the keys' topics.

Planted structure (all but ``tiny``):

* keys: a bank of 256 topic vectors per space (64-dim proxy space, 192-dim K
  space); block r draws a topic z_r and every token of the block adds
  0.5 * bank[z_r] to its proxy key and to its K (all groups);
* queries: tokens of one 64-token segment share a per-(segment, group, head)
  indexer query direction u and head weight; each token adds its own noise
  (0.3 * N(0,1)).  Adjacent queries therefore select overlapping blocks, the
  property the second page reports for real queries.

Transforms: K and Q are RMS-normalised per head vector then get neox-style
rotary (base 10000) on their first 64 dims; V is RMS-normalised; indexer
queries are RMS-normalised, proxy keys layer-normalised (no affine), both with
rotary on their first 32 dims; compression logits are N(0,1); head weights
fp32.  Everything else is BF16.
"""
from __future__ import annotations

import dataclasses
import hashlib

import torch

N_TOPICS = 256
TOPIC_SCALE = 0.5
QUERY_SEGMENT = 64
QUERY_NOISE = 0.3


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seq_len: int            # tokens of context per sequence (cache length)
    num_seqs: int = 1
    q_start: int = 0        # position of the first query
    n_queries: int = 0      # queries per sequence (0 -> seq_len - q_start)
    chunk: int = 8192       # queries per call
    groups: int = 4
    heads_per_group: int = 16
    head_dim: int = 192
    idx_heads: int = 8
    idx_dim: int = 64
    block: int = 8
    topk: int = 512
    seed: int = 0
    fp32_inputs: bool = False   # tiny: every input drawn as fp32 N(0,1)
    structured: bool = True     # planted topics / query segments / norms / rotary
    query_overlap: bool = True  # queries of a 64-token segment share a direction (structured only)

    @property
    def nq(self) -> int:
        return self.n_queries or (self.seq_len - self.q_start)

    @property
    def n_heads(self) -> int:
        return self.groups * self.heads_per_group


WORKLOADS = {
    "tiny": Workload("tiny", 256, chunk=256, groups=1, idx_heads=4, topk=8, seed=0,
                     fp32_inputs=True, structured=False),
    "prefill8k": Workload("prefill8k", 8192, seed=1),
    "prefill128k": Workload("prefill128k", 131072, seed=2),
    "decode": Workload("decode", 262144, num_seqs=16, q_start=262143, n_queries=1, chunk=1, seed=3),
    "prefill1m": Workload("prefill1m", 1048576, seed=4),
    "prefill1m_b1": Workload("prefill1m_b1", 1048576, block=1, topk=2048, seed=4),
    "prefill128k_indep": Workload("prefill128k_indep", 131072, seed=2, query_overlap=False),
}


def _seed(*parts) -> int:
    h = hashlib.sha256(("/".join(str(p) for p in parts)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _randn(shape, device, *tag) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*tag))
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _randint(high, shape, device, *tag) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*tag))
    return torch.randint(0, high, shape, generator=g, device=device)


def _rms(x: torch.Tensor) -> torch.Tensor:
    return x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True))


def _layernorm(x: torch.Tensor) -> torch.Tensor:
    x = x - x.mean(-1, keepdim=True)
    return x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + 1e-6)


def _rotary(x: torch.Tensor, pos: torch.Tensor, span: int, base: float = 10000.0) -> torch.Tensor:
    """neox-style rotary on the first ``span`` dims; pos has x's leading dim."""
    half = span // 2
    inv = base ** (-torch.arange(half, device=x.device, dtype=torch.float64) * 2.0 / span)
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    shape = [ang.shape[0]] + [1] * (x.dim() - 2) + [half]
    cos = torch.cos(ang).to(torch.float32).reshape(shape)
    sin = torch.sin(ang).to(torch.float32).reshape(shape)
    x1, x2, rest = x[..., :half], x[..., half:span], x[..., span:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin, rest], dim=-1)


def _store_dtype(wl: Workload):
    return torch.float32 if wl.fp32_inputs else torch.bfloat16


def make_cache(wl: Workload, device, seq: int = 0, rows: int = 65536):
    """Per-sequence cache tensors: proxy keys and logits [L, Di]; K, V [L, G, D]."""
    L, G, D, Di = wl.seq_len, wl.groups, wl.head_dim, wl.idx_dim
    dt = _store_dtype(wl)
    kp = torch.empty((L, Di), dtype=dt, device=device)
    c = torch.empty((L, Di), dtype=dt, device=device)
    k = torch.empty((L, G, D), dtype=dt, device=device)
    v = torch.empty((L, G, D), dtype=dt, device=device)
    if wl.structured:
        pbank = _randn((N_TOPICS, Di), device, wl.seed, "pbank")
        kbank = _randn((N_TOPICS, D), device, wl.seed, "kbank")
        nblk = (L + wl.block - 1) // wl.block
        topic = _randint(N_TOPICS, (nblk,), device, wl.seed, "ztopic", seq)
    for r0 in range(0, L, rows):
        r1 = min(L, r0 + rows)
        n = r1 - r0
        tag = (wl.seed, seq, r0)
        kp_ = _randn((n, Di), device, *tag, "kp")
        c_ = _randn((n, Di), device, *tag, "c")
        k_ = _randn((n, G, D), device, *tag, "k")
        v_ = _randn((n, G, D), device, *tag, "v")
        if wl.structured:
            pos = torch.arange(r0, r1, device=device)
            z = topic[pos // wl.block]
            kp_ = _rotary(_layernorm(kp_ + TOPIC_SCALE * pbank[z]), pos, 32)
            k_ = _rotary(_rms(k_ + TOPIC_SCALE * kbank[z][:, None, :]), pos, 64)
            v_ = _rms(v_)
        kp[r0:r1] = kp_.to(dt)
        c[r0:r1] = c_.to(dt)
        k[r0:r1] = k_.to(dt)
        v[r0:r1] = v_.to(dt)
    return {"kp": kp, "c": c, "k": k, "v": v}


def make_queries(wl: Workload, device, pos0: int, n: int, seq: int = 0):
    """Query-side tensors for positions [pos0, pos0+n) of one sequence.

    q [n, G*Hg, D]; idx_q [n, G, H, Di]; idx_w [n, G, H] (fp32).  Rows are drawn
    per 64-token segment from (seed, sequence, segment), so any chunk of a
    sequence can be generated on its own and always gives the same values.
    """
    G, Hg, D, H, Di = wl.groups, wl.heads_per_group, wl.head_dim, wl.idx_heads, wl.idx_dim
    dt = _store_dtype(wl)
    seg0 = pos0 // QUERY_SEGMENT
    seg1 = (pos0 + n - 1) // QUERY_SEGMENT + 1
    q = torch.empty((n, G * Hg, D), dtype=dt, device=device)
    iq = torch.empty((n, G, H, Di), dtype=dt, device=device)
    iw = torch.empty((n, G, H), dtype=torch.float32, device=device)
    step = 128  # segments per draw
    for s0 in range(seg0, seg1, step):
        s1 = min(seg1, s0 + step)
        a = max(pos0, s0 * QUERY_SEGMENT)
        b = min(pos0 + n, s1 * QUERY_SEGMENT)
        m = (s1 - s0) * QUERY_SEGMENT
        tag = (wl.seed, seq, s0, "q")
        q_ = _randn((m, G * Hg, D), device, *tag, "main")
        iq_ = _randn((m, G, H, Di), device, *tag, "idx")
        iw_ = _randn((m, G, H), device, *tag, "w")
        if wl.structured:
            pos = torch.arange(s0 * QUERY_SEGMENT, s1 * QUERY_SEGMENT, device=device)
            if wl.query_overlap:
                u = _randn((s1 - s0, G, H, Di), device, *tag, "u")
                uw = _randn((s1 - s0, G, H), device, *tag, "uw")
                rep = torch.arange(m, device=device) // QUERY_SEGMENT
                iq_ = _rotary(_rms(u[rep] + QUERY_NOISE * iq_), pos, 32)
                iw_ = uw[rep] + QUERY_NOISE * iw_
            else:
                iq_ = _rotary(_rms(iq_), pos, 32)
            q_ = _rotary(_rms(q_), pos, 64)
        lo, hi = a - s0 * QUERY_SEGMENT, b - s0 * QUERY_SEGMENT
        q[a - pos0:b - pos0] = q_[lo:hi].to(dt)
        iq[a - pos0:b - pos0] = iq_[lo:hi].to(dt)
        iw[a - pos0:b - pos0] = iw_[lo:hi]
    return {"q": q, "idx_q": iq, "idx_w": iw}


def make_gate(wl: Workload, device, pos0: int, n: int, seq: int = 0) -> torch.Tensor:
    """Head-wise output-gate logits [n, G*Hg] (bf16) for positions [pos0, pos0+n):
    2 * N(0,1), so that the gate's sigmoid spans most of (0, 1)."""
    return (2.0 * _randn((n, wl.n_heads), device, wl.seed, seq, pos0, "gate")).to(torch.bfloat16)


def make_selection(wl: Workload, device, pos0: int, n: int, num_seqs: int = 1, seed: int = 0):
    """A random valid selection input (for exercising attention on its own).

    For query t and group g: min(k, floor(t/B)) distinct block ids < floor(t/B),
    ascending, padded with -1; counts [S, n, G].  Queries of one 64-token
    segment rank blocks by a shared random preference plus their own noise,
    so adjacent queries overlap as real selections do.
    """
    G, k, B = wl.groups, wl.topk, wl.block
    sel = torch.full((num_seqs, n, G, k), -1, dtype=torch.int32, device=device)
    cnt = torch.empty((num_seqs, n, G), dtype=torch.int32, device=device)
    tmax = pos0 + n - 1
    rmax = max(tmax // B, 1)
    for s in range(num_seqs):
        for r0 in range(0, n, 256):
            r1 = min(n, r0 + 256)
            t = torch.arange(pos0 + r0, pos0 + r1, device=device)
            ncand = t // B
            seg = t // QUERY_SEGMENT
            pref = _randn((int(seg.max() - seg.min()) + 1, G, rmax), device, wl.seed, seed, s, "selpref", r0)
            noise = _randn((r1 - r0, G, rmax), device, wl.seed, seed, s, "selnoise", r0)
            sc = pref[seg - seg.min()] + 0.5 * noise
            valid = torch.arange(rmax, device=device)[None, None, :] < ncand[:, None, None]
            sc = torch.where(valid, sc, torch.full_like(sc, -float("inf")))
            kk = min(k, rmax)
            top = torch.topk(sc, kk, dim=-1).indices
            take = torch.arange(kk, device=device)[None, None, :] < torch.clamp(ncand, max=k)[:, None, None]
            ids = torch.where(take, top, torch.full_like(top, 1 << 30))
            ids = torch.sort(ids, dim=-1).values
            ids = torch.where(ids == (1 << 30), torch.full_like(ids, -1), ids)
            sel[s, r0:r1, :, :kk] = ids.to(torch.int32)
            cnt[s, r0:r1] = torch.clamp(ncand, max=k).to(torch.int32)[:, None]
    return sel, cnt
