"""Test harness: run the CUDA path through the C ABI and the CPU oracle side by side.

Test infrastructure only.  Inputs come from ``sparse_long_context_sgqa_b200.inputs``
(shared by both sides); the oracle receives host copies of those inputs and
never any output of the CUDA path.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

from oracle import sgqa_oracle as O
from sparse_long_context_sgqa_b200 import inputs as I

MERGE_RTOL = 1e-3        # merged keys, fp32 vs exact
MERGE_ATOL = 1e-6        # absolute floor for values near zero
TIE_RTOL = 1e-5          # selection differences allowed only between near-equal scores
ATTN_ATOL = 2e-2         # max-abs on unit-scale bf16 outputs


def params_for(wl: I.Workload):
    from sparse_long_context_sgqa_b200.binding import Params
    return Params(num_kv_groups=wl.groups, heads_per_group=wl.heads_per_group, head_dim=wl.head_dim,
                  idx_heads=wl.idx_heads, idx_dim=wl.idx_dim, block_size=wl.block, topk=wl.topk,
                  merge_in_f32=1 if wl.fp32_inputs else 0)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


@dataclasses.dataclass
class Run:
    wl: I.Workload
    cache: dict            # device tensors, per-sequence stacked [S, L, ...]
    queries: dict          # device tensors [S, nq, ...] for positions q_start..
    store: torch.Tensor    # [S, L/B, Di] uint8 (GPU)
    merged: torch.Tensor   # [S, L/B, Di] fp32 (GPU)
    sel: torch.Tensor      # [S, nq, G, k]
    cnt: torch.Tensor      # [S, nq, G]
    out: torch.Tensor      # [S, nq, 64, 192]


def make_inputs(wl: I.Workload, device, seqs=None):
    seqs = range(wl.num_seqs) if seqs is None else seqs
    caches = [I.make_cache(wl, device, seq=s) for s in seqs]
    qs = [I.make_queries(wl, device, wl.q_start, wl.nq, seq=s) for s in seqs]
    cache = {k: torch.stack([c[k] for c in caches]) for k in caches[0]}
    queries = {k: torch.stack([q[k] for q in qs]) for k in qs[0]}
    if wl.fp32_inputs:  # the attention and indexer kernels take BF16 operands
        for k in ("k", "v"):
            cache[k] = bf16(cache[k])
        for k in ("q", "idx_q"):
            queries[k] = bf16(queries[k])
    return cache, queries


def run_forward(wl: I.Workload, device, cache=None, queries=None, premerge=True) -> Run:
    """The CUDA path as bench.py drives it: chunked sgqa_forward calls."""
    from sparse_long_context_sgqa_b200 import binding as Bd
    if cache is None:
        cache, queries = make_inputs(wl, device)
    p = params_for(wl)
    S, L, B = cache["kp"].shape[0], wl.seq_len, wl.block
    nblk = L // B
    store = torch.zeros((S, nblk, wl.idx_dim), dtype=torch.uint8, device=device)
    merged = torch.zeros((S, nblk, wl.idx_dim), dtype=torch.float32, device=device)
    nq = wl.nq
    sel = torch.full((S, nq, wl.groups, wl.topk), -7, dtype=torch.int32, device=device)
    cnt = torch.full((S, nq, wl.groups), -7, dtype=torch.int32, device=device)
    out = torch.zeros((S, nq, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=device)
    if premerge and wl.q_start // B > 0:
        Bd.sgqa_merge_blocks(p, S, L, cache["kp"], cache["c"], 0, wl.q_start // B, merged, store)
    chunk = min(wl.chunk, nq)
    ws = Bd.alloc_workspace(p, S, chunk, wl.q_start + nq, device)
    for c0 in range(0, nq, chunk):
        n = min(chunk, nq - c0)
        sl = slice(c0, c0 + n)
        sel_c = torch.empty((S, n, wl.groups, wl.topk), dtype=torch.int32, device=device)
        cnt_c = torch.empty((S, n, wl.groups), dtype=torch.int32, device=device)
        out_c = torch.empty((S, n, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=device)
        Bd.sgqa_forward(p, S, wl.q_start + c0, n,
                        queries["q"][:, sl].contiguous(), queries["idx_q"][:, sl].contiguous(),
                        queries["idx_w"][:, sl].contiguous(), L, L, cache["kp"], cache["c"],
                        cache["k"], cache["v"], merged, store, sel_c, cnt_c, out_c, ws)
        sel[:, sl] = sel_c
        cnt[:, sl] = cnt_c
        out[:, sl] = out_c
    Bd.sgqa_check()
    return Run(wl, cache, queries, store, merged, sel, cnt, out)


# ---------------------------------------------------------------------------
# comparisons
# ---------------------------------------------------------------------------

def store_mismatch_ok(gpu_codes: np.ndarray, merged_exact: np.ndarray, kp: np.ndarray = None,
                      block: int = None) -> np.ndarray:
    """Boolean mask of GPU store codes that are explained by FP32 rounding.

    Both sides decide the code in the same precision (the merged value in
    FP32, then BF16, then E4M3), but the GPU's FP32 value carries the rounding
    error of its merge arithmetic (B exponentials, B multiply-adds, a sum and
    a division).  A code may differ from the oracle's only where the exact
    merged value lies within that error of a rounding boundary: within
    1e-6 relative, plus (given the block's proxy keys kp) 16 FP32 ulps of the
    block's largest proxy-key magnitude in that coordinate, the absolute error
    a weighted sum of B terms of at most that size can carry (it dominates
    where the terms cancel and the merged value is near zero).
    """
    delta = 1e-6 * np.abs(merged_exact)
    if kp is not None:
        nb = merged_exact.shape[0]
        absmax = np.abs(kp[:nb * block].reshape(nb, block, -1)).max(axis=1)
        delta = delta + 2.0 ** -20 * absmax
    ok = O.store_codes(merged_exact) == gpu_codes
    ok |= O.store_codes(merged_exact - delta) == gpu_codes
    ok |= O.store_codes(merged_exact + delta) == gpu_codes
    return ok


def oracle_keys(kp_np, c_np, block):
    merged = O.merge_blocks(kp_np, c_np, block)
    codes = O.store_codes(merged)
    return merged, codes, O.e4m3_decode(codes)


def check_selection(gpu_ids, scores, k):
    """Compare a GPU selection with the oracle's scores; returns number of tie swaps."""
    n = scores.shape[0]
    ref = O.select_topk(scores, k)
    gpu_ids = np.asarray(gpu_ids, dtype=np.int64)
    assert len(gpu_ids) == len(ref) == min(k, n), (len(gpu_ids), len(ref), n)
    assert np.all(np.diff(gpu_ids) > 0), "selection must be strictly ascending"
    assert len(gpu_ids) == 0 or (gpu_ids[0] >= 0 and gpu_ids[-1] < n)
    if np.array_equal(gpu_ids, ref):
        return 0
    order = np.lexsort((np.arange(n), -scores))
    theta = scores[order[k - 1]]
    diff = np.setxor1d(gpu_ids, ref)
    for r in diff:
        tol = TIE_RTOL * max(abs(scores[r]), abs(theta), 1e-30)
        assert abs(scores[r] - theta) <= tol, f"block {r}: score {scores[r]!r} vs k-th {theta!r}"
    return len(diff) // 2


def sample_rows(wl: I.Workload, n_rows: int, seed: int = 0):
    """Query indices (within the call's queries) to check: edges plus a random spread."""
    nq = wl.nq
    rng = np.random.default_rng(seed)
    pick = {0, nq - 1, nq // 2}
    for t in (1, 5, 7, 8, 9, 15, 16, 63, 64, 4095, 4096, 4097, 4103, 4104):
        i = t - wl.q_start
        if 0 <= i < nq:
            pick.add(i)
    extra = rng.choice(nq, size=min(nq, max(0, n_rows - len(pick))), replace=False)
    pick.update(int(x) for x in extra)
    return sorted(pick)


def scale_of(wl):
    return 1.0 / math.sqrt(wl.head_dim)
