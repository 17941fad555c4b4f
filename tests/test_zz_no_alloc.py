"""sgqa_sparse_attn_noalloc: decode attention without a caller workspace.

Some callers cannot allocate device memory when they call (a host runtime
that fixed its device memory at start-up, a plugin reached through a plain C
interface with no allocator handle).  This entry point serves them from a
static scratch array inside the library.  Block sizes 1, 2 and 4 keep their
split-K partials in that array; block size 8 combines its splits on chip and
uses none of it.  Each call's output must match sgqa_sparse_attn, which takes
a workspace, on the same inputs -- including on later calls of other shapes,
after an earlier call has left its partials in the shared array -- and the
oracle on sampled rows.

The file is named so that pytest collects it last.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import sgqa_oracle as O
from sparse_long_context_sgqa_b200 import inputs as I
from tests import _harness as Hn

pytestmark = pytest.mark.gpu


def _case(wl, device, q_pos0, nq, num_seqs, seed):
    cache, _ = Hn.make_inputs(wl, device, seqs=range(num_seqs))
    qs = [I.make_queries(wl, device, q_pos0, nq, seq=s) for s in range(num_seqs)]
    q = torch.stack([x["q"] for x in qs]).to(torch.bfloat16).contiguous()
    sel, cnt = I.make_selection(wl, device, q_pos0, nq, num_seqs=num_seqs, seed=seed)
    return cache, q, sel, cnt


def _oracle_rows(wl, cache, q, sel, cnt, got, q_pos0, picks):
    worst = 0.0
    for s, i, g in picks:
        t = q_pos0 + i
        ids = sel[s, i, g, :cnt[s, i, g]].cpu().numpy()
        pos = O.attended_positions(t, ids, wl.block)
        hs = slice(g * wl.heads_per_group, (g + 1) * wl.heads_per_group)
        ref = O.sparse_attention(Hn.to_np(q[s, i, hs]), Hn.to_np(cache["k"][s, pos, g]),
                                 Hn.to_np(cache["v"][s, pos, g]), Hn.scale_of(wl))
        worst = max(worst, float(np.abs(got[s, i, hs].float().cpu().numpy() - ref).max()))
    return worst


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row(cuda_device):
    from sparse_long_context_sgqa_b200 import binding as Bd
    base = dataclasses.replace(I.WORKLOADS["prefill8k"], name="noalloc")
    # (workload, q_pos0, nq, num_seqs): block sizes 2, 1 and 4 use the static
    # array (each call after the first finds the previous call's partials
    # there); block size 8 does not, at a size whose partials would not fit it
    calls = [
        (dataclasses.replace(base, seq_len=20000, block=2, topk=100, seed=11), 19995, 5, 3),
        (dataclasses.replace(base, seq_len=9000, block=1, topk=256, seed=12), 8990, 10, 2),
        (dataclasses.replace(base, seq_len=12000, block=4, topk=64, seed=13), 11968, 32, 2),
        (dataclasses.replace(base, seq_len=20000, block=2, topk=100, seed=11), 19995, 5, 3),
        (dataclasses.replace(base, seq_len=4096, block=8, topk=512, seed=14), 4088, 8, 64),
    ]
    rng = np.random.default_rng(5)
    for n_call, (wl, q0, nq, S) in enumerate(calls):
        cache, q, sel, cnt = _case(wl, cuda_device, q0, nq, S, seed=n_call)
        p = Hn.params_for(wl)
        L = wl.seq_len
        ref = torch.zeros((S, nq, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=cuda_device)
        ws = Bd.alloc_workspace(p, S, nq, q0 + nq, cuda_device)
        Bd.sgqa_sparse_attn(p, S, q0, nq, q, L, L, cache["k"], cache["v"], sel, cnt, ref, ws)
        got = torch.full_like(ref, float("nan"))
        Bd.sgqa_sparse_attn_noalloc(p, S, q0, nq, q, L, L, cache["k"], cache["v"], sel, cnt, got)
        Bd.sgqa_check()
        diff = (got.float() - ref.float()).abs().max().item()
        assert np.isfinite(diff) and diff <= Hn.ATTN_ATOL, (n_call, diff)
        picks = {(0, 0, 0), (S - 1, nq - 1, wl.groups - 1)}
        picks.update((int(rng.integers(S)), int(rng.integers(nq)), int(rng.integers(wl.groups))) for _ in range(6))
        worst = _oracle_rows(wl, cache, q, sel, cnt, got, q0, sorted(picks))
        assert worst <= Hn.ATTN_ATOL, (n_call, worst)


def test_noalloc_rejects_calls_beyond_its_scratch(cuda_device):
    from sparse_long_context_sgqa_b200 import binding as Bd
    dummy = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    idx = torch.zeros(16, dtype=torch.int32, device=cuda_device)
    wl = dataclasses.replace(I.WORKLOADS["prefill8k"], seq_len=64, name="big")
    with pytest.raises(Bd.SgqaError) as e:  # more queries than the decode path takes
        Bd.sgqa_sparse_attn_noalloc(Hn.params_for(wl), 1, 0, 64, dummy, 64, 64, dummy, dummy, idx, idx, dummy)
    assert e.value.code == 2
    # block size 2: split partials of 4096 x 8 x 4 rows are larger than the static array
    p = Hn.params_for(dataclasses.replace(wl, block=2, topk=16))
    with pytest.raises(Bd.SgqaError) as e:
        Bd.sgqa_sparse_attn_noalloc(p, 4096, 0, 8, dummy, 64, 64, dummy, dummy, idx, idx, dummy)
    assert e.value.code == 2
