"""sgqa_sparse_attn_noalloc: decode attention without a caller workspace.

Some callers cannot allocate device memory when they call (a host runtime
that fixed its device memory at start-up, a plugin reached through a plain C
interface with no allocator handle).  This entry point serves them from a
static scratch array inside the library; its output must match
sgqa_sparse_attn, which takes a workspace, on the same inputs -- including on
a second call, after the first has left its partials in the shared array.

The file is named so that pytest collects it last.
"""
import dataclasses

import numpy as np
import pytest
import torch

from sparse_long_context_sgqa_b200 import inputs as I
from tests import _harness as Hn

pytestmark = pytest.mark.gpu


def _case(wl, device, q_pos0, nq, num_seqs, seed):
    cache, _ = Hn.make_inputs(wl, device, seqs=range(num_seqs))
    qs = [I.make_queries(wl, device, q_pos0, nq, seq=s) for s in range(num_seqs)]
    q = torch.stack([x["q"] for x in qs]).to(torch.bfloat16).contiguous()
    sel, cnt = I.make_selection(wl, device, q_pos0, nq, num_seqs=num_seqs, seed=seed)
    return cache, q, sel, cnt


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    from sparse_long_context_sgqa_b200 import binding as Bd
    base = dataclasses.replace(I.WORKLOADS["prefill8k"], name="noalloc")
    calls = [
        (dataclasses.replace(base, seq_len=20000, seed=11), 19995, 5, 3),
        (dataclasses.replace(base, seq_len=9000, seed=12), 8990, 10, 2),
    ]
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


def test_noalloc_rejects_calls_beyond_its_scratch(cuda_device):
    from sparse_long_context_sgqa_b200 import binding as Bd
    wl = dataclasses.replace(I.WORKLOADS["prefill8k"], seq_len=64, name="big")
    p = Hn.params_for(wl)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    idx = torch.zeros(16, dtype=torch.int32, device=cuda_device)
    with pytest.raises(Bd.SgqaError) as e:  # more queries than the decode path takes
        Bd.sgqa_sparse_attn_noalloc(p, 1, 0, 64, dummy, 64, 64, dummy, dummy, idx, idx, dummy)
    assert e.value.code == 2
    with pytest.raises(Bd.SgqaError) as e:  # split partials larger than the static array
        Bd.sgqa_sparse_attn_noalloc(p, 4096, 0, 8, dummy, 64, 64, dummy, dummy, idx, idx, dummy)
    assert e.value.code == 2
