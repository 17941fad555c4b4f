"""Host logic of SparseGQA.prefill on CPU, with the library calls replaced by a
stand-in that checks what each call receives: chunks of a batch of several
sequences must reach the C ABI as contiguous tensors holding exactly that
chunk, and the outputs must land back in place."""
import torch

from sparse_long_context_sgqa_b200 import api
from sparse_long_context_sgqa_b200.binding import Params


def _fake_forward(calls):
    def run(p, S, q_pos0, nq, q, idx_q, idx_w, cap, clen, kp, c, k, v, merged, store, sel, cnt, *rest):
        gate, out = (rest[0], rest[1]) if len(rest) == 4 else (None, rest[0])
        for t in (q, idx_q, idx_w, sel, cnt, out) + ((gate,) if gate is not None else ()):
            assert t.is_contiguous()
        assert q.shape[:2] == (S, nq) and sel.shape[:2] == (S, nq) and out.shape[:2] == (S, nq)
        calls.append((q_pos0, nq, q.clone(), None if gate is None else gate.clone()))
        # a recognisable result: the query plus its position, per head
        out.copy_(q + q_pos0)
        sel.fill_(q_pos0)
        cnt.fill_(nq)
    return run


def test_prefill_chunks_of_a_batch_are_contiguous_and_land_in_place(monkeypatch):
    calls = []
    monkeypatch.setattr(api.Bd, "sgqa_forward", _fake_forward(calls))
    monkeypatch.setattr(api.Bd, "sgqa_forward_gated", _fake_forward(calls))
    p = Params(num_kv_groups=1, topk=4)
    S, N, chunk = 2, 10, 4  # chunks of 4, 4 and 2 queries
    model = api.SparseGQA(p, S, 64, chunk, "cpu")
    q = torch.arange(S * N * 16 * 3, dtype=torch.float32).view(S, N, 16, 3)
    idx_q = torch.zeros((S, N, 1, 8, 64))
    idx_w = torch.zeros((S, N, 1, 8))
    gate = torch.arange(S * N * 16, dtype=torch.float32).view(S, N, 16)
    out = torch.zeros_like(q)
    sel = torch.full((S, N, 1, 4), -1, dtype=torch.int32)
    cnt = torch.zeros((S, N, 1), dtype=torch.int32)
    model.prefill(q, idx_q, idx_w, out, sel, cnt, q_pos0=100, gate=gate)
    assert [(c[0], c[1]) for c in calls] == [(100, 4), (104, 4), (108, 2)]
    for (pos, n, qc, gc), c0 in zip(calls, (0, 4, 8)):
        assert torch.equal(qc, q[:, c0:c0 + n]) and torch.equal(gc, gate[:, c0:c0 + n])
        assert torch.equal(out[:, c0:c0 + n], q[:, c0:c0 + n] + pos)
        assert (sel[:, c0:c0 + n] == pos).all() and (cnt[:, c0:c0 + n] == n).all()
