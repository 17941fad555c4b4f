"""User-facing API: one object that owns the caches and workspace of a batch of
sequences and runs the hot path chunk by chunk through the C ABI.

``SparseGQA.forward`` (one call: a decode step or one chunk) and ``prefill``
(all chunks) take device tensors; ``forward_host`` takes pinned host tensors
and copies them in and the result out (the end-to-end path).  All arithmetic
runs in ``libsgqa.so``.
"""
from __future__ import annotations

import torch

from . import binding as Bd


class SparseGQA:
    def __init__(self, params: Bd.Params, num_seqs: int, capacity: int, chunk: int, device,
                 keep_merged_f32: bool = False):
        self.p = params
        self.S = num_seqs
        self.cap = capacity
        self.chunk = chunk
        self.device = torch.device(device)
        G, D, Di, B = params.num_kv_groups, params.head_dim, params.idx_dim, params.block_size
        in_dt = torch.float32 if params.merge_in_f32 else torch.bfloat16
        self.kp = torch.empty((num_seqs, capacity, Di), dtype=in_dt, device=device)
        self.c = torch.empty((num_seqs, capacity, Di), dtype=in_dt, device=device)
        self.k = torch.empty((num_seqs, capacity, G, D), dtype=torch.bfloat16, device=device)
        self.v = torch.empty((num_seqs, capacity, G, D), dtype=torch.bfloat16, device=device)
        self.store = torch.zeros((num_seqs, capacity // B, Di), dtype=torch.uint8, device=device)
        self.merged = (torch.zeros((num_seqs, capacity // B, Di), dtype=torch.float32, device=device)
                       if keep_merged_f32 else None)
        self.ws = Bd.alloc_workspace(params, num_seqs, chunk, capacity, device)

    def forward(self, q_pos0, q, idx_q, idx_w, sel, sel_count, out, cache_len=None, stream=None, gate=None):
        """One call of the hot path for queries [q_pos0, q_pos0 + nq) (nq <= chunk).

        Every tensor is contiguous with the layouts of include/sgqa.h; gate
        ([S, nq, G*Hg] bf16 logits) applies the head-wise sigmoid output gate.
        """
        nq = q.shape[1]
        clen = self.cap if cache_len is None else cache_len
        if gate is None:
            Bd.sgqa_forward(self.p, self.S, q_pos0, nq, q, idx_q, idx_w, self.cap, clen, self.kp, self.c, self.k,
                            self.v, self.merged, self.store, sel, sel_count, out, self.ws, stream)
        else:
            Bd.sgqa_forward_gated(self.p, self.S, q_pos0, nq, q, idx_q, idx_w, self.cap, clen, self.kp, self.c,
                                  self.k, self.v, self.merged, self.store, sel, sel_count, gate, out, self.ws, stream)

    def prefill(self, q, idx_q, idx_w, out, sel=None, sel_count=None, q_pos0=0, stream=None, gate=None):
        """Chunked prefill of all queries in q ([S, N, G*Hg, D]); caches already hold their K/V.

        A chunk of a batch of several sequences is not contiguous in q: it is
        copied into a contiguous tensor before the call.
        """
        S, N = q.shape[0], q.shape[1]
        G, k = self.p.num_kv_groups, self.p.topk
        if self.device.type != "cuda":  # host-side use (tests with a stand-in library)
            self._prefill_chunks(q, idx_q, idx_w, out, sel, sel_count, q_pos0, stream, gate, S, N, G, k)
            return
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        with torch.cuda.stream(st):  # the chunk copies run on the calls' stream
            self._prefill_chunks(q, idx_q, idx_w, out, sel, sel_count, q_pos0, st, gate, S, N, G, k)

    def _prefill_chunks(self, q, idx_q, idx_w, out, sel, sel_count, q_pos0, stream, gate, S, N, G, k):
        for c0 in range(0, N, self.chunk):
            n = min(self.chunk, N - c0)
            s_sel = sel[:, c0:c0 + n] if sel is not None and S == 1 else torch.empty(
                (S, n, G, k), dtype=torch.int32, device=self.device)
            s_cnt = sel_count[:, c0:c0 + n] if sel_count is not None and S == 1 else torch.empty(
                (S, n, G), dtype=torch.int32, device=self.device)
            o = out[:, c0:c0 + n] if S == 1 else torch.empty((S, n) + tuple(out.shape[2:]),
                                                             dtype=out.dtype, device=self.device)
            self.forward(q_pos0 + c0, q[:, c0:c0 + n].contiguous(), idx_q[:, c0:c0 + n].contiguous(),
                         idx_w[:, c0:c0 + n].contiguous(), s_sel, s_cnt, o, stream=stream,
                         gate=None if gate is None else gate[:, c0:c0 + n].contiguous())
            if S != 1:
                out[:, c0:c0 + n] = o
                if sel is not None:
                    sel[:, c0:c0 + n] = s_sel
                if sel_count is not None:
                    sel_count[:, c0:c0 + n] = s_cnt

    def forward_host(self, host: dict, out_host: torch.Tensor, stream=None):
        """End to end from pinned host memory: copy the inputs in, run, copy the output out.

        host holds pinned tensors with the cache layouts (kp, c, k, v) and the query
        layouts (q, idx_q, idx_w) of a full prefill; out_host receives [S, N, G*Hg, D].
        The copies are pipelined with the chunks: chunk c needs only the cache
        positions before its last query and its own queries, so while chunk c
        runs, chunk c+1's inputs are copied in on one stream and chunk c-1's
        output is copied out on another (the two PCIe directions run at once).
        Work is enqueued only; the given stream (default: the current one) waits
        for the last copy out.  Returns (bytes copied host->device, bytes copied
        device->host).
        """
        cur = torch.cuda.current_stream(self.device) if stream is None else stream
        if not hasattr(self, "_copy_streams"):
            self._copy_streams = (torch.cuda.Stream(device=self.device), torch.cuda.Stream(device=self.device))
        h2d_s, d2h_s = self._copy_streams
        S, N = host["q"].shape[0], host["q"].shape[1]
        G, k = self.p.num_kv_groups, self.p.topk
        with torch.cuda.stream(cur):  # the buffers belong to the calls' stream (and the two copy streams below)
            dq = {n: torch.empty(host[n].shape, dtype=host[n].dtype, device=self.device)
                  for n in ("q", "idx_q", "idx_w")}
            out = torch.empty(out_host.shape, dtype=out_host.dtype, device=self.device)
            sel = torch.empty((S, self.chunk, G, k), dtype=torch.int32, device=self.device)
            cnt = torch.empty((S, self.chunk, G), dtype=torch.int32, device=self.device)
        h2d_s.wait_stream(cur)
        d2h_s.wait_stream(cur)
        for c0 in range(0, N, self.chunk):
            n = min(self.chunk, N - c0)
            with torch.cuda.stream(h2d_s):
                for s in range(S):
                    for name in ("kp", "c", "k", "v"):
                        getattr(self, name)[s, c0:c0 + n].copy_(host[name][s, c0:c0 + n], non_blocking=True)
                    for name in ("q", "idx_q", "idx_w"):
                        dq[name][s, c0:c0 + n].copy_(host[name][s, c0:c0 + n], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(h2d_s)
            cur.wait_event(ready)
            with torch.cuda.stream(cur):  # the chunk's own copies run on the calls' stream
                o = out[:, c0:c0 + n] if S == 1 else torch.empty((S, n) + tuple(out.shape[2:]), dtype=out.dtype,
                                                                 device=self.device)
                if S == 1 or n == self.chunk:
                    c_sel, c_cnt = sel[:, :n], cnt[:, :n]
                else:  # a short last chunk of several sequences: contiguous scratch of its own
                    c_sel = torch.empty((S, n, G, k), dtype=torch.int32, device=self.device)
                    c_cnt = torch.empty((S, n, G), dtype=torch.int32, device=self.device)
                self.forward(c0, dq["q"][:, c0:c0 + n].contiguous(), dq["idx_q"][:, c0:c0 + n].contiguous(),
                             dq["idx_w"][:, c0:c0 + n].contiguous(), c_sel, c_cnt, o, stream=cur)
                if S != 1:
                    out[:, c0:c0 + n] = o
            done = torch.cuda.Event()
            done.record(cur)
            d2h_s.wait_event(done)
            with torch.cuda.stream(d2h_s):
                for s in range(S):
                    out_host[s, c0:c0 + n].copy_(out[s, c0:c0 + n], non_blocking=True)
        for t in list(dq.values()) + [out, sel, cnt]:
            t.record_stream(h2d_s)
            t.record_stream(d2h_s)
        cur.wait_stream(d2h_s)
        h2d = sum(host[n].numel() * host[n].element_size() for n in ("kp", "c", "k", "v", "q", "idx_q", "idx_w"))
        return h2d, out_host.numel() * out_host.element_size()
