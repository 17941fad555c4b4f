"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Tolerances: merged keys 1e-3 relative (1e-6 absolute floor) in FP32; store
codes bit-exact except where FP32 rounding of the exact merged value decides a
boundary; selections bit-exact except swaps between scores within 1e-5
relative of the k-th score; attention outputs 2e-2 max-abs on bf16 outputs.
"""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import sgqa_oracle as O
from sparse_long_context_sgqa_b200 import inputs as I
from tests import _harness as Hn

pytestmark = pytest.mark.gpu

WL = I.WORKLOADS
SMALL8 = dataclasses.replace(WL["prefill8k"], name="prefill2k", seq_len=2048)


def _bd():
    from sparse_long_context_sgqa_b200 import binding
    return binding


def test_library_loads(cuda_device):
    assert "sm_100a" in _bd().version()


def test_e4m3_store_exhaustive_over_bf16(cuda_device):
    """B=1 merge is the identity, so the store path sees every BF16 value."""
    bits = (np.arange(2 ** 16, dtype=np.uint32) << np.uint32(16)).view(np.float32)
    vals = bits[np.isfinite(bits)]
    n = (len(vals) + 63) // 64 * 64
    x = np.zeros(n, dtype=np.float32)
    x[:len(vals)] = vals
    kp = torch.from_numpy(x.reshape(-1, 64)).to(cuda_device)
    c = torch.zeros_like(kp)
    p = _bd().Params(num_kv_groups=1, idx_heads=4, block_size=1, topk=8, merge_in_f32=1)
    L = kp.shape[0]
    store = torch.zeros((L, 64), dtype=torch.uint8, device=cuda_device)
    merged = torch.zeros((L, 64), dtype=torch.float32, device=cuda_device)
    _bd().sgqa_merge_blocks(p, 1, L, kp, c, 0, L, merged, store)
    torch.cuda.synchronize()
    assert torch.equal(merged.cpu(), kp.cpu())
    ref = O.e4m3_encode(O.round_e4m3(x.astype(np.float64)))
    got = store.cpu().numpy().reshape(-1)
    bad = np.nonzero(got != ref)[0]
    detail = [(float(x[j]), int(got[j]), int(ref[j])) for j in bad[:12]]
    assert len(bad) == 0, f"{len(bad)} codes differ (value, gpu, oracle): {detail}"



@pytest.mark.parametrize("wl", [WL["tiny"], SMALL8,
                                dataclasses.replace(SMALL8, block=4, name="b4"),
                                dataclasses.replace(SMALL8, block=1, name="b1"),
                                WL["prefill8k"]], ids=lambda w: w.name)
def test_merge_parity(cuda_device, wl):
    cache, _ = Hn.make_inputs(wl, cuda_device)
    p = Hn.params_for(wl)
    L, B = wl.seq_len, wl.block
    store = torch.zeros((1, L // B, 64), dtype=torch.uint8, device=cuda_device)
    merged = torch.zeros((1, L // B, 64), dtype=torch.float32, device=cuda_device)
    # two calls: [0, a) then [a, L/B) -- ranges must not disturb other rows
    a = (L // B) // 3
    _bd().sgqa_merge_blocks(p, 1, L, cache["kp"], cache["c"], 0, a, merged, store)
    _bd().sgqa_merge_blocks(p, 1, L, cache["kp"], cache["c"], a, L // B, merged, store)
    torch.cuda.synchronize()
    exact = O.merge_blocks(Hn.to_np(cache["kp"][0]), Hn.to_np(cache["c"][0]), B)
    got = merged[0].cpu().double().numpy()
    assert np.all(np.abs(got - exact) <= Hn.MERGE_RTOL * np.abs(exact) + Hn.MERGE_ATOL)
    codes = store[0].cpu().numpy()
    ok = Hn.store_mismatch_ok(codes, exact, Hn.to_np(cache["kp"][0]), B)
    assert ok.all(), f"{(~ok).sum()} store codes differ beyond FP32 rounding"
    flips = (codes != O.store_codes(exact)).sum()
    assert flips <= max(2, 1e-4 * codes.size)


def _index_isolated(wl, device, q_pos0, nq, rows):
    cache, _ = Hn.make_inputs(wl, device)
    qs = I.make_queries(wl, device, q_pos0, nq)
    if wl.fp32_inputs:
        qs["idx_q"] = qs["idx_q"].to(torch.bfloat16)
    _, codes, keys = Hn.oracle_keys(Hn.to_np(cache["kp"][0]), Hn.to_np(cache["c"][0]), wl.block)
    L = wl.seq_len
    store = torch.from_numpy(codes).to(device)[None].contiguous()
    p = Hn.params_for(wl)
    sel = torch.full((1, nq, wl.groups, wl.topk), -7, dtype=torch.int32, device=device)
    cnt = torch.full((1, nq, wl.groups), -7, dtype=torch.int32, device=device)
    ws = _bd().alloc_workspace(p, 1, nq, q_pos0 + nq, device)
    _bd().sgqa_index_topk(p, 1, q_pos0, nq, qs["idx_q"][None].contiguous(), qs["idx_w"][None].contiguous(),
                          L, store, sel, cnt, ws)
    _bd().sgqa_check()
    sel, cnt = sel[0].cpu().numpy(), cnt[0].cpu().numpy()
    t = q_pos0 + np.arange(nq)
    assert np.array_equal(cnt, np.minimum(wl.topk, t // wl.block)[:, None].repeat(wl.groups, 1))
    iq, iw = Hn.to_np(qs["idx_q"]), Hn.to_np(qs["idx_w"])
    ties = 0
    for i in rows:
        for g in range(wl.groups):
            tt = q_pos0 + i
            sc = O.index_scores(iq[i, g], iw[i, g], keys[:tt // wl.block])
            c = cnt[i, g]
            assert np.all(sel[i, g, c:] == -1)
            ties += Hn.check_selection(sel[i, g, :c], sc, wl.topk)
    return ties


@pytest.mark.parametrize("case", ["tiny", "prefill8k", "unaligned_chunk", "b1", "b4_k64", "decode_short",
                                  "decode_mid"])
def test_index_topk_parity(cuda_device, case):
    """decode_short / decode_mid: calls of at most 32 queries (the decode path,
    one cluster per query scoring and selecting on chip) with 512..515 and
    9000..9002 candidates: rows just above k, where the last CTAs of a cluster
    own no candidate, and rows that split unevenly over the cluster."""
    if case == "decode_short":
        wl = dataclasses.replace(SMALL8, name="dec_short", seq_len=4224); q0, nq = 4100, 24; rows = range(nq)
    elif case == "decode_mid":
        wl = dataclasses.replace(SMALL8, name="dec_mid", seq_len=72192); q0, nq = 72000, 24; rows = range(nq)
    elif case == "tiny":
        wl = WL["tiny"]; q0, nq = 0, 256; rows = range(256)
    elif case == "prefill8k":
        wl = WL["prefill8k"]; q0, nq = 0, 8192; rows = Hn.sample_rows(wl, 48)
    elif case == "unaligned_chunk":
        wl = SMALL8; q0, nq = 1029, 611; rows = list(range(0, nq, 13)) + [nq - 1]
    elif case == "b1":
        wl = dataclasses.replace(SMALL8, block=1, topk=256); q0, nq = 0, 2048; rows = list(range(0, 2048, 37)) + [2047]
    else:
        wl = dataclasses.replace(SMALL8, block=4, topk=64); q0, nq = 512, 1536; rows = list(range(0, nq, 29)) + [nq - 1]
    ties = _index_isolated(wl, cuda_device, q0, nq, rows)
    assert ties <= 2 * len(rows)


@pytest.mark.parametrize("case", ["short_rows", "filtered_rows", "filtered_rows_65k", "dup_short", "dup_long",
                                  "decode_rows", "dup_decode", "filtered_k2048", "dup_k2048", "zeros_k2048"])
def test_index_topk_exact_ties(cuda_device, case):
    """Exact score ties, which the selection must break toward smaller block ids.

    short_rows / filtered_rows: zero head weights make every score of every
    third row exactly 0, so the only valid selection is the k smallest ids.
    short_rows has 600..2903 candidates per row (the shared-memory histogram
    kernel: a zero row falls in one bin and one sub-bin, overflows the boundary
    buffer and is redone by the radix kernel); filtered_rows has 16384..16895
    (the sampled-threshold path: every zero row keeps all of its candidates,
    overflows the kept list and is recomputed for the radix kernel);
    filtered_rows_65k has 65536..66559, rows of the length a 512K-token context
    reaches (the filtered path and its fallback at 1M-context row lengths);
    decode_rows has 32 queries at 32762..32765 candidates (the decode path:
    each row selected by a cluster of CTAs; a zero row's single boundary bin
    overflows the cluster's buffers and goes to the radix kernel).

    dup_short / dup_long: the store repeats 211 distinct keys (block r holds
    the codes of block r mod 211), so every row's scores come in groups of
    equal values and the k-th position falls inside a group of about n / 211
    equal scores: the histogram kernel resolves those ties itself (groups up
    to 64 by ranking, larger ones by the warp radix select).  The selected
    members of the boundary group must be its smallest ids.  dup_short has
    600..2903 candidates per row, dup_long 15360..16383, dup_decode 32762..32765
    (the cluster select ranks each boundary group itself).

    filtered_k2048 / dup_k2048: B = 1 and top-2048 (the 1M-context B = 1
    variant's selection) at 32768..33023 candidates: the filtered path with
    kept lists of 2k and the select for k above 512, which merges the four
    ascending lists' taken ids.

    zeros_k2048: the same rows over the 211-key store, with head weights
    (-1, -1, 0, ...) in every third row: every score is <= 0 and a candidate
    scores exactly 0 when both weighted heads' ReLU inputs are <= 0, about a
    quarter of them (5k..12k per row).  The k-th best falls inside that group
    of exact zeros, which fills one histogram bin and one sub-bin beyond the
    boundary buffer, and is resolved by the key / id threshold searches; the
    selection must be the group's 2048 smallest ids."""
    dup = case.startswith("dup") or case == "zeros_k2048"
    if case in ("filtered_k2048", "dup_k2048", "zeros_k2048"):
        wl = dataclasses.replace(WL["prefill8k"], name="ties_k2048", seq_len=40960, block=1, topk=2048)
        q0, nq = 32768, 256  # candidates 32768 .. 33023 per query (B = 1)
    elif case in ("decode_rows", "dup_decode"):
        wl = dataclasses.replace(WL["prefill8k"], name="ties_decode", seq_len=262144, topk=512)
        q0, nq = 262100, 32  # candidates 32762 .. 32765 per query, the decode path
    elif case in ("short_rows", "dup_short"):
        wl = dataclasses.replace(WL["prefill8k"], name="ties", seq_len=24576, topk=512)
        q0, nq = 4800, 16384 + 2048  # candidates 600 .. 2903 per query (B = 8)
    elif case == "dup_long":
        wl = dataclasses.replace(WL["prefill8k"], name="ties_dup_long", seq_len=131072, topk=512)
        q0, nq = 122880, 8192  # candidates 15360 .. 16383 per query
    elif case == "filtered_rows_65k":
        wl = dataclasses.replace(WL["prefill8k"], name="ties_65k", seq_len=532480, topk=512)
        q0, nq = 524288, 8192  # candidates 65536 .. 66559 per query
    else:
        wl = dataclasses.replace(WL["prefill8k"], name="ties_long", seq_len=139264, topk=512)
        q0, nq = 131072, 4096  # candidates 16384 .. 16895 per query
    cache, _ = Hn.make_inputs(wl, cuda_device)
    qs = I.make_queries(wl, cuda_device, q0, nq)
    zero = torch.zeros(nq, dtype=torch.bool, device=cuda_device)
    neg = torch.zeros(nq, dtype=torch.bool, device=cuda_device)
    if not dup:
        zero[::3] = True
        qs["idx_w"][zero] = 0.0
    if case == "zeros_k2048":
        neg[::3] = True
        qs["idx_w"][neg] = 0.0
        qs["idx_w"][neg, :, :2] = -1.0
    _, codes, keys = Hn.oracle_keys(Hn.to_np(cache["kp"][0]), Hn.to_np(cache["c"][0]), wl.block)
    if dup:
        codes = np.ascontiguousarray(codes[np.arange(codes.shape[0]) % 211])
        keys = O.e4m3_decode(codes)
    store = torch.from_numpy(codes).to(cuda_device)[None].contiguous()
    p = Hn.params_for(wl)
    sel = torch.full((1, nq, wl.groups, wl.topk), -7, dtype=torch.int32, device=cuda_device)
    cnt = torch.full((1, nq, wl.groups), -7, dtype=torch.int32, device=cuda_device)
    ws = _bd().alloc_workspace(p, 1, nq, q0 + nq, cuda_device)
    _bd().sgqa_index_topk(p, 1, q0, nq, qs["idx_q"][None].contiguous(), qs["idx_w"][None].contiguous(),
                          wl.seq_len, store, sel, cnt, ws)
    _bd().sgqa_check()
    sel, cnt = sel[0].cpu().numpy(), cnt[0].cpu().numpy()
    assert np.all(cnt == wl.topk)
    zero_np = zero.cpu().numpy()
    assert np.all(sel[zero_np] == np.arange(wl.topk, dtype=np.int32))
    iq, iw = Hn.to_np(qs["idx_q"]), Hn.to_np(qs["idx_w"])
    ties = 0
    step = {"short_rows": 397, "dup_short": 397, "filtered_rows_65k": 397, "decode_rows": 2, "dup_decode": 2,
            "filtered_k2048": 19, "dup_k2048": 19, "zeros_k2048": 19}.get(case, 97)
    rows = [i for i in range(1, nq, step) if not zero_np[i]] + [nq - 1]
    if case == "zeros_k2048":
        rows = list(range(0, nq, 3 * 7))  # weight-(-1, -1) rows only
        wide = 0
        for i in rows:
            for g in range(wl.groups):
                cand = keys[:(q0 + i) // wl.block]
                dots = cand.astype(np.float64) @ iq[i, g, :2].astype(np.float64).T
                if np.abs(dots).min() < 1e-3:  # a sign the fp32 sums might not share
                    continue
                grp = np.flatnonzero(np.all(dots <= 0.0, axis=1))
                if grp.size < wl.topk:  # the zeros and the best of the rest
                    ties += Hn.check_selection(sel[i, g], O.index_scores(iq[i, g], iw[i, g], cand), wl.topk)
                    continue
                wide += grp.size > 4096
                assert np.array_equal(sel[i, g], grp[:wl.topk]), (i, g)
        assert wide > 0 and ties <= 2 * len(rows)
        return
    for i in rows:
        for g in range(wl.groups):
            sc = O.index_scores(iq[i, g], iw[i, g], keys[:(q0 + i) // wl.block])
            ties += Hn.check_selection(sel[i, g], sc, wl.topk)
            if dup:
                order = np.lexsort((np.arange(sc.shape[0]), -sc))
                group = np.flatnonzero(sc == sc[order[wl.topk - 1]])
                assert group.size > 1
                chosen = np.intersect1d(sel[i, g], group)
                assert np.array_equal(chosen, group[:chosen.size]), (i, g)
    assert ties <= 2 * len(rows)


@pytest.mark.parametrize("case", ["short", "long"])
def test_index_topk_outlier_keys(cuda_device, case):
    """Blocks 2 and 37 of the store hold the E4M3 code of 240 in every
    dimension, so in many rows one candidate's score lies hundreds of times
    the typical spread away from the rest.  The linear bins of the histogram
    top-k then crowd every other candidate into a few bins: the sample's and
    the exact step's second histogram levels must separate them.  Block 2 is
    in the sample (float4 0), block 37 is not.  Selections are checked against
    the oracle (exact up to near-ties).  short: 600..2903 candidates per row,
    long: 15360..16383."""
    if case == "short":
        wl = dataclasses.replace(WL["prefill8k"], name="outlier", seq_len=24576, topk=512)
        q0, nq, step = 4800, 16384 + 2048, 397
    else:
        wl = dataclasses.replace(WL["prefill8k"], name="outlier_long", seq_len=131072, topk=512)
        q0, nq, step = 122880, 8192, 97
    cache, _ = Hn.make_inputs(wl, cuda_device)
    qs = I.make_queries(wl, cuda_device, q0, nq)
    _, codes, _ = Hn.oracle_keys(Hn.to_np(cache["kp"][0]), Hn.to_np(cache["c"][0]), wl.block)
    codes = codes.copy()
    codes[[2, 37]] = 119  # E4M3 code of 240.0
    keys = O.e4m3_decode(codes)
    assert keys[2, 0] == 240.0
    store = torch.from_numpy(codes).to(cuda_device)[None].contiguous()
    p = Hn.params_for(wl)
    sel = torch.full((1, nq, wl.groups, wl.topk), -7, dtype=torch.int32, device=cuda_device)
    cnt = torch.full((1, nq, wl.groups), -7, dtype=torch.int32, device=cuda_device)
    ws = _bd().alloc_workspace(p, 1, nq, q0 + nq, cuda_device)
    _bd().sgqa_index_topk(p, 1, q0, nq, qs["idx_q"][None].contiguous(), qs["idx_w"][None].contiguous(),
                          wl.seq_len, store, sel, cnt, ws)
    _bd().sgqa_check()
    sel, cnt = sel[0].cpu().numpy(), cnt[0].cpu().numpy()
    assert np.all(cnt == wl.topk)
    iq, iw = Hn.to_np(qs["idx_q"]), Hn.to_np(qs["idx_w"])
    rows = list(range(1, nq, step)) + [nq - 1]
    ties, skewed = 0, 0
    for i in rows:
        for g in range(wl.groups):
            sc = O.index_scores(iq[i, g], iw[i, g], keys[:(q0 + i) // wl.block])
            ties += Hn.check_selection(sel[i, g], sc, wl.topk)
            rest = np.delete(sc, [2, 37])
            skewed += sc.max() - np.median(rest) > 100 * (np.sort(rest)[-1] - np.median(rest))
    assert ties <= 2 * len(rows)
    assert skewed > 0  # the planted outliers did skew some of the checked rows


def _attn_isolated(wl, device, q_pos0, nq, rows, num_seqs=1, groups=None, gated=False):
    cache, _ = Hn.make_inputs(wl, device, seqs=range(num_seqs))
    qs = [I.make_queries(wl, device, q_pos0, nq, seq=s) for s in range(num_seqs)]
    q = torch.stack([x["q"] for x in qs]).to(torch.bfloat16).contiguous()
    sel, cnt = I.make_selection(wl, device, q_pos0, nq, num_seqs=num_seqs)
    p = Hn.params_for(wl)
    L = wl.seq_len
    out = torch.zeros((num_seqs, nq, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=device)
    ws = _bd().alloc_workspace(p, num_seqs, nq, q_pos0 + nq, device)
    gate = None
    if gated:
        gate = torch.stack([I.make_gate(wl, device, q_pos0, nq, seq=s) for s in range(num_seqs)]).contiguous()
        _bd().sgqa_sparse_attn_gated(p, num_seqs, q_pos0, nq, q, L, L, cache["k"], cache["v"], sel, cnt, gate, out,
                                     ws)
    else:
        _bd().sgqa_sparse_attn(p, num_seqs, q_pos0, nq, q, L, L, cache["k"], cache["v"], sel, cnt, out, ws)
    _bd().sgqa_check()
    worst = 0.0
    for s in range(num_seqs):
        K, V = Hn.to_np(cache["k"][s]), Hn.to_np(cache["v"][s])
        qn = Hn.to_np(q[s])
        seln, cntn = sel[s].cpu().numpy(), cnt[s].cpu().numpy()
        on = out[s].float().cpu().numpy()
        for i in rows:
            for g in (range(wl.groups) if groups is None else groups):
                t = q_pos0 + i
                ids = seln[i, g, :cntn[i, g]]
                pos = O.attended_positions(t, ids, wl.block)
                hs = slice(g * 16, (g + 1) * 16)
                ref = O.sparse_attention(qn[i, hs], K[pos, g], V[pos, g], Hn.scale_of(wl))
                if gate is not None:
                    ref = O.gated_head_output(ref, Hn.to_np(gate[s, i, hs]))
                worst = max(worst, float(np.abs(on[i, hs] - ref).max()))
    assert worst <= Hn.ATTN_ATOL, worst
    return worst


@pytest.mark.parametrize("case", ["prefill8k", "decode_path", "b1", "b2_decode"])
def test_sparse_attn_gated_parity(cuda_device, case):
    """The head-wise sigmoid output gate fused into each attention kernel's
    normalisation: tcgen05 prefill (B = 8), TMA decode with the cluster combine
    (B = 8), the warp-MMA prefill (B = 1) and the split-K decode with its
    combine kernel (B = 2)."""
    if case == "prefill8k":
        _attn_isolated(WL["prefill8k"], cuda_device, 0, 8192, Hn.sample_rows(WL["prefill8k"], 24), gated=True)
    elif case == "decode_path":
        wl = dataclasses.replace(SMALL8, seq_len=20000, name="dec")
        _attn_isolated(wl, cuda_device, 19990, 10, range(10), num_seqs=3, gated=True)
    elif case == "b1":
        wl = dataclasses.replace(SMALL8, block=1, topk=2048)
        _attn_isolated(wl, cuda_device, 0, 2048, list(range(0, 2048, 97)) + [2047], gated=True)
    else:
        wl = dataclasses.replace(SMALL8, seq_len=20000, name="dec2", block=2, topk=100)
        _attn_isolated(wl, cuda_device, 19990, 10, range(10), num_seqs=2, gated=True)


def _paged_pool(k, v, rng, spare=37):
    """Pools of 16-token pages [num_pages, G, 16, D] holding every sequence's
    cache in shuffled pages (group-major inside a page)."""
    S, L, G, D = k.shape
    per = (L + 15) // 16
    num_pages = S * per + spare
    perm = torch.from_numpy(rng.permutation(num_pages)[:S * per].astype(np.int32)).to(k.device)
    table = perm.view(S, per).contiguous()
    kp = torch.zeros((num_pages, G, 16, D), dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    pad = per * 16 - L
    kpad = torch.nn.functional.pad(k, (0, 0, 0, 0, 0, pad)).view(S * per, 16, G, D).permute(0, 2, 1, 3)
    vpad = torch.nn.functional.pad(v, (0, 0, 0, 0, 0, pad)).view(S * per, 16, G, D).permute(0, 2, 1, 3)
    kp[table.view(-1).long()] = kpad
    vp[table.view(-1).long()] = vpad
    return kp, vp, table


def test_sparse_attn_paged_equals_contiguous(cuda_device):
    """A paged cache (16-token pages in shuffled order, spare pages) gives the
    contiguous path's output bit for bit, gated, and the oracle's."""
    wl = dataclasses.replace(SMALL8, seq_len=20000, name="dec")
    S, q0, nq, L = 3, 19990, 10, 20000
    cache, _ = Hn.make_inputs(wl, cuda_device, seqs=range(S))
    qs = [I.make_queries(wl, cuda_device, q0, nq, seq=s) for s in range(S)]
    q = torch.stack([x["q"] for x in qs]).to(torch.bfloat16).contiguous()
    sel, cnt = I.make_selection(wl, cuda_device, q0, nq, num_seqs=S)
    gate = torch.stack([I.make_gate(wl, cuda_device, q0, nq, seq=s) for s in range(S)]).contiguous()
    p = Hn.params_for(wl)
    out_c = torch.zeros((S, nq, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=cuda_device)
    out_p = torch.zeros_like(out_c)
    ws = _bd().alloc_workspace(p, S, nq, q0 + nq, cuda_device)
    _bd().sgqa_sparse_attn_gated(p, S, q0, nq, q, L, L, cache["k"], cache["v"], sel, cnt, gate, out_c, ws)
    kpool, vpool, table = _paged_pool(cache["k"], cache["v"], np.random.default_rng(5))
    _bd().sgqa_sparse_attn_paged(p, S, q0, nq, q, kpool, vpool, table, L, sel, cnt, out_p, gate=gate)
    _bd().sgqa_check()
    assert torch.equal(out_p, out_c)
    worst = 0.0
    for s in range(S):
        K, V = Hn.to_np(cache["k"][s]), Hn.to_np(cache["v"][s])
        seln, cntn = sel[s].cpu().numpy(), cnt[s].cpu().numpy()
        on, qn, gn = out_p[s].float().cpu().numpy(), Hn.to_np(q[s]), Hn.to_np(gate[s])
        for i in range(nq):
            for g in range(wl.groups):
                pos = O.attended_positions(q0 + i, seln[i, g, :cntn[i, g]], wl.block)
                hs = slice(g * 16, (g + 1) * 16)
                ref = O.gated_head_output(O.sparse_attention(qn[i, hs], K[pos, g], V[pos, g], Hn.scale_of(wl)), gn[i, hs])
                worst = max(worst, float(np.abs(on[i, hs] - ref).max()))
    assert worst <= Hn.ATTN_ATOL, worst


def test_sparse_attn_paged_prefill_equals_contiguous(cuda_device):
    """Prefill-sized calls (the tensor-core kernel) over a paged cache give the
    contiguous path's output bit for bit (gated), and the oracle's: a chunk of
    1536 queries with selections of up to 512 blocks, two sequences."""
    wl = dataclasses.replace(SMALL8, seq_len=6144, name="pf_paged")
    S, q0, nq, L = 2, 4608, 1536, 6144
    cache, _ = Hn.make_inputs(wl, cuda_device, seqs=range(S))
    qs = [I.make_queries(wl, cuda_device, q0, nq, seq=s) for s in range(S)]
    q = torch.stack([x["q"] for x in qs]).to(torch.bfloat16).contiguous()
    sel, cnt = I.make_selection(wl, cuda_device, q0, nq, num_seqs=S)
    gate = torch.stack([I.make_gate(wl, cuda_device, q0, nq, seq=s) for s in range(S)]).contiguous()
    p = Hn.params_for(wl)
    out_c = torch.zeros((S, nq, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=cuda_device)
    out_p = torch.zeros_like(out_c)
    ws = _bd().alloc_workspace(p, S, nq, q0 + nq, cuda_device)
    _bd().sgqa_sparse_attn_gated(p, S, q0, nq, q, L, L, cache["k"], cache["v"], sel, cnt, gate, out_c, ws)
    kpool, vpool, table = _paged_pool(cache["k"], cache["v"], np.random.default_rng(9))
    _bd().sgqa_sparse_attn_paged(p, S, q0, nq, q, kpool, vpool, table, L, sel, cnt, out_p, gate=gate, workspace=ws)
    _bd().sgqa_check()
    assert torch.equal(out_p, out_c)
    rng = np.random.default_rng(3)
    worst = 0.0
    for _ in range(24):
        s, i, g = int(rng.integers(S)), int(rng.integers(nq)), int(rng.integers(wl.groups))
        ids = sel[s, i, g, :cnt[s, i, g]].cpu().numpy()
        pos = O.attended_positions(q0 + i, ids, wl.block)
        hs = slice(g * 16, (g + 1) * 16)
        ref = O.gated_head_output(O.sparse_attention(Hn.to_np(q[s, i, hs]), Hn.to_np(cache["k"][s, pos, g]),
                                                     Hn.to_np(cache["v"][s, pos, g]), Hn.scale_of(wl)),
                                  Hn.to_np(gate[s, i, hs]))
        worst = max(worst, float(np.abs(out_p[s, i, hs].float().cpu().numpy() - ref).max()))
    assert worst <= Hn.ATTN_ATOL, worst


def test_sparse_attn_paged_bad_page_is_reported(cuda_device):
    """A page-table entry outside the pool is caught by the kernel's check
    (the copy reads zeros) and reported by sgqa_check as a device error."""
    wl = dataclasses.replace(SMALL8, seq_len=4096, name="dec_bad")
    S, q0, nq, L = 1, 4090, 4, 4096
    cache, _ = Hn.make_inputs(wl, cuda_device, seqs=range(S))
    q = I.make_queries(wl, cuda_device, q0, nq)["q"][None].to(torch.bfloat16).contiguous()
    sel, cnt = I.make_selection(wl, cuda_device, q0, nq, num_seqs=S)
    kpool, vpool, table = _paged_pool(cache["k"], cache["v"], np.random.default_rng(6), spare=0)
    table[0, 255] = kpool.shape[0] + 3  # the page of the current block (tokens 4080..4095)
    out = torch.zeros((S, nq, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=cuda_device)
    p = Hn.params_for(wl)
    _bd().sgqa_sparse_attn_paged(p, S, q0, nq, q, kpool, vpool, table, L, sel, cnt, out)
    with pytest.raises(_bd().SgqaError) as err:
        _bd().sgqa_check()
    assert err.value.code == 6  # SGQA_ERR_DEVICE
    _bd().sgqa_check()  # the status word was cleared


def test_forward_gated_equals_gate_times_forward(cuda_device):
    """sgqa_forward_gated = sigmoid(gate) * sgqa_forward, head by head (same
    inputs, one 2048-token prefill chunk)."""
    wl = SMALL8
    run = Hn.run_forward(wl, cuda_device)
    p = Hn.params_for(wl)
    S, nq, L = 1, wl.nq, wl.seq_len
    gate = I.make_gate(wl, cuda_device, wl.q_start, nq)[None].contiguous()
    out = torch.zeros_like(run.out)
    sel, cnt = torch.empty_like(run.sel), torch.empty_like(run.cnt)
    store = torch.empty_like(run.store)
    ws = _bd().alloc_workspace(p, S, nq, wl.q_start + nq, cuda_device)
    _bd().sgqa_forward_gated(p, S, wl.q_start, nq, run.queries["q"], run.queries["idx_q"], run.queries["idx_w"], L, L,
                             run.cache["kp"], run.cache["c"], run.cache["k"], run.cache["v"], None, store, sel, cnt,
                             gate, out, ws)
    _bd().sgqa_check()
    assert torch.equal(sel, run.sel) and torch.equal(cnt, run.cnt)
    sig = torch.sigmoid(gate.float())[..., None]
    diff = (out.float() - sig * run.out.float()).abs().max().item()
    assert diff <= Hn.ATTN_ATOL, diff


@pytest.mark.parametrize("case", ["tiny", "prefill8k", "unaligned_chunk", "decode_path", "b1", "b2"])
def test_sparse_attn_parity(cuda_device, case):
    if case == "tiny":
        _attn_isolated(WL["tiny"], cuda_device, 0, 256, range(256))
    elif case == "prefill8k":
        _attn_isolated(WL["prefill8k"], cuda_device, 0, 8192, Hn.sample_rows(WL["prefill8k"], 40))
    elif case == "unaligned_chunk":
        _attn_isolated(SMALL8, cuda_device, 1029, 611, list(range(0, 611, 7)) + [610])
    elif case == "decode_path":
        wl = dataclasses.replace(SMALL8, seq_len=20000, name="dec")
        _attn_isolated(wl, cuda_device, 19990, 10, range(10), num_seqs=3)
    elif case == "b1":
        wl = dataclasses.replace(SMALL8, block=1, topk=2048)
        _attn_isolated(wl, cuda_device, 0, 2048, list(range(0, 2048, 41)) + [2047])
    else:
        wl = dataclasses.replace(SMALL8, block=2, topk=100)
        _attn_isolated(wl, cuda_device, 0, 2048, list(range(0, 2048, 41)) + [2047])


def _e2e(wl, device, rows, seqs=(0,)):
    run = Hn.run_forward(wl, device)
    B = wl.block
    stats = {"rows": 0, "tie_rows": 0, "flip_rows": 0, "worst": 0.0}
    for s in seqs:
        kp_np = Hn.to_np(run.cache["kp"][s])
        exact = O.merge_blocks(kp_np, Hn.to_np(run.cache["c"][s]), B)
        codes = O.store_codes(exact)
        gpu_codes = run.store[s].cpu().numpy()
        assert Hn.store_mismatch_ok(gpu_codes, exact, kp_np, B).all()
        del kp_np
        flipped = set(np.nonzero((gpu_codes != codes).any(axis=1))[0].tolist())
        keys = O.e4m3_decode(codes)
        K, V = run.cache["k"][s], run.cache["v"][s]  # rows gathered per checked query (long contexts)
        q, iq, iw = (Hn.to_np(run.queries[x][s]) for x in ("q", "idx_q", "idx_w"))
        sel, cnt = run.sel[s].cpu().numpy(), run.cnt[s].cpu().numpy()
        out = run.out[s].float().cpu().numpy()
        for i in rows:
            t = wl.q_start + i
            for g in range(wl.groups):
                stats["rows"] += 1
                sc = O.index_scores(iq[i, g], iw[i, g], keys[:t // B])
                ref_sel = O.select_topk(sc, wl.topk)
                gsel = sel[i, g, :cnt[i, g]]
                assert cnt[i, g] == len(ref_sel)
                if not np.array_equal(gsel, ref_sel):
                    diff = set(np.setxor1d(gsel, ref_sel).tolist())
                    if diff & flipped:
                        stats["flip_rows"] += 1
                        continue
                    Hn.check_selection(gsel, sc, wl.topk)
                    stats["tie_rows"] += 1
                    continue
                pos = O.attended_positions(t, ref_sel, B)
                hs = slice(g * 16, (g + 1) * 16)
                pos_d = torch.from_numpy(np.asarray(pos, dtype=np.int64)).to(K.device)
                ref = O.sparse_attention(q[i, hs], Hn.to_np(K[pos_d, g]), Hn.to_np(V[pos_d, g]), Hn.scale_of(wl))
                stats["worst"] = max(stats["worst"], float(np.abs(out[i, hs] - ref).max()))
    assert stats["worst"] <= Hn.ATTN_ATOL, stats
    assert stats["flip_rows"] + stats["tie_rows"] <= max(2, 0.05 * stats["rows"]), stats
    return stats


def test_forward_host_pipelined_matches_device_path(cuda_device):
    """SparseGQA.forward_host copies each chunk's inputs in and output out on
    side streams while other chunks run; its output must equal the chunked
    device-resident path bit for bit (same kernels on the same inputs)."""
    from sparse_long_context_sgqa_b200.api import SparseGQA
    wl = dataclasses.replace(WL["prefill8k"], name="e2e", seq_len=3072, chunk=1024)
    run = Hn.run_forward(wl, cuda_device)
    p = Hn.params_for(wl)
    model = SparseGQA(p, 1, wl.seq_len, wl.chunk, cuda_device)
    host = {n: run.cache[n].cpu().pin_memory() for n in ("kp", "c", "k", "v")}
    for n in ("q", "idx_q", "idx_w"):
        host[n] = run.queries[n].cpu().pin_memory()
    out_host = torch.empty(run.out.shape, dtype=run.out.dtype).pin_memory()
    h2d, d2h = model.forward_host(host, out_host)
    torch.cuda.synchronize()
    _bd().sgqa_check()
    assert h2d == sum(host[n].numel() * host[n].element_size() for n in host)
    assert d2h == out_host.numel() * out_host.element_size()
    assert torch.equal(out_host, run.out.cpu())
    assert torch.equal(model.store.cpu(), run.store.cpu())


def test_forward_tiny_all_rows(cuda_device):
    _e2e(WL["tiny"], cuda_device, range(256))


def test_forward_prefill8k_sampled(cuda_device):
    _e2e(WL["prefill8k"], cuda_device, Hn.sample_rows(WL["prefill8k"], 40))


def test_full_topk_equals_dense_causal_attention(cuda_device):
    """k >= number of blocks: the sparse path is textbook causal attention."""
    wl = dataclasses.replace(WL["tiny"], topk=32, name="tiny_dense")
    run = Hn.run_forward(wl, cuda_device)
    q = Hn.to_np(run.queries["q"][0]).transpose(1, 0, 2)       # [16, N, D]
    k = Hn.to_np(run.cache["k"][0, :, 0])[None].repeat(16, 0)
    v = Hn.to_np(run.cache["v"][0, :, 0])[None].repeat(16, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True).numpy()
    got = run.out[0].float().cpu().numpy().transpose(1, 0, 2)
    assert np.abs(got - ref).max() <= Hn.ATTN_ATOL


def test_forward_decode_workload_full_size(cuda_device):
    """16 sequences x 262144 cached tokens, one query each; two sequences checked."""
    wl = WL["decode"]
    _e2e(wl, cuda_device, [0], seqs=(0, 11))


def test_forward_prefill128k_last_chunk(cuda_device):
    wl = dataclasses.replace(WL["prefill128k"], q_start=131072 - 8192)
    _e2e(wl, cuda_device, Hn.sample_rows(wl, 24))


def test_forward_prefill1m_last_chunk(cuda_device):
    """The last 8192-query chunk of the 1M-token prefill (B = 8, top-512
    blocks): rows of 130048..131071 candidates take the sampled-threshold
    filtered index path; blocks below the chunk are merged beforehand."""
    wl = dataclasses.replace(WL["prefill1m"], q_start=1048576 - 8192)
    _e2e(wl, cuda_device, Hn.sample_rows(wl, 64))


def test_forward_prefill1m_b1_last_chunk(cuda_device):
    """The last 8192-query chunk of the 1M-token prefill with B = 1 and
    top-2048 tokens (the pages' comparison variant): rows of
    1040384..1048575 candidates take the filtered path with kept lists of 2k
    and the select for k above 512; the union of 8 queries' tokens spans a
    1M-token range (the bitmap planner with its compact prefix) and the
    attention gathers token rows by cp.async."""
    wl = dataclasses.replace(WL["prefill1m_b1"], q_start=1048576 - 8192)
    _e2e(wl, cuda_device, Hn.sample_rows(wl, 24))


def test_forward_prefill1m_mid_chunk(cuda_device):
    """A chunk in the middle of the 1M-token prefill: queries 327680..335871,
    rows of 40960..41983 candidates."""
    wl = dataclasses.replace(WL["prefill1m"], seq_len=335872, q_start=327680)
    _e2e(wl, cuda_device, Hn.sample_rows(wl, 48))


def test_decode_steps_across_block_boundaries(cuda_device):
    """Consecutive one-token sgqa_forward calls at t = 8m-1 .. 8m+8 for two
    sequences: each call merges the block its token completes (t = 8m-1 and
    8m+7 complete blocks m-1 and m; the others merge nothing), selects from
    the blocks before floor(t/8) and attends to its own block up to t.  Every
    step is checked against the oracle: the store after the step, the
    selection (up to near-ties) and the attention output."""
    from sparse_long_context_sgqa_b200 import binding as Bd
    wl = dataclasses.replace(SMALL8, name="decode_steps", seq_len=3328)
    S, m, B = 2, 400, 8
    t0, t1 = 8 * m - 1, 8 * m + 8
    cache, _ = Hn.make_inputs(wl, cuda_device, seqs=range(S))
    qs = [I.make_queries(wl, cuda_device, t0, t1 - t0 + 1, seq=s) for s in range(S)]
    queries = {n: torch.stack([x[n] for x in qs]).contiguous() for n in qs[0]}
    p = Hn.params_for(wl)
    L = wl.seq_len
    store = torch.zeros((S, L // B, wl.idx_dim), dtype=torch.uint8, device=cuda_device)
    Bd.sgqa_merge_blocks(p, S, L, cache["kp"], cache["c"], 0, t0 // B, None, store)
    ws = Bd.alloc_workspace(p, S, 1, t1 + 1, cuda_device)
    kps = [Hn.to_np(cache["kp"][s]) for s in range(S)]
    exact = [O.merge_blocks(kps[s], Hn.to_np(cache["c"][s]), B) for s in range(S)]
    merged_blocks = t0 // B
    skipped = 0
    for t in range(t0, t1 + 1):
        i = t - t0
        sel = torch.full((S, 1, wl.groups, wl.topk), -7, dtype=torch.int32, device=cuda_device)
        cnt = torch.full((S, 1, wl.groups), -7, dtype=torch.int32, device=cuda_device)
        out = torch.zeros((S, 1, wl.n_heads, wl.head_dim), dtype=torch.bfloat16, device=cuda_device)
        Bd.sgqa_forward(p, S, t, 1, queries["q"][:, i:i + 1].contiguous(), queries["idx_q"][:, i:i + 1].contiguous(),
                        queries["idx_w"][:, i:i + 1].contiguous(), L, t + 1, cache["kp"], cache["c"], cache["k"],
                        cache["v"], None, store, sel, cnt, out, ws)
        Bd.sgqa_check()
        merged_blocks = max(merged_blocks, (t + 1) // B)
        for s in range(S):
            codes = store[s].cpu().numpy()
            assert Hn.store_mismatch_ok(codes[:merged_blocks], exact[s][:merged_blocks], kps[s], B).all(), (t, s)
            assert not codes[merged_blocks:].any(), (t, s)  # blocks not yet complete stay unmerged
            ref_codes = O.store_codes(exact[s][:t // B])
            flipped = set(np.nonzero((codes[:t // B] != ref_codes).any(axis=1))[0].tolist())
            keys = O.e4m3_decode(ref_codes)
            for g in range(wl.groups):
                c = int(cnt[s, 0, g])
                assert c == min(wl.topk, t // B)
                got = sel[s, 0, g, :c].cpu().numpy()
                assert np.all(sel[s, 0, g, c:].cpu().numpy() == -1)
                sc = O.index_scores(Hn.to_np(queries["idx_q"][s, i, g]), Hn.to_np(queries["idx_w"][s, i, g]), keys)
                ref_sel = O.select_topk(sc, wl.topk)
                if not np.array_equal(got, ref_sel):
                    # only near-ties or a block whose stored code sits on a rounding boundary may differ
                    if not (set(np.setxor1d(got, ref_sel).tolist()) & flipped):
                        Hn.check_selection(got, sc, wl.topk)
                    skipped += 1
                    continue
                pos = O.attended_positions(t, ref_sel, B)
                hs = slice(g * 16, (g + 1) * 16)
                ref = O.sparse_attention(Hn.to_np(queries["q"][s, i, hs]), Hn.to_np(cache["k"][s, pos, g]),
                                         Hn.to_np(cache["v"][s, pos, g]), Hn.scale_of(wl))
                err = float(np.abs(out[s, 0, hs].float().cpu().numpy() - ref).max())
                assert err <= Hn.ATTN_ATOL, (t, s, g, err)
    assert skipped <= 4, skipped  # of 10 steps x 2 sequences x 4 groups
