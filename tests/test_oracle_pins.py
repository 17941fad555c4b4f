"""Pins for the CPU oracle: closed forms, invariants, library routines, brute force.

Each test fixes a part of ``oracle.sgqa_oracle`` against something other than
the oracle itself, chosen so that a plausible slip (a dropped term, a wrong
sign or index, a transposed operand) fails at least one of them.  Sources: the
page "Step-5-Preview: Sparse Reads Are Not a Compressed KV Cache", sections
cited per test.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import sgqa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            lhs, _ = line.split("|", 1)
            k, v = lhs.split("=")
            vals[k.strip()] = float(v)
    return vals


# --------------------------------------------------------------------------
# Roundings: BF16 and OCP E4M3 against torch's casts (library routines)
# --------------------------------------------------------------------------

def test_bf16_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200000)
    bits = rng.integers(0, 2 ** 32, 50000, dtype=np.uint64).astype(np.uint32)
    halfway = ((bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, halfway[np.isfinite(halfway)], np.float32([0.0, -0.0, 1.0, -1.0])])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x)
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))


def _all_bf16_values():
    bits = np.arange(2 ** 16, dtype=np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return bits.view(np.float32).astype(np.float64)


def test_e4m3_matches_torch_cast_exhaustive_bf16():
    x = _all_bf16_values()
    ok = np.isfinite(x) & (np.abs(x) < 464.0)
    ref = torch.from_numpy(x[ok]).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.round_e4m3(x[ok])
    assert np.array_equal(got, ref)
    # torch maps values at or above 464 to NaN; the store is saturating (satfinite).
    big = np.isfinite(x) & (np.abs(x) >= 464.0)
    assert np.all(np.abs(O.round_e4m3(x[big])) == 448.0)
    assert np.isnan(O.round_e4m3(np.nan))


def test_e4m3_codes_roundtrip_and_torch_decode():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(vals), np.isnan(ref))
    fin = ~np.isnan(vals)
    assert np.array_equal(vals[fin], ref[fin])
    assert np.array_equal(O.e4m3_encode(vals[fin]), codes[fin])
    # spec points: largest finite, smallest normal, smallest subnormal
    assert O.e4m3_encode(448.0) == 0x7E and O.e4m3_encode(-448.0) == 0xFE
    assert O.e4m3_encode(2.0 ** -6) == 0x08 and O.e4m3_encode(2.0 ** -9) == 0x01
    # round half to even
    assert O.round_e4m3(1.0625) == 1.0 and O.round_e4m3(1.1875) == 1.25
    assert O.round_e4m3(2.0 ** -10) == 0.0 and O.round_e4m3(3 * 2.0 ** -10) == 2.0 ** -8


def test_store_codes_double_rounding():
    # x = 1 + 2**-4 + 2**-12 is exact in fp32.  BF16 keeps 7 fraction bits, and
    # 2**-12 is below half a BF16 ulp, so BF16 gives 1.0625.  In E4M3 1.0625 is
    # the midpoint of 1.0 and 1.125 and goes to the even 1.0, whereas rounding x
    # straight to E4M3 gives 1.125: the BF16 step changes the stored code.
    x = 1.0 + 2.0 ** -4 + 2.0 ** -12
    assert O.round_bf16(x) == 1.0625
    assert O.e4m3_decode(O.store_codes(np.array([x])))[0] == 1.0
    assert O.round_e4m3(x) == 1.125


# --------------------------------------------------------------------------
# Merge: section "Eight tokens become one search key, coordinate by coordinate"
# --------------------------------------------------------------------------

def test_merge_identical_tokens_give_that_token():
    rng = np.random.default_rng(1)
    tok = rng.standard_normal(64)
    kp = np.tile(tok, (8, 1))
    c = rng.standard_normal((8, 64)) * 5
    assert np.allclose(O.merge_block(kp, c), tok, rtol=0, atol=1e-14)


def test_merge_equal_logits_give_coordinate_mean():
    rng = np.random.default_rng(2)
    kp = rng.standard_normal((8, 64))
    c = np.tile(rng.standard_normal(64), (8, 1))
    assert np.allclose(O.merge_block(kp, c), kp.mean(axis=0), rtol=0, atol=1e-14)


def test_merge_dominant_logit_picks_that_coordinate():
    rng = np.random.default_rng(3)
    kp = rng.standard_normal((8, 64))
    c = np.zeros((8, 64))
    winner = rng.integers(0, 8, 64)
    c[winner, np.arange(64)] = 1000.0  # exp(-1000) underflows: exactly one weight
    assert np.array_equal(O.merge_block(kp, c), kp[winner, np.arange(64)])


def test_merge_closed_form_log_logits():
    # logits ln(j+1): weights (j+1)/36 exactly; merged = sum (j+1) k_j / 36.
    kp = np.array([[float(j * j - 3 * j + 1), float(-j)] for j in range(8)])
    c = np.log(np.arange(1, 9, dtype=np.float64))[:, None].repeat(2, axis=1)
    expect = [float(sum(Fraction(j + 1, 36) * Fraction(int(kp[j, d])) for j in range(8))) for d in range(2)]
    assert np.allclose(O.merge_block(kp, c), expect, rtol=1e-14, atol=0)


def test_merge_shift_and_permutation_invariance_and_range():
    rng = np.random.default_rng(4)
    kp = rng.standard_normal((8, 64))
    c = rng.standard_normal((8, 64)) * 3
    m = O.merge_block(kp, c)
    shift = rng.standard_normal(64) * 50
    assert np.allclose(O.merge_block(kp, c + shift), m, rtol=1e-12, atol=1e-12)
    perm = rng.permutation(8)
    assert np.allclose(O.merge_block(kp[perm], c[perm]), m, rtol=1e-12, atol=1e-13)
    assert np.all(m >= kp.min(axis=0) - 1e-12) and np.all(m <= kp.max(axis=0) + 1e-12)
    # per-coordinate weights: changing coordinate 0's logits leaves the others
    c2 = c.copy()
    c2[:, 0] = rng.standard_normal(8) * 3
    m2 = O.merge_block(kp, c2)
    assert np.array_equal(m2[1:], m[1:])


def test_merge_not_in_convex_hull_of_whole_vectors():
    # Two tokens in 2-D: coordinate 0 weights token 0, coordinate 1 weights token 1.
    kp = np.array([[1.0, 0.0], [0.0, 1.0]])
    c = np.array([[100.0, -100.0], [-100.0, 100.0]])
    m = O.merge_block(kp, c)
    assert np.allclose(m, [1.0, 1.0])  # hull of (1,0),(0,1) has x+y = 1
    assert m.sum() > 1.5


def test_merge_blocks_block_size_one_is_identity_and_uses_completed_blocks():
    rng = np.random.default_rng(5)
    kp = rng.standard_normal((13, 64))
    c = rng.standard_normal((13, 64))
    assert np.array_equal(O.merge_blocks(kp, c, 1), kp)
    mb = O.merge_blocks(kp, c, 8)
    assert mb.shape == (1, 64)  # the 5-token tail is not a completed block
    assert np.array_equal(mb[0], O.merge_block(kp[:8], c[:8]))


# --------------------------------------------------------------------------
# Score: section "Selection is a weighted ReLU score, not attention softmax"
# --------------------------------------------------------------------------

def test_score_on_basis_keys_reads_query_entries():
    # keys[r] = e_r: q_i . keys[r] = q[i, r]; score = sum_i w_i max(0, q[i, r]).
    q = np.array([[2.0, -1.0, 0.5, 0.0], [-3.0, 4.0, 1.0, -2.0], [1.0, 1.0, -1.0, 3.0]])
    w = np.array([0.5, -2.0, 1.0])
    keys = np.eye(4)
    expect = [0.5 * 2.0 + 1.0 * 1.0,            # r0: heads 0 and 2 positive
              -2.0 * 4.0 + 1.0 * 1.0,           # r1: heads 1 and 2
              0.5 * 0.5 - 2.0 * 1.0,            # r2: heads 0 and 1
              1.0 * 3.0]                        # r3: head 2
    assert np.allclose(O.index_scores(q, w, keys), expect, rtol=0, atol=1e-15)


def test_score_relu_is_inside_the_sum_and_no_softmax():
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([1.0, 1.0])
    k = np.array([[3.0, -5.0]])      # head dots 3 and -5: ReLU gives 3, not -2
    assert O.index_scores(q, w, k)[0] == 3.0
    k = np.array([[-1.0, -1.0]])     # every dot negative: exactly zero
    assert O.index_scores(q, w, k)[0] == 0.0
    # signed weights make negative scores possible
    assert O.index_scores(q, np.array([-1.0, 0.5]), np.array([[2.0, 0.0]]))[0] == -2.0
    # positive homogeneity (ReLU) and permutation equivariance over candidates
    rng = np.random.default_rng(6)
    q = rng.standard_normal((8, 64)); w = rng.standard_normal(8); keys = rng.standard_normal((50, 64))
    s = O.index_scores(q, w, keys)
    assert np.allclose(O.index_scores(2.5 * q, w, keys), 2.5 * s)
    perm = rng.permutation(50)
    assert np.allclose(O.index_scores(q, w, keys[perm]), s[perm])
    assert not np.allclose(O.index_scores(-q, w, keys), -s)


# --------------------------------------------------------------------------
# Selection: ties to the smaller id, causal candidates, budget
# --------------------------------------------------------------------------

def test_select_topk_against_python_sorted_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(200):
        n = int(rng.integers(1, 300))
        k = int(rng.integers(1, 64))
        s = np.round(rng.standard_normal(n) * 3) / 2.0   # many exact ties
        s[rng.random(n) < 0.1] = -0.0
        s[rng.random(n) < 0.1] = 0.0
        ref = sorted(sorted(range(n), key=lambda r: (-float(s[r]), r))[:k])
        assert list(O.select_topk(s, k)) == ref


def test_select_fewer_candidates_than_k_takes_all():
    assert list(O.select_topk(np.array([1.0, -2.0, 0.5]), 8)) == [0, 1, 2]
    assert list(O.select_topk(np.array([]), 8)) == []


def test_attended_positions_budget_and_current_block():
    g = _golden("page_figures.txt")
    B, k = int(g["block_size"]), int(g["historical_blocks"])
    t = 1048575
    sel = np.arange(k) * 7
    pos = O.attended_positions(t, sel, B)
    assert len(pos) == k * B + B == int(g["max_tokens_read_per_group"])
    assert len(set(pos.tolist())) == len(pos)
    assert round(g["context_T"] / len(pos), 1) == g["read_ratio_T_over_4104"]
    # the last query of a 1M prefill sees floor((T-1)/8) candidate summaries
    assert (int(g["context_T"]) - 1) // B == int(g["summaries_at_1M"])
    gib = int(g["context_T"]) * int(g["summaries_at_1M"]) * 4 / 2 ** 30
    assert round(gib, 6) == g["score_matrix_gib_tp8"]
    assert 2 * 4 * 192 * 2 == int(g["kv_bytes_per_token_layer"])
    # t < B: only the current block's positions 0..t
    assert list(O.attended_positions(5, np.array([], dtype=np.int64), 8)) == [0, 1, 2, 3, 4, 5]
    # the current block is restricted to positions <= t
    assert list(O.attended_positions(19, np.array([0]), 8)) == list(range(8)) + [16, 17, 18, 19]


# --------------------------------------------------------------------------
# Attention against torch's scaled_dot_product_attention (library routine)
# --------------------------------------------------------------------------

def _tiny_problem(seed, L=64, G=2, Hg=4, D=32, H=3, Di=16, B=8):
    rng = np.random.default_rng(seed)
    return dict(
        q=rng.standard_normal((L, G * Hg, D)), k=rng.standard_normal((L, G, D)),
        v=rng.standard_normal((L, G, D)), idx_q=rng.standard_normal((L, G, H, Di)),
        idx_w=rng.standard_normal((L, G, H)), kp=rng.standard_normal((L, Di)),
        c=rng.standard_normal((L, Di)), L=L, G=G, Hg=Hg, D=D, B=B)


def _sdpa(q, k, v, scale, mask=None, causal=False):
    qt = torch.from_numpy(np.ascontiguousarray(q))[None]
    kt = torch.from_numpy(np.ascontiguousarray(k))[None]
    vt = torch.from_numpy(np.ascontiguousarray(v))[None]
    am = None if mask is None else torch.from_numpy(mask)[None]
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=am, is_causal=causal, scale=scale)[0].numpy()


@pytest.mark.parametrize("B", [8, 1, 4])
def test_full_topk_equals_dense_causal_attention(B):
    p = _tiny_problem(10, B=B)
    keys = O.merge_blocks(p["kp"], p["c"], B)
    rows = [(i, g) for i in range(p["L"]) for g in range(p["G"])]
    res = O.forward_rows(rows, q=p["q"], k=p["k"], v=p["v"], idx_q=p["idx_q"], idx_w=p["idx_w"],
                         keys=keys, block=B, topk=10 ** 6, heads_per_group=p["Hg"])
    scale = 1.0 / math.sqrt(p["D"])
    for g in range(p["G"]):
        hs = slice(g * p["Hg"], (g + 1) * p["Hg"])
        dense = _sdpa(p["q"][:, hs].transpose(1, 0, 2),
                      np.repeat(p["k"][None, :, g], p["Hg"], 0),
                      np.repeat(p["v"][None, :, g], p["Hg"], 0), scale, causal=True)
        for i in range(p["L"]):
            assert np.allclose(res[(i, g)][1], dense[:, i], rtol=1e-10, atol=1e-12)


def test_sparse_attention_equals_masked_sdpa():
    p = _tiny_problem(11, L=96)
    B, k = 8, 3
    keys = O.merge_blocks(p["kp"], p["c"], B)
    rows = [(i, g) for i in range(p["L"]) for g in range(p["G"])]
    res = O.forward_rows(rows, q=p["q"], k=p["k"], v=p["v"], idx_q=p["idx_q"], idx_w=p["idx_w"],
                         keys=keys, block=B, topk=k, heads_per_group=p["Hg"])
    scale = 1.0 / math.sqrt(p["D"])
    for g in range(p["G"]):
        mask = np.zeros((p["L"], p["L"]), dtype=bool)
        for i in range(p["L"]):
            sel = set(res[(i, g)][0].tolist())
            assert len(sel) == min(k, i // B)
            for s in range(p["L"]):
                mask[i, s] = (s // B in sel) or (B * (i // B) <= s <= i)
        hs = slice(g * p["Hg"], (g + 1) * p["Hg"])
        ref = _sdpa(p["q"][:, hs].transpose(1, 0, 2), np.repeat(p["k"][None, :, g], p["Hg"], 0),
                    np.repeat(p["v"][None, :, g], p["Hg"], 0), scale, mask=mask[None].repeat(p["Hg"], 0))
        for i in range(p["L"]):
            assert np.allclose(res[(i, g)][1], ref[:, i], rtol=1e-10, atol=1e-12)


def test_selection_has_no_future_leak():
    p = _tiny_problem(12, L=80)
    B, k = 8, 2
    for t in [7, 8, 15, 37, 63, 79]:
        keys = O.merge_blocks(p["kp"], p["c"], B)
        base = O.forward_rows([(t, 0)], q=p["q"], k=p["k"], v=p["v"], idx_q=p["idx_q"],
                              idx_w=p["idx_w"], keys=keys, block=B, topk=k, heads_per_group=p["Hg"])
        kp2, c2 = p["kp"].copy(), p["c"].copy()
        cut = B * (t // B)
        kp2[cut:] += 100.0
        c2[cut:] = -c2[cut:]
        keys2 = O.merge_blocks(kp2, c2, B)
        pert = O.forward_rows([(t, 0)], q=p["q"], k=p["k"], v=p["v"], idx_q=p["idx_q"],
                              idx_w=p["idx_w"], keys=keys2, block=B, topk=k, heads_per_group=p["Hg"])
        assert np.array_equal(base[(t, 0)][0], pert[(t, 0)][0])
        assert np.array_equal(base[(t, 0)][1], pert[(t, 0)][1])


def test_selection_tie_goes_to_smaller_block_id():
    # duplicate merged keys give exactly equal scores: the smaller ids win
    rng = np.random.default_rng(13)
    keys = np.repeat(rng.standard_normal((1, 16)), 10, axis=0)
    s = O.index_scores(rng.standard_normal((3, 16)), rng.standard_normal(3), keys)
    assert np.all(s == s[0])
    assert list(O.select_topk(s, 4)) == [0, 1, 2, 3]


# --------------------------------------------------------------------------
# Head-wise sigmoid output gate (section "Main attention still reads original K/V")
# --------------------------------------------------------------------------

def test_gate_closed_forms():
    """sigmoid(0) = 1/2 exactly; sigmoid(g) + sigmoid(-g) = 1; saturation at
    large |g| (a wrong sign or a missing gate fails one of these)."""
    rng = np.random.default_rng(11)
    out = rng.standard_normal((5, 3, 192))
    assert np.array_equal(O.gated_head_output(out, np.zeros((5, 3))), 0.5 * out)
    g = rng.standard_normal((5, 3)) * 3.0
    np.testing.assert_allclose(O.gated_head_output(out, g) + O.gated_head_output(out, -g), out, rtol=0, atol=1e-14)
    np.testing.assert_allclose(O.gated_head_output(out, np.full((5, 3), 40.0)), out, rtol=1e-15, atol=0)
    assert np.abs(O.gated_head_output(out, np.full((5, 3), -40.0))).max() < 1e-16 * np.abs(out).max()
    # one logit scales its whole head vector, and only that head's
    g1 = np.zeros((5, 3)); g1[2, 1] = math.log(3.0)   # sigmoid = 3/4
    got = O.gated_head_output(out, g1)
    np.testing.assert_allclose(got[2, 1], 0.75 * out[2, 1], rtol=1e-15)
    mask = np.ones((5, 3), bool); mask[2, 1] = False
    assert np.array_equal(got[mask], 0.5 * out[mask])


def test_gate_on_single_token_attention_is_gated_value_row():
    """Attention over one token returns that token's V row; the gate scales it."""
    rng = np.random.default_rng(12)
    q = rng.standard_normal((16, 192)); k = rng.standard_normal((1, 192)); v = rng.standard_normal((1, 192))
    att = O.sparse_attention(q, k, v, 192 ** -0.5)
    g = rng.standard_normal(16)
    np.testing.assert_allclose(O.gated_head_output(att, g), (1 / (1 + np.exp(-g)))[:, None] * v[0][None, :],
                               rtol=1e-13, atol=0)


# --------------------------------------------------------------------------
# Token coverage (this build's reading of the second page's undefined measure)
# --------------------------------------------------------------------------

def test_token_coverage_invariants_and_torch_softmax():
    """All positions cover 1; a set and its complement sum to 1; equal logits
    give |A| / (t + 1); the value matches torch's softmax mass directly."""
    rng = np.random.default_rng(13)
    q = rng.standard_normal((16, 192))
    k = rng.standard_normal((40, 192))
    scale = 192 ** -0.5
    allpos = np.arange(40)
    assert abs(O.token_coverage(q, k, allpos, scale) - 1.0) < 1e-14
    a = rng.choice(40, size=17, replace=False)
    comp = np.setdiff1d(allpos, a)
    assert abs(O.token_coverage(q, k, a, scale) + O.token_coverage(q, k, comp, scale) - 1.0) < 1e-14
    assert O.token_coverage(np.zeros((16, 192)), k, a, scale) == pytest.approx(17 / 40, abs=1e-15)
    p = torch.softmax(torch.from_numpy(q @ k.T * scale), dim=1)
    ref = float(p[:, torch.from_numpy(a)].sum(dim=1).mean())
    assert O.token_coverage(q, k, a, scale) == pytest.approx(ref, abs=1e-13)

