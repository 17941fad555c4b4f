"""CPU oracle for the Sparse GQA global-attention hot path (test infrastructure).

This module is TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  The product path (the
CUDA library and its Python binding) never imports or calls it, and shares no
code with it.

It restates, in plain numpy with float64 arithmetic, what the method computes.
Source: the page "Step-5-Preview: Sparse Reads Are Not a Compressed KV Cache"
(flozi.net), cited below by section title, and the page "Step 5 Preview
architecture blog details Sparse GQA with block-wise token merging cutting
indexer cost 8x" (agihunt.info).  The page's display equations were lost in
extraction; the formulas below are the readings of the surrounding prose:

* merge      -- section "Eight tokens become one search key, coordinate by
                coordinate": for each completed block r and proxy coordinate d,
                a softmax over the block's B compression logits of that
                coordinate (common maximum subtracted) weights the block's B
                proxy-key coordinates.  FP32 accumulation, then storage rounding
                FP32 -> BF16 -> E4M3.
* score      -- section "Selection is a weighted ReLU score, not attention
                softmax": I[t,g,r] = sum_i w[t,g,i] * ReLU(q[t,g,i] . Q8(k_r)),
                Q8 = the E4M3 store value widened losslessly to BF16.  No
                softmax, no extra scale.
* selection  -- same section: only blocks r < floor(t/B) compete; top-k by
                score, equal scores resolved by ascending block id; t's own
                block is added on top, limited to positions <= t.
* attention  -- section "Main attention still reads original K/V": head h uses
                group g(h) = floor(h / heads_per_group); plain scaled
                dot-product scores and an exact softmax over the group's
                selected original tokens.
* gate       -- same section: each head's result scaled by the sigmoid of its
                own gate logit (one per token and head).

Inputs are taken exactly as the GPU sees them (BF16 or FP32 values widened to
float64).  All accumulation is float64.

Parity pins: every function here is pinned by tests under ``tests/`` against
closed forms, invariants, library routines (torch's BF16/E4M3 casts, torch's
scaled_dot_product_attention, Python's sorted) or brute force.  No function is
parity unpinned; ``token_coverage`` implements this build's reading of a
measure the pages leave undefined (see its docstring).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_fp32", "round_bf16", "round_e4m3", "e4m3_encode", "e4m3_decode",
    "merge_block", "merge_blocks", "store_codes", "index_scores",
    "select_topk", "attended_positions", "sparse_attention", "gated_head_output",
    "forward_rows", "token_coverage", "E4M3_MAX",
]

E4M3_MAX = 448.0          # OCP FP8 E4M3: largest finite magnitude 1.75 * 2**8
E4M3_MIN_NORMAL_EXP = -6  # OCP FP8 E4M3: exponent bias 7, smallest normal 2**-6
E4M3_MANT_BITS = 3


# ---------------------------------------------------------------------------
# Storage roundings (section "Eight tokens become one search key ...": FP32
# accumulation, rounded through BF16 into E4M3 for storage).
# ---------------------------------------------------------------------------

def round_fp32(x) -> np.ndarray:
    """Round to IEEE binary32 (round to nearest even), returned as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round to BF16 with round-to-nearest-even, returned as float64.

    The value is first rounded to binary32 (BF16 conversion is defined from
    binary32), then its low 16 mantissa bits are rounded away: add 0x7FFF plus
    the lowest kept bit, truncate.  NaN stays NaN.
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    rounded = ((bits + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    out = rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(np.isnan(f), np.nan, out)


def round_e4m3(x) -> np.ndarray:
    """Round to OCP FP8 E4M3 ("fn": no infinities), nearest-even, saturating.

    E4M3 has exponent bias 7, three mantissa bits, subnormals with quantum
    2**-9, and largest finite magnitude 448.  Magnitudes above 448 saturate to
    448 (the "satfinite" store); NaN stays NaN.  Within a binade [2**e, 2**(e+1))
    (e >= -6) the quantum is 2**(e-3); below 2**-6 it is 2**-9.  Division by a
    power of two is exact in float64, and np.rint rounds halves to even.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, E4M3_MIN_NORMAL_EXP)
    quantum = np.exp2(e - E4M3_MANT_BITS)
    q = np.rint(a / quantum) * quantum
    q = np.minimum(q, E4M3_MAX)
    out = np.copysign(q, x)
    return np.where(np.isnan(x), np.nan, out)


def e4m3_encode(v) -> np.ndarray:
    """Bit pattern (uint8) of E4M3 values (inputs must already be E4M3 values)."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint8) << 7
    a = np.abs(v)
    sub = a < 2.0 ** E4M3_MIN_NORMAL_EXP
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.floor(np.log2(np.where(sub, 1.0, a)))
        mant_norm = np.rint((a / np.exp2(e) - 1.0) * 8.0)
    exp_field = np.where(sub, 0, e + 7)
    mant = np.where(sub, np.rint(a / 2.0 ** -9), mant_norm)
    code = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(np.isnan(v), 0x7F, code)
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """Value (float64) of E4M3 bit patterns; 0x7F/0xFF decode to NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.exp2(ef - 7.0) * (1.0 + m / 8.0)
    sub = m * 2.0 ** -9
    val = s * np.where(ef == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


# ---------------------------------------------------------------------------
# Stage 1: block-wise token merging
# ---------------------------------------------------------------------------

def merge_block(kp_blk, c_blk) -> np.ndarray:
    """Merge one completed block: [B, Di] proxy keys and logits -> [Di].

    Section "Eight tokens become one search key, coordinate by coordinate":
    for each coordinate d separately, weights softmax_j(c[j, d]) with the
    common maximum max_j c[j, d] subtracted before exponentiation, applied to
    the proxy-key coordinates kp[j, d].
    """
    kp_blk = np.asarray(kp_blk, dtype=np.float64)
    c_blk = np.asarray(c_blk, dtype=np.float64)
    m = c_blk.max(axis=0, keepdims=True)
    e = np.exp(c_blk - m)
    return (e * kp_blk).sum(axis=0) / e.sum(axis=0)


def merge_blocks(kp, c, block) -> np.ndarray:
    """Merge every completed block of a sequence: [L, Di] -> [L // B, Di]."""
    kp = np.asarray(kp, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    n_blocks = kp.shape[0] // block
    out = np.empty((n_blocks, kp.shape[1]), dtype=np.float64)
    for r in range(n_blocks):
        out[r] = merge_block(kp[r * block:(r + 1) * block], c[r * block:(r + 1) * block])
    return out


def store_codes(merged) -> np.ndarray:
    """E4M3 storage codes of merged keys: FP32 result -> BF16 -> E4M3 (uint8).

    Section "Eight tokens become one search key ...": the reduction is held in
    FP32 and rounded through BF16 into E4M3 for storage.
    """
    return e4m3_encode(round_e4m3(round_bf16(round_fp32(merged))))


# ---------------------------------------------------------------------------
# Stage 2: weighted-ReLU indexer score
# ---------------------------------------------------------------------------

def index_scores(q_idx, w_idx, keys) -> np.ndarray:
    """Scores of one (query t, group g) against candidate keys.

    q_idx [H, Di] indexer query heads, w_idx [H] signed head weights (prescale
    already inside), keys [R, Di] widened store values.  Section "Selection is
    a weighted ReLU score, not attention softmax":
        I[r] = sum_i w[i] * max(0, sum_d q[i, d] * keys[r, d]).
    """
    q_idx = np.asarray(q_idx, dtype=np.float64)
    w_idx = np.asarray(w_idx, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    dots = keys @ q_idx.T                      # [R, H]
    return np.maximum(dots, 0.0) @ w_idx       # [R]


# ---------------------------------------------------------------------------
# Stage 3: causal top-k selection, ties to the smaller block id
# ---------------------------------------------------------------------------

def select_topk(scores, k) -> np.ndarray:
    """Ascending ids of the k best candidates (score descending, id ascending).

    ``scores`` holds the scores of candidates 0..n-1 (already restricted to the
    causal candidates r < floor(t/B)).  With fewer than k candidates every
    candidate is selected.  -0.0 and +0.0 compare equal (float comparison).
    """
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    ids = np.arange(n)
    # np.lexsort sorts by the last key first: primary -score, secondary id.
    order = np.lexsort((ids, -scores + 0.0))
    return np.sort(order[:min(k, n)]).astype(np.int64)


def attended_positions(t, sel, block) -> np.ndarray:
    """Token positions attended by query t: selected blocks plus the current one.

    Section "Selection is a weighted ReLU score ...": every token of each
    selected historical block, then the block containing t restricted to its
    causally visible positions B*floor(t/B) .. t.
    """
    sel = np.asarray(sel, dtype=np.int64)
    hist = (sel[:, None] * block + np.arange(block)[None, :]).reshape(-1)
    cur = np.arange(block * (t // block), t + 1)
    return np.concatenate([hist, cur])


# ---------------------------------------------------------------------------
# Stage 4: exact softmax attention over the selected original tokens
# ---------------------------------------------------------------------------

def sparse_attention(q_heads, k_rows, v_rows, scale) -> np.ndarray:
    """Attention of a group's query heads over gathered original K/V rows.

    q_heads [Hg, D], k_rows/v_rows [S, D] (the attended positions of the
    group).  Section "Main attention still reads original K/V": scaled dot
    products, softmax over the selected tokens only, weighted sum of V.
    """
    q_heads = np.asarray(q_heads, dtype=np.float64)
    k_rows = np.asarray(k_rows, dtype=np.float64)
    v_rows = np.asarray(v_rows, dtype=np.float64)
    logits = (q_heads @ k_rows.T) * scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v_rows


def gated_head_output(head_out, gate_logit) -> np.ndarray:
    """Head-wise sigmoid gate on the attention output.

    Section "Main attention still reads original K/V": the attention result of
    a head is sigmoid-gated before the heads are concatenated and projected.
    Reading (the section gives no shape): one gate logit per (token, head),
    as the head-wise attention gate of the same vendor's Step 3.5 Flash
    configuration table ("Every architecture field") states.
    head_out [..., D], gate_logit [...] -> sigmoid(gate_logit) * head_out.
    """
    g = np.asarray(gate_logit, dtype=np.float64)
    return (1.0 / (1.0 + np.exp(-g)))[..., None] * np.asarray(head_out, dtype=np.float64)


# ---------------------------------------------------------------------------
# The whole path for a set of query rows
# ---------------------------------------------------------------------------

def forward_rows(rows, *, q, k, v, idx_q, idx_w, keys, block, topk,
                 heads_per_group, scale=None, q_pos0=0):
    """Selection and output for chosen query rows of one sequence.

    rows      iterable of (i, g): query index within the arrays below and KV group
    q         [nq, G*Hg, D] main queries (query i sits at position q_pos0 + i)
    k, v      [L, G, D] original cache (L >= q_pos0 + nq)
    idx_q     [nq, G, H, Di], idx_w [nq, G, H]
    keys      [R, Di] widened store values (E4M3 decoded), R >= floor(t/B)
    Returns {(i, g): (sel ids, out [Hg, D])}.
    """
    D = q.shape[-1]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    res = {}
    for (i, g) in rows:
        t = q_pos0 + i
        n_cand = t // block
        scores = index_scores(idx_q[i, g], idx_w[i, g], keys[:n_cand])
        sel = select_topk(scores, topk)
        pos = attended_positions(t, sel, block)
        hs = slice(g * heads_per_group, (g + 1) * heads_per_group)
        out = sparse_attention(q[i, hs], k[pos, g], v[pos, g], scale)
        res[(i, g)] = (sel, out)
    return res


def token_coverage(q_heads, k_all, positions, scale) -> float:
    """Dense-softmax mass that the attended positions capture.

    The second page reports token coverage for B=8,k=4096 against B=1,k=2048
    without defining it.  Reading adopted here: for one query row, the mean over
    the group's heads of the causal dense softmax probability mass that falls on
    the attended positions.  k_all holds the K rows of positions 0..t.  The
    definition is this reading; the pins check its implementation (full set,
    complements, equal logits, torch's softmax).
    """
    q_heads = np.asarray(q_heads, dtype=np.float64)
    k_all = np.asarray(k_all, dtype=np.float64)
    logits = (q_heads @ k_all.T) * scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return float(p[:, np.asarray(positions)].sum(axis=1).mean())
