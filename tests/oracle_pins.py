"""Pins for the fp64 oracle: facts the pages and the mathematics fix.

Every pin takes an ``oracle.Oracle`` handle and raises ``AssertionError`` when
the handle disagrees with the fact.  ``test_oracle_pins.py`` runs them on the
real oracle; ``test_oracle_mutants.py`` runs them on copies of the oracle with
a planted mistake and requires that each mistake fails at least one pin.

None of these re-types the oracle's formula: each one checks a closed form, a
count the pages state, an invariant, a hand-derived value (``golden/``), or a
special case that a library routine (torch's scaled_dot_product_attention in
float64) computes on its own.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NEG_INF = -math.inf


def _rng(seed):
    return np.random.default_rng(seed)


def _visible_count(p, window, k_len):
    """Keys visible from absolute position p: interval [max(0,p-w+1), min(p, k_len-1)]."""
    lo = max(0, p - window + 1) if window > 0 else 0
    hi = min(p, k_len - 1)
    return max(0, hi - lo + 1)


# --------------------------------------------------------------------------------------
# mlx-arsenal "Attention" page: causal_mask / sliding_window_mask
# --------------------------------------------------------------------------------------

def pin_causal_mask_shape_and_rows(orc):
    """Shape (1,1,S,offset+S); entries 0/-inf; lower-triangular with a KV offset:
    row i sees the offset cached keys plus queries 0..i, so offset+i+1 zeros that
    form a prefix, and the last row sees every key."""
    for S in range(1, 13):
        for offset in range(0, 6):
            m = orc.causal_mask(S, offset)
            assert m.shape == (1, 1, S, offset + S)
            m = m[0, 0]
            assert np.all((m == 0.0) | (m == NEG_INF))
            for i in range(S):
                zeros = np.flatnonzero(m[i] == 0.0)
                assert len(zeros) == offset + i + 1, (S, offset, i, len(zeros))
                assert np.array_equal(zeros, np.arange(offset + i + 1))
            assert np.all(m[S - 1] == 0.0)


def pin_sliding_window_rows(orc):
    """Each row sees at most window_size keys, itself included, ending on its own
    position; a window at least as long as the sequence is the causal mask."""
    for S in range(1, 11):
        for offset in range(0, 4):
            for w in range(1, S + offset + 2):
                m = orc.sliding_window_mask(S, w, offset)
                assert m.shape == (1, 1, S, offset + S)
                m = m[0, 0]
                assert np.all((m == 0.0) | (m == NEG_INF))
                for i in range(S):
                    zeros = np.flatnonzero(m[i] == 0.0)
                    assert len(zeros) == min(w, offset + i + 1), (S, offset, w, i)
                    assert zeros[-1] == offset + i
                    assert np.all(np.diff(zeros) == 1)
                if w >= S + offset:
                    assert np.array_equal(m, orc.causal_mask(S, offset)[0, 0])


# --------------------------------------------------------------------------------------
# Tylo.jl "Primitives" page: attention!
# --------------------------------------------------------------------------------------

def pin_two_key_golden(orc):
    """Hand-derived values in golden/two_key_softmax.json."""
    with open(os.path.join(GOLDEN, "two_key_softmax.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], dtype=np.float64)[None, None]          # (1,1,1,1)
    k = np.array(g["k"], dtype=np.float64)[None, None]          # (1,1,2,1)
    v = np.array(g["v"], dtype=np.float64)[None, None]
    for case in g["cases"]:
        O, L = orc.attn_fwd(q, k, v, math.log(3.0), causal=case["causal"],
                            input_pos=case["input_pos"])
        assert abs(O[0, 0, 0, 0] - case["O"][0]) < 1e-12, (case, O)
        assert abs(L[0, 0, 0] - math.log(case["LSE_is_ln"])) < 1e-12, (case, L)


def pin_probability_rows(orc):
    """With V = identity the output rows are the probability rows: each sums to 1,
    is >= 0, and is exactly 0 where the page-1 mask is -inf."""
    rng = _rng(1)
    for causal, window, offset, S in [(True, 0, 0, 7), (True, 0, 3, 6), (True, 3, 2, 8),
                                      (False, 0, 0, 5), (True, 1, 4, 4)]:
        Sk = offset + S
        D = Sk
        Q = rng.standard_normal((1, 2, S, D))
        K = rng.standard_normal((1, 1, Sk, D))
        V = np.eye(Sk)[None, None]
        O, _ = orc.attn_fwd(Q, K, V, 0.7, causal=causal, window=window, input_pos=offset)
        P = O
        assert np.all(P >= 0.0)
        assert np.allclose(P.sum(-1), 1.0, atol=1e-12, rtol=0)
        if causal:
            m = (orc.sliding_window_mask(S, window, offset) if window
                 else orc.causal_mask(S, offset))[0, 0]
            assert np.all(P[0, :, m == NEG_INF] == 0.0)
            assert np.all(P[0, :, m == 0.0] > 0.0)


def pin_constant_v(orc):
    """A constant V row gives that row as output for every row that sees a key."""
    rng = _rng(2)
    B, Hq, Hkv, S, D = 2, 4, 2, 9, 5
    vrow = rng.standard_normal(D)
    Q = rng.standard_normal((B, Hq, S, D))
    K = rng.standard_normal((B, Hkv, S, D))
    V = np.broadcast_to(vrow, (B, Hkv, S, D)).copy()
    for causal, window in [(False, 0), (True, 0), (True, 3)]:
        O, _ = orc.attn_fwd(Q, K, V, 0.9, causal=causal, window=window)
        assert np.allclose(O, vrow, atol=1e-12, rtol=0)


def pin_causal_row0(orc):
    """Causal, input_pos 0: query row 0 sees only key 0, so O[0] = V[0] exactly."""
    rng = _rng(3)
    Q = rng.standard_normal((1, 3, 6, 4))
    K = rng.standard_normal((1, 3, 6, 4))
    V = rng.standard_normal((1, 3, 6, 4))
    O, L = orc.attn_fwd(Q, K, V, 0.5, causal=True)
    assert np.array_equal(O[0, :, 0, :], V[0, :, 0, :])
    s00 = 0.5 * np.einsum("hd,hd->h", Q[0, :, 0], K[0, :, 0])
    assert np.allclose(L[0, :, 0], s00, atol=1e-12, rtol=0)


def pin_uniform_attention(orc):
    """K = 0 makes every visible score equal, so O_i is the mean of the visible V
    rows and LSE_i = ln(number of visible keys); rows that see nothing give O = 0
    and LSE = -inf.  Counts come from interval arithmetic on the definitions."""
    rng = _rng(4)
    B, Hq, Hkv, Sq, Sk, D = 3, 4, 2, 11, 14, 3
    Q = rng.standard_normal((B, Hq, Sq, D))
    K = np.zeros((B, Hkv, Sk, D))
    V = rng.standard_normal((B, Hkv, Sk, D))
    k_len = np.array([14, 5, 0], dtype=np.int32)
    q_len = np.array([11, 7, 11], dtype=np.int32)
    for causal, window, input_pos in [(False, 0, 0), (True, 0, 3), (True, 4, 2), (True, 1, 0)]:
        O, L = orc.attn_fwd(Q, K, V, 1.3, causal=causal, window=window, input_pos=input_pos,
                            k_lengths=k_len, q_lengths=q_len)
        for b in range(B):
            for hq in range(Hq):
                hkv = hq // (Hq // Hkv)
                for i in range(Sq):
                    p = input_pos + i
                    if i >= q_len[b]:
                        n = 0
                    elif causal:
                        n = _visible_count(p, window, min(k_len[b], Sk))
                        lo = max(0, p - window + 1) if window > 0 else 0
                    else:
                        n = int(min(k_len[b], Sk))
                        lo = 0
                    if n == 0:
                        assert np.all(O[b, hq, i] == 0.0) and L[b, hq, i] == NEG_INF
                        continue
                    mean = V[b, hkv, lo:lo + n].mean(0)
                    assert np.allclose(O[b, hq, i], mean, atol=1e-12, rtol=0), (b, hq, i)
                    assert abs(L[b, hq, i] - math.log(n)) < 1e-12


def pin_gqa_repeat(orc):
    """GQA equals MHA on K/V heads repeated Hq/Hkv times (consecutive groups)."""
    rng = _rng(5)
    B, Hq, Hkv, Sq, Sk, D = 2, 6, 2, 5, 8, 4
    Q = rng.standard_normal((B, Hq, Sq, D))
    K = rng.standard_normal((B, Hkv, Sk, D))
    V = rng.standard_normal((B, Hkv, Sk, D))
    Kr = np.repeat(K, Hq // Hkv, axis=1)
    Vr = np.repeat(V, Hq // Hkv, axis=1)
    for causal, window, input_pos in [(False, 0, 0), (True, 0, 3), (True, 2, 3)]:
        O1, L1 = orc.attn_fwd(Q, K, V, 0.8, causal=causal, window=window, input_pos=input_pos)
        O2, L2 = orc.attn_fwd(Q, Kr, Vr, 0.8, causal=causal, window=window, input_pos=input_pos)
        assert np.allclose(O1, O2, atol=1e-13, rtol=0)
        assert np.allclose(L1, L2, atol=1e-13, rtol=0)


def _sdpa(Q, K, V, scale, allowed):
    q = torch.from_numpy(Q)
    k = torch.from_numpy(K)
    v = torch.from_numpy(V)
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=torch.from_numpy(allowed), scale=scale).numpy()


def pin_library_sdpa(orc):
    """Against torch's scaled_dot_product_attention in float64 with the page-1
    masks (causal_mask / sliding_window_mask with the KV offset) as the boolean
    mask, on rows that see at least one key; K/V heads repeated for GQA."""
    rng = _rng(6)
    cases = [  # B, Hq, Hkv, S, offset, D, causal, window
        (2, 4, 2, 9, 0, 16, False, 0),
        (1, 4, 1, 7, 5, 8, True, 0),
        (2, 2, 2, 12, 0, 8, True, 4),
        (1, 6, 3, 6, 9, 32, True, 5),
    ]
    for B, Hq, Hkv, S, offset, D, causal, window in cases:
        Sk = offset + S
        Q = rng.standard_normal((B, Hq, S, D))
        K = rng.standard_normal((B, Hkv, Sk, D))
        V = rng.standard_normal((B, Hkv, Sk, D))
        scale = 1.0 / math.sqrt(D)
        O, _ = orc.attn_fwd(Q, K, V, scale, causal=causal, window=window, input_pos=offset)
        if causal:
            m = (orc.sliding_window_mask(S, window, offset) if window
                 else orc.causal_mask(S, offset))[0, 0]
            allowed = (m == 0.0)
        else:
            allowed = np.ones((S, Sk), dtype=bool)
        ref = _sdpa(Q, np.repeat(K, Hq // Hkv, 1), np.repeat(V, Hq // Hkv, 1), scale, allowed)
        assert np.allclose(O, ref, atol=1e-12, rtol=0), np.abs(O - ref).max()


def pin_lse_matches_probabilities(orc):
    """LSE is the log normaliser: P_ij = exp(s_ij - LSE_i) for the probabilities read
    out with V = identity, and max_j s_ij <= LSE_i <= max_j s_ij + ln(n_i)."""
    rng = _rng(7)
    S, offset = 6, 2
    Sk = S + offset
    D = Sk
    Q = rng.standard_normal((1, 1, S, D))
    K = rng.standard_normal((1, 1, Sk, D))
    P, L = orc.attn_fwd(Q, K, np.eye(Sk)[None, None], 1.1, causal=True, input_pos=offset)
    s = 1.1 * (Q[0, 0] @ K[0, 0].T)
    for i in range(S):
        vis = np.arange(Sk) <= offset + i
        assert np.all(P[0, 0, i, vis] > 0.0)
        logp = np.log(P[0, 0, i, vis])
        assert np.allclose(logp + L[0, 0, i], s[i, vis], atol=1e-12, rtol=0)
        smax = s[i, vis].max()
        assert smax - 1e-12 <= L[0, 0, i] <= smax + math.log(vis.sum()) + 1e-12


def pin_lengths_are_prefixes(orc):
    """k_lengths = L equals dropping keys L.. ; rows at or past q_lengths are O = 0,
    LSE = -inf, and the rows before them are unchanged."""
    rng = _rng(8)
    B, Hq, Hkv, S, D = 2, 2, 1, 10, 6
    Q = rng.standard_normal((B, Hq, S, D))
    K = rng.standard_normal((B, Hkv, S, D))
    V = rng.standard_normal((B, Hkv, S, D))
    k_len = np.array([6, 10], dtype=np.int32)
    q_len = np.array([10, 4], dtype=np.int32)
    for causal in (False, True):
        O, L = orc.attn_fwd(Q, K, V, 0.6, causal=causal, k_lengths=k_len, q_lengths=q_len)
        for b in range(B):
            Ob, Lb = orc.attn_fwd(Q[b:b + 1], K[b:b + 1, :, :k_len[b]], V[b:b + 1, :, :k_len[b]],
                                  0.6, causal=causal)
            ql = q_len[b]
            assert np.allclose(O[b, :, :ql], Ob[0, :, :ql], atol=1e-13, rtol=0)
            assert np.allclose(L[b, :, :ql], Lb[0, :, :ql], atol=1e-13, rtol=0)
            assert np.all(O[b, :, ql:] == 0.0) and np.all(L[b, :, ql:] == NEG_INF)


def pin_row_subset(orc):
    """Computing a subset of query rows gives those rows of the full result."""
    rng = _rng(9)
    B, Hq, Hkv, S, D = 1, 4, 2, 13, 4
    Q = rng.standard_normal((B, Hq, S, D))
    K = rng.standard_normal((B, Hkv, S, D))
    V = rng.standard_normal((B, Hkv, S, D))
    rows = np.array([0, 5, 12, 7], dtype=np.int32)
    O, L = orc.attn_fwd(Q, K, V, 0.4, causal=True, window=3, input_pos=2)
    Os, Ls = orc.attn_fwd(Q[:, :, rows], K, V, 0.4, causal=True, window=3, input_pos=2,
                          rows=rows, Sq=S)
    assert np.array_equal(Os, O[:, :, rows]) and np.array_equal(Ls, L[:, :, rows])


# --------------------------------------------------------------------------------------
# Tylo.jl "Primitives" page: decode_attention!
# --------------------------------------------------------------------------------------

def pin_decode_is_last_row_of_prefill(orc):
    """Single-token decode is causal attention of one query at absolute position
    len-1 over the first len cached keys, with the default scale 1/sqrt(D)."""
    rng = _rng(10)
    B, Hq, Hkv, S_cap, D = 3, 4, 2, 12, 8
    Q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, S_cap, D))
    V = rng.standard_normal((B, Hkv, S_cap, D))
    lengths = np.array([12, 1, 7], dtype=np.int32)
    O, L = orc.decode(Q, K, V, lengths)
    for b in range(B):
        n = int(lengths[b])
        Op, Lp = orc.attn_fwd(Q[b:b + 1, :, None, :], K[b:b + 1], V[b:b + 1],
                              1.0 / math.sqrt(D), causal=True, input_pos=n - 1)
        assert np.allclose(O[b], Op[0, :, 0], atol=1e-13, rtol=0)
        assert np.allclose(L[b], Lp[0, :, 0], atol=1e-13, rtol=0)


def pin_decode_closed_forms(orc):
    """Decode with K = 0 averages the first len V rows (LSE = ln len); a constant V
    comes back unchanged; len = 0 gives O = 0, LSE = -inf; the scale is 1/sqrt(D)
    (a single key with q.k = sqrt(D) has LSE exactly 1)."""
    rng = _rng(11)
    B, Hq, Hkv, S_cap, D = 3, 2, 1, 9, 16
    Q = rng.standard_normal((B, Hq, D))
    V = rng.standard_normal((B, Hkv, S_cap, D))
    lengths = np.array([9, 3, 0], dtype=np.int32)
    O, L = orc.decode(Q, np.zeros((B, Hkv, S_cap, D)), V, lengths)
    for b in range(B):
        n = int(lengths[b])
        if n == 0:
            assert np.all(O[b] == 0.0) and np.all(L[b] == NEG_INF)
            continue
        assert np.allclose(O[b], V[b, 0, :n].mean(0), atol=1e-12, rtol=0)
        assert np.allclose(L[b], math.log(n), atol=1e-12, rtol=0)
    vrow = rng.standard_normal(D)
    Vc = np.broadcast_to(vrow, (B, Hkv, S_cap, D)).copy()
    O, _ = orc.decode(Q, rng.standard_normal((B, Hkv, S_cap, D)), Vc, np.array([9, 4, 1]))
    assert np.allclose(O, vrow, atol=1e-12, rtol=0)
    # q = 1, k0 = 1/sqrt(D): q.k0 = sqrt(D), times the scale 1/sqrt(D) gives 1, and
    # one visible key makes LSE equal to that score.
    q1 = np.ones((1, 1, D))
    k1 = np.zeros((1, 1, 2, D))
    k1[0, 0, 0] = 1.0 / math.sqrt(D)
    _, L1 = orc.decode(q1, k1, np.zeros((1, 1, 2, D)), np.array([1]))
    assert abs(L1[0, 0] - 1.0) < 1e-12, L1


# --------------------------------------------------------------------------------------
# Tylo.jl "Primitives" page: flex_attention! score and mask mods
# --------------------------------------------------------------------------------------

def pin_flex_golden(orc):
    """Hand-derived soft-cap and ALiBi values in golden/flex_score_mods.json."""
    with open(os.path.join(GOLDEN, "flex_score_mods.json")) as f:
        g = json.load(f)
    sc = g["softcap"]
    q = np.array(sc["q"], dtype=np.float64)[None, None]
    k = np.array(sc["k"], dtype=np.float64)[None, None]
    v = np.array(sc["v"], dtype=np.float64)[None, None]
    ln3 = math.log(3.0)
    O, L = orc.flex_fwd(q, k, v, ln3 * ln3, softcap=2.0 * ln3)
    assert abs(O[0, 0, 0, 0] - sc["O"][0]) < 1e-12, O
    assert abs(L[0, 0, 0] - math.log(sc["LSE_is_ln"])) < 1e-12, L
    al = g["alibi"]
    Sk, row = al["Sk"], al["row"]
    slopes = np.array(al["slopes_in_units_of_ln2"]) * math.log(2.0)
    Q = np.zeros((1, 2, Sk, Sk))
    K = np.zeros((1, 1, Sk, Sk))
    V = np.eye(Sk)[None, None]
    O, L = orc.flex_fwd(Q, K, V, 0.7, causal=True, alibi_slopes=slopes)
    for h in range(2):
        assert np.allclose(O[0, h, row], al["p"][h], rtol=0, atol=1e-12), (h, O[0, h, row])
        assert abs(L[0, h, row] - math.log(al["LSE_is_ln"][h])) < 1e-12, (h, L[0, h, row])


def pin_flex_softcap_limits(orc):
    """A cap far above every score changes nothing (cap * tanh(s / cap) -> s): the
    result equals attention! without a score mod.  A cap far below every score
    flattens them to ~0: uniform weights over the visible keys, LSE = ln(count)."""
    rng = _rng(21)
    Q, K, V = rng.standard_normal((2, 4, 9, 8)), rng.standard_normal((2, 2, 11, 8)), \
        rng.standard_normal((2, 2, 11, 8))
    O0, L0 = orc.attn_fwd(Q, K, V, 0.4, causal=True, input_pos=2)
    O1, L1 = orc.flex_fwd(Q, K, V, 0.4, causal=True, input_pos=2, softcap=1e9)
    assert np.max(np.abs(O1 - O0)) < 1e-9 and np.max(np.abs(L1 - L0)) < 1e-9
    O2, L2 = orc.flex_fwd(Q, K, V, 0.4, causal=True, input_pos=2, softcap=1e-12)
    for i in range(9):
        n = i + 3  # keys 0 .. input_pos + i
        mean = V[:, :, :n].mean(axis=2)  # (B, Hkv, D)
        assert np.allclose(O2[:, :, i], np.repeat(mean, 2, axis=1), rtol=0, atol=1e-9)
        assert np.allclose(L2[:, :, i], math.log(n), rtol=0, atol=1e-9)


def pin_flex_alibi_geometric(orc):
    """With K = 0 the ALiBi scores are slope * (q - j): the weights over the visible
    keys of a causal row are geometric, p_j = r^(q-j) / sum_k r^(q-k) with
    r = exp(slope), and LSE = ln sum_k r^(q-k).  Checked per query head (GQA group
    of 3 sharing one KV head, three different slopes) and with input_pos > 0."""
    Sk, input_pos, Sq = 7, 3, 4
    slopes = np.array([0.35, -0.6, 1.1])
    Q = np.zeros((1, 3, Sq, Sk))
    K = np.zeros((1, 1, Sk, Sk))
    V = np.eye(Sk)[None, None]
    O, L = orc.flex_fwd(Q, K, V, 1.3, causal=True, input_pos=input_pos, alibi_slopes=slopes)
    for h in range(3):
        r = math.exp(slopes[h])
        for i in range(Sq):
            q = input_pos + i
            w = np.array([r ** (q - j) if j <= q else 0.0 for j in range(Sk)])
            assert np.allclose(O[0, h, i], w / w.sum(), rtol=0, atol=1e-12), (h, i)
            assert abs(L[0, h, i] - math.log(w.sum())) < 1e-12, (h, i)


def pin_flex_document_blocks(orc):
    """DocumentMask over contiguous documents (ids per position) with the causal
    mask is block-diagonal: each document's rows equal attention! run on that
    document alone (its own queries, keys and values, causal, input_pos 0).
    Also with GQA (4 query heads on 2 KV heads) and a sliding window."""
    rng = _rng(22)
    lens = [5, 1, 9, 3, 6]
    S = sum(lens)
    doc = np.repeat(np.arange(len(lens)), lens)
    Q, K, V = rng.standard_normal((2, 4, S, 8)), rng.standard_normal((2, 2, S, 8)), \
        rng.standard_normal((2, 2, S, 8))
    for window in (0, 4):
        O, L = orc.flex_fwd(Q, K, V, 0.35, causal=True, window=window, doc_q=doc, doc_kv=doc)
        a = 0
        for n in lens:
            sl = slice(a, a + n)
            Od, Ld = orc.attn_fwd(Q[:, :, sl], K[:, :, sl], V[:, :, sl], 0.35, causal=True,
                                  window=window)
            assert np.max(np.abs(O[:, :, sl] - Od)) < 1e-12, (window, a, n)
            assert np.max(np.abs(L[:, :, sl] - Ld)) < 1e-12, (window, a, n)
            a += n


# --------------------------------------------------------------------------------------
# vllm-mlx "attention" page: paged KV cache (num_blocks, block_size, num_kv_heads,
# head_size) with block tables, decoded with decode_attention!
# --------------------------------------------------------------------------------------

def _scatter_paged(K, V, lengths, block_size, rng, extra_blocks=3):
    """Scatter contiguous caches (B, Hkv, S_cap, D) into a shuffled block pool."""
    B, Hkv, S_cap, D = K.shape
    max_blocks = -(-S_cap // block_size)
    n_blocks = B * max_blocks + extra_blocks
    perm = rng.permutation(n_blocks)[:B * max_blocks].reshape(B, max_blocks)
    Kc = rng.standard_normal((n_blocks, block_size, Hkv, D))
    Vc = rng.standard_normal((n_blocks, block_size, Hkv, D))
    for b in range(B):
        for lb in range(max_blocks):
            j0, j1 = lb * block_size, min((lb + 1) * block_size, S_cap)
            Kc[perm[b, lb], :j1 - j0] = K[b, :, j0:j1].transpose(1, 0, 2)
            Vc[perm[b, lb], :j1 - j0] = V[b, :, j0:j1].transpose(1, 0, 2)
    return Kc, Vc, perm.astype(np.int32)


def pin_paged_equals_contiguous(orc):
    """A cache scattered into shuffled blocks and read back through the block table
    decodes exactly like the contiguous cache (decode_attention!), for several
    block sizes, with GQA, and for lengths 0, 1, block edges and the capacity."""
    rng = _rng(31)
    B, Hq, Hkv, S_cap, D = 5, 6, 2, 37, 8
    Q = rng.standard_normal((B, Hq, D))
    K, V = rng.standard_normal((B, Hkv, S_cap, D)), rng.standard_normal((B, Hkv, S_cap, D))
    lengths = np.array([0, 1, 16, 33, 37], dtype=np.int32)
    O0, L0 = orc.decode(Q, K, V, lengths)
    for bs in (1, 4, 16, 64):
        Kc, Vc, bt = _scatter_paged(K, V, lengths, bs, rng)
        O1, L1 = orc.decode_paged(Q, Kc, Vc, bt, lengths)
        assert np.max(np.abs(O1 - O0)) < 1e-12, bs
        assert np.array_equal(np.isneginf(L1), np.isneginf(L0))
        fin = ~np.isneginf(L0)
        assert np.max(np.abs(L1[fin] - L0[fin])) < 1e-12, bs


def pin_paged_reads_only_listed_slots(orc):
    """Blocks the table does not reach, and slots past a sequence's length, may hold
    anything (here NaN): the result stays finite and equal."""
    rng = _rng(32)
    B, Hq, Hkv, S_cap, D, bs = 3, 4, 4, 20, 8, 8
    Q = rng.standard_normal((B, Hq, D))
    K, V = rng.standard_normal((B, Hkv, S_cap, D)), rng.standard_normal((B, Hkv, S_cap, D))
    lengths = np.array([5, 20, 9], dtype=np.int32)
    Kc, Vc, bt = _scatter_paged(K, V, lengths, bs, rng)
    O0, L0 = orc.decode_paged(Q, Kc, Vc, bt, lengths)
    used = np.zeros(Kc.shape[:2], dtype=bool)
    for b in range(B):
        for j in range(lengths[b]):
            used[bt[b, j // bs], j % bs] = True
    Kc[~used] = np.nan
    Vc[~used] = np.nan
    O1, L1 = orc.decode_paged(Q, Kc, Vc, bt, lengths)
    assert np.all(np.isfinite(O1)) and np.array_equal(O1, O0) and np.array_equal(L1, L0)


# --------------------------------------------------------------------------------------
# mlx-arsenal "Radius-bounded block scores (RBS)" page: block scores and block mask;
# block-sparse attention from a per-head block mask
# --------------------------------------------------------------------------------------

def pin_rbs_closed_form(orc):
    """Key blocks built as c_b +/- delta_b e_1 (32 keys each way) have centroid c_b and
    radius delta_b exactly; a query block of 64 identical tokens q scores
    ln 64 + <q, c_b>/sqrt(D) (base) and ln 64 + (<q, c_b> + |q| delta_b beta_b)/sqrt(D)
    (rescue), beta from the median and 90th percentile of the radii (numpy's
    linear-interpolation quantile) clipped to [0, 1].  GQA: both query heads of
    the KV head, with different q."""
    rng = _rng(41)
    D, nkb = 16, 10
    deltas = np.arange(1, nkb + 1, dtype=np.float64) * 0.5
    rng.shuffle(deltas)
    cents = rng.standard_normal((nkb, D))
    K = np.empty((1, 1, 64 * nkb, D))
    for b in range(nkb):
        sign = np.where(np.arange(64) % 2 == 0, 1.0, -1.0)
        K[0, 0, 64 * b:64 * b + 64] = cents[b] + np.outer(sign, np.eye(D)[0]) * deltas[b]
    qs = rng.standard_normal((2, D))
    Q = np.repeat(qs[None, :, None, :], 64, axis=2)  # (1, 2, 64, D)
    base, rescue = orc.rbs_block_scores(Q, K)
    lo, hi = np.quantile(deltas, 0.5), np.quantile(deltas, 0.9)
    beta = np.clip((deltas - lo) / (hi - lo), 0.0, 1.0)
    for h in range(2):
        q = qs[h]
        want_b = math.log(64) + cents @ q / math.sqrt(D)
        want_r = math.log(64) + (cents @ q + np.linalg.norm(q) * deltas * beta) / math.sqrt(D)
        assert np.allclose(base[0, h, 0], want_b, rtol=0, atol=1e-10), h
        assert np.allclose(rescue[0, h, 0], want_r, rtol=0, atol=1e-10), h


def pin_rbs_degenerate_and_gqa(orc):
    """Equal radii (the two quantiles coincide): no block is strictly wider, beta = 0,
    rescue = base.  GQA: scores with 4 query heads on 2 KV heads equal those with the
    KV heads repeated (4 on 4).  A short last block (Sq, Sk not multiples of 64)."""
    rng = _rng(42)
    D = 8
    K = np.tile(rng.standard_normal((1, 1, 1, D)), (1, 1, 130, 1))  # every block radius 0
    Q = rng.standard_normal((1, 2, 100, D))
    base, rescue = orc.rbs_block_scores(Q, K)
    assert np.array_equal(base, rescue)
    Q = rng.standard_normal((2, 4, 150, D))
    K = rng.standard_normal((2, 2, 200, D))
    b1, r1 = orc.rbs_block_scores(Q, K)
    b2, r2 = orc.rbs_block_scores(Q, np.repeat(K, 2, axis=1))
    assert np.max(np.abs(b1 - b2)) < 1e-12 and np.max(np.abs(r1 - r2)) < 1e-12


def pin_rbs_relative_mask_golden(orc):
    """Hand-derived union of the two relative masks and the band
    (golden/rbs_relative_mask.json)."""
    with open(os.path.join(GOLDEN, "rbs_relative_mask.json")) as f:
        g = json.load(f)
    base = np.log(np.array(g["base_ratio"], dtype=np.float64))[None, None]
    rescue = np.log(np.array(g["rescue_ratio"], dtype=np.float64))[None, None]
    keep = orc.rbs_block_mask(base, rescue, g["alpha_base"], g["alpha_rescue"], g["diagonal"])
    assert np.array_equal(keep[0, 0], np.array(g["keep"], dtype=np.uint8)), keep


def pin_block_sparse_attention(orc):
    """Keeping every block is attention!; keeping only the 64x64 diagonal blocks is
    attention! on each 64-token block alone (per head: head 1 keeps everything)."""
    rng = _rng(43)
    S, D = 150, 8
    Q, K, V = rng.standard_normal((1, 2, S, D)), rng.standard_normal((1, 2, S, D)), \
        rng.standard_normal((1, 2, S, D))
    nb = (S + 63) // 64
    keep = np.ones((1, 2, nb, nb), dtype=np.uint8)
    O0, L0 = orc.attn_fwd(Q, K, V, 0.3)
    O1, L1 = orc.flex_fwd(Q, K, V, 0.3, block_keep=keep)
    assert np.max(np.abs(O1 - O0)) < 1e-12 and np.max(np.abs(L1 - L0)) < 1e-12
    keep[0, 0] = np.eye(nb, dtype=np.uint8)
    O2, L2 = orc.flex_fwd(Q, K, V, 0.3, block_keep=keep)
    assert np.max(np.abs(O2[0, 1] - O0[0, 1])) < 1e-12
    for a in range(0, S, 64):
        sl = slice(a, min(a + 64, S))
        Ob, Lb = orc.attn_fwd(Q[:, :1, sl], K[:, :1, sl], V[:, :1, sl], 0.3)
        assert np.max(np.abs(O2[:, :1, sl] - Ob)) < 1e-12 and np.max(np.abs(L2[:, :1, sl] - Lb)) < 1e-12


# --------------------------------------------------------------------------------------
# Tylo.jl "Primitives" page: ∇attention!
# --------------------------------------------------------------------------------------

def pin_bwd_finite_differences(orc):
    """Every gradient element equals the central difference of the loss sum(O * dO)
    through the forward oracle (causal with input_pos, a window, ragged lengths,
    GQA), to 1e-6."""
    rng = _rng(51)
    B, Hq, Hkv, Sq, Sk, D = 2, 2, 1, 4, 6, 3
    Q, K, V = rng.standard_normal((B, Hq, Sq, D)), rng.standard_normal((B, Hkv, Sk, D)), \
        rng.standard_normal((B, Hkv, Sk, D))
    dO = rng.standard_normal((B, Hq, Sq, D))
    kl, ql = np.array([6, 4], np.int32), np.array([4, 3], np.int32)
    for causal, window, ip in ((True, 0, 2), (True, 3, 1), (False, 0, 0)):
        kw = dict(causal=causal, window=window, input_pos=ip, k_lengths=kl, q_lengths=ql)
        dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, 0.6, **kw)

        def loss(Q_, K_, V_):
            O, _ = orc.attn_fwd(Q_, K_, V_, 0.6, **kw)
            return float((O * dO).sum())
        h = 1e-6
        for X, G, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
            for idx in np.ndindex(X.shape):
                Xp, Xm = X.copy(), X.copy()
                Xp[idx] += h
                Xm[idx] -= h
                args_p = [Q, K, V]
                args_m = [Q, K, V]
                args_p[which], args_m[which] = Xp, Xm
                fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
                assert abs(fd - G[idx]) < 1e-6, (causal, window, which, idx, fd, G[idx])


def pin_bwd_gqa_and_uniform(orc):
    """GQA: dK / dV of a KV head are the sums of the MHA gradients of its query heads
    on repeated K / V, and dQ is unchanged.  K = 0: uniform weights 1/n_i over the
    visible keys, so dV_j = sum over rows i that see j of dO_i / n_i and dQ = 0."""
    rng = _rng(52)
    B, Hq, Hkv, S, D = 1, 4, 2, 7, 5
    Q, K, V = rng.standard_normal((B, Hq, S, D)), rng.standard_normal((B, Hkv, S, D)), \
        rng.standard_normal((B, Hkv, S, D))
    dO = rng.standard_normal((B, Hq, S, D))
    dQ, dK, dV = orc.attn_bwd(Q, K, V, dO, 0.4, causal=True)
    mQ, mK, mV = orc.attn_bwd(Q, np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1), dO, 0.4,
                              causal=True)
    assert np.max(np.abs(dQ - mQ)) < 1e-12
    assert np.max(np.abs(dK - mK.reshape(B, Hkv, 2, S, D).sum(2))) < 1e-12
    assert np.max(np.abs(dV - mV.reshape(B, Hkv, 2, S, D).sum(2))) < 1e-12
    Kz = np.zeros_like(K)
    dQ, dK, dV = orc.attn_bwd(Q, Kz, V, dO, 0.4, causal=True, input_pos=2)
    assert np.max(np.abs(dQ)) < 1e-12
    want = np.zeros_like(V)
    for h in range(Hq):
        for i in range(S):
            n = i + 3  # keys 0 .. input_pos + i, capped by S
            n = min(n, S)
            want[0, h // 2, :n] += dO[0, h, i] / n
    assert np.max(np.abs(dV - want)) < 1e-12


def pin_visibility(orc):
    """attn_visible (the key set each row's scores keep) against three things:
    the page-1 causal_mask / sliding_window_mask of the same shape (visible ⇔
    entry 0); the keys attn_fwd itself weighs, read off with K = 0 and V = I (O[i,
    j] ≠ 0 ⇔ key j carries weight), with GQA, lengths, input_pos, a window and
    a row subset; and the decode key set, the first lengths[b] keys."""
    for S in range(1, 10):
        for offset in range(0, 4):
            vis = orc.attn_visible(1, S, offset + S, causal=True, input_pos=offset)[0]
            assert np.array_equal(vis == 1, orc.causal_mask(S, offset)[0, 0] == 0.0)
            for w in range(1, S + offset + 1):
                vis = orc.attn_visible(1, S, offset + S, causal=True, window=w,
                                       input_pos=offset)[0]
                m = orc.sliding_window_mask(S, w, offset)[0, 0]
                assert np.array_equal(vis == 1, m == 0.0), (S, offset, w)
    rng = _rng(31)
    B, Hq, Hkv, Sq, Sk = 3, 4, 2, 9, 13
    Q = rng.standard_normal((B, Hq, Sq, Sk))
    K = np.zeros((B, Hkv, Sk, Sk))
    V = np.broadcast_to(np.eye(Sk), (B, Hkv, Sk, Sk)).copy()
    k_len = np.array([13, 6, 0], dtype=np.int32)
    q_len = np.array([9, 4, 9], dtype=np.int32)
    for causal, window, input_pos, rows in [(False, 0, 0, None), (True, 0, 4, None),
                                            (True, 3, 2, None), (True, 1, 0, [0, 5, 8]),
                                            (True, 0, 0, [8, 2])]:
        kw = dict(causal=causal, window=window, input_pos=input_pos, k_lengths=k_len,
                  q_lengths=q_len)
        Qr = Q if rows is None else Q[:, :, rows]
        O, L = orc.attn_fwd(Qr, K, V, 0.7, rows=rows, Sq=Sq, **kw)
        vis = orc.attn_visible(B, Sq, Sk, rows=rows, **kw)
        n_rows = Sq if rows is None else len(rows)
        assert vis.shape == (B, n_rows, Sk) and vis.dtype == np.uint8
        assert set(np.unique(vis)) <= {0, 1}
        for hq in range(Hq):
            assert np.array_equal(O[:, hq] != 0.0, vis == 1), (causal, window, input_pos, hq)
        cnt = vis.sum(-1)
        for b in range(B):
            for r in range(n_rows):
                i = r if rows is None else rows[r]
                if i >= q_len[b]:
                    want = 0
                elif causal:
                    want = _visible_count(input_pos + i, window, int(k_len[b]))
                else:
                    want = int(k_len[b])
                assert cnt[b, r] == want, (b, i)
    lengths = np.array([0, 1, 7, 20], dtype=np.int32)
    vis = orc.attn_visible(4, 1, 20, k_lengths=lengths)
    for b, n in enumerate(lengths):
        assert np.array_equal(vis[b, 0], (np.arange(20) < n).astype(np.uint8))


PINS = [
    pin_visibility,
    pin_causal_mask_shape_and_rows,
    pin_sliding_window_rows,
    pin_two_key_golden,
    pin_probability_rows,
    pin_constant_v,
    pin_causal_row0,
    pin_uniform_attention,
    pin_gqa_repeat,
    pin_library_sdpa,
    pin_lse_matches_probabilities,
    pin_lengths_are_prefixes,
    pin_row_subset,
    pin_decode_is_last_row_of_prefill,
    pin_decode_closed_forms,
    pin_flex_golden,
    pin_flex_softcap_limits,
    pin_flex_alibi_geometric,
    pin_flex_document_blocks,
    pin_paged_equals_contiguous,
    pin_paged_reads_only_listed_slots,
    pin_rbs_closed_form,
    pin_rbs_degenerate_and_gqa,
    pin_rbs_relative_mask_golden,
    pin_block_sparse_attention,
    pin_bwd_finite_differences,
    pin_bwd_gqa_and_uniform,
]
