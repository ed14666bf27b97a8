"""Pins of the CPU oracle: checks that tie it to something other than itself.

Each ``pin_*`` takes an ``oracle.Oracle`` handle and raises AssertionError on a
mismatch. They use closed forms, hand-worked fixtures (tests/golden/),
invariants, brute force over all subsets, and library routines (numpy sums,
sorts and matrix products) — never the oracle's own code. The mutation test
runs every pin against deliberately broken copies of the oracle and requires
each copy to fail at least one.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 to bf16 (nearest-even) and return the bit patterns."""
    f = np.asarray(x, np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# fine score
# --------------------------------------------------------------------------
def pin_fine_score_worked(orc):
    g = _load("fine_score_worked.json")
    q = np.array(g["q"], np.int8)
    w = np.array(g["w"], np.int32)
    for case in g["cases"]:
        got = orc.fine_score(q, w, np.array(case["k"], np.int8))
        assert got == case["score"], (case, got)


def pin_fine_score_unit_vectors(orc):
    """q_h = a e_i, k = b e_j gives w_h * max(0, a b) when i == j, else 0."""
    H_I, d_I = 3, 5
    w = np.array([2, 5, 7], np.int32)
    for h in range(H_I):
        for i in range(d_I):
            for j in range(d_I):
                for a, b in ((3, 4), (-3, 4), (5, -2), (-6, -7)):
                    q = np.zeros((H_I, d_I), np.int8)
                    k = np.zeros(d_I, np.int8)
                    q[h, i] = a
                    k[j] = b
                    want = int(w[h]) * max(0, a * b) if i == j else 0
                    got = orc.fine_score(q, w, k)
                    assert got == want, (h, i, j, a, b, got, want)


def pin_fine_score_negative_part(orc):
    """score(k) - score(-k) = sum_h w_h (q_h . k): the ReLU splits a signed dot
    into its positive and negative parts (checked with numpy's matmul)."""
    rng = _rng(1)
    for _ in range(50):
        H_I, d_I = int(rng.integers(1, 6)), int(rng.integers(1, 40))
        q = rng.integers(-128, 128, (H_I, d_I)).astype(np.int8)
        k = rng.integers(-127, 128, d_I).astype(np.int8)
        w = rng.integers(1, 9, H_I).astype(np.int32)
        lin = int(w.astype(np.int64) @ (q.astype(np.int64) @ k.astype(np.int64)))
        got = orc.fine_score(q, w, k) - orc.fine_score(q, w, (-k.astype(np.int16)).astype(np.int8))
        assert got == lin, (got, lin)


def pin_fine_score_weight_additivity(orc):
    """Scores are linear in the head weights and homogeneous in the key."""
    rng = _rng(2)
    for _ in range(50):
        H_I, d_I = int(rng.integers(1, 8)), int(rng.integers(1, 33))
        q = rng.integers(-128, 128, (H_I, d_I)).astype(np.int8)
        k = rng.integers(-40, 41, d_I).astype(np.int8)
        w1 = rng.integers(0, 9, H_I).astype(np.int32)
        w2 = rng.integers(0, 9, H_I).astype(np.int32)
        s12 = orc.fine_score(q, w1 + w2, k)
        assert s12 == orc.fine_score(q, w1, k) + orc.fine_score(q, w2, k)
        assert orc.fine_score(q, w1, 3 * k) == 3 * orc.fine_score(q, w1, k)
        # one head alone equals its own weighted ReLU computed with numpy
        for h in range(H_I):
            wh = np.zeros(H_I, np.int32)
            wh[h] = 1
            dot = int(q[h].astype(np.int64) @ k.astype(np.int64))
            assert orc.fine_score(q, wh, k) == max(0, dot)


# --------------------------------------------------------------------------
# block sums and coarse score
# --------------------------------------------------------------------------
def pin_block_sums_numpy(orc):
    rng = _rng(3)
    for L, d_I, B in ((1, 4, 1), (7, 3, 2), (64, 8, 16), (100, 32, 7), (130, 16, 64), (37, 5, 64)):
        k = rng.integers(-128, 128, (L, d_I)).astype(np.int8)
        nblk = -(-L // B)
        pad = np.zeros((nblk * B, d_I), np.int64)
        pad[:L] = k
        want = pad.reshape(nblk, B, d_I).sum(axis=1)
        got = orc.block_sums(k, B)
        assert got.shape == want.shape and np.array_equal(got, want), (L, d_I, B)
    k = rng.integers(-128, 128, (9, 4)).astype(np.int8)
    assert np.array_equal(orc.block_sums(k, 1), k.astype(np.int64))


def pin_coarse_is_fine_on_single_key(orc):
    """A block holding one key (S_b = k) scores exactly like that key, and a
    block of n copies of k scores n times as much."""
    rng = _rng(4)
    for _ in range(30):
        H_I, d_I = int(rng.integers(1, 6)), int(rng.integers(1, 20))
        q = rng.integers(-128, 128, (H_I, d_I)).astype(np.int8)
        w = rng.integers(1, 9, H_I).astype(np.int32)
        k = rng.integers(-128, 128, d_I).astype(np.int8)
        fine = orc.fine_score(q, w, k)
        assert orc.coarse_score(q, w, k.astype(np.int64)) == fine
        n = int(rng.integers(2, 300))
        assert orc.coarse_score(q, w, n * k.astype(np.int64)) == n * fine


# --------------------------------------------------------------------------
# index sets
# --------------------------------------------------------------------------
def pin_index_worked(orc):
    g = _load("index_worked.json")
    q = np.array(g["q"], np.int8)
    w = np.array(g["w"], np.int32)
    k = np.array(g["k"], np.int8)
    for c in g["cases"]:
        got = orc.index_query(q, w, k, g["L"], c["sink"], c["window"], c["topk"], c["hi_block"], c["hi_topblocks"])
        assert got.tolist() == c["set"], (c, got.tolist())


def _middle(L, sink, window):
    s = min(sink, L)
    ws = max(s, L - window)
    return s, ws


def _np_scores(q, w, k):
    """Fine scores of every key with numpy's matmul (a library routine)."""
    dots = k.astype(np.int64) @ q.astype(np.int64).T          # [L, H_I]
    return np.maximum(dots, 0) @ w.astype(np.int64)            # [L]


def pin_index_subset_dominance(orc):
    """Brute force over every subset: the selected middle tokens are the one
    topk-subset that dominates the rest under (score desc, position asc)."""
    rng = _rng(5)
    for trial in range(40):
        L = int(rng.integers(1, 13))
        sink, window = int(rng.integers(0, 3)), int(rng.integers(0, 3))
        topk = int(rng.integers(0, 6))
        H_I, d_I = 2, 3
        q = rng.integers(-2, 3, (H_I, d_I)).astype(np.int8)   # tiny values: many ties
        w = rng.integers(1, 3, H_I).astype(np.int32)
        k = rng.integers(-2, 3, (L, d_I)).astype(np.int8)
        got = orc.index_query(q, w, k, L, sink, window, topk)
        s, ws = _middle(L, sink, window)
        mid = list(range(s, ws))
        sc = _np_scores(q, w, k)
        m = min(topk, len(mid))
        winners = []
        for sub in itertools.combinations(mid, m):
            inside = set(sub)
            ok = all((sc[i] > sc[j]) or (sc[i] == sc[j] and i < j)
                     for i in inside for j in mid if j not in inside)
            if ok:
                winners.append(sub)
        assert len(winners) == 1, (trial, winners)
        want = sorted(list(range(s)) + list(winners[0]) + list(range(ws, L)))
        want += [-1] * (sink + window + topk - len(want))
        assert got.tolist() == want, (trial, got.tolist(), want)


def pin_index_equal_keys(orc):
    """All keys equal: every middle score ties, so the lowest positions win."""
    L, sink, window, topk = 50, 3, 7, 9
    q = np.array([[1, -2, 3]], np.int8)
    w = np.array([4], np.int32)
    k = np.tile(np.array([[2, 1, 1]], np.int8), (L, 1))
    got = orc.index_query(q, w, k, L, sink, window, topk)
    want = list(range(0, 3)) + list(range(3, 12)) + list(range(43, 50))
    assert got.tolist() == want


def _check_si_invariants(got, L, sink, window, topk):
    budget = sink + window + topk
    s, ws = _middle(L, sink, window)
    valid = [x for x in got.tolist() if x != -1]
    n = len(valid)
    assert got.shape[0] == budget
    assert all(x == -1 for x in got.tolist()[n:]), "padding must be a -1 tail"
    assert s + (L - ws) <= n <= s + (L - ws) + min(topk, ws - s)
    assert all(0 <= x < L for x in valid)
    assert all(a < b for a, b in zip(valid, valid[1:])), "strictly ascending"
    sv = set(valid)
    assert set(range(s)) <= sv and set(range(ws, L)) <= sv, "sink and window always kept"
    assert n <= budget


def pin_index_si_invariants(orc):
    rng = _rng(6)
    for _ in range(60):
        L = int(rng.integers(1, 400))
        sink, window, topk = (int(x) for x in rng.integers(0, 40, 3))
        H_I, d_I = int(rng.integers(1, 5)), 8
        q = rng.integers(-128, 128, (H_I, d_I)).astype(np.int8)
        w = rng.integers(1, 9, H_I).astype(np.int32)
        k = rng.integers(-128, 128, (L, d_I)).astype(np.int8)
        hb = int(rng.choice([0, 1, 4, 16]))
        ht = int(rng.integers(0, 10))
        got = orc.index_query(q, w, k, L, sink, window, topk, hb, ht)
        _check_si_invariants(got, L, sink, window, topk)
        if hb == 0:
            assert len([x for x in got if x != -1]) == min(L, sink + window + topk)


def pin_index_dense_when_budget_covers(orc):
    rng = _rng(7)
    for _ in range(30):
        L = int(rng.integers(1, 200))
        sink, window = int(rng.integers(0, 50)), int(rng.integers(0, 50))
        topk = max(0, L - sink - window) + int(rng.integers(0, 5))
        q = rng.integers(-128, 128, (2, 4)).astype(np.int8)
        w = np.array([1, 2], np.int32)
        k = rng.integers(-128, 128, (L, 4)).astype(np.int8)
        got = orc.index_query(q, w, k, L, sink, window, topk)
        assert [x for x in got if x != -1] == list(range(L))


def pin_index_topk_by_sort(orc):
    """The selection equals a numpy lexsort of (position asc within score desc)."""
    rng = _rng(8)
    for _ in range(40):
        L = int(rng.integers(1, 3000))
        sink, window, topk = int(rng.integers(0, 70)), int(rng.integers(0, 200)), int(rng.integers(0, 300))
        H_I, d_I = 4, 16
        q = rng.integers(-8, 8, (H_I, d_I)).astype(np.int8)
        w = rng.integers(1, 5, H_I).astype(np.int32)
        k = rng.integers(-8, 8, (L, d_I)).astype(np.int8)
        got = orc.index_query(q, w, k, L, sink, window, topk)
        s, ws = _middle(L, sink, window)
        sc = _np_scores(q, w, k)
        mid = np.arange(s, ws)
        order = np.lexsort((mid, -sc[mid]))
        sel = mid[order[:topk]]
        want = sorted(list(range(s)) + sel.tolist() + list(range(ws, L)))
        want += [-1] * (sink + window + topk - len(want))
        assert got.tolist() == want


def pin_hi_all_blocks_kept_is_flat(orc):
    rng = _rng(9)
    for _ in range(30):
        L = int(rng.integers(1, 600))
        sink, window, topk = int(rng.integers(0, 30)), int(rng.integers(0, 60)), int(rng.integers(0, 80))
        B = int(rng.choice([1, 3, 16, 64]))
        q = rng.integers(-16, 16, (3, 8)).astype(np.int8)
        w = rng.integers(1, 9, 3).astype(np.int32)
        k = rng.integers(-16, 16, (L, 8)).astype(np.int8)
        flat = orc.index_query(q, w, k, L, sink, window, topk)
        hi = orc.index_query(q, w, k, L, sink, window, topk, B, (L + B - 1) // B)
        assert np.array_equal(flat, hi)


def pin_hi_unit_blocks_is_flat(orc):
    """hi_block = 1 makes each block sum a key, so the coarse pass is the fine
    pass; keeping at least topk blocks then reproduces the flat selection."""
    rng = _rng(10)
    for _ in range(30):
        L = int(rng.integers(1, 500))
        sink, window, topk = int(rng.integers(0, 20)), int(rng.integers(0, 40)), int(rng.integers(0, 60))
        q = rng.integers(-16, 16, (2, 8)).astype(np.int8)
        w = rng.integers(1, 9, 2).astype(np.int32)
        k = rng.integers(-16, 16, (L, 8)).astype(np.int8)
        flat = orc.index_query(q, w, k, L, sink, window, topk)
        hi = orc.index_query(q, w, k, L, sink, window, topk, 1, topk + int(rng.integers(0, 5)))
        assert np.array_equal(flat, hi)


def pin_hi_restricts_to_kept_blocks(orc):
    """With HI on, every selected middle token lies in one of the hi_topblocks
    blocks with the best coarse scores (numpy block sums and matmul)."""
    rng = _rng(11)
    for _ in range(30):
        L = int(rng.integers(20, 800))
        sink, window, topk = int(rng.integers(0, 10)), int(rng.integers(0, 30)), int(rng.integers(1, 100))
        B = int(rng.choice([4, 16, 32]))
        ht = int(rng.integers(1, 8))
        q = rng.integers(-16, 16, (2, 8)).astype(np.int8)
        w = rng.integers(1, 9, 2).astype(np.int32)
        k = rng.integers(-16, 16, (L, 8)).astype(np.int8)
        got = orc.index_query(q, w, k, L, sink, window, topk, B, ht)
        s, ws = _middle(L, sink, window)
        nblk = -(-L // B)
        pad = np.zeros((nblk * B, 8), np.int64)
        pad[:L] = k
        S = pad.reshape(nblk, B, 8).sum(axis=1)
        coarse = np.maximum(S @ q.astype(np.int64).T, 0) @ w.astype(np.int64)
        cand = [b for b in range(nblk) if b * B < ws and min((b + 1) * B, L) > s]
        order = sorted(cand, key=lambda b: (-coarse[b], b))
        kept = set(order[:ht])
        mid_sel = [x for x in got.tolist() if x != -1 and s <= x < ws]
        assert all(x // B in kept for x in mid_sel)
        pool = [t for t in range(s, ws) if t // B in kept]
        assert len(mid_sel) == min(topk, len(pool))
        sc = _np_scores(q, w, k)
        rest = [t for t in pool if t not in set(mid_sel)]
        for i in mid_sel:
            for j in rest:
                assert sc[i] > sc[j] or (sc[i] == sc[j] and i < j)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def _dense_attention(qf, kf, vf, H_kv):
    """Textbook causal-free softmax attention over all rows, fp64 numpy."""
    H_q, d = qf.shape
    out = np.zeros((H_q, d))
    for h in range(H_q):
        kvh = h * H_kv // H_q
        logits = kf[:, kvh, :] @ qf[h] / math.sqrt(d)
        e = np.exp(logits - logits.max())
        out[h] = (e / e.sum()) @ vf[:, kvh, :]
    return out


def pin_attend_single_token(orc):
    rng = _rng(12)
    H_q, H_kv, d, L = 4, 2, 16, 9
    q = _bf16_bits(rng.standard_normal((H_q, d)))
    k = _bf16_bits(rng.standard_normal((L, H_kv, d)))
    v = _bf16_bits(rng.standard_normal((L, H_kv, d)))
    for t in range(L):
        out = orc.attend_query(q, k, v, np.array([t, -1, -1], np.int32))
        for h in range(H_q):
            assert np.array_equal(out[h], _bits_to_f64(v[t, h * H_kv // H_q]))


def pin_attend_identical_keys_mean(orc):
    rng = _rng(13)
    H_q, H_kv, d, L = 2, 1, 8, 20
    q = _bf16_bits(rng.standard_normal((H_q, d)))
    k = np.tile(_bf16_bits(rng.standard_normal((1, H_kv, d))), (L, 1, 1))
    v = _bf16_bits(rng.standard_normal((L, H_kv, d)))
    sel = np.array([1, 4, 5, 11, 19, -1], np.int32)
    out = orc.attend_query(q, k, v, sel)
    want = _bits_to_f64(v[[1, 4, 5, 11, 19], 0]).mean(axis=0)
    for h in range(H_q):
        assert np.allclose(out[h], want, rtol=0, atol=1e-14)


def pin_attend_two_token_closed_form(orc):
    """Two rows: o = sigma(z0 - z1) v0 + sigma(z1 - z0) v1, z = q.k / sqrt(d)."""
    q = _bf16_bits(np.array([[1.0, 1.0]]))
    k = _bf16_bits(np.array([[[1.0, 0.0]], [[0.0, 2.0]]]))
    v = _bf16_bits(np.array([[[2.0, 0.0]], [[0.0, 4.0]]]))
    out = orc.attend_query(q, k, v, np.array([0, 1], np.int32))
    z0, z1 = 1 / math.sqrt(2), 2 / math.sqrt(2)
    p0 = 1 / (1 + math.exp(z1 - z0))
    want = np.array([2 * p0, 4 * (1 - p0)])
    assert np.allclose(out[0], want, rtol=1e-15, atol=1e-15), (out, want)


def pin_attend_gqa_mapping(orc):
    """Contiguous GQA groups: with H_q=6, H_kv=3, heads 0-1 read kv head 0,
    2-3 read 1, 4-5 read 2 (each kv head's V is a distinct constant)."""
    rng = _rng(14)
    H_q, H_kv, d, L = 6, 3, 4, 5
    q = _bf16_bits(rng.standard_normal((H_q, d)))
    k = _bf16_bits(rng.standard_normal((L, H_kv, d)))
    vals = np.zeros((L, H_kv, d))
    for j, c in enumerate((-3.0, 7.0, 0.5)):
        vals[:, j, :] = c
    v = _bf16_bits(vals)
    out = orc.attend_query(q, k, v, np.arange(L, dtype=np.int32))
    for h, c in enumerate((-3.0, -3.0, 7.0, 7.0, 0.5, 0.5)):
        assert np.allclose(out[h], c, rtol=0, atol=1e-14), (h, out[h])


def pin_attend_dense_equivalence(orc):
    """Budget covering the context: the index set is 0..L-1 and the attention
    equals a separately written dense softmax attention."""
    rng = _rng(15)
    for L in (1, 2, 17, 130):
        H_q, H_kv, d = 8, 2, 32
        qi = rng.integers(-8, 8, (4, 16)).astype(np.int8)
        wi = rng.integers(1, 5, 4).astype(np.int32)
        ki = rng.integers(-8, 8, (L, 16)).astype(np.int8)
        sel = orc.index_query(qi, wi, ki, L, 4, 16, max(0, L - 20) + 3)
        assert [x for x in sel if x != -1] == list(range(L))
        q = _bf16_bits(rng.standard_normal((H_q, d)))
        k = _bf16_bits(rng.standard_normal((L, H_kv, d)))
        v = _bf16_bits(rng.standard_normal((L, H_kv, d)))
        got = orc.attend_query(q, k, v, sel)
        want = _dense_attention(_bits_to_f64(q), _bits_to_f64(k), _bits_to_f64(v), H_kv)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def pin_attend_padding_and_empty(orc):
    rng = _rng(16)
    H_q, H_kv, d, L = 2, 1, 8, 10
    q = _bf16_bits(rng.standard_normal((H_q, d)))
    k = _bf16_bits(rng.standard_normal((L, H_kv, d)))
    v = _bf16_bits(rng.standard_normal((L, H_kv, d)))
    a = orc.attend_query(q, k, v, np.array([2, 3, 9], np.int32))
    b = orc.attend_query(q, k, v, np.array([2, 3, 9, -1, -1, -1], np.int32))
    assert np.array_equal(a, b)
    want = _dense_attention(_bits_to_f64(q), _bits_to_f64(k[[2, 3, 9]]), _bits_to_f64(v[[2, 3, 9]]), H_kv)
    assert np.allclose(a, want, rtol=1e-12, atol=1e-12)
    z = orc.attend_query(q, k, v, np.array([-1, -1], np.int32))
    assert np.array_equal(z, np.zeros((H_q, d)))


# --------------------------------------------------------------------------
# batch drivers (packed sequences, CLI)
# --------------------------------------------------------------------------
def pin_batch_matches_single_queries(orc):
    rng = _rng(17)
    lens = [5, 40, 1, 77]
    d_I, H_I = 8, 2
    T = sum(lens)
    offs = np.cumsum([0] + lens[:-1]).astype(np.int64)
    k = rng.integers(-16, 16, (T, d_I)).astype(np.int8)
    # two queries per sequence at different visible lengths (prefill-like)
    q_seq = np.array([0, 1, 1, 2, 3, 3], np.int32)
    q_len = np.array([5, 40, 12, 1, 77, 30], np.int32)
    n_q = len(q_seq)
    qi = rng.integers(-16, 16, (n_q, H_I, d_I)).astype(np.int8)
    wi = rng.integers(1, 9, (n_q, H_I)).astype(np.int32)
    for hb, ht in ((0, 0), (4, 3)):
        sets = orc.lsa_index(qi, k, wi, offs, q_seq, q_len, 2, 4, 6, hb, ht, n_threads=2)
        for r in range(n_q):
            base = offs[q_seq[r]]
            one = orc.index_query(qi[r], wi[r], k[base:base + lens[q_seq[r]]], q_len[r], 2, 4, 6, hb, ht)
            assert np.array_equal(sets[r], one)
            assert all(x < q_len[r] for x in sets[r])
    H_q, H_kv, d, G = 4, 2, 8, 3
    qs = [_bf16_bits(rng.standard_normal((n_q, H_q, d))) for _ in range(G)]
    ks = [_bf16_bits(rng.standard_normal((T, H_kv, d))) for _ in range(G)]
    vs = [_bf16_bits(rng.standard_normal((T, H_kv, d))) for _ in range(G)]
    outs = orc.lsa_attend(qs, ks, vs, sets, offs, q_seq, n_threads=3)
    for g in range(G):
        # CLI with G layers equals G separate single-layer calls on the same set
        one = orc.lsa_attend([qs[g]], [ks[g]], [vs[g]], sets, offs, q_seq)[0]
        assert np.array_equal(outs[g], one)
        for r in range(n_q):
            base = offs[q_seq[r]]
            L = lens[q_seq[r]]
            want = orc.attend_query(qs[g][r], ks[g][base:base + L], vs[g][base:base + L], sets[r])
            assert np.array_equal(outs[g][r], want)


# ---- FP8 KV cache --------------------------------------------------------
def _e4m3_torch(codes: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _e4m3_to_bf16_bits(codes: np.ndarray, scale: float) -> np.ndarray:
    import torch
    vals = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float32) * scale
    bits = vals.to(torch.bfloat16)
    assert torch.equal(bits.to(torch.float32), vals)  # an E4M3 value times a power of two is a bf16
    return bits.view(torch.int16).numpy().view(np.uint16)


def _fp8_case(seed, L=40, H_q=8, H_kv=2, d=128):
    import torch
    rng = _rng(seed)
    q = _bf16_bits(rng.standard_normal((H_q, d)))
    k = torch.from_numpy(rng.standard_normal((L, H_kv, d)).astype(np.float32)).to(torch.float8_e4m3fn)
    v = torch.from_numpy(rng.standard_normal((L, H_kv, d)).astype(np.float32)).to(torch.float8_e4m3fn)
    s = np.array([0, 3, 4, -1, 17, 18, 19, 39, -1, -1], np.int32)
    return q, k.view(torch.uint8).numpy(), v.view(torch.uint8).numpy(), s


def pin_fp8_decode_matches_torch_on_every_code(orc):
    """E4M3 decode of all 256 codes against torch's float8_e4m3fn type."""
    codes = np.arange(256, dtype=np.uint8)
    want = _e4m3_torch(codes)
    got = np.array([orc.e4m3_value(c) for c in codes])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(got[~nan], want[~nan])


def pin_fp8_decode_closed_forms(orc):
    """Values the format's definition fixes (bias 7, subnormals m/8 * 2^-6)."""
    assert orc.e4m3_value(0x00) == 0.0
    assert orc.e4m3_value(0x38) == 1.0
    assert orc.e4m3_value(0xB8) == -1.0
    assert orc.e4m3_value(0x7E) == 448.0
    assert orc.e4m3_value(0x08) == 2.0 ** -6
    assert orc.e4m3_value(0x01) == 2.0 ** -9
    assert orc.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert np.isnan(orc.e4m3_value(0x7F))


def pin_fp8_attention_is_bf16_attention_on_the_values(orc):
    """FP8 attention = the bf16 attention on the decoded, scaled values."""
    q, k8, v8, s = _fp8_case(1)
    for ks, vs in ((1.0, 1.0), (0.5, 2.0), (0.125, 0.25)):
        got = orc.attend_query_fp8(q, k8, v8, ks, vs, s)
        want = orc.attend_query(q, _e4m3_to_bf16_bits(k8, ks), _e4m3_to_bf16_bits(v8, vs), s)
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def pin_fp8_attention_scales(orc):
    """Linear in v_scale; k_scale = 0 gives the plain mean of the selected V rows;
    an empty set gives zeros."""
    q, k8, v8, s = _fp8_case(2)
    base = orc.attend_query_fp8(q, k8, v8, 0.7, 1.0, s)
    np.testing.assert_allclose(orc.attend_query_fp8(q, k8, v8, 0.7, 3.0, s), 3.0 * base, rtol=1e-13, atol=1e-13)
    flat = orc.attend_query_fp8(q, k8, v8, 0.0, 1.0, s)
    vals = _e4m3_torch(v8)
    rows = s[s >= 0]
    for h in range(q.shape[0]):
        kvh = h * k8.shape[1] // q.shape[0]
        np.testing.assert_allclose(flat[h], vals[rows, kvh].mean(axis=0), rtol=1e-13, atol=1e-13)
    assert not orc.attend_query_fp8(q, k8, v8, 1.0, 1.0, np.full(6, -1, np.int32)).any()


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
