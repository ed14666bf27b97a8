"""The context-parallel kernels on the GPU through the C ABI: candidate keys of
given positions and blocks against the oracle's scores, the exact merge of
packed candidates against a sort, and the whole protocol for two token
ranges of one sequence (the two ranks' exchanges done in one process) against
the oracle's index set and lsa_index's."""
import numpy as np
import pytest
import torch

import oracle
import parity
from long_context_sparse_lsa_b200 import binding as lsa
from long_context_sparse_lsa_b200 import context_parallel as cp
from long_context_sparse_lsa_b200 import workloads as wls
from long_context_sparse_lsa_b200.pipeline import LsaStep

pytestmark = pytest.mark.gpu
DEV = "cuda"
BASE = wls.small(wls.BATCH128K, name="cpg", lens=(3000,), G=1)


def _sorted_best(values: np.ndarray, k: int):
    x = values[values != 0].view(np.uint64) if values.dtype != np.uint64 else values[values != 0]
    best = np.sort(x)[::-1][:k]
    return np.sort((cp.ID_MASK - (best & np.uint64(cp.ID_MASK))).astype(np.int64))


def test_merge_pairs_matches_a_sort_with_ties_and_short_rows():
    rng = np.random.default_rng(5)
    rows, cap, k = 6, 5000, 700
    vals = np.zeros((rows, cap), np.int64)
    counts = np.zeros(rows, np.int32)
    for r in range(rows):
        n = [cap, 3000, 700, 10, 0, 4321][r]
        keys = rng.integers(1, 4 if r % 2 else 1 << 30, size=n)   # odd rows: heavy ties
        ids = rng.permutation(1 << 20)[:n]
        vals[r, :n] = cp.pack(torch.from_numpy(keys), torch.from_numpy(ids)).numpy()
        counts[r] = n
    v = torch.from_numpy(vals).to(DEV)
    out = torch.empty((rows, k), dtype=torch.int32, device=DEV)
    kept = torch.empty((rows, k), dtype=torch.int64, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lsa.lsa_merge_pairs(v, torch.from_numpy(counts).to(DEV), k, out, kept, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got, gk = out.cpu().numpy(), kept.cpu().numpy()
    for r in range(rows):
        want = _sorted_best(vals[r, :counts[r]].view(np.uint64), k)
        np.testing.assert_array_equal(got[r, :len(want)], want)
        assert np.all(got[r, len(want):] == -1)
        # the kept values are the entries of those ids
        ids_of = (cp.ID_MASK - (gk[r, :len(want)].view(np.uint64) & np.uint64(cp.ID_MASK))).astype(np.int64)
        np.testing.assert_array_equal(ids_of, want)


def test_point_scores_match_the_oracle():
    wl = wls.small(BASE, lens=(3000, 1200), hi_block=64, hi_topblocks=8, seed=81)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    torch.cuda.synchronize()
    orc = oracle.get()
    rng = np.random.default_rng(2)
    offs = parity.host(t.kv_offset)
    boffs = parity.host(t.blk_offset)
    q_seq = parity.host(t.q_seq)
    n = 300
    pos = np.stack([rng.integers(0, L, n) for L in wl.lens]).astype(np.int32)
    pos[0, 7] = -1
    keys = torch.empty((wl.n_q, n), dtype=torch.int32, device=DEV)
    lsa.lsa_score_tokens(t.q_idx, t.k_idx, t.w, wl.w_max, torch.from_numpy(offs[q_seq]).to(DEV),
                         torch.from_numpy(pos).to(DEV), keys)
    nb = 20
    blk = np.stack([rng.integers(0, (L + 63) // 64, nb) for L in wl.lens]).astype(np.int32)
    bkeys = torch.empty((wl.n_q, nb), dtype=torch.int64, device=DEV)
    lsa.lsa_score_blocks(t.q_idx, t.w, wl.w_max, st.block_sums, torch.from_numpy(boffs[q_seq]).to(DEV),
                         torch.from_numpy(blk).to(DEV), bkeys)
    torch.cuda.synchronize()
    k_all = parity.host(t.k_idx)
    kk, bk = keys.cpu().numpy().view(np.uint32), bkeys.cpu().numpy()
    for r in range(wl.n_q):
        q, w = parity.host(t.q_idx[r]), parity.host(t.w[r])
        kseq = k_all[offs[q_seq[r]]:offs[q_seq[r]] + wl.lens[q_seq[r]]]
        sums = orc.block_sums(kseq, 64)
        for j in range(n):
            p = int(pos[r, j])
            assert kk[r, j] == (0 if p < 0 else orc.fine_score(q, w, kseq[p]) + 1)
        for j in range(nb):
            assert bk[r, j] == orc.coarse_score(q, w, sums[int(blk[r, j])]) + 1


@pytest.mark.parametrize("hi", [True, False])
def test_two_token_ranges_give_the_whole_sequence_set(hi):
    kw = dict(hi_block=64, hi_topblocks=24) if hi else dict(hi_block=0, hi_topblocks=0)
    wl = wls.small(BASE, lens=(9000,), sink=32, window=200, topk=800, seed=83, **kw)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    torch.cuda.synchronize()
    L = wl.lens[0]
    B = wl.hi_block
    bounds = cp.shard_bounds(L, 2, B if hi else 1)
    budget = cp.Budget(wl.sink, wl.window, wl.topk, B, wl.hi_topblocks)
    ranks = [cp.ContextParallelIndex(bounds, r, budget, wl.w_max) for r in range(2)]
    shard = []
    for r, (lo, hi_) in enumerate(bounds):
        sums = st.block_sums[lo // B:(hi_ + B - 1) // B].contiguous() if hi else None
        shard.append((t.k_idx[lo:hi_].contiguous(), sums))
    q, w = t.q_idx[0], t.w[0]
    kept = None
    if hi:
        loc = [ix.local_best(ix.block_candidates(q, w, shard[r][1], L), wl.hi_topblocks) for r, ix in enumerate(ranks)]
        kept = ranks[0].global_best(torch.cat(loc), wl.hi_topblocks)
    loc = [ix.local_best(ix.token_candidates(q, w, shard[r][0], L, kept), wl.topk) for r, ix in enumerate(ranks)]
    got = ranks[0].assemble(L, ranks[0].global_best(torch.cat(loc), wl.topk))
    torch.cuda.synchronize()
    want = parity.oracle_sets(wl, t)[0]
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    np.testing.assert_array_equal(parity.host(st.sets)[0], want)


def _f64(t: torch.Tensor) -> np.ndarray:
    return (parity.u16(t).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _lse_fp64(q, k, sets, kv_off, q_seq):
    """ln sum_j exp(q . k_j / sqrt(d)) per (row, head) in fp64 from the bf16 values."""
    qq, kk = _f64(q), _f64(k)
    n_q, H_q, d = qq.shape
    ratio = H_q // kk.shape[1]
    out = np.full((n_q, H_q), -np.inf)
    for r in range(n_q):
        e = sets[r][sets[r] >= 0].astype(np.int64) + int(kv_off[q_seq[r]])
        if e.size == 0:
            continue
        for h in range(H_q):
            s = kk[e, h // ratio] @ qq[r, h] / np.sqrt(d)
            m = s.max()
            out[r, h] = m + np.log(np.exp(s - m).sum())
    return out


def test_shard_sets_bit_exact():
    rng = np.random.default_rng(11)
    n_q, budget = 7, 3000
    sets = np.full((n_q, budget), -1, np.int32)
    for r in range(n_q):
        n = [budget, 2000, 0, 1, 2999, 1500, 64][r]
        sets[r, :n] = np.sort(rng.choice(1 << 16, size=n, replace=False))
    sets[5, 10] = -1  # a hole inside the row is dropped too
    d = torch.from_numpy(sets).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for lo, hi in ((0, 1 << 16), (0, 20000), (20000, 40000), (65000, 1 << 20), (5, 5)):
        got = torch.empty_like(d)
        lsa.lsa_shard_sets(d, lo, hi, got, status)
        torch.cuda.synchronize()
        want = np.full_like(sets, -1)
        for r in range(n_q):
            keep = sets[r][(sets[r] >= lo) & (sets[r] < hi)] - lo
            want[r, :keep.size] = keep
        np.testing.assert_array_equal(got.cpu().numpy(), want)
    assert int(status.item()) == 0


@pytest.mark.parametrize("topk", [16, 2400])  # one split (direct output) and several (merge kernel)
def test_attend_lse_matches_the_definition(topk):
    wl = wls.small(BASE, lens=(3000, 2500), drafts=2, hi_block=0, hi_topblocks=0, sink=8, window=32, topk=topk,
                   G=2, seed=85)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.index()
    sets = st.sets.clone()
    sets[1] = -1  # an empty set: zero output, lse -inf
    n_q, H_q, d = t.q[0].shape
    out = [torch.empty((n_q, H_q, d), dtype=torch.float32, device=DEV) for _ in range(wl.G)]
    lse = [torch.empty((n_q, H_q), dtype=torch.float32, device=DEV) for _ in range(wl.G)]
    batch = st.batch
    ws = torch.empty(max(1, lsa.lsa_attend_workspace_size(batch, H_q, t.k[0].shape[1], d, sets.shape[1], wl.G)),
                     dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lsa.lsa_attend_lse(t.q, t.k, t.v, sets, batch, out, lse, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    hs = parity.host(sets)
    want = parity.oracle_attend_full(t, hs)
    for g in range(wl.G):
        parity.check_attention(out[g].cpu().numpy(), want[g], f"layer {g}")
        got_lse = lse[g].cpu().numpy().astype(np.float64)
        ref = _lse_fp64(t.q[g], t.k[g], hs, parity.host(t.kv_offset), parity.host(t.q_seq))
        assert np.all(np.isneginf(got_lse[1])) and np.all(np.isneginf(ref[1]))
        fin = np.isfinite(ref)
        np.testing.assert_array_equal(np.isfinite(got_lse), fin)
        assert np.abs(got_lse[fin] - ref[fin]).max() < 1e-3


def test_combine_matches_the_definition():
    rng = np.random.default_rng(12)
    P, rows, d = 5, 300, 128
    o = rng.normal(size=(P, rows, d)).astype(np.float32)
    lse = (rng.normal(size=(P, rows)) * 20).astype(np.float32)
    lse[1:, 7] = -np.inf          # one part only
    lse[:, 9] = -np.inf           # every part empty
    lse[:, 11] = 3.0              # equal weights
    out = torch.empty((rows, d), dtype=torch.float32, device=DEV)
    lse_out = torch.empty(rows, dtype=torch.float32, device=DEV)
    lsa.lsa_combine(torch.from_numpy(o).to(DEV), torch.from_numpy(lse).to(DEV), out, lse_out)
    torch.cuda.synchronize()
    l64 = lse.astype(np.float64)
    M = np.max(l64, axis=0)
    Mf = np.where(np.isfinite(M), M, 0.0)
    wgt = np.where(np.isfinite(l64), np.exp(l64 - Mf), 0.0)
    den = wgt.sum(0)
    want = (wgt[..., None] * o).sum(0) / np.where(den > 0, den, 1.0)[:, None]
    want_lse = np.where(den > 0, Mf + np.log(np.where(den > 0, den, 1.0)), -np.inf)
    got, got_lse = out.cpu().numpy(), lse_out.cpu().numpy()
    np.testing.assert_allclose(got, want, atol=1e-5, rtol=1e-5)
    np.testing.assert_allclose(got[7], o[0, 7])
    assert np.all(got[9] == 0.0) and np.isneginf(got_lse[9])
    np.testing.assert_allclose(got[11], o[:, 11].mean(0), atol=1e-5)
    fin = np.isfinite(want_lse)
    np.testing.assert_allclose(got_lse[fin], want_lse[fin], atol=1e-4, rtol=1e-6)


def test_two_ranks_attention_equals_the_whole_set():
    wl = wls.small(BASE, lens=(9000,), drafts=3, hi_block=64, hi_topblocks=24, sink=32, window=200, topk=800,
                   G=2, seed=86)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    torch.cuda.synchronize()
    L = wl.lens[0]
    bounds = cp.shard_bounds(L, 2, wl.hi_block)
    parts = []
    for r, (lo, hi) in enumerate(bounds):
        att = cp.ContextParallelAttention(bounds, r, exchange=lambda x: x)
        local = att.shard(st.sets, lo, hi)
        parts.append(att.partial(t.q, [x[lo:hi].contiguous() for x in t.k], [x[lo:hi].contiguous() for x in t.v],
                                 local, hi - lo))
    o_parts = torch.stack([p[0] for p in parts])
    lse_parts = torch.stack([p[1] for p in parts])
    got = cp.ContextParallelAttention._gpu_combine(o_parts, lse_parts)
    torch.cuda.synchronize()
    want = parity.oracle_attend_full(t, parity.host(st.sets))
    for g in range(wl.G):
        parity.check_attention(got[g].cpu().numpy(), want[g], f"layer {g}")
