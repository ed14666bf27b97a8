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
