"""Draft rows attended together (lsa_attend_grouped) on the GPU: every row's
output against the oracle's attention over that row's own set, for groups of
1, 2, 4 and 8 draft rows, one split and several, sets that are not ascending,
invalid rows, groups naming two sequences, and the full-size 4 x 4 draft
workload in the launch configuration the bench times."""
import numpy as np
import pytest
import torch

import parity
from long_context_sparse_lsa_b200 import binding as lsa
from long_context_sparse_lsa_b200 import workloads as wls
from long_context_sparse_lsa_b200.pipeline import LsaStep

pytestmark = pytest.mark.gpu
DEV = "cuda"
BASE = wls.small(wls.DRAFTS128K, name="drafts_small", lens=(5000, 3300, 4100), G=2)


def _grouped(st: LsaStep, sets: torch.Tensor, D: int):
    t = st.t
    n_q, H_q, d = t.q[0].shape
    H_kv = t.k[0].shape[1]
    out = [torch.full((n_q, H_q, d), 7.0, dtype=torch.float32, device=DEV) for _ in t.q]
    need = lsa.lsa_attend_grouped_workspace_size(st.batch, H_q, H_kv, d, sets.shape[1], len(t.q), D)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    lsa.lsa_attend_grouped(t.q, t.k, t.v, sets, st.batch, D, out, ws, status)
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in out], int(status.item())


def _union_sizes(sets: np.ndarray, D: int):
    return [len(np.unique(g[g >= 0])) for g in sets.reshape(-1, D * sets.shape[1])]


@pytest.mark.parametrize("D,topk,share", [(1, 300, 0), (2, 300, 0), (4, 300, 75), (8, 120, 90), (1, 16, 0)])
def test_grouped_rows_match_the_oracle(D, topk, share):
    wl = wls.small(BASE, drafts=D, topk=topk, draft_share=share, sink=16, window=64 if topk > 16 else 16,
                   hi_block=64, hi_topblocks=12, seed=90 + D)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    torch.cuda.synchronize()
    sets = parity.host(st.sets)
    np.testing.assert_array_equal(sets, parity.oracle_sets(wl, t))
    got, status = _grouped(st, st.sets, D)
    assert status == 0
    want = parity.oracle_attend_full(t, sets)
    for g in range(wl.G):
        parity.check_attention(got[g], want[g], f"layer {g}")
    if D > 1:
        assert max(_union_sizes(sets, D)) < D * wl.budget  # the sink runs at least are shared


def test_any_sets_rows_and_groups_are_lsa_attends():
    """Whatever the sets, rows and groups hold, the output is lsa_attend's:
    repeated entries count twice, entries past q_len are flagged and
    skipped, sets out of order are attended as they are, an invalid row is
    zero, and a group whose rows name two sequences attends each row over its
    own sequence."""
    D = 4
    wl = wls.small(BASE, drafts=D, topk=200, sink=8, window=32, hi_block=0, hi_topblocks=0, seed=97)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.index()
    torch.cuda.synchronize()
    h = parity.host(st.sets).copy()
    q_len = parity.host(t.q_len)
    h[1, 5] = h[1, 4]              # repeated
    h[1, 6] = q_len[1] + 3          # past q_len: flagged, skipped
    h[6, 10:20] = h[6, 10:20][::-1].copy()  # out of order
    h[9, 40:] = -1                  # a short set
    sets = torch.from_numpy(h).to(DEV)
    got, status = _grouped(st, sets, D)
    assert status & lsa.LSA_DEV_BAD_INDEX
    fixed = h.copy()
    fixed[1, 6] = -1
    want = parity.oracle_attend_full(t, fixed)
    for g in range(wl.G):
        parity.check_attention(got[g], want[g], f"layer {g}")
    # an invalid row (q_len past its sequence): zero output, the rest as before
    bad_len = t.q_len.clone()
    bad_len[2] = 10 ** 7
    saved = st.batch.q_len
    st.batch.q_len = bad_len
    got2, status2 = _grouped(st, st.sets, D)
    st.batch.q_len = saved
    assert status2 & lsa.LSA_DEV_BAD_LENGTH
    want2 = parity.oracle_attend_full(t, parity.host(st.sets))
    for g in range(wl.G):
        assert np.all(got2[g][2] == 0.0)
        keep = [r for r in range(wl.n_q) if r != 2]
        parity.check_attention(got2[g][keep], want2[g][keep], f"layer {g}")
    # a group whose rows name two sequences: each row over its own sequence
    # (row 5's set, drawn for sequence 1, is valid in sequence 2 too: lens 3300 < 4100)
    bad_seq = t.q_seq.clone()
    bad_seq[5] = 2
    saved = st.batch.q_seq
    st.batch.q_seq = bad_seq
    got3, status3 = _grouped(st, st.sets, D)
    st.batch.q_seq = saved
    assert status3 == 0
    t3 = wls.Tensors(**{**t.__dict__, "q_seq": bad_seq})
    want3 = parity.oracle_attend_full(t3, parity.host(st.sets))
    for g in range(wl.G):
        parity.check_attention(got3[g], want3[g], f"layer {g}")


def test_fullsize_draft_step_every_row():
    """The 4 x 4 draft workload at full size: every row's set bit-exact and
    every row's attention (grouped, as the bench times it) against the
    oracle's."""
    wl = wls.DRAFTS128K
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    torch.cuda.synchronize()
    sets = parity.host(st.sets)
    parity.check_sets(sets, parity.oracle_sets(wl, t), "draft sets")
    got, status = _grouped(st, st.sets, wl.drafts)
    assert status == 0
    rows = list(range(wl.n_q))
    want = parity.oracle_attend_rows(t, sets, rows)
    for g in range(wl.G):
        parity.check_attention(got[g], want[g], f"layer {g}")
    sizes = _union_sizes(sets, wl.drafts)
    assert sum(sizes) < wl.n_q * wl.budget, sizes
