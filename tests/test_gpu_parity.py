"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs. Index sets must match bit for bit; attention must satisfy
max|err| <= 5e-3 and rel-L2 <= 1e-3 (tests/parity.py). Sizes span several
tiles, clusters and ragged tails; the edge cases of the method (empty middle,
budget covering the context, SI-only budgets, HI keeping every block, ties)
each have a case."""
import numpy as np
import pytest
import torch

import oracle
import parity
from long_context_sparse_lsa_b200 import binding as lsa
from long_context_sparse_lsa_b200 import workloads as wls
from long_context_sparse_lsa_b200.pipeline import LsaStep

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_case(wl, check_attn=True, layers=None):
    t = wls.make(wl, DEV, layers=layers)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    want = parity.oracle_sets(wl, t)
    parity.check_sets(parity.host(st.sets), want, wl.name)
    if check_attn:
        ref = parity.oracle_attend_full(t, want)
        for g in range(len(t.q)):
            parity.check_attention(parity.host(st.out[g]), ref[g], f"{wl.name} layer {g}")
    return st, t


def test_tiny_decode_workload():
    run_case(wls.TINY)


BASE = wls.small(wls.BATCH128K, name="small", lens=(3000,), G=1)

CASES = {
    # HI off, several clusters' worth of tiles and ragged lengths
    "flat_ragged": dict(lens=(37, 1, 4096, 513, 2049), hi_block=0, hi_topblocks=0, sink=16, window=64, topk=300),
    "flat_long": dict(lens=(40000,), hi_block=0, hi_topblocks=0),
    # HI on with partial last blocks and blocks that straddle sink/window
    "hi_ragged": dict(lens=(5000, 777, 64, 12001), hi_block=64, hi_topblocks=8, sink=70, window=100, topk=200),
    "hi_b16": dict(lens=(6000, 3333), hi_block=16, hi_topblocks=40, topk=300, window=50, sink=3),
    "hi_b128_many": dict(lens=(70000,), hi_block=128, hi_topblocks=300, topk=2048, window=2048, sink=64),
    "hi_b256": dict(lens=(20000, 9000), hi_block=256, hi_topblocks=20, topk=1000, window=300, sink=10),
    "hi_all_blocks_kept": dict(lens=(4000,), hi_block=64, hi_topblocks=4096, topk=500, window=100, sink=10),
    "hi_b1_like_flat": dict(lens=(3000,), hi_block=1, hi_topblocks=600, topk=500, window=100, sink=10),
    # budgets: covering the context, SI only, no sink / no window
    "dense_equivalent": dict(lens=(900, 50, 1), hi_block=0, hi_topblocks=0, sink=64, window=512, topk=400),
    "si_only": dict(lens=(5000,), hi_block=0, hi_topblocks=0, sink=32, window=256, topk=0),
    "no_sink_no_window": dict(lens=(3000, 2000), hi_block=0, hi_topblocks=0, sink=0, window=0, topk=777),
    "hi_empty_middle": dict(lens=(1000,), hi_block=64, hi_topblocks=4, sink=600, window=600, topk=100),
    # ties: a tiny value range makes many equal scores
    "ties": dict(lens=(9000,), hi_block=0, hi_topblocks=0, qk_lo=-1, qk_hi=1, w_hi=1, topk=1000),
    "ties_hi": dict(lens=(9000,), hi_block=32, hi_topblocks=50, qk_lo=-1, qk_hi=1, w_hi=1, topk=1000),
    # selection paths: every key equal and large (the threshold bin overflows
    # the candidate list), keys small enough to be their own histogram bins,
    # and rows too long to stage in shared memory (several compaction chunks)
    "all_equal_big": dict(lens=(9000,), qk_lo=3, qk_hi=3, hi_block=0, hi_topblocks=0, topk=1500),
    "all_equal_big_hi": dict(lens=(9000,), qk_lo=3, qk_hi=3, hi_block=32, hi_topblocks=60, topk=1500),
    "small_keys": dict(lens=(6000,), H_I=1, d_I=32, qk_lo=0, qk_hi=1, w_hi=1, hi_block=0, hi_topblocks=0,
                       topk=700),
    "flat_60k": dict(lens=(60000, 45000), hi_block=0, hi_topblocks=0, topk=3000),
    # indexer head counts and key widths
    "heads1_d32": dict(lens=(5000,), H_I=1, d_I=32, qk_lo=-128, qk_hi=127, w_hi=16, hi_block=0, hi_topblocks=0),
    "heads20_d64": dict(lens=(7000, 100), H_I=20, d_I=64, hi_block=32, hi_topblocks=30),
    "heads64": dict(lens=(4000,), H_I=64, d_I=128, qk_lo=-16, qk_hi=15, w_hi=4, hi_block=0, hi_topblocks=0),
    "full_int8_range": dict(lens=(6000,), H_I=8, d_I=128, qk_lo=-128, qk_hi=127, w_hi=2, hi_block=64,
                            hi_topblocks=16),
    # attention shapes: GQA ratios and kv-head counts
    "gqa_1to1": dict(lens=(2000,), H_q=4, H_kv=4, hi_block=0, hi_topblocks=0),
    "gqa_16": dict(lens=(2000, 300), H_q=32, H_kv=2, hi_block=0, hi_topblocks=0),
    "gqa_kv8": dict(lens=(2500,), H_q=16, H_kv=8, hi_block=0, hi_topblocks=0),
    "gqa_kv1": dict(lens=(2500,), H_q=4, H_kv=1, hi_block=0, hi_topblocks=0),
    # cross-layer indexing: one set, three layers
    "cli_g3": dict(lens=(3000, 1500), G=3, hi_block=64, hi_topblocks=10),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_small_cases(name):
    kw = dict(CASES[name])
    kw.setdefault("seed", 100 + sorted(CASES).index(name))
    wl = wls.small(BASE, name=name, **kw)
    run_case(wl)


def test_prefill_rows_through_decode_kernel():
    """Rows of one sequence with causal visible lengths, too few for the dense
    path: scored row by row."""
    wl = wls.small(wls.PREFILL, name="prefill_small", lens=(3000 + 40,), prefill_new=40, seed=7)
    st, _ = run_case(wl)
    assert not lsa.lsa_index_uses_tensor_cores(st.batch, wl.H_I, wl.d_I, st.budget)


# Prefill chunks of one sequence (HI off, 64 rows or more): the fine scores
# come from the tensor-core contraction. Row counts that leave a partial
# 16-row tile, caches that are not a whole number of 128-token tiles, rows
# whose middle is empty or shorter than the sink, and a second sequence
# (which sends the chunk back to the per-row kernel).
PREFILL_CASES = {
    "tc_ragged_rows": dict(lens=(5000 + 77,), prefill_new=77),
    "tc_short_cache": dict(lens=(40 + 300,), prefill_new=300, sink=16, window=64, topk=100),
    "tc_wide_window": dict(lens=(1500 + 130,), prefill_new=130, sink=64, window=1400, topk=50),
    "tc_full_range": dict(lens=(3000 + 96,), prefill_new=96, qk_lo=-128, qk_hi=127, w_hi=4, topk=500),
    "tc_ties": dict(lens=(4000 + 64,), prefill_new=64, qk_lo=-1, qk_hi=1, w_hi=1, topk=700),
    # wider query/key ranges and weights than the default draw
    "tc_qk32_w4": dict(lens=(3000 + 80,), prefill_new=80, qk_lo=-32, qk_hi=31, w_hi=4, topk=400),
    "tc_qk64_w3": dict(lens=(3000 + 80,), prefill_new=80, qk_lo=-64, qk_hi=63, w_hi=3, topk=400),
}


@pytest.mark.parametrize("name", sorted(PREFILL_CASES))
def test_prefill_chunks_tensor_core_scores(name):
    kw = dict(PREFILL_CASES[name])
    kw.setdefault("seed", 300 + sorted(PREFILL_CASES).index(name))
    wl = wls.small(wls.PREFILL, name=name, **kw)
    st, _ = run_case(wl)
    assert lsa.lsa_index_uses_tensor_cores(st.batch, wl.H_I, wl.d_I, st.budget)


def test_dense_equivalence_matches_textbook_attention():
    wl = wls.small(BASE, name="dense", lens=(600,), hi_block=0, hi_topblocks=0, sink=8, window=100, topk=600,
                   seed=11)
    st, t = run_case(wl, check_attn=False)
    sets = parity.host(st.sets)
    assert [x for x in sets[0] if x >= 0] == list(range(600))
    q = parity.u16(t.q[0])[0]
    k = parity.u16(t.k[0])
    v = parity.u16(t.v[0])
    f = lambda b: (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)
    qf, kf, vf = f(q), f(k), f(v)
    H_q, H_kv = qf.shape[0], kf.shape[1]
    want = np.zeros_like(qf)
    for h in range(H_q):
        kvh = h * H_kv // H_q
        z = kf[:, kvh] @ qf[h] / np.sqrt(128.0)
        p = np.exp(z - z.max())
        want[h] = p @ vf[:, kvh] / p.sum()
    parity.check_attention(parity.host(st.out[0])[0], want, "dense textbook")


def test_block_sums_exact_and_append_update():
    wl = wls.small(BASE, name="bsums", lens=(1000, 64, 1, 5000), hi_block=64, hi_topblocks=8, seed=21)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    torch.cuda.synchronize()
    orc = oracle.get()
    got = parity.decode_block_sums(st.block_sums, wl.d_I)
    k = parity.host(t.k_idx)
    offs = parity.host(t.kv_offset)
    boffs = parity.host(t.blk_offset)
    for b, L in enumerate(wl.lens):
        want = orc.block_sums(k[offs[b]:offs[b] + L], wl.hi_block)
        np.testing.assert_array_equal(got[boffs[b]:boffs[b] + want.shape[0]], want)
    # overwrite the last 3 tokens of every sequence, refresh with n_new = 3
    for b, L in enumerate(wl.lens):
        lo = max(0, L - 3)
        t.k_idx[offs[b] + lo:offs[b] + L] = 7
    st.update_block_sums(3)
    torch.cuda.synchronize()
    got = parity.decode_block_sums(st.block_sums, wl.d_I)
    k = parity.host(t.k_idx)
    for b, L in enumerate(wl.lens):
        want = orc.block_sums(k[offs[b]:offs[b] + L], wl.hi_block)
        np.testing.assert_array_equal(got[boffs[b]:boffs[b] + want.shape[0]], want)


@pytest.mark.parametrize("n_new,hi_block", [(1, 64), (70, 64), (5, 0)])
def test_append_writes_rows_and_refreshes_block_sums(n_new, hi_block):
    """The decode append writes each sequence's newest n_new tokens (keys and
    both layers' K/V rows) and, with HI on, re-sums their blocks: the caches
    equal a host-side copy of the rows into place and the block sums equal
    the oracle's sums of the updated cache; nothing else changes."""
    wl = wls.small(BASE, name="append", lens=(1000, 71, 130, 5000), hi_block=hi_block,
                   hi_topblocks=8 if hi_block else 0, G=2, seed=31)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    gen = torch.Generator().manual_seed(1000 + n_new)
    n_seq = wl.n_seq
    k_idx_new = torch.randint(-16, 16, (n_seq, n_new, wl.d_I), dtype=torch.int8, generator=gen)
    k_new = [torch.randn((n_seq, n_new, wl.H_kv, wl.d), generator=gen).to(torch.bfloat16) for _ in range(wl.G)]
    v_new = [torch.randn((n_seq, n_new, wl.H_kv, wl.d), generator=gen).to(torch.bfloat16) for _ in range(wl.G)]
    want_k = parity.host(t.k_idx).copy()
    want_K = [parity.u16(x).copy() for x in t.k]
    want_V = [parity.u16(x).copy() for x in t.v]
    offs = parity.host(t.kv_offset)
    for b, L in enumerate(wl.lens):
        lo = offs[b] + L - n_new
        want_k[lo:lo + n_new] = k_idx_new[b].numpy()
        for g in range(wl.G):
            want_K[g][lo:lo + n_new] = k_new[g][b].view(torch.int16).numpy().view(np.uint16)
            want_V[g][lo:lo + n_new] = v_new[g][b].view(torch.int16).numpy().view(np.uint16)
    lsa.lsa_append(k_idx_new.to(DEV), t.k_idx, [x.to(DEV) for x in k_new], [x.to(DEV) for x in v_new], t.k, t.v,
                   hi_block, st.block_sums, st.batch, n_new, st.status)
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    np.testing.assert_array_equal(parity.host(t.k_idx), want_k)
    for g in range(wl.G):
        np.testing.assert_array_equal(parity.u16(t.k[g]), want_K[g])
        np.testing.assert_array_equal(parity.u16(t.v[g]), want_V[g])
    if hi_block:
        orc = oracle.get()
        got = parity.decode_block_sums(st.block_sums, wl.d_I)
        boffs = parity.host(t.blk_offset)
        for b, L in enumerate(wl.lens):
            want = orc.block_sums(want_k[offs[b]:offs[b] + L], hi_block)
            np.testing.assert_array_equal(got[boffs[b]:boffs[b] + want.shape[0]], want)


APPEND_INDEX_CASES = {
    # HI on, the new tokens inside every window: the append runs in the block selection (8-CTA clusters)
    "fused_b64": dict(lens=(3000, 71, 130, 5000, 2600, 4100, 900, 3500, 1200), hi_block=64, hi_topblocks=8,
                      window=100, sink=16, topk=300, n_new=1),
    "fused_b64_nnew4": dict(lens=(3000, 5000, 2600, 4100, 900, 3500, 1200, 6000), hi_block=64, hi_topblocks=6,
                            window=67, sink=8, topk=200, n_new=4),
    # few rows: separate coarse scores, 16-CTA clusters, two blocks of new tokens
    "fused_one_row_b128": dict(lens=(40000,), hi_block=128, hi_topblocks=40, window=260, sink=64, topk=1024,
                               n_new=130),
    # draft rows (q_len < seq_lens), n_new = drafts
    "fused_drafts": dict(lens=(4000, 6000), hi_block=64, hi_topblocks=10, window=80, sink=16, topk=300, n_new=4,
                         drafts=4),
    # not fusable: a new token's block meets the middle (window < hi_block + n_new - 1), HI off
    "sequential_window": dict(lens=(3000, 5000), hi_block=64, hi_topblocks=8, window=40, sink=16, topk=300,
                              n_new=1),
    "sequential_flat": dict(lens=(3000, 5000), hi_block=0, hi_topblocks=0, window=64, sink=16, topk=300, n_new=3),
}


@pytest.mark.parametrize("case", list(APPEND_INDEX_CASES))
def test_append_index_equals_append_then_index(case):
    """lsa_append_index: the caches hold the new rows, the block sums are the
    oracle's sums of the updated cache and the index sets are the oracle's
    sets over it, bit for bit, whether the append runs inside the block
    selection or as its own launch."""
    kw = dict(APPEND_INDEX_CASES[case])
    n_new = kw.pop("n_new")
    wl = wls.small(BASE, name=case, G=2, seed=41, **kw)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    fused = wl.hi_block > 0 and wl.window >= wl.hi_block + n_new - 1
    n_idx = lsa.lsa_index_launches(st.batch, wl.H_I, wl.d_I, st.budget)
    assert lsa.lsa_append_index_launches(st.batch, wl.H_I, wl.d_I, st.budget, n_new) == n_idx + (0 if fused else 1)
    gen = torch.Generator().manual_seed(2000 + n_new)
    n_seq = wl.n_seq
    k_idx_new = torch.randint(-16, 16, (n_seq, n_new, wl.d_I), dtype=torch.int8, generator=gen)
    k_new = [torch.randn((n_seq, n_new, wl.H_kv, wl.d), generator=gen).to(torch.bfloat16) for _ in range(wl.G)]
    v_new = [torch.randn((n_seq, n_new, wl.H_kv, wl.d), generator=gen).to(torch.bfloat16) for _ in range(wl.G)]
    want_k = parity.host(t.k_idx).copy()
    want_K = [parity.u16(x).copy() for x in t.k]
    want_V = [parity.u16(x).copy() for x in t.v]
    offs = parity.host(t.kv_offset)
    for b, L in enumerate(wl.lens):
        lo = offs[b] + L - n_new
        want_k[lo:lo + n_new] = k_idx_new[b].numpy()
        for g in range(wl.G):
            want_K[g][lo:lo + n_new] = k_new[g][b].view(torch.int16).numpy().view(np.uint16)
            want_V[g][lo:lo + n_new] = v_new[g][b].view(torch.int16).numpy().view(np.uint16)
    st.sets.fill_(-7)
    lsa.lsa_append_index(k_idx_new.to(DEV), [x.to(DEV) for x in k_new], [x.to(DEV) for x in v_new], t.k, t.v, n_new,
                         t.q_idx, t.k_idx, t.w, wl.w_max, st.batch, st.budget, st.sets, st.block_sums, st.ws_index,
                         st.status)
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    np.testing.assert_array_equal(parity.host(t.k_idx), want_k)
    for g in range(wl.G):
        np.testing.assert_array_equal(parity.u16(t.k[g]), want_K[g])
        np.testing.assert_array_equal(parity.u16(t.v[g]), want_V[g])
    if wl.hi_block:
        orc = oracle.get()
        got = parity.decode_block_sums(st.block_sums, wl.d_I)
        boffs = parity.host(t.blk_offset)
        for b, L in enumerate(wl.lens):
            want = orc.block_sums(want_k[offs[b]:offs[b] + L], wl.hi_block)
            np.testing.assert_array_equal(got[boffs[b]:boffs[b] + want.shape[0]], want)
    parity.check_sets(parity.host(st.sets), parity.oracle_sets(wl, t), wl.name)


def test_append_index_appends_to_sequences_without_rows():
    """The fused append covers every sequence of the batch, also one that no
    query row reads (rows of sequences 0 and 2 only): its new rows and block
    sum are written, and the rows' sets equal the oracle's on the updated
    cache."""
    wl = wls.small(BASE, name="ai_norows", lens=(3000, 5000, 2600), hi_block=64, hi_topblocks=8, window=100,
                   sink=16, topk=300, G=1, seed=47)
    t = wls.make(wl, DEV)
    t.q_seq.copy_(torch.tensor([0, 0, 2], dtype=torch.int32))
    t.q_len.copy_(torch.tensor([3000, 2990, 2600], dtype=torch.int32))
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    n_new = 2
    gen = torch.Generator().manual_seed(49)
    k_idx_new = torch.randint(-16, 16, (wl.n_seq, n_new, wl.d_I), dtype=torch.int8, generator=gen)
    kn = [torch.randn((wl.n_seq, n_new, wl.H_kv, wl.d), generator=gen).to(torch.bfloat16)]
    vn = [torch.randn((wl.n_seq, n_new, wl.H_kv, wl.d), generator=gen).to(torch.bfloat16)]
    want_k = parity.host(t.k_idx).copy()
    want_V = parity.u16(t.v[0]).copy()
    offs = parity.host(t.kv_offset)
    for b, L in enumerate(wl.lens):
        lo = offs[b] + L - n_new
        want_k[lo:lo + n_new] = k_idx_new[b].numpy()
        want_V[lo:lo + n_new] = vn[0][b].view(torch.int16).numpy().view(np.uint16)
    assert lsa.lsa_append_index_launches(st.batch, wl.H_I, wl.d_I, st.budget, n_new) == \
        lsa.lsa_index_launches(st.batch, wl.H_I, wl.d_I, st.budget)
    lsa.lsa_append_index(k_idx_new.to(DEV), [x.to(DEV) for x in kn], [x.to(DEV) for x in vn], t.k, t.v, n_new,
                         t.q_idx, t.k_idx, t.w, wl.w_max, st.batch, st.budget, st.sets, st.block_sums, st.ws_index,
                         st.status)
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    np.testing.assert_array_equal(parity.host(t.k_idx), want_k)
    np.testing.assert_array_equal(parity.u16(t.v[0]), want_V)
    orc = oracle.get()
    got = parity.decode_block_sums(st.block_sums, wl.d_I)
    boffs = parity.host(t.blk_offset)
    for b, L in enumerate(wl.lens):
        want = orc.block_sums(want_k[offs[b]:offs[b] + L], wl.hi_block)
        np.testing.assert_array_equal(got[boffs[b]:boffs[b] + want.shape[0]], want)
    parity.check_sets(parity.host(st.sets), parity.oracle_sets(wl, t), wl.name)


def test_append_index_flags_a_bad_sequence():
    """A sequence whose new tokens outnumber its tokens is skipped and flagged
    by the fused append (LSA_DEV_BAD_LENGTH); the other sequences' rows are
    still written."""
    wl = wls.small(BASE, name="ai_bad", lens=(3000, 5000), hi_block=64, hi_topblocks=8, window=100, sink=16,
                   topk=300, G=1, seed=43)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    n_new = 1
    k_idx_new = torch.full((wl.n_seq, n_new, wl.d_I), 5, dtype=torch.int8, device=DEV)
    kn = [torch.zeros((wl.n_seq, n_new, wl.H_kv, wl.d), dtype=torch.bfloat16, device=DEV)]
    t.seq_lens[0] = 0  # sequence 0 now holds no token
    lsa.lsa_append_index(k_idx_new, kn, kn, t.k, t.v, n_new, t.q_idx, t.k_idx, t.w, wl.w_max, st.batch, st.budget,
                         st.sets, st.block_sums, st.ws_index, st.status)
    torch.cuda.synchronize()
    assert st.status_bits() & lsa.LSA_DEV_BAD_LENGTH
    offs = parity.host(t.kv_offset)
    assert np.all(parity.host(t.k_idx)[offs[1] + 5000 - 1] == 5)


def test_extreme_block_sums_hi_block_256():
    """|S| reaches 128 * 256 = 32768: the byte planes stay exact."""
    wl = wls.small(BASE, name="bs_extreme", lens=(512,), hi_block=256, hi_topblocks=1, seed=3)
    t = wls.make(wl, DEV)
    t.k_idx[:256] = -128
    t.k_idx[256:] = 127
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    torch.cuda.synchronize()
    got = parity.decode_block_sums(st.block_sums, wl.d_I)
    assert np.all(got[0] == -32768) and np.all(got[1] == 127 * 256)


def test_device_status_flags():
    wl = wls.small(BASE, name="status", lens=(2000, 3000), hi_block=0, hi_topblocks=0, seed=5)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    # a query whose visible length exceeds its sequence
    st.t.q_len[1] = 5000
    st.index()
    torch.cuda.synchronize()
    assert st.status_bits() & lsa.LSA_DEV_BAD_LENGTH
    assert np.all(parity.host(st.sets)[1] == -1)
    # corrupted index-set entries are skipped and flagged
    st.t.q_len[1] = 3000
    st.status.zero_()
    st.index()
    sets = st.sets.clone()
    sets[0, 5] = 999999
    sets[0, 6] = -7
    lsa.lsa_attend(t.q, t.k, t.v, sets, st.batch, st.out, st.ws_attend, st.status)
    torch.cuda.synchronize()
    assert st.status_bits() & lsa.LSA_DEV_BAD_INDEX
    assert np.all(np.isfinite(parity.host(st.out[0])))
    # head weight above w_max
    st.status.zero_()
    t.w[0, 0] = wl.w_max + 1
    st.index()
    torch.cuda.synchronize()
    assert st.status_bits() & lsa.LSA_DEV_BAD_WEIGHT


def test_repeated_calls_are_deterministic():
    wl = wls.small(BASE, name="det", lens=(20000, 17000), hi_block=64, hi_topblocks=32, seed=9)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    outs, sets = [], []
    for _ in range(3):
        st.index()
        st.attend()
        torch.cuda.synchronize()
        sets.append(parity.host(st.sets).copy())
        outs.append(parity.host(st.out[0]).copy())
    assert all(np.array_equal(sets[0], s) for s in sets)
    assert all(np.array_equal(outs[0], o) for o in outs)


def test_draft_rows_per_sequence():
    """Several draft tokens per sequence in one decode step (MTP-style): row j
    of a sequence of L tokens sees L - 3 + j of them. Every row through the
    decode kernels, HI on, two layers per index set."""
    wl = wls.small(BASE, name="drafts", lens=(40000, 25000, 61000), drafts=4, hi_block=64, hi_topblocks=256,
                   G=2, seed=23)
    t = wls.make(wl, DEV)
    assert wl.n_q == 12 and parity.host(t.q_len).tolist()[:4] == [39997, 39998, 39999, 40000]
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    rows = np.arange(wl.n_q)
    want = parity.oracle_sets(wl, t, rows=rows)
    parity.check_sets(parity.host(st.sets), want, wl.name)
    ref = parity.oracle_attend_rows(t, want, rows)
    for g in range(wl.G):
        parity.check_attention(parity.host(st.out[g]), ref[g], f"{wl.name} layer {g}")


@pytest.mark.parametrize("lens,hi,G", [((6000,) * 16, False, 2), ((37, 1, 4096, 513, 2049), False, 1),
                                       ((20000, 17000, 9000), True, 2)])
def test_fp8_kv_attention(lens, hi, G):
    """Attention over FP8 E4M3 K/V caches with per-layer scales against the
    oracle's FP8 attention: 16 rows split 9 ways (two layers), ragged short
    rows including a one-token sequence, and an HI-selected set."""
    kw = dict(hi_block=64, hi_topblocks=64) if hi else dict(hi_block=0, hi_topblocks=0)
    wl = wls.small(BASE, name="fp8", lens=lens, G=G, seed=41, **kw)
    t = wls.make(wl, DEV, with_kv=False)
    st = LsaStep(wl, t, DEV, kv_fp8=True)
    st.build_block_sums()
    st.index()
    st.out[0].fill_(float("nan"))
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    rows = np.arange(wl.n_q)
    want = parity.oracle_sets(wl, t, rows=rows)
    parity.check_sets(parity.host(st.sets), want, wl.name)
    ref = parity.oracle_attend_rows_fp8(st, want, rows)
    for g in range(G):
        parity.check_attention(parity.host(st.out[g]), ref[g], f"fp8 layer {g}")


def test_graph_replay_matches_eager():
    wl = wls.small(BASE, name="graph", lens=(30000, 4000, 9000), hi_block=64, hi_topblocks=64, G=2, seed=13)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.step()
    torch.cuda.synchronize()
    sets0 = parity.host(st.sets).copy()
    outs0 = [parity.host(o).copy() for o in st.out]
    st.pack_io()  # the graphs then read and write the packed input and output buffers
    st.capture()
    st.sets.fill_(-5)
    for o in st.out:
        o.fill_(float("nan"))
    for _ in range(2):
        st.replay()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    np.testing.assert_array_equal(parity.host(st.sets), sets0)
    for g in range(len(outs0)):
        np.testing.assert_array_equal(parity.host(st.out[g]), outs0[g])
    # the step graph with timing events inside computes the same and times both calls
    st.sets.fill_(-5)
    for o in st.out:
        o.fill_(float("nan"))
    st.replay("step_timed")
    torch.cuda.synchronize()
    np.testing.assert_array_equal(parity.host(st.sets), sets0)
    for g in range(len(outs0)):
        np.testing.assert_array_equal(parity.host(st.out[g]), outs0[g])
    ms = st.call_ms()
    assert 0.0 < ms["index"] < 1000.0 and 0.0 < ms["attend"] < 1000.0
    parity.check_sets(sets0, parity.oracle_sets(wl, t), "graph")
    # the e2e graph: inputs from pinned host memory (the queries on a second
    # stream), outputs back to it; the device buffers start cleared
    h_in = st.in_buf.cpu().pin_memory()
    h_out = torch.zeros(st.out_buf.shape, dtype=torch.uint8, pin_memory=True)
    st.capture_e2e(h_in, h_out)
    st.in_buf.zero_()
    st.out_buf.zero_()
    st.sets.fill_(-5)
    st.replay("e2e")
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    np.testing.assert_array_equal(parity.host(st.sets), sets0)
    assert torch.equal(st.in_buf.cpu(), h_in)
    for g in range(len(outs0)):
        lo = st.out[g].data_ptr() - st.out_buf.data_ptr()
        got = h_out[lo:lo + st.out[g].numel() * 4].view(torch.float32).view(st.out[g].shape).numpy()
        np.testing.assert_array_equal(got, outs0[g])


# HI rows that see fewer tokens than their sequence holds, with a window
# shorter than a block: the candidate block holding a row's last visible
# token must be summed over the tokens the row sees (the oracle's block sums
# over [b*B, min((b+1)*B, L))), not taken from the stored sum of the whole
# cached block. Draft rows (more rows than sequences: coarse scores inside
# the block selection), causal prefill rows, and rows whose q_len was moved
# below seq_lens with as many rows as sequences (the separate coarse kernel).
R5_CASES = {
    "drafts_short_window": dict(lens=(5000, 3000, 7001), drafts=4, hi_block=64, hi_topblocks=16, sink=8,
                                window=10, topk=300, G=2),
    "drafts_one_seq_b128": dict(lens=(9000,), drafts=4, hi_block=128, hi_topblocks=12, sink=4, window=0,
                                topk=500),
    "prefill_rows_b32": dict(lens=(3000 + 40,), prefill_new=40, hi_block=32, hi_topblocks=20, sink=4, window=5,
                             topk=200),
}


@pytest.mark.parametrize("name", sorted(R5_CASES))
def test_hi_rows_shorter_than_their_sequence(name):
    kw = dict(R5_CASES[name])
    kw.setdefault("seed", 500 + sorted(R5_CASES).index(name))
    wl = wls.small(BASE, name=name, **kw)
    st, _ = run_case(wl)
    assert st.status_bits() == 0


def test_hi_q_len_below_seq_lens_one_row_per_sequence():
    wl = wls.small(BASE, name="r5_qlen", lens=(4000, 6000, 2500), hi_block=64, hi_topblocks=10, sink=16, window=20,
                   topk=250, seed=510)
    t = wls.make(wl, DEV)
    t.q_len.copy_(torch.tensor([3950, 5999, 2431], dtype=torch.int32, device=DEV))
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    want = parity.oracle_sets(wl, t)
    parity.check_sets(parity.host(st.sets), want, wl.name)
    ref = parity.oracle_attend_full(t, want)
    parity.check_attention(parity.host(st.out[0]), ref[0], wl.name)


def test_fp8_query_outside_fp16_range_is_flagged():
    """lsa_attend_fp8 multiplies on fp16 tensor cores: a bf16 query element
    of magnitude 65536 or more has no fp16 value, so the call flags the row
    (LSA_DEV_BAD_QUERY) instead of returning a silently wrong output; queries
    inside the range leave the status clear."""
    wl = wls.small(BASE, name="fp8_qrange", lens=(3000, 2000), hi_block=0, hi_topblocks=0, seed=43)
    t = wls.make(wl, DEV, with_kv=False)
    st = LsaStep(wl, t, DEV, kv_fp8=True)
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    t.q[0][1, 3, 17] = 65280.0  # the largest bf16 below 65504: still an fp16
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    t.q[0][1, 3, 17] = -70000.0
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() & lsa.LSA_DEV_BAD_QUERY


# lsa_attend_si on prefill chunks: the sink and window runs as dense tiles,
# the selected entries gathered per row, against the oracle's attention over
# the whole set and against lsa_attend on the same sets. Budgets with empty
# runs, rows shorter than the budget, row counts off the 16-row tiles, G = 2.
SI_CASES = {
    "si_default": dict(lens=(5000 + 77,), prefill_new=77),
    "si_short_rows": dict(lens=(40 + 300,), prefill_new=300, sink=16, window=64, topk=100),
    "si_no_sink": dict(lens=(3000 + 50,), prefill_new=50, sink=0, window=128, topk=200),
    "si_no_window": dict(lens=(3000 + 33,), prefill_new=33, sink=32, window=0, topk=200),
    "si_no_topk": dict(lens=(2000 + 40,), prefill_new=40, sink=16, window=300, topk=0),
    "si_wide_window": dict(lens=(1500 + 130,), prefill_new=130, sink=64, window=1400, topk=50),
    "si_two_layers": dict(lens=(4000 + 48,), prefill_new=48, G=2),
}


@pytest.mark.parametrize("name", sorted(SI_CASES))
def test_si_attention_on_prefill_chunks(name):
    wl = wls.small(wls.PREFILL, name=name, seed=61, **SI_CASES[name])
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    assert st.si_attend
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    sets = parity.host(st.sets)
    parity.check_sets(sets, parity.oracle_sets(wl, t), name)
    ref = parity.oracle_attend_full(t, sets)
    got = [parity.host(o).copy() for o in st.out]
    for g in range(len(t.q)):
        parity.check_attention(got[g], ref[g], f"{name} layer {g}")
    # the same sets through lsa_attend
    plain = LsaStep(wl, t, DEV, si_attend=False)
    plain.sets.copy_(st.sets)
    plain.attend()
    torch.cuda.synchronize()
    for g in range(len(t.q)):
        parity.check_attention(got[g], parity.host(plain.out[g]).astype(np.float64), f"{name} vs lsa_attend")


def test_si_attention_flags_values_beyond_fp16():
    """A V element of magnitude >= 65520 inside a window run cannot enter the
    fp16 P V of the dense tiles: LSA_DEV_BAD_VALUE."""
    wl = wls.small(wls.PREFILL, name="si_big_v", lens=(2000 + 32,), prefill_new=32, seed=62)
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.index()
    t.v[0][wl.lens[0] - wl.prefill_new - 5, 0, 3] = 1.0e6  # inside every row's window run
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() & lsa.LSA_DEV_BAD_VALUE


def test_si_attention_on_a_2048_row_chunk():
    """lsa_attend_si on 2048 rows of a 65,536-token cache (128 dense tiles of
    16 rows per kv head): 64 rows spread over the chunk (first and last
    included) against the oracle."""
    wl = wls.PREFILL_PROFILE
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    assert st.si_attend
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    rows = sorted(set(np.linspace(0, wl.n_q - 1, 64).astype(int).tolist()))
    sets = parity.host(st.sets)[rows]
    want = parity.oracle_attend_rows(t, sets, rows)
    for g in range(len(t.q)):
        parity.check_attention(parity.host(st.out[g])[rows], want[g], f"2048-row chunk layer {g}")
