"""Host logic on CPU: the bench's algorithmic byte counts, the draft-row
layout, and the decode step's sequencing rules (which calls may overlap, how
many kernels a step launches) for small workloads built on the CPU device."""
from __future__ import annotations

import pytest
import torch

import bench
from long_context_sparse_lsa_b200 import workloads as wls
from long_context_sparse_lsa_b200.pipeline import LsaStep


def test_step_bytes_of_the_batched_128k_decode():
    b = bench.step_bytes(wls.BATCH128K)
    # per query: 3136 entries x (K + V) x 4 kv heads x 256 B, q (bf16), out (f32), set (int32)
    per_q = 2 * 3136 * 1024 + 32 * 128 * 2 + 32 * 128 * 4 + 3136 * 4
    assert b["attend"] == 16 * per_q == 103_354_368
    # per query: the block sums of the middle's blocks, the kept keys, q, w, the set write
    nb = (131072 - 1024 + 63) // 64 - 64 // 64
    per_i = nb * 256 + 256 * 64 * 128 + 16 * 128 + 16 * 4 + 3136 * 4
    assert b["index"] == 16 * per_i
    # per sequence: the new token's key and K/V rows read and written, one block re-read, its sums written
    assert b["append"] == 16 * (2 * (128 + 2 * 1024) + 64 * 128 + 256)
    assert b["total"] == b["attend"] + b["index"] + b["append"]


def test_fp8_caches_halve_the_attention_rows():
    b16, b8 = bench.step_bytes(wls.BATCH128K), bench.step_bytes(wls.BATCH128K, kv_fp8=True)
    assert b16["attend"] - b8["attend"] == 16 * 3136 * 1024  # (K + V) x 512 B saved per entry
    assert b8["index"] == b16["index"]


def test_cold_build_reads_every_key_once():
    wl = wls.BATCH128K
    assert bench.cold_block_sum_bytes(wl) == 16 * 131072 * 128 + 16 * 2048 * 256
    assert bench.cold_block_sum_bytes(wls.PREFILL) == 0  # HI off: no block sums


def test_draft_rows_layout_and_row_lengths():
    wl = wls.small(wls.BATCH128K, lens=(100, 50), drafts=3)
    assert wl.n_q == 6
    off, lens, boff, q_seq, q_len, nb = wls.layout(wl, "cpu")
    assert q_seq.tolist() == [0, 0, 0, 1, 1, 1]
    assert q_len.tolist() == [98, 99, 100, 48, 49, 50]
    assert bench._rows(wl) == [98, 99, 100, 48, 49, 50]


def _step(wl, **kw):
    t = wls.make(wl, "cpu", with_kv=not kw.get("kv_fp8", False))
    return LsaStep(wl, t, "cpu", **kw)


def test_append_overlaps_the_index_call_only_on_disjoint_rows():
    base = wls.small(wls.BATCH128K, lens=(3000, 2000), seed=3)
    # HI on: the append rewrites the newest tokens' block; coarse scores read blocks before the window
    assert _step(wls.small(base, window=1024, hi_block=64)).overlap_ok()
    assert _step(wls.small(base, window=64, hi_block=64)).overlap_ok()          # window >= B + n_new - 1
    assert not _step(wls.small(base, window=62, hi_block=64)).overlap_ok()
    assert not _step(wls.small(base, window=65, hi_block=64, drafts=4)).overlap_ok()
    # HI off: only the new tokens' keys must lie in the window
    flat = wls.small(base, hi_block=0, hi_topblocks=0)
    assert _step(wls.small(flat, window=1)).overlap_ok()
    assert not _step(wls.small(flat, window=1, drafts=2)).overlap_ok()
    # a prefill chunk has no append
    st = _step(wls.small(wls.PREFILL, lens=(3000,), prefill_new=100))
    assert st.n_new == 0 and not st.overlap_ok()


def test_new_rows_are_the_newest_cached_tokens():
    wl = wls.small(wls.BATCH128K, lens=(300, 70), drafts=2, G=2, seed=5)
    st = _step(wl)
    t = st.t
    for b, (o, L) in enumerate(zip(t.kv_offset.tolist(), t.seq_lens.tolist())):
        assert torch.equal(st.k_idx_new[b], t.k_idx[o + L - 2:o + L])
        for g in range(2):
            assert torch.equal(st.k_new[g][b], t.k[g][o + L - 2:o + L])
            assert torch.equal(st.v_new[g][b], t.v[g][o + L - 2:o + L])
    st8 = _step(wl, kv_fp8=True)
    assert st8.k8[0].dtype == torch.uint8 and st8.k_new[0].dtype == torch.uint8
    o, L = t.kv_offset.tolist()[1], t.seq_lens.tolist()[1]
    assert torch.equal(st8.v_new[1][1], st8.v8[1][o + L - 2:o + L])


@pytest.mark.parametrize("wl,n,fuse", [(wls.BATCH128K, 5, True), (wls.CTX1M, 6, True), (wls.BATCH128K, 6, False),
                                       (wls.CTX1M, 7, False)])
def test_kernels_per_step(wl, n, fuse):
    """16 rows: block selection with the coarse scores and the append inside, fine scores,
    token selection, attention, merge; one 1M row adds the separate coarse-score kernel;
    without the fused call the append is a launch of its own."""
    small = wls.small(wl, lens=tuple(min(L, 4096) for L in wl.lens))
    st = _step(small, fuse_append=fuse)
    # the plan depends on the shape's host fields only; use the real lengths for it
    st.batch.max_len = max(wl.lens)
    assert st.kernels_per_step() == n


@pytest.mark.parametrize("kv_fp8", [False, True])
def test_pack_io_keeps_values_in_one_aligned_buffer(kv_fp8):
    """pack_io: the per-step inputs and the outputs become 256-byte aligned
    views of one buffer each, with their values unchanged."""
    wl = wls.small(wls.BATCH128K, lens=(300, 70), drafts=2, G=2, seed=7)
    st = _step(wl, kv_fp8=kv_fp8)
    t = st.t
    before = [x.clone() for x in [t.q_idx, t.w, *t.q, st.k_idx_new, *st.k_new, *st.v_new]]
    st.pack_io()
    after = [t.q_idx, t.w, *t.q, st.k_idx_new, *st.k_new, *st.v_new]
    lo = st.in_buf.data_ptr()
    hi = lo + st.in_buf.numel()
    for b, a in zip(before, after):
        assert torch.equal(a, b) and a.dtype == b.dtype and a.is_contiguous()
        assert (a.data_ptr() - lo) % 256 == 0 and lo <= a.data_ptr() and a.data_ptr() + a.numel() * a.element_size() <= hi
    # the views do not overlap: writing one leaves the others unchanged
    t.w.fill_(-1)
    assert torch.equal(t.q_idx, before[0]) and torch.equal(t.q[0], before[2])
    olo = st.out_buf.data_ptr()
    assert len(st.out) == 2
    for o in st.out:
        assert o.dtype == torch.float32 and o.shape == (wl.n_q, wl.H_q, wl.d)
        assert (o.data_ptr() - olo) % 256 == 0
    assert st.out[1].data_ptr() - st.out[0].data_ptr() >= st.out[0].numel() * 4


def test_pageable_host_memory_is_not_written_by_kernels():
    """The e2e graph lets the attention write into a host buffer only when the
    device can address it at its own address; pageable memory never can."""
    from long_context_sparse_lsa_b200.pipeline import _device_addressable
    assert not _device_addressable(torch.empty(4096, dtype=torch.uint8))
