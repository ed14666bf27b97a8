"""Parity at the full workload sizes, in the launch configuration the bench
times: the step graph captured through the C ABI (block-sum append update,
index, attend) replayed once on seeded inputs.

  * batched decode, 16 sequences x 131072 tokens, HI 64 x 256: every row;
  * 1M-token decode with one index set for G = 4 layers, HI 128 x 512: the row
    and all four layers;
  * 64 ragged sequences (lognormal lengths, G = 2): every row;
  * a causal prefill chunk of 8192 rows on a 262144-token cache (HI off): 64
    rows spanning the chunk.

Index sets are compared bit-exact with the oracle; attention within
max|err| 5e-3 and rel-L2 1e-3 of its fp64 evaluation on the K/V rows the
oracle's own sets name.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import parity
from long_context_sparse_lsa_b200 import binding as lsa
from long_context_sparse_lsa_b200 import workloads as wls
from long_context_sparse_lsa_b200.pipeline import LsaStep

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_graph(wl):
    t = wls.make(wl, DEV)
    st = LsaStep(wl, t, DEV)
    st.build_block_sums()
    torch.cuda.synchronize()
    st.capture()
    st.sets.fill_(-7)
    st.replay()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    return st, t


def _check(wl, st, t, rows):
    rows = np.asarray(rows)
    want = parity.oracle_sets(wl, t, rows=rows)
    parity.check_sets(parity.host(st.sets)[rows], want, wl.name)
    ref = parity.oracle_attend_rows(t, want, rows)
    for g in range(len(t.q)):
        parity.check_attention(parity.host(st.out[g])[rows], ref[g], f"{wl.name} layer {g}")


def _free():
    """Return the cached device memory once the caller has dropped its last
    references to a workload's buffers (``del st, t`` first)."""
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_batched_decode_128k_every_row():
    wl = wls.BATCH128K
    st, t = _run_graph(wl)
    _check(wl, st, t, np.arange(wl.n_q))
    del st, t
    _free()


def test_1m_cross_layer_decode_every_layer():
    wl = wls.CTX1M
    st, t = _run_graph(wl)
    assert len(t.q) == 4
    _check(wl, st, t, np.arange(wl.n_q))
    del st, t
    _free()


def test_ragged_batch_every_row():
    wl = wls.ragged()
    st, t = _run_graph(wl)
    _check(wl, st, t, np.arange(wl.n_q))
    del st, t
    _free()


def test_fp8_kv_decode_128k_sample():
    """The 16 x 131072 decode with FP8 E4M3 K/V caches, through the step graph
    the bench times: index sets bit-exact on every row, the FP8 attention of a
    sample of rows against the oracle's."""
    wl = wls.BATCH128K
    t = wls.make(wl, DEV, with_kv=False)
    st = LsaStep(wl, t, DEV, kv_fp8=True)
    st.build_block_sums()
    torch.cuda.synchronize()
    st.capture()
    st.sets.fill_(-7)
    st.replay()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    rows = np.arange(wl.n_q)
    want = parity.oracle_sets(wl, t, rows=rows)
    parity.check_sets(parity.host(st.sets), want, wl.name)
    sample = np.array([0, 5, 11, 15])
    ref = parity.oracle_attend_rows_fp8(st, want[sample], sample)
    parity.check_attention(parity.host(st.out[0])[sample], ref[0], "fp8 128k")
    del st, t
    _free()


def test_prefill_chunk_sample():
    wl = wls.PREFILL
    st, t = _run_graph(wl)
    assert lsa.lsa_index_uses_tensor_cores(st.batch, wl.H_I, wl.d_I, st.budget)
    n = wl.n_q
    # 64 rows spread over the chunk (both ends, every 1/62 of it between)
    rows = sorted({0, 1, n - 2, n - 1} | {int(x) for x in np.linspace(2, n - 3, 60)})
    assert len(rows) == 64
    _check(wl, st, t, rows)
    del st, t
    _free()
