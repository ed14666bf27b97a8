"""The allocation-free attention entry point.

Callers that cannot call cudaMalloc on this path (an engine whose device
memory is owned by its own pool allocator, a decode loop that must not run an
allocation) use lsa_attend_noalloc, whose scratch is a fixed static array in
the library. It must give what lsa_attend gives with a caller workspace, on
consecutive calls that share the array, and refuse shapes that do not fit.

This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
from long_context_sparse_lsa_b200 import binding as lsa
from long_context_sparse_lsa_b200 import workloads as wls
from long_context_sparse_lsa_b200.pipeline import LsaStep

pytestmark = pytest.mark.gpu


def _reference(wl):
    t = wls.make(wl, "cuda")
    st = LsaStep(wl, t, "cuda")
    st.build_block_sums()
    st.index()
    st.attend()
    torch.cuda.synchronize()
    assert st.status_bits() == 0
    return t, st, [parity.host(o).copy() for o in st.out]


@pytest.mark.parametrize("wl", [
    wls.small(wls.BATCH128K, name="noalloc_hi_g2", lens=(20000, 7000, 513), hi_topblocks=32, G=2, seed=31),
    wls.small(wls.TINY, name="noalloc_tiny", seed=32),
], ids=lambda w: w.name)
def test_noalloc_matches_workspace_version_twice(wl):
    t, st, want = _reference(wl)
    need = lsa.lsa_attend_workspace_size(st.batch, wl.H_q, wl.H_kv, wl.d, st.budget.length, len(t.q))
    assert 0 < need <= (8 << 20)
    # the oracle's attention over the oracle's own sets (the GPU sets match them bit for bit)
    sets = parity.oracle_sets(wl, t)
    parity.check_sets(parity.host(st.sets), sets, wl.name)
    ref = parity.oracle_attend_full(t, sets)
    for call in range(2):
        outs = [torch.full_like(o, float("nan")) for o in st.out]
        lsa.lsa_attend_noalloc(t.q, t.k, t.v, st.sets, st.batch, outs, st.status)
        torch.cuda.synchronize()
        assert st.status_bits() == 0
        for g in range(len(outs)):
            got = parity.host(outs[g])
            parity.check_attention(got, want[g], f"{wl.name} call {call} layer {g} vs lsa_attend")
            parity.check_attention(got, ref[g], f"{wl.name} call {call} layer {g} vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 8 rows x 8 layers with 16384-entry sets are split four ways; the split
    # partials of 64 query heads need more than the static scratch holds
    n_q, G, H_q, H_kv, budget = 8, 8, 64, 4, 16384
    dev = "cuda"
    batch = lsa.Batch(torch.zeros(1, dtype=torch.int64, device=dev), torch.full((1,), 100000, dtype=torch.int32,
                      device=dev), torch.zeros(n_q, dtype=torch.int32, device=dev),
                      torch.full((n_q,), 100000, dtype=torch.int32, device=dev), 100000, 100000)
    need = lsa.lsa_attend_workspace_size(batch, H_q, H_kv, 128, budget, G)
    assert need > (8 << 20)
    q = [torch.zeros((n_q, H_q, 128), dtype=torch.bfloat16, device=dev) for _ in range(G)]
    kv = [torch.zeros((16, H_kv, 128), dtype=torch.bfloat16, device=dev) for _ in range(G)]
    out = [torch.zeros((n_q, H_q, 128), dtype=torch.float32, device=dev) for _ in range(G)]
    sets = torch.full((n_q, budget), -1, dtype=torch.int32, device=dev)  # nothing would be read
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_attend_noalloc(q, kv, kv, sets, batch, out)
    assert e.value.status == 2  # LSA_ERR_UNSUPPORTED
