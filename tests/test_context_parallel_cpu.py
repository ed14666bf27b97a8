"""Context parallelism on CPU: one sequence's index set computed by two gloo
ranks, each holding one token range of the caches, through the exchange and
stage logic of long_context_sparse_lsa_b200.context_parallel, must equal the
single-device oracle's set bit for bit, including when many scores tie
across the two ranges (the lower position must win across ranks too).

The library's kernels need a GPU; here each rank's scores come from the
oracle (its fine and coarse score functions on the rank's own keys) and the
merge of packed candidate values is a plain numpy sort — the test checks the
protocol (shard bounds, candidate packing, one all-gather per stage, the
global choice from the union of the ranks' best) and the exactness of
choosing from that union, not the kernels (tests/test_gpu_parity.py does)."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from long_context_sparse_lsa_b200 import context_parallel as cp
from long_context_sparse_lsa_b200 import workloads as wls


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def numpy_merge(values: torch.Tensor, k: int):
    """The k best packed values of each row (0 = empty): ids ascending with -1
    after, and the kept values in id order with 0 after."""
    v = values.numpy().astype(np.int64).view(np.uint64)
    rows = v.shape[0]
    ids = np.full((rows, k), -1, np.int32)
    kept = np.zeros((rows, k), np.uint64)
    for r in range(rows):
        x = v[r][v[r] != 0]
        best = np.sort(x)[::-1][:k]
        i = (cp.ID_MASK - (best & np.uint64(cp.ID_MASK))).astype(np.int64)
        order = np.argsort(i)
        ids[r, : len(best)] = i[order]
        kept[r, : len(best)] = best[order]
    return torch.from_numpy(ids), torch.from_numpy(kept.view(np.int64))


def _cases():
    base = wls.small(wls.BATCH128K, name="cp", lens=(3000,), G=1)
    return {
        # tiny score range: many equal scores across the two ranges
        "hi_ties": wls.small(base, lens=(3000,), hi_block=64, hi_topblocks=12, sink=16, window=100, topk=300,
                             qk_lo=-1, qk_hi=1, w_hi=1, seed=71),
        "hi_random": wls.small(base, lens=(5003,), hi_block=32, hi_topblocks=40, sink=10, window=77, topk=500,
                               seed=72),
        "flat_ties": wls.small(base, lens=(2500,), hi_block=0, hi_topblocks=0, sink=8, window=64, topk=400,
                               qk_lo=-1, qk_hi=1, w_hi=1, seed=73),
        "hi_all_blocks": wls.small(base, lens=(1500,), hi_block=64, hi_topblocks=4096, sink=4, window=30, topk=200,
                                   seed=74),
    }


def _rank_main(rank: int, world: int, port: int, name: str, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _cases()[name]
        t = wls.make(wl, "cpu")
        orc = oracle.get()
        L = wl.lens[0]
        B = wl.hi_block
        bounds = cp.shard_bounds(L, world, B if B > 0 else 1)
        lo, hi = bounds[rank]
        k_all = t.k_idx.numpy()
        k_mine = k_all[lo:hi]
        q = t.q_idx[0].numpy()
        w = t.w[0].numpy()
        sums = orc.block_sums(k_mine, B) if B > 0 else None  # this rank's blocks only

        def score_blocks(q_idx, w_, block_sums, blocks_local):
            keys = [orc.coarse_score(q, w, block_sums[int(b)]) + 1 for b in blocks_local.tolist()]
            return torch.tensor(keys, dtype=torch.int64)

        def score_tokens(q_idx, w_, k_idx, pos_local):
            keys = [orc.fine_score(q, w, k_idx[int(p)]) + 1 for p in pos_local.tolist()]
            return torch.tensor(keys, dtype=torch.int64)

        idx = cp.ContextParallelIndex(bounds, rank, cp.Budget(wl.sink, wl.window, wl.topk, B, wl.hi_topblocks),
                                      wl.w_max, merge=numpy_merge, score_blocks=score_blocks,
                                      score_tokens=score_tokens)
        got = idx.index(t.q_idx[0], t.w[0], k_mine, sums, L).numpy()
        want = orc.index_query(q, w, k_all, L, wl.sink, wl.window, wl.topk, B, wl.hi_topblocks)
        out.put((rank, got.tolist(), want.tolist(), bounds))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(_cases()))
def test_two_ranks_give_the_single_device_set(name):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, got0, want, bounds), (_, got1, _, _) = res
    assert bounds[0][1] == bounds[1][0] and bounds[0][0] == 0  # two non-empty token ranges
    assert got0 == got1                                        # every rank holds the same set
    assert got0 == want                                        # ... the single-device oracle's


def test_shard_bounds_are_block_aligned_and_cover_the_sequence():
    for L, world, align in ((3000, 2, 64), (5003, 3, 32), (7, 4, 1), (128, 2, 128)):
        b = cp.shard_bounds(L, world, align)
        assert b[0][0] == 0 and b[-1][1] == L
        assert all(lo % align == 0 for lo, _ in b)
        assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))


def test_pack_orders_by_key_then_lower_id():
    keys = torch.tensor([5, 5, 7, 0], dtype=torch.int64)
    ids = torch.tensor([10, 3, 99, 1], dtype=torch.int64)
    v = cp.pack(keys, ids).numpy().view(np.uint64)
    assert v[3] == 0                          # no candidate
    assert v[2] > v[1] > v[0]                 # key 7 first, then key 5 with the lower id
    ids_out, _ = numpy_merge(cp.pack(keys, ids)[None], 2)
    assert ids_out.tolist() == [[3, 99]]
