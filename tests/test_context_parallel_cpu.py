"""Context parallelism on CPU: one sequence's index set computed by two gloo
ranks, each holding one token range of the caches, through the exchange and
stage logic of long_context_sparse_lsa_b200.context_parallel, must equal the
single-device oracle's set bit for bit, including when many scores tie
across the two ranges (the lower position must win across ranks too); and
the attention over such a set, each rank attending over its own entries and
the partials combined by their log-sum-exp after one all-gather, must equal
the oracle's attention over the whole set.

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


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def numpy_shard(sets: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
    s = sets.numpy()
    out = np.full_like(s, -1)
    for r in range(s.shape[0]):
        keep = s[r][(s[r] >= lo) & (s[r] < hi)] - lo
        out[r, : keep.size] = keep
    return torch.from_numpy(out)


def numpy_partial(q, k, v, local_sets, n_tokens):
    """Softmax attention over each row's local entries in fp64 (scale
    1/sqrt(d), q head h -> kv head h // (H_q / H_kv)): the normalised output
    and ln of the denominator (-inf and zeros for no entry)."""
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k[0].shape[1]
    ratio = H_q // H_kv
    out = np.zeros((G, n_q, H_q, d))
    lse = np.full((G, n_q, H_q), -np.inf)
    s = local_sets.numpy()
    for g in range(G):
        qg, kg, vg = (bf16_to_f64(x[g].view(torch.int16).numpy().view(np.uint16)) for x in (q, k, v))
        for r in range(n_q):
            e = s[r][s[r] >= 0]
            if e.size == 0:
                continue
            for h in range(H_q):
                sc = kg[e, h // ratio] @ qg[r, h] / np.sqrt(d)
                m = sc.max()
                p = np.exp(sc - m)
                out[g, r, h] = p @ vg[e, h // ratio] / p.sum()
                lse[g, r, h] = m + np.log(p.sum())
    return torch.from_numpy(out), torch.from_numpy(lse)


def numpy_combine(o_parts: torch.Tensor, lse_parts: torch.Tensor) -> torch.Tensor:
    o, l = o_parts.numpy(), lse_parts.numpy()
    M = l.max(axis=0)
    wgt = np.where(np.isfinite(l), np.exp(l - np.where(np.isfinite(M), M, 0.0)), 0.0)
    den = wgt.sum(axis=0)
    out = (wgt[..., None] * o).sum(axis=0) / np.where(den > 0, den, 1.0)[..., None]
    return torch.from_numpy(out)


def _attend_rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # one sequence of 3000 tokens, G = 2, three decode rows whose sets
        # (from the oracle's index) spread over both token ranges; a fourth
        # row's set holds only sink tokens (rank 1 has none of them)
        base = wls.small(wls.BATCH128K, name="cpa", lens=(3000,), G=2)
        wl = wls.small(base, lens=(3000,), drafts=3, hi_block=64, hi_topblocks=10, sink=16, window=64, topk=200,
                       seed=75)
        t = wls.make(wl, "cpu")
        orc = oracle.get()
        L = wl.lens[0]
        sets = []
        for r in range(wl.n_q):
            Lr = int(t.q_len[r])
            sets.append(orc.index_query(t.q_idx[r].numpy(), t.w[r].numpy(), t.k_idx.numpy(), Lr, wl.sink,
                                        wl.window, wl.topk, wl.hi_block, wl.hi_topblocks))
        sink_only = np.full_like(sets[0], -1)
        sink_only[:5] = np.arange(5)
        sets = np.stack(sets + [sink_only]).astype(np.int32)
        q = [torch.cat([x, x[:1]]) for x in t.q]  # the fourth row reuses row 0's query
        bounds = cp.shard_bounds(L, world, 64)
        lo, hi = bounds[rank]
        att = cp.ContextParallelAttention(bounds, rank, shard=numpy_shard, partial=numpy_partial,
                                          combine=numpy_combine)
        got = att.attend(q, [x[lo:hi] for x in t.k], [x[lo:hi] for x in t.v], torch.from_numpy(sets)).numpy()
        want = []
        for g in range(wl.G):
            kk, vv = (x[g].view(torch.int16).numpy().view(np.uint16) for x in (t.k, t.v))
            qq = q[g].view(torch.int16).numpy().view(np.uint16)
            want.append(np.stack([orc.attend_query(qq[r], kk, vv, sets[r]) for r in range(sets.shape[0])]))
        out.put((rank, float(np.abs(got - np.stack(want)).max())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_attention_equals_the_whole_set():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_attend_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the combination is exact: the fp64 partials combine to the oracle's
    # fp64 attention up to rounding
    assert all(err < 1e-9 for _, err in res), res


def test_combine_of_one_part_is_that_part_and_empty_parts_drop_out():
    rng = np.random.default_rng(3)
    o = torch.from_numpy(rng.normal(size=(3, 5, 8)))
    lse = torch.from_numpy(rng.normal(size=(3, 5)))
    lse[1] = -np.inf
    lse[2] = -np.inf
    np.testing.assert_allclose(numpy_combine(o, lse).numpy(), o[0].numpy())
    # two parts with equal lse: the mean of their outputs
    lse2 = torch.zeros((2, 5), dtype=torch.float64)
    np.testing.assert_allclose(numpy_combine(o[:2], lse2).numpy(), o[:2].mean(0).numpy())


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
