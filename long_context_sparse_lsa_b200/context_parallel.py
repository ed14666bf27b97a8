"""Context parallelism for one long sequence: its caches split by token range
over the ranks of a process group, one GPU each, with exact merges.

LSA's selections are global over a row's middle (the HI block top-k, then
the token top-k: "LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
Attention 문제"; "LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적
특징", HI and SI bullets). Split over ranks they stay exact: every member of
the global top-k, under the total order (score descending, lower id first),
is also among the top-k of its own rank's candidates under the same order.
So each rank

  1. scores the candidate HI blocks of its token range (lsa_score_blocks),
     keeps its own best hi_topblocks (lsa_merge_pairs) and all-gathers them;
     the best hi_topblocks of the union (lsa_merge_pairs) are the kept blocks,
     the same on every rank;
  2. scores the middle tokens of the kept blocks inside its range
     (lsa_score_tokens), keeps its own best topk, all-gathers them, and the
     best topk of the union are the selected tokens;
  3. assembles the index set [0, s) + selected + [ws, L), -1 padded.

The attention over that set splits the same way (ContextParallelAttention):
each rank takes the entries in its range (lsa_shard_sets), attends over them
with its own K/V rows (lsa_attend_lse: normalised output and the log of the
softmax denominator), all-gathers the partials in one collective, and the
log-sum-exp combination of the partials (lsa_combine) is the attention over
the whole set.

Candidates travel as packed 64-bit values, key << ID_BITS | (2^ID_BITS - 1 -
id) (key = score + 1), so that larger values rank first and ties go to the
lower id; a zero is an empty slot. Only the caller's device buffers, the
library's kernels and one all-gather per stage are used; the rank-local data
never leaves its GPU. Shard boundaries are multiples of hi_block, so no HI
block straddles two ranks.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as lsa

ID_BITS = lsa.MERGE_ID_BITS
ID_MASK = (1 << ID_BITS) - 1


def shard_bounds(L: int, world: int, align: int = 1) -> list[tuple[int, int]]:
    """Contiguous token ranges [lo, hi), one per rank, covering [0, L):
    equal numbers of `align`-token blocks per rank (the last may hold fewer,
    and the ragged tail of the last block); boundaries are multiples of align."""
    align = max(1, align)
    nb = (L + align - 1) // align
    per = (nb + world - 1) // world
    return [(min(r * per * align, L), min((r + 1) * per * align, L)) for r in range(world)]


def pack(keys: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
    """Packed candidate values (int64 bit patterns): key << ID_BITS |
    (ID_MASK - id); 0 where key is 0 (no candidate). keys < 2^39 (the index
    call's score bounds), 0 <= ids < 2^ID_BITS."""
    keys = keys.to(torch.int64)
    ids = ids.to(torch.int64)
    return torch.where(keys > 0, (keys << ID_BITS) | (ID_MASK - ids), torch.zeros_like(keys))


def gpu_merge(values: torch.Tensor, k: int) -> tuple[torch.Tensor, torch.Tensor]:
    """The k best packed values of each row of `values` (int64 [rows, cap],
    0 = empty) with lsa_merge_pairs: (ids int32 [rows, k] ascending, -1 after;
    the kept values int64 [rows, k], 0 after)."""
    rows, cap = values.shape
    counts = torch.full((rows,), cap, dtype=torch.int32, device=values.device)
    ids = torch.empty((rows, k), dtype=torch.int32, device=values.device)
    kept = torch.empty((rows, k), dtype=torch.int64, device=values.device)
    lsa.lsa_merge_pairs(values.contiguous(), counts, k, ids, kept)
    return ids, kept


def dist_exchange(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's equally long candidate vector (one
    collective); the ranks' vectors concatenated in rank order."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.cat(parts)


@dataclass
class Budget:
    sink: int
    window: int
    topk: int
    hi_block: int = 0
    hi_topblocks: int = 0

    @property
    def length(self) -> int:
        return self.sink + self.window + self.topk


class ContextParallelIndex:
    """The index set of one decode row whose caches are split over ranks.

    The rank holds positions [lo, hi) of the sequence: k_idx int8 [hi - lo,
    d_I] and (HI on) the block sums of its blocks, int8 [ceil((hi - lo) / B),
    2 d_I] (byte planes, as lsa_hi_block_sums writes them). score_blocks,
    score_tokens, merge and exchange default to the library's kernels and to
    an all-gather over `group`; they are parameters so that the exchange
    logic can be exercised without GPUs."""

    def __init__(self, bounds: list[tuple[int, int]], rank: int, budget: Budget, w_max: int, group=None,
                 merge=None, exchange=None, score_blocks=None, score_tokens=None):
        self.bounds = bounds
        self.rank = rank
        self.b = budget
        self.w_max = w_max
        self.group = group
        self.merge = merge or gpu_merge
        self.exchange = exchange or (lambda x: dist_exchange(x, group))
        self.score_blocks = score_blocks or self._gpu_score_blocks
        self.score_tokens = score_tokens or self._gpu_score_tokens
        lo, hi = bounds[rank]
        if budget.hi_block > 0 and lo % budget.hi_block != 0:
            raise ValueError("shard boundaries must be multiples of hi_block")

    # -- the library's kernels -------------------------------------------------
    def _gpu_score_blocks(self, q_idx, w, block_sums, blocks_local):
        dev = q_idx.device
        keys = torch.zeros((1, blocks_local.numel()), dtype=torch.int64, device=dev)
        if blocks_local.numel():
            lsa.lsa_score_blocks(q_idx[None].contiguous(), w[None].contiguous(), self.w_max, block_sums,
                                 torch.zeros(1, dtype=torch.int64, device=dev),
                                 blocks_local.to(torch.int32)[None].contiguous(), keys)
        return keys[0]

    def _gpu_score_tokens(self, q_idx, w, k_idx, pos_local):
        dev = q_idx.device
        keys = torch.zeros((1, pos_local.numel()), dtype=torch.int32, device=dev)
        if pos_local.numel():
            lsa.lsa_score_tokens(q_idx[None].contiguous(), k_idx, w[None].contiguous(), self.w_max,
                                 torch.zeros(1, dtype=torch.int64, device=dev),
                                 pos_local.to(torch.int32)[None].contiguous(), keys)
        return keys[0].to(torch.int64) & 0xFFFFFFFF

    # -- the stages --------------------------------------------------------------
    def middle(self, L: int) -> tuple[int, int]:
        s = min(self.b.sink, L)
        return s, max(s, L - self.b.window)

    def local_best(self, values: torch.Tensor, k: int) -> torch.Tensor:
        """This rank's k best candidates (packed, 0-padded to k)."""
        if k == 0:
            return torch.zeros(0, dtype=torch.int64, device=values.device)
        if values.numel() == 0:
            return torch.zeros(k, dtype=torch.int64, device=values.device)
        return self.merge(values[None], k)[1][0]

    def global_best(self, gathered: torch.Tensor, k: int) -> torch.Tensor:
        """The ids of the k best of the gathered candidates, ascending."""
        if k == 0 or gathered.numel() == 0:
            return torch.zeros(0, dtype=torch.int64, device=gathered.device)
        ids = self.merge(gathered[None], k)[0][0].to(torch.int64)
        return ids[ids >= 0]

    def block_candidates(self, q_idx, w, block_sums, L: int) -> torch.Tensor:
        """Packed keys of this rank's candidate blocks (those meeting the middle)."""
        B = self.b.hi_block
        lo, hi = self.bounds[self.rank]
        s, ws = self.middle(L)
        dev = q_idx.device
        b0 = max(s // B, lo // B)
        b1 = min((ws + B - 1) // B, (min(hi, L) + B - 1) // B) if ws > s else b0
        blocks = torch.arange(b0, max(b0, b1), dtype=torch.int64, device=dev)
        keys = self.score_blocks(q_idx, w, block_sums, blocks - lo // B)
        return pack(keys, blocks)

    def token_candidates(self, q_idx, w, k_idx, L: int, kept_blocks: torch.Tensor | None) -> torch.Tensor:
        """Packed keys of this rank's candidate tokens: the middle tokens of
        its range (inside the kept blocks when HI is on)."""
        lo, hi = self.bounds[self.rank]
        s, ws = self.middle(L)
        dev = q_idx.device
        a, b = max(s, lo), min(ws, hi)
        if self.b.hi_block > 0:
            B = self.b.hi_block
            mine = kept_blocks[(kept_blocks * B < b) & ((kept_blocks + 1) * B > a)]
            pos = (mine[:, None] * B + torch.arange(B, device=dev)[None]).reshape(-1)
            pos = pos[(pos >= a) & (pos < b)]
        else:
            pos = torch.arange(a, max(a, b), dtype=torch.int64, device=dev)
        keys = self.score_tokens(q_idx, w, k_idx, pos - lo)
        return pack(keys, pos)

    def assemble(self, L: int, selected: torch.Tensor) -> torch.Tensor:
        """[0, s) + selected + [ws, L), -1 padded to the budget."""
        s, ws = self.middle(L)
        dev = selected.device
        out = torch.cat([torch.arange(0, s, device=dev), selected.to(torch.int64), torch.arange(ws, L, device=dev)])
        pad = torch.full((self.b.length - out.numel(),), -1, dtype=torch.int64, device=dev)
        return torch.cat([out, pad]).to(torch.int32)

    def index(self, q_idx, w, k_idx, block_sums, L: int) -> torch.Tensor:
        """The row's index set, identical on every rank."""
        kept = None
        if self.b.hi_block > 0:
            local = self.local_best(self.block_candidates(q_idx, w, block_sums, L), self.b.hi_topblocks)
            kept = self.global_best(self.exchange(local), self.b.hi_topblocks)
        local = self.local_best(self.token_candidates(q_idx, w, k_idx, L, kept), self.b.topk)
        selected = self.global_best(self.exchange(local), self.b.topk)
        return self.assemble(L, selected)


class ContextParallelAttention:
    """Attention of decode rows of one sequence whose K/V caches are split
    over ranks by token range.

    The rank holds positions [lo, hi) of every layer's K and V (bf16 [hi - lo,
    H_kv, d]). Every rank passes the same index sets (int32 [n_q, budget],
    positions relative to the sequence start, e.g. from
    ContextParallelIndex); every rank returns the same output. shard,
    partial, combine and exchange default to the library's kernels and an
    all-gather over `group`; they are parameters so that the exchange logic
    can be exercised without GPUs."""

    def __init__(self, bounds: list[tuple[int, int]], rank: int, group=None, shard=None, partial=None,
                 combine=None, exchange=None):
        self.bounds = bounds
        self.rank = rank
        self.group = group
        self.shard = shard or self._gpu_shard
        self.partial = partial or self._gpu_partial
        self.combine = combine or self._gpu_combine
        self.exchange = exchange or (lambda x: dist_exchange(x, group))
        lo, hi = bounds[rank]
        if hi <= lo:
            raise ValueError("every rank needs a non-empty token range")

    # -- the library's kernels -------------------------------------------------
    @staticmethod
    def _gpu_shard(sets: torch.Tensor, lo: int, hi: int) -> torch.Tensor:
        local = torch.empty_like(sets)
        lsa.lsa_shard_sets(sets.contiguous(), lo, hi, local)
        return local

    @staticmethod
    def _gpu_partial(q: list, k: list, v: list, local_sets: torch.Tensor, n_tokens: int):
        dev = q[0].device
        n_q, H_q, d = q[0].shape
        H_kv = k[0].shape[1]
        batch = lsa.Batch(kv_offset=torch.zeros(1, dtype=torch.int64, device=dev),
                          seq_lens=torch.full((1,), n_tokens, dtype=torch.int32, device=dev),
                          q_seq=torch.zeros(n_q, dtype=torch.int32, device=dev),
                          q_len=torch.full((n_q,), n_tokens, dtype=torch.int32, device=dev),
                          max_len=n_tokens, total_tokens=n_tokens)
        G = len(q)
        ws = torch.empty(max(1, lsa.lsa_attend_workspace_size(batch, H_q, H_kv, d, local_sets.shape[1], G)),
                         dtype=torch.uint8, device=dev)
        out = torch.empty((G, n_q, H_q, d), dtype=torch.float32, device=dev)
        lse = torch.empty((G, n_q, H_q), dtype=torch.float32, device=dev)
        lsa.lsa_attend_lse(q, k, v, local_sets, batch, list(out.unbind(0)), list(lse.unbind(0)), ws)
        return out, lse

    @staticmethod
    def _gpu_combine(o_parts: torch.Tensor, lse_parts: torch.Tensor) -> torch.Tensor:
        out = torch.empty(o_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
        lsa.lsa_combine(o_parts.contiguous(), lse_parts.contiguous(), out)
        return out

    # -- the steps -------------------------------------------------------------
    def attend(self, q: list, k: list, v: list, sets: torch.Tensor) -> torch.Tensor:
        """Every layer's output (fp32 [G, n_q, H_q, d]) over the whole set.

        q: G tensors bf16 [n_q, H_q, d] (the same on every rank); k, v: this
        rank's G tensors bf16 [hi - lo, H_kv, d]."""
        lo, hi = self.bounds[self.rank]
        local = self.shard(sets, lo, hi)
        o, lse = self.partial(q, k, v, local, hi - lo)
        n_o = o.numel()
        # one collective: every rank's outputs and lse values in one vector
        gathered = self.exchange(torch.cat([o.reshape(-1), lse.reshape(-1)]))
        world = gathered.numel() // (n_o + lse.numel())
        parts = gathered.reshape(world, -1)
        o_parts = parts[:, :n_o].reshape((world,) + tuple(o.shape))
        lse_parts = parts[:, n_o:].reshape((world,) + tuple(lse.shape))
        return self.combine(o_parts, lse_parts)
