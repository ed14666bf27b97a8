"""The synthetic workloads of the LSA hot path and their seeded tensors.

Shapes follow the pages' serving picture (a 69B / 3B-active MoE with native
1,024K context served on one node: "LongCat-Flash-Lite-Sparse (aitrends.kr)",
TL;DR and "알아두면 좋은 것"); the pages publish no kernel workload, so the
sizes below are this library's stand-ins. Inputs are drawn by ``inputs``;
this module only lays them out (no arithmetic of the method).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import inputs as gen


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    lens: tuple[int, ...]          # tokens per sequence (decode: incl. the current one)
    H_I: int
    d_I: int
    qk_lo: int
    qk_hi: int
    w_hi: int
    sink: int
    window: int
    topk: int
    hi_block: int                  # 0 = HI off
    hi_topblocks: int
    H_q: int
    H_kv: int
    d: int
    G: int                         # layers sharing one index set
    prefill_new: int = 0           # > 0: a causal prefill chunk of this many tokens on sequence 0
    drafts: int = 1                # decode rows per sequence (several draft tokens, MTP-style):
                                   # row j of a sequence of L tokens sees L - drafts + 1 + j
    draft_share: int = 0           # percent of each later draft row's indexer-query elements (and all of
                                   # its head weights, when > 0) taken from the sequence's first draft row
    note: str = field(default="", compare=False)

    @property
    def budget(self) -> int:
        return self.sink + self.window + self.topk

    @property
    def n_seq(self) -> int:
        return len(self.lens)

    @property
    def total_tokens(self) -> int:
        return sum(self.lens)

    @property
    def n_q(self) -> int:
        return self.prefill_new if self.prefill_new else self.n_seq * self.drafts

    @property
    def w_max(self) -> int:
        return self.w_hi


def _ragged_lens(seed: int) -> tuple[int, ...]:
    return tuple(gen.lognormal_lengths(64, 32768.0, 1.0, 8192, 1 << 20, 12 << 20, seed, gen.STREAM_LENS))


TINY = Workload("tiny_decode_4k", 0, (4096,), 4, 32, -8, 7, 4, 4, 128, 256, 0, 0, 8, 1, 128, 1,
                note="tiny decode, 1 seq x 4096, HI off")
BATCH128K = Workload("decode_b16_128k_hi64x256", 1, (131072,) * 16, 16, 128, -16, 15, 8, 64, 1024, 2048,
                     64, 256, 32, 4, 128, 1, note="batched decode, 16 seqs x 131072, HI 64x256")
CTX1M = Workload("decode_b1_1m_cli4_hi128x512", 2, (1048576,), 16, 128, -16, 15, 8, 64, 2048, 2048,
                 128, 512, 32, 4, 128, 4, note="1M decode, G=4 layers per index set, HI 128x512")
# Draft rows: 4 sequences x 4 draft tokens on the 128K shape (16 decode rows,
# as the batched case); later drafts share 75% of the first draft's indexer
# query elements.
DRAFTS128K = Workload("decode_b4x4_128k_drafts_hi64x256", 5, (131072,) * 4, 16, 128, -16, 15, 8, 64, 1024, 2048,
                      64, 256, 32, 4, 128, 1, drafts=4, draft_share=75,
                      note="4 seqs x 4 draft rows, 131072 tokens, HI 64x256, drafts share 75% of the indexer query")
PREFILL = Workload("prefill_8192_on_262144", 3, (262144 + 8192,), 16, 128, -16, 15, 8, 64, 1024, 2048,
                   0, 0, 32, 4, 128, 1, prefill_new=8192,
                   note="causal prefill chunk of 8192 tokens on a 262144-token cache, HI off")


# The batched-decode shape on a 32768-token context: the same per-query
# attention and fine-index work as the 128K case on a 4x smaller cache, for
# profiler captures that must stay a few GB on the device.
PROFILE32K = Workload("decode_b16_32k_hi64x256", 1, (32768,) * 16, 16, 128, -16, 15, 8, 64, 1024, 2048,
                      64, 256, 32, 4, 128, 1, note="batched decode, 16 seqs x 32768, HI 64x256 (profiling size)")


# A smaller prefill chunk (2048 rows on a 65536-token cache, same heads and
# budget) for profiler captures of the tensor-core indexer.
PREFILL_PROFILE = Workload("prefill_2048_on_65536", 3, (65536 + 2048,), 16, 128, -16, 15, 8, 64, 1024, 2048,
                           0, 0, 32, 4, 128, 1, prefill_new=2048,
                           note="causal prefill chunk of 2048 tokens on a 65536-token cache, HI off (profiling size)")


def ragged() -> Workload:
    return Workload("ragged_decode_64seq_lognormal", 4, _ragged_lens(4), 16, 128, -16, 15, 8, 64, 1024, 2048,
                    64, 256, 32, 4, 128, 2, note="64 ragged seqs, lognormal median 32768, G=2, HI 64x256")


def all_workloads() -> list[Workload]:
    return [TINY, BATCH128K, CTX1M, PREFILL, ragged(), PROFILE32K, PREFILL_PROFILE, DRAFTS128K]


def by_name(name: str) -> Workload:
    for w in all_workloads():
        if w.name == name:
            return w
    raise KeyError(name)


@dataclass
class Tensors:
    """Device (or host) tensors of one workload draw."""
    q_idx: torch.Tensor        # int8 [n_q, H_I, d_I]
    k_idx: torch.Tensor        # int8 [T, d_I]
    w: torch.Tensor            # int32 [n_q, H_I]
    q: list                    # G x bf16 [n_q, H_q, d]
    k: list                    # G x bf16 [T, H_kv, d]
    v: list                    # G x bf16 [T, H_kv, d]
    kv_offset: torch.Tensor    # int64 [n_seq]
    seq_lens: torch.Tensor     # int32 [n_seq]
    blk_offset: torch.Tensor   # int64 [n_seq] (rows of the block-sum cache)
    q_seq: torch.Tensor        # int32 [n_q]
    q_len: torch.Tensor        # int32 [n_q]
    n_blk_rows: int            # rows of the block-sum cache


def layout(wl: Workload, device, hi_block: int | None = None):
    """Sequence offsets, query rows and block-sum rows of a workload."""
    hb = wl.hi_block if hi_block is None else hi_block
    lens = list(wl.lens)
    offs, acc = [], 0
    for L in lens:
        offs.append(acc)
        acc += L
    boffs, bacc = [], 0
    for L in lens:
        boffs.append(bacc)
        bacc += (L + hb - 1) // hb if hb > 0 else 0
    if wl.prefill_new:
        C = lens[0] - wl.prefill_new
        q_seq = [0] * wl.prefill_new
        q_len = [C + i + 1 for i in range(wl.prefill_new)]
    else:
        D = wl.drafts
        q_seq = [b for b in range(len(lens)) for _ in range(D)]
        q_len = [L - D + 1 + j for L in lens for j in range(D)]
    t = lambda x, dt: torch.tensor(x, dtype=dt, device=device)
    return (t(offs, torch.int64), t(lens, torch.int32), t(boffs, torch.int64), t(q_seq, torch.int32),
            t(q_len, torch.int32), bacc)


def make(wl: Workload, device, layers: int | None = None, with_kv: bool = True) -> Tensors:
    """Draw every tensor of a workload on ``device``."""
    G = wl.G if layers is None else layers
    s = wl.seed
    T = wl.total_tokens
    n_q = wl.n_q
    q_idx = gen.uniform_int8((n_q, wl.H_I, wl.d_I), wl.qk_lo, wl.qk_hi, s, gen.STREAM_Q_IDX, device)
    k_idx = gen.uniform_int8((T, wl.d_I), wl.qk_lo, wl.qk_hi, s, gen.STREAM_K_IDX, device)
    w = gen.uniform_weights((n_q, wl.H_I), wl.w_hi, s, gen.STREAM_W, device)
    if wl.drafts > 1 and wl.draft_share > 0 and not wl.prefill_new:
        # draft tokens of one sequence ask for similar context: later drafts
        # copy a share of the first draft's indexer query and its weights
        D = wl.drafts
        pick = gen.uniform_int8((n_q, wl.H_I, wl.d_I), 0, 99, s, gen.STREAM_DRAFT, device) < wl.draft_share
        first = torch.arange(n_q, device=device) // D * D
        q_idx = torch.where(pick, q_idx[first], q_idx)
        w = w[first].clone()
    q, k, v = [], [], []
    for g in range(G):
        q.append(gen.normal_bf16((n_q, wl.H_q, wl.d), s, gen.STREAM_Q + g, device))
        if with_kv:
            k.append(gen.normal_bf16((T, wl.H_kv, wl.d), s, gen.STREAM_K + g, device))
            v.append(gen.normal_bf16((T, wl.H_kv, wl.d), s, gen.STREAM_V + g, device))
    kv_offset, seq_lens, blk_offset, q_seq, q_len, nb = layout(wl, device)
    return Tensors(q_idx, k_idx, w, q, k, v, kv_offset, seq_lens, blk_offset, q_seq, q_len, nb)


def small(wl: Workload, **changes) -> Workload:
    """A reduced copy of a workload (same generator, different sizes)."""
    fields = dict(wl.__dict__)
    fields.update(changes)
    return Workload(**fields)
