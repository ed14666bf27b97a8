"""A decode step of the LSA hot path over one workload, through the C ABI.

Allocation and call sequencing only (device buffers via torch, calls via
``binding``): the HI block-sum append update, one ``lsa_index`` per group of
G layers (Cross-Layer Indexing) and one ``lsa_attend`` for the G layers.
"""
from __future__ import annotations

import torch

from . import binding as lsa
from .workloads import Tensors, Workload


class LsaStep:
    def __init__(self, wl: Workload, t: Tensors, device="cuda"):
        self.wl = wl
        self.t = t
        self.device = device
        self.G = len(t.q)
        self.batch = lsa.Batch(t.kv_offset, t.seq_lens, t.q_seq, t.q_len, max(wl.lens), wl.total_tokens,
                               t.blk_offset if wl.hi_block > 0 else None)
        self.budget = lsa.Budget(wl.sink, wl.window, wl.topk, wl.hi_block, wl.hi_topblocks)
        n_q = wl.n_q
        self.sets = torch.empty((n_q, self.budget.length), dtype=torch.int32, device=device)
        self.out = [torch.empty((n_q, wl.H_q, wl.d), dtype=torch.float32, device=device) for _ in range(self.G)]
        self.block_sums = None
        if wl.hi_block > 0:
            self.block_sums = torch.zeros((max(1, t.n_blk_rows), 2 * wl.d_I), dtype=torch.int8, device=device)
        ws_i = lsa.lsa_index_workspace_size(self.batch, wl.H_I, wl.d_I, self.budget)
        self.ws_index = torch.empty(max(1, ws_i), dtype=torch.uint8, device=device) if ws_i else None
        ws_a = lsa.lsa_attend_workspace_size(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget.length, self.G)
        self.ws_attend = torch.zeros(max(256, ws_a), dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    # -- the three calls --------------------------------------------------------
    def build_block_sums(self, stream=None):
        if self.block_sums is not None:
            lsa.lsa_hi_block_sums(self.t.k_idx, self.wl.hi_block, self.batch, self.block_sums, 0, self.status, stream)

    def update_block_sums(self, n_new: int = 1, stream=None):
        if self.block_sums is not None:
            lsa.lsa_hi_block_sums(self.t.k_idx, self.wl.hi_block, self.batch, self.block_sums, n_new, self.status,
                                  stream)

    def index(self, stream=None):
        lsa.lsa_index(self.t.q_idx, self.t.k_idx, self.t.w, self.wl.w_max, self.batch, self.budget, self.sets,
                      self.block_sums, self.ws_index, self.status, stream)

    def attend(self, stream=None):
        lsa.lsa_attend(self.t.q, self.t.k, self.t.v, self.sets, self.batch, self.out, self.ws_attend, self.status,
                       stream)

    def step(self, stream=None):
        """One decode step: append update of the block sums, index, attend."""
        self.update_block_sums(1, stream)
        self.index(stream)
        self.attend(stream)

    def overlap_ok(self, n_new: int = 1) -> bool:
        """True when the block-sum append update may run beside the index call.

        The update rewrites only the blocks holding the n_new newest tokens;
        the coarse HI scores read only blocks that end before the window
        start. With window >= hi_block + n_new - 1 those blocks lie inside the
        window and the two calls touch disjoint rows."""
        wl = self.wl
        return self.block_sums is not None and wl.window >= wl.hi_block + n_new - 1

    def status_bits(self) -> int:
        return int(self.status.item())

    # -- CUDA graphs ------------------------------------------------------------
    def capture(self):
        """Capture the three calls as CUDA graphs (block-sum append update,
        index, attend), and the whole step as one more graph ("step") in which
        the block-sum update runs on a forked stream beside the index call when
        overlap_ok(). A step then replays without host launch overhead. The
        graphs keep this object's buffers; changing their contents between
        replays is how new inputs enter."""
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):  # one eager pass fills the launch-plan caches
            self.step()
        torch.cuda.current_stream(self.device).wait_stream(side)
        torch.cuda.synchronize(self.device)
        self.graphs = {}
        for name, fn in (("block_sums", lambda: self.update_block_sums(1)), ("index", self.index),
                         ("attend", self.attend)):
            if name == "block_sums" and self.block_sums is None:
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                fn()
            self.graphs[name] = g
        g = torch.cuda.CUDAGraph()
        fork = torch.cuda.Stream(self.device)
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            cur = torch.cuda.current_stream(self.device)
            if self.overlap_ok(1):
                fork.wait_stream(cur)
                with torch.cuda.stream(fork):
                    self.update_block_sums(1)
                self.index()
                cur.wait_stream(fork)
                self.attend()
            else:
                self.step()
        self.graphs["step"] = g
        # the same step with timing events recorded around the index and
        # attention calls inside the graph: their durations within a step,
        # without the launch of a graph of their own
        ev = lambda: torch.cuda.Event(enable_timing=True, external=True)
        self.call_events = {"index": (ev(), ev()), "attend": (ev(), ev())}
        (ix0, ix1), (at0, at1) = self.call_events["index"], self.call_events["attend"]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            cur = torch.cuda.current_stream(self.device)
            overlap = self.overlap_ok(1)
            if overlap:
                fork.wait_stream(cur)
                with torch.cuda.stream(fork):
                    self.update_block_sums(1)
            else:
                self.update_block_sums(1)
            ix0.record(cur)
            self.index()
            ix1.record(cur)
            if overlap:
                cur.wait_stream(fork)
            at0.record(cur)
            self.attend()
            at1.record(cur)
        self.graphs["step_timed"] = g
        torch.cuda.synchronize(self.device)
        return self.graphs

    def call_ms(self) -> dict:
        """Index and attention durations (ms) inside the last replay of the
        "step_timed" graph; call after it has completed."""
        return {k: a.elapsed_time(b) for k, (a, b) in self.call_events.items()}

    def replay(self, name: str | None = None):
        """Replay one captured graph, or the whole step when name is None."""
        name = name if name is not None else "step"
        if name in self.graphs:
            self.graphs[name].replay()

    def kernels_per_step(self) -> int:
        """Kernel launches of one step: the block-sum update (HI) and the
        launches the index and attention calls report for this shape."""
        wl = self.wl
        n_idx = lsa.lsa_index_launches(self.batch, wl.H_I, wl.d_I, self.budget)
        n_att = lsa.lsa_attend_launches(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget.length, self.G)
        return (1 if self.block_sums is not None else 0) + n_idx + n_att
