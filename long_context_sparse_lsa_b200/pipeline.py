"""A decode step of the LSA hot path over one workload, through the C ABI.

Allocation and call sequencing only (device buffers via torch, calls via
``binding``): the decode append (the newest tokens' keys and K/V rows written
into the caches, their blocks' HI sums refreshed), one ``lsa_index`` per
group of G layers (Cross-Layer Indexing) and one ``lsa_attend`` for the G
layers. A prefill chunk (``wl.prefill_new``) has no append: its rows are
already in the caches.
"""
from __future__ import annotations

import torch

from . import binding as lsa
from . import inputs as gen
from .workloads import Tensors, Workload


def _device_addressable(t: torch.Tensor) -> bool:
    """True when the pinned host tensor t can be written by a kernel at its
    own address (unified addressing maps page-locked host memory into the
    device's address space); checked with cudaPointerGetAttributes."""
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        return False
    err, attr = rt.cudaPointerGetAttributes(t.data_ptr())
    return (err == rt.cudaError_t.cudaSuccess and attr.type == rt.cudaMemoryType.cudaMemoryTypeHost
            and int(attr.devicePointer) == t.data_ptr())


def _pack(tensors, device):
    """One contiguous uint8 device buffer holding copies of `tensors`, each
    at a 256-byte aligned offset, and the views of it that replace them."""
    offs, total = [], 0
    for x in tensors:
        offs.append(total)
        total += (x.numel() * x.element_size() + 255) // 256 * 256
    buf = torch.empty(max(total, 256), dtype=torch.uint8, device=device)
    views = []
    for x, o in zip(tensors, offs):
        v = buf[o:o + x.numel() * x.element_size()].view(x.dtype).view(x.shape)
        v.copy_(x)
        views.append(v)
    return buf, views


class LsaStep:
    def __init__(self, wl: Workload, t: Tensors, device="cuda", kv_fp8: bool = False, grouped: bool = False,
                 si_attend: bool | None = None, fuse_append: bool = True):
        """kv_fp8: the K/V caches are FP8 E4M3 codes (drawn here, per layer,
        with scales k_scale / v_scale) and the attention is lsa_attend_fp8;
        the bf16 caches of `t` are then unused and may be empty.
        grouped: the decode rows of each sequence (wl.drafts of them) attend
        through lsa_attend_grouped (the rows of a group in one CTA).
        si_attend: attend through lsa_attend_si (sink and window runs as dense
        tiles); by default for a prefill chunk with bf16 caches.
        fuse_append: a decode step's append and index calls go through
        lsa_append_index (the append inside the block selection when the new
        tokens lie in every window); otherwise lsa_append, then lsa_index."""
        self.wl = wl
        self.t = t
        self.device = device
        self.G = len(t.q)
        self.kv_fp8 = kv_fp8
        self.grouped = grouped
        if grouped and (kv_fp8 or wl.prefill_new):
            raise ValueError("grouped attention serves bf16 decode rows")
        if si_attend is None:
            si_attend = bool(wl.prefill_new) and not kv_fp8 and not grouped and wl.n_seq == 1
        self.si_attend = si_attend
        self.fuse_append = fuse_append
        if kv_fp8:
            shape = (wl.total_tokens, wl.H_kv, wl.d)
            self.k8 = [gen.normal_e4m3(shape, wl.seed, gen.STREAM_K8 + g, device) for g in range(self.G)]
            self.v8 = [gen.normal_e4m3(shape, wl.seed, gen.STREAM_V8 + g, device) for g in range(self.G)]
            self.k_scale = [0.75 + 0.25 * g for g in range(self.G)]
            self.v_scale = [1.5 - 0.25 * g for g in range(self.G)]
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
        if grouped:
            ws_a = lsa.lsa_attend_grouped_workspace_size(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget.length,
                                                         self.G, wl.drafts)
        elif si_attend:
            ws_a = lsa.lsa_attend_si_workspace_size(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget, self.G)
        else:
            ws_a = lsa.lsa_attend_workspace_size(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget.length, self.G)
        self.ws_attend = torch.zeros(max(256, ws_a), dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        # the tokens a decode step appends: each sequence's newest `drafts`
        # tokens, whose rows the step writes (the synthetic draw already holds
        # them, so the caches keep their contents)
        self.n_new = 0 if wl.prefill_new else wl.drafts
        if self.n_new:
            offs, lens = t.kv_offset.tolist(), t.seq_lens.tolist()
            pos = torch.tensor([o + L - self.n_new + j for o, L in zip(offs, lens) for j in range(self.n_new)],
                               dtype=torch.int64, device=device)
            n_seq = len(lens)
            self.k_idx_new = t.k_idx.index_select(0, pos).view(n_seq, self.n_new, wl.d_I).clone()
            kc, vc = self.kv_caches()
            self.k_new = [x.index_select(0, pos).view(n_seq, self.n_new, wl.H_kv, wl.d).clone() for x in kc]
            self.v_new = [x.index_select(0, pos).view(n_seq, self.n_new, wl.H_kv, wl.d).clone() for x in vc]

    # -- the three calls --------------------------------------------------------
    def build_block_sums(self, stream=None):
        if self.block_sums is not None:
            lsa.lsa_hi_block_sums(self.t.k_idx, self.wl.hi_block, self.batch, self.block_sums, 0, self.status, stream)

    def update_block_sums(self, n_new: int = 1, stream=None):
        if self.block_sums is not None:
            lsa.lsa_hi_block_sums(self.t.k_idx, self.wl.hi_block, self.batch, self.block_sums, n_new, self.status,
                                  stream)

    def pack_io(self):
        """Place the step's per-step inputs (indexer queries and weights, the
        queries of every layer, the appended tokens' rows) in one contiguous
        device buffer `in_buf` and its outputs in another, `out_buf`, so that a
        serving loop moves them with one host-to-device and one device-to-host
        copy per step. The tensors keep their values and become views of the
        buffers. Call before capture(): the graphs keep these addresses."""
        t, G = self.t, self.G
        # the index call's inputs first, the attention's queries last: the
        # e2e graph copies the two parts on two streams (capture_e2e)
        ins = [t.q_idx, t.w]
        if self.n_new:
            ins += [self.k_idx_new, *self.k_new, *self.v_new]
        n_head = len(ins)
        ins += list(t.q)
        self.in_buf, v = _pack(ins, self.device)
        t.q_idx, t.w = v[0], v[1]
        if self.n_new:
            self.k_idx_new = v[2]
            self.k_new = list(v[3:3 + G])
            self.v_new = list(v[3 + G:3 + 2 * G])
        t.q = list(v[n_head:])
        self.in_split = t.q[0].data_ptr() - self.in_buf.data_ptr()  # first byte of the queries
        self.out_buf, self.out = _pack(self.out, self.device)

    def kv_caches(self):
        """The K and V caches the attention reads (FP8 codes or bf16)."""
        return (self.k8, self.v8) if self.kv_fp8 else (self.t.k, self.t.v)

    def append(self, stream=None):
        """The decode append: write the newest tokens' keys and K/V rows and
        refresh the block sums of their blocks (one launch)."""
        if self.n_new:
            kc, vc = self.kv_caches()
            lsa.lsa_append(self.k_idx_new, self.t.k_idx, self.k_new, self.v_new, kc, vc,
                           self.wl.hi_block, self.block_sums, self.batch, self.n_new, self.status, stream)

    def append_index(self, stream=None):
        """The append and the index call in one: lsa_append_index."""
        kc, vc = self.kv_caches()
        lsa.lsa_append_index(self.k_idx_new, self.k_new, self.v_new, kc, vc, self.n_new, self.t.q_idx, self.t.k_idx,
                             self.t.w, self.wl.w_max, self.batch, self.budget, self.sets, self.block_sums,
                             self.ws_index, self.status, stream)

    def index(self, stream=None):
        lsa.lsa_index(self.t.q_idx, self.t.k_idx, self.t.w, self.wl.w_max, self.batch, self.budget, self.sets,
                      self.block_sums, self.ws_index, self.status, stream)

    def attend(self, stream=None):
        if self.kv_fp8:
            lsa.lsa_attend_fp8(self.t.q, self.k8, self.v8, self.k_scale, self.v_scale, self.sets, self.batch,
                               self.out, self.ws_attend, self.status, stream)
        elif self.grouped:
            lsa.lsa_attend_grouped(self.t.q, self.t.k, self.t.v, self.sets, self.batch, self.wl.drafts, self.out,
                                   self.ws_attend, self.status, stream)
        elif self.si_attend:
            lsa.lsa_attend_si(self.t.q, self.t.k, self.t.v, self.sets, self.budget, self.batch, self.out,
                              self.ws_attend, self.status, stream)
        else:
            lsa.lsa_attend(self.t.q, self.t.k, self.t.v, self.sets, self.batch, self.out, self.ws_attend,
                           self.status, stream)

    def step(self, stream=None):
        """One decode step: append, index, attend."""
        if self.n_new and self.fuse_append:
            self.append_index(stream)
        else:
            self.append(stream)
            self.index(stream)
        self.attend(stream)

    def overlap_ok(self) -> bool:
        """True when the append may run beside the index call.

        The append writes the n_new newest tokens' rows and, with HI on, the
        sums of the blocks that hold them. The index call reads keys of the
        middle only (positions below the window start) and, with HI on, the
        sums of the blocks that meet the middle. With window >= n_new (HI
        off) or window >= hi_block + n_new - 1 (HI on) none of those is
        written, so the two calls touch disjoint memory; the attention, which
        reads the new K/V rows, runs after both."""
        wl = self.wl
        if not self.n_new:
            return False
        need = wl.hi_block + self.n_new - 1 if wl.hi_block > 0 else self.n_new
        return wl.window >= need

    def status_bits(self) -> int:
        return int(self.status.item())

    # -- CUDA graphs ------------------------------------------------------------
    def capture(self, fork_append: bool = False):
        """Capture the three calls as CUDA graphs (append, index, attend), and
        the whole step as one more graph ("step"). In the step graph the three
        calls follow each other on one stream, so every kernel boundary keeps
        its programmatic (early) launch; with fork_append (and overlap_ok())
        the append runs on a forked stream beside the index call instead,
        which turns the attention's dependence on the index call into a full
        graph edge. A step then replays without host launch overhead. Two
        more graphs serve measurement: "step_timed" (the step with timing
        events around the index and attention calls) and, with HI on, "cold"
        (a full block-sum build, then index and attention). The graphs keep
        this object's buffers; changing their contents between replays is how
        new inputs enter."""
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):  # one eager pass fills the launch-plan caches
            self.step()
        torch.cuda.current_stream(self.device).wait_stream(side)
        torch.cuda.synchronize(self.device)
        self.graphs = {}
        for name, fn in (("append", self.append), ("index", self.index), ("attend", self.attend)):
            if name == "append" and not self.n_new:
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                fn()
            self.graphs[name] = g
        g = torch.cuda.CUDAGraph()
        fork = torch.cuda.Stream(self.device)
        fork_ok = fork_append and self.overlap_ok() and not self.fuse_append
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            cur = torch.cuda.current_stream(self.device)
            if fork_ok:
                fork.wait_stream(cur)
                with torch.cuda.stream(fork):
                    self.append()
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
            overlap = fork_ok
            fused = bool(self.n_new) and self.fuse_append
            if overlap:
                fork.wait_stream(cur)
                with torch.cuda.stream(fork):
                    self.append()
            elif not fused:
                self.append()
            ix0.record(cur)
            if fused:
                self.append_index()  # the index call's time then includes the append
            else:
                self.index()
            ix1.record(cur)
            if overlap:
                cur.wait_stream(fork)
            at0.record(cur)
            self.attend()
            at1.record(cur)
        self.graphs["step_timed"] = g
        if self.block_sums is not None:
            # a cold step: the block sums rebuilt from the whole key cache first
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                self.build_block_sums()
                self.index()
                self.attend()
            self.graphs["cold"] = g
        torch.cuda.synchronize(self.device)
        return self.graphs

    def capture_e2e(self, h_in: torch.Tensor, h_out: torch.Tensor):
        """Capture graph "e2e": one step with its host copies, for a serving
        loop whose inputs and outputs live in pinned host memory (h_in, h_out:
        uint8, the sizes of in_buf and out_buf; call pack_io() first). The
        index call's inputs are copied first; the queries (read only by the
        attention) are copied on a second stream while the index call runs,
        and the attention waits for them. The bf16 attention writes its
        outputs straight into h_out when the device can address it (the
        result crosses to the host as the kernel stores it); otherwise they
        are copied back last."""
        cut = self.in_split
        direct = not (self.kv_fp8 or self.grouped or self.si_attend) and _device_addressable(h_out)
        host_out = []
        if direct:
            for o in self.out:
                lo = o.data_ptr() - self.out_buf.data_ptr()
                host_out.append(h_out[lo:lo + o.numel() * o.element_size()].view(o.dtype).view(o.shape))
        side = torch.cuda.Stream(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            cur = torch.cuda.current_stream(self.device)
            side.wait_stream(cur)
            with torch.cuda.stream(side):
                self.in_buf[cut:].copy_(h_in[cut:], non_blocking=True)
            self.in_buf[:cut].copy_(h_in[:cut], non_blocking=True)
            if self.n_new and self.fuse_append:
                self.append_index()
            else:
                if self.n_new:
                    self.append()
                self.index()
            cur.wait_stream(side)
            if direct:
                lsa.lsa_attend(self.t.q, self.t.k, self.t.v, self.sets, self.batch, host_out, self.ws_attend,
                               self.status)
            else:
                self.attend()
                h_out.copy_(self.out_buf, non_blocking=True)
        self.e2e_direct_out = direct
        self.graphs["e2e"] = g
        torch.cuda.synchronize(self.device)
        return g

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
        """Kernel launches of one step: the append (decode) and the launches
        the index and attention calls report for this shape."""
        wl = self.wl
        if self.n_new and self.fuse_append:
            n_idx = lsa.lsa_append_index_launches(self.batch, wl.H_I, wl.d_I, self.budget, self.n_new)
        else:
            n_idx = (1 if self.n_new else 0) + lsa.lsa_index_launches(self.batch, wl.H_I, wl.d_I, self.budget)
        if self.grouped:
            n_att = lsa.lsa_attend_grouped_launches(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget.length, self.G,
                                                    wl.drafts)
        elif self.si_attend:
            n_att = lsa.lsa_attend_si_launches(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget, self.G)
        else:
            n_att = lsa.lsa_attend_launches(self.batch, wl.H_q, wl.H_kv, wl.d, self.budget.length, self.G)
        return n_idx + n_att
