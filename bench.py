"""Benchmark of the LSA decode hot path (one JSON line on rank 0).

A step is one decode step of the batched 128K workload (16 sequences x
131072 tokens, HI 64x256, sink/window/topk 64/1024/2048, 32 q heads over 4
kv heads): the HI block-sum append update, the indexer (coarse scores, HI
block selection, fine scores, top-k and SI assembly) and the split-K sparse
attention with its merge. Inputs are seeded synthetic tensors resident in
HBM. L2 is flushed (a 2 x L2-size write) before every timed step, outside the
timed interval; every step is timed with CUDA events on the launching
stream. On one GPU the line also carries the 1M-token decode (one index set
for G = 4 layers) and the 8192-token causal prefill chunk under "secondary".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference]

With torchrun (N > 1) every rank runs its own independent batch (weak
scaling, no collective on the data path); the step time is the max over
ranks. ``--impl reference`` times the CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_lsa_b200 import workloads as wls  # noqa: E402

METRIC = "LSA decode queries/s at 128K & 1M ctx; achieved HBM GB/s vs B200 peak"
UNIT = "queries/s"
PROFILES = os.path.join(ROOT, "profiles")


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move; nothing avoided by HI counted)
# ---------------------------------------------------------------------------
def step_bytes(wl, kv_fp8: bool = False) -> dict:
    n_q, G = wl.n_q, wl.G
    kv_row = wl.H_kv * wl.d * (1 if kv_fp8 else 2)  # bytes of one token's K (or V) in one layer
    rows = _rows(wl)
    attend = 0
    for L in rows:
        e = min(L, wl.budget)
        attend += G * (2 * e * kv_row + wl.H_q * wl.d * 2 + wl.H_q * wl.d * 4 + wl.budget * 4)
    index = 0
    for L in rows:
        s = min(wl.sink, L)
        ws = max(s, L - wl.window)
        if wl.hi_block > 0:
            B = wl.hi_block
            nb = (ws + B - 1) // B - s // B if ws > s else 0
            kept = min(nb, wl.hi_topblocks)
            index += nb * 2 * wl.d_I + kept * B * wl.d_I  # block sums read + kept keys
        else:
            index += (ws - s) * wl.d_I
        index += wl.H_I * wl.d_I + wl.H_I * 4 + wl.budget * 4  # q, w, index-set write
    if wl.prefill_new:  # one cache shared by every row of the chunk: read it once
        index = wl.lens[0] * wl.d_I + n_q * (wl.H_I * wl.d_I + wl.H_I * 4 + wl.budget * 4)
    # decode append per sequence: the new tokens' key and K/V rows read and
    # written once; with HI on, one block of keys re-read and its sum written
    app = 0
    if not wl.prefill_new:
        for L in wl.lens:
            app += 2 * wl.drafts * (wl.d_I + 2 * G * kv_row)
            if wl.hi_block > 0:
                app += wl.hi_block * wl.d_I + 2 * wl.d_I
    return {"attend": attend, "index": index, "append": app, "total": attend + index + app}


def cold_block_sum_bytes(wl) -> int:
    """Bytes of a full block-sum build: every cached key read once, every
    block's two byte planes written once."""
    if wl.hi_block <= 0:
        return 0
    nb = sum((L + wl.hi_block - 1) // wl.hi_block for L in wl.lens)
    return wl.total_tokens * wl.d_I + nb * 2 * wl.d_I


def _rows(wl):
    """Visible length of every query row."""
    if wl.prefill_new:
        C = wl.lens[0] - wl.prefill_new
        return [C + i + 1 for i in range(wl.prefill_new)]
    return [L - wl.drafts + 1 + j for L in wl.lens for j in range(wl.drafts)]


def attend_flops(wl) -> int:
    """Multiply-adds x 2 of the attention: q.k and p.v over every selected
    entry, every query head and layer (4 * d flop per head and entry)."""
    tot = 0
    for L in _rows(wl):
        tot += min(L, wl.budget)
    return 4 * wl.d * wl.H_q * wl.G * tot


def prefill_unique_kv_bytes(wl) -> int:
    """Bytes of the distinct K and V rows a prefill chunk's sets can name: at
    most the whole cache the chunk sees (every token once per layer)."""
    kv_row = wl.H_kv * wl.d * 2
    return 2 * wl.G * wl.lens[0] * kv_row


def index_int8_ops(wl) -> int:
    """Multiply-adds x 2 of the fine scores (every middle token of every row)."""
    tot = 0
    for L in _rows(wl):
        s = min(wl.sink, L)
        ws = max(s, L - wl.window)
        tot += ws - s
    return 2 * tot * wl.H_I * wl.d_I


# ---------------------------------------------------------------------------
def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get("hbm_gbs", 6650.0)), "measured"
    return 6650.0, "fallback"


def _bf16_sustained():
    """Dense bf16 tensor rate in TFLOP/s for kernels timed inside a long step:
    the measured sustained cuBLAS rate, else the profiling fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return float(d["bf16_tflops_sustained"]), "measured (sustained cuBLAS bf16)"
    return 1400.0, "fallback (sustained bf16)"


def measure_int8_peak(dev, n: int = 8192, reps: int = 20) -> dict:
    """Dense int8 tensor rate of this GPU, measured: a library int8 GEMM
    (torch._int_mm, n x n x n, int32 accumulate) run back to back; best of
    three bursts of `reps` (CUDA events). Only a denominator: the indexer
    itself never calls it."""
    a = torch.randint(-16, 16, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-16, 16, (n, n), dtype=torch.int8, device=dev)
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    best = None
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        best = ms if best is None else min(best, ms)
    del a, b
    return {"tops": 2.0 * n ** 3 / (best / 1000.0) / 1e12, "kind": f"measured: torch._int_mm {n}^3 int8 GEMM, best "
            f"of 3 bursts of {reps}", "ms": best}


ATTEND_SOURCES = ("attend.cu", "common.cuh")
INDEX_SOURCES = ("index_select.cu", "index_score.cu", "index_common.cuh", "append.cuh", "common.cuh", "internal.h")


def _kernel_hash(files=ATTEND_SOURCES) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "long_context_sparse_lsa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _ncu_traffic(kernel_hash: str, workload: str, kind: str = "attend"):
    """DRAM bytes per launch of the call's kernels (kind "attend": the attention
    kernel; "index": the index call's kernels) from the committed ncu summary,
    if it was taken on this exact kernel source and workload."""
    p = os.path.join(PROFILES, f"{kind}_{workload}.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_hash:
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms (the bench
    samples over a 0.6 s burst of replayed steps just before the timed steps
    and through them)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
def cpu_baseline(wl, t, max_seconds=20.0, max_queries=None, min_seconds=0.0):
    """The oracle (one thread) on a bounded sample of the workload's queries:
    index + G-layer attention per query; only the oracle calls are timed, and
    the result is scaled to queries/s. The queries are taken in order (and
    again from the first, until at least `min_seconds` of oracle time) and
    the sample stops once `max_seconds` are spent. ``t`` may live on any
    device: each query's keys and the K/V rows its oracle set names are copied
    to the host before its timed calls."""
    import numpy as np

    import oracle

    orc = oracle.get()
    u16 = lambda x: x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    kv_off = t.kv_offset.cpu().numpy()
    q_seq = t.q_seq.cpu().numpy()
    q_len = t.q_len.cpu().numpy()
    n = len(q_seq) if max_queries is None else min(max_queries, len(q_seq))
    done, busy, passes = 0, 0.0, 0
    while True:
        for r in range(n):
            base = int(kv_off[q_seq[r]])
            L = int(q_len[r])
            kseq = t.k_idx[base:base + L].cpu().numpy()
            qi = t.q_idx[r].cpu().numpy()
            wr = t.w[r].cpu().numpy()
            c0 = time.perf_counter()
            s = orc.index_query(qi, wr, kseq, L, wl.sink, wl.window, wl.topk, wl.hi_block, wl.hi_topblocks)
            busy += time.perf_counter() - c0
            valid = s[s >= 0]
            local = np.full(s.shape[0], -1, np.int32)
            local[: valid.shape[0]] = np.arange(valid.shape[0], dtype=np.int32)
            rows = torch.as_tensor(valid.astype(np.int64) + base, device=t.k[0].device)
            for g in range(len(t.q)):
                kr, vr, qg = u16(t.k[g].index_select(0, rows)), u16(t.v[g].index_select(0, rows)), u16(t.q[g][r])
                c0 = time.perf_counter()
                orc.attend_query(qg, kr, vr, local)
                busy += time.perf_counter() - c0
            done += 1
            if busy > max_seconds:
                break
        passes += 1
        if busy > max_seconds or busy >= min_seconds or done == 0:
            break
    return {"value": done / busy, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} query evaluations ({passes} pass(es) over {n} of the {wl.n_q} queries) of {wl.name} "
                      f"(index + {len(t.q)}-layer attention each), single-threaded C oracle, {busy:.1f} s of "
                      f"oracle time"}


def host_cpu() -> dict:
    """The host's CPU model, its logical CPU count and the CPUs this process may run on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count() or 1
    return {"cpu_model": model, "nproc": os.cpu_count(), "usable_cpus": usable}


class OracleStep:
    """One step of the workload evaluated by the oracle on host threads: the
    index sets of every query row (oracle lsa_index), then the G-layer
    attention of every row (oracle lsa_attend). The K/V rows each set names are
    gathered once, outside the timed calls, into a packed per-row copy (the
    oracle reads exactly those rows); only the two oracle calls are timed."""

    def __init__(self, wl, t, n_threads: int):
        import numpy as np

        import oracle

        self.np = np
        self.orc = oracle.get()
        self.wl = wl
        self.n_threads = n_threads
        h = lambda x: x.contiguous().cpu().numpy()
        self.q_idx, self.k_idx, self.w = h(t.q_idx), h(t.k_idx), h(t.w)
        self.kv_offset, self.q_seq, self.q_len = h(t.kv_offset), h(t.q_seq), h(t.q_len)
        u16 = lambda x: x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        self.q = [u16(x) for x in t.q]
        sets = self.index()
        n_q, budget = sets.shape
        rows = np.zeros((n_q, budget), np.int64)
        self.local = np.full((n_q, budget), -1, np.int32)
        for r in range(n_q):
            v = sets[r][sets[r] >= 0].astype(np.int64)
            rows[r, : v.shape[0]] = v + self.kv_offset[self.q_seq[r]]
            self.local[r, : v.shape[0]] = np.arange(v.shape[0], dtype=np.int32)
        idx = torch.as_tensor(rows.reshape(-1), device=t.k[0].device)
        self.k = [u16(x.index_select(0, idx)) for x in t.k]
        self.v = [u16(x.index_select(0, idx)) for x in t.v]
        self.offs = np.arange(n_q, dtype=np.int64) * budget
        self.rows = np.arange(n_q, dtype=np.int32)

    def index(self):
        wl = self.wl
        return self.orc.lsa_index(self.q_idx, self.k_idx, self.w, self.kv_offset, self.q_seq, self.q_len, wl.sink,
                                  wl.window, wl.topk, wl.hi_block, wl.hi_topblocks, n_threads=self.n_threads)

    def run(self) -> float:
        """Seconds of one step (index + attention of every row)."""
        c0 = time.perf_counter()
        self.index()
        self.orc.lsa_attend(self.q, self.k, self.v, self.local, self.offs, self.rows, n_threads=self.n_threads)
        return time.perf_counter() - c0


def cpu_baseline_all_cores(wl, t, max_seconds=10.0):
    """The oracle on every usable host CPU (one thread per CPU, the queries of
    a step spread over them), whole steps repeated until `max_seconds` of
    oracle time."""
    cpu = host_cpu()
    n = max(1, cpu["usable_cpus"])
    step = OracleStep(wl, t, n)
    busy, steps = 0.0, 0
    while busy < max_seconds or steps == 0:
        busy += step.run()
        steps += 1
    return {"value": steps * wl.n_q / busy, "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"{steps} whole steps of {wl.name} ({wl.n_q} query rows each: index + {len(t.q)}-layer "
                      f"attention), C oracle on {n} threads, {busy:.1f} s of oracle time",
            **cpu}


def reference_sample(wl):
    """The reference arm's bounded sample: a step's worth of query rows on the
    workload's first sequence (decode: n_q draft-layout rows seeing the last
    n_q positions of that sequence; prefill: the chunk's first 16 rows), drawn
    on the host."""
    if wl.prefill_new:
        n = min(wl.prefill_new, 16)
        C = wl.lens[0] - wl.prefill_new
        return wls.small(wl, lens=(C + n,), prefill_new=n)
    return wls.small(wl, lens=wl.lens[:1], drafts=wl.n_q)


def run_reference(args, wl):
    """--impl reference: the CPU oracle as it stands, on the host cores. A step
    evaluates the sample's query rows once (index + attention, every usable
    CPU); ms_per_step is the measured time of one such step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sample = reference_sample(wl)
    t = wls.make(sample, "cpu")
    cpu = host_cpu()
    n_threads = max(1, cpu["usable_cpus"])
    step = OracleStep(sample, t, n_threads)
    for _ in range(args.warmup):
        step.run()
    times = [step.run() for _ in range(args.steps)]
    ms = 1000.0 * statistics.median(times)
    value = sample.n_q / (ms / 1000.0)
    desc = (f"{sample.n_q} query rows per step on the first sequence of {wl.name} "
            f"(context {min(sample.lens[0], max(_rows(sample)))}), index + {sample.G}-layer attention, "
            f"C oracle on {n_threads} threads; {args.steps} timed steps of {ms:.1f} ms (median)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64+f64",
            "data": "synthetic (seeded SplitMix64 draws)",
            "config": {"workload": wl.name, "n_queries": wl.n_q, "context": max(wl.lens), "layers_per_index": wl.G,
                       "queries_per_step": sample.n_q},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_threads, "kind": "oracle", "sample": desc,
                             **cpu},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# multi-GPU plumbing (replicas: no collective on the data path)
# ---------------------------------------------------------------------------
def rank_workload(wl, rank: int):
    """Each rank draws its own independent batch of the same shape (weak
    scaling): rank 0 the workload's seed, rank i > 0 seed + 1000 i."""
    return wls.small(wl, seed=wl.seed + 1000 * rank) if rank else wl


def max_over_ranks(x: float, dist, device) -> float:
    """A time the job reports: the maximum of the ranks' times (one
    all-reduce of a scalar; the bench issues no other collective)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed / the max-over-ranks time."""
    return units_per_rank * world / (ms / 1000.0)


# ---------------------------------------------------------------------------
def time_workload(wl, dev, flush, stream, steps, warmup, pg=None, clocks=None, kv_fp8=False, grouped=False,
                  fuse_append=True):
    """Draws the workload, captures its step graphs and times `steps` steps
    (after `warmup`), each after an L2 flush: the whole step graph for the
    headline, then the three calls one by one for the breakdown."""
    from long_context_sparse_lsa_b200.pipeline import LsaStep

    t = wls.make(wl, dev, with_kv=not kv_fp8)
    st = LsaStep(wl, t, dev, kv_fp8=kv_fp8, grouped=grouped, fuse_append=fuse_append)
    st.pack_io()  # one input and one output buffer per step (the e2e leg copies each once)
    st.build_block_sums()
    torch.cuda.synchronize()
    st.capture()

    def one_step(evs):
        """The timed step: the captured step graph (the append beside
        the index call when the two touch disjoint rows, then attention)."""
        flush.fill_(1)
        evs[0].record(stream)
        st.replay()
        evs[1].record(stream)

    def split_step(evs):
        """The three calls one after another, for the per-call breakdown."""
        flush.fill_(1)
        evs[0].record(stream)
        st.replay("append")
        evs[1].record(stream)
        st.replay("index")
        evs[2].record(stream)
        st.replay("attend")
        evs[3].record(stream)

    ev = lambda n: [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for _ in range(warmup):
        one_step(ev(2))
        split_step(ev(4))
    torch.cuda.synchronize()
    if st.status_bits() != 0:
        raise RuntimeError(f"device status {st.status_bits():#x} after warm-up ({wl.name})")
    if clocks is not None:
        # the timed steps last milliseconds, nvidia-smi samples every 200 ms:
        # sample over ~0.6 s of the same step replayed back to back right
        # before the timed steps, and through them
        clocks.start()
        t_end = time.perf_counter() + 0.6
        while time.perf_counter() < t_end:
            for _ in range(64):
                st.replay()
            torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    evs = [ev(2) for _ in range(steps)]
    for i in range(steps):
        one_step(evs[i])
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clk = clocks.stop() if clocks is not None else None
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    # per-call breakdown (outside the timed region)
    sevs = [ev(4) for _ in range(steps)]
    for i in range(steps):
        split_step(sevs[i])
    torch.cuda.synchronize()
    # the calls' durations inside the step: the step graph with timing
    # events around the index and attention calls, one replay at a time
    in_step = []
    for i in range(steps):
        flush.fill_(1)
        st.replay("step_timed")
        torch.cuda.synchronize()
        in_step.append(st.call_ms())
    # cold steps: the block sums rebuilt from the whole key cache inside each
    # step (nothing resident between steps), then index and attention
    cold = []
    if "cold" in st.graphs:
        cevs = [ev(2) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(1)
            cevs[i][0].record(stream)
            st.replay("cold")
            cevs[i][1].record(stream)
        torch.cuda.synchronize()
        cold = [e[0].elapsed_time(e[1]) for e in cevs]
    if st.status_bits() != 0:
        raise RuntimeError(f"device status {st.status_bits():#x} after timing ({wl.name})")
    return {"st": st, "t": t, "ms": ms, "clocks": clk, "n_kernels": st.kernels_per_step(), "cold": cold,
            "bs": [e[0].elapsed_time(e[1]) for e in sevs], "ix": [e[1].elapsed_time(e[2]) for e in sevs],
            "at": [e[2].elapsed_time(e[3]) for e in sevs],
            "ix_in_step": [c["index"] for c in in_step], "at_in_step": [c["attend"] for c in in_step],
            "fused_append": bool(st.n_new) and st.fuse_append}


def draft_union_entries(sets: torch.Tensor, drafts: int) -> int:
    """Distinct positions over each sequence's draft rows, summed: the K/V rows
    a step must read from HBM per kv head and layer."""
    total = 0
    for grp in sets.view(-1, drafts * sets.shape[1]):
        total += int(torch.unique(grp[grp >= 0]).numel())
    return total


def cold_line(wl, cold_ms, world, pg, dev):
    """The cold-step numbers (block sums rebuilt inside every step), or None
    when the workload has HI off."""
    if not cold_ms:
        return None
    ms = max_over_ranks(sum(cold_ms) / len(cold_ms), pg, dev)
    byts = step_bytes(wl)["total"] - step_bytes(wl)["append"] + cold_block_sum_bytes(wl)
    return {"value": job_rate(wl.n_q, world, ms), "unit": UNIT, "ms_per_step": ms,
            "algorithmic_bytes_per_step": byts, "step_gbs": byts / (ms / 1000.0) / 1e9,
            "note": "block sums rebuilt from the whole key cache inside every step (full build, "
                    "then index, then attention; one CUDA graph, L2 flushed before each step)"}


def secondary(dev, flush, stream, steps, warmup, peak, fuse_append=True):
    """The 1M-token decode (G = 4) and the 8192-token prefill chunk, each
    measured like the headline (step graph, L2 flush, CUDA events)."""
    from long_context_sparse_lsa_b200 import binding as lsa

    out = {}
    mean = lambda xs: sum(xs) / len(xs)
    try:
        int8 = measure_int8_peak(dev)
    except Exception as exc:  # reported, never silently replaced by an assumed figure
        int8 = {"tops": None, "kind": f"int8 GEMM unavailable: {exc!r}"}
    for wl, fp8 in ((wls.CTX1M, False), (wls.PREFILL, False), (wls.BATCH128K, True), (wls.ragged(), False),
                    (wls.DRAFTS128K, False)):
        drafts = wl.drafts > 1
        run = time_workload(wl, dev, flush, stream, steps, warmup, kv_fp8=fp8, fuse_append=fuse_append)
        st = run["st"]
        ms = run["ms"]
        byts = step_bytes(wl, kv_fp8=fp8)
        if drafts:
            # concurrent draft rows of a sequence read each K/V row they share
            # from HBM once (L2 holds it for the others): count the union
            union = draft_union_entries(st.sets, wl.drafts)
            kv_row = wl.H_kv * wl.d * 2
            byts = dict(byts)
            byts["attend"] = wl.G * (2 * union * kv_row + wl.n_q * (wl.H_q * wl.d * 6 + wl.budget * 4))
            byts["total"] = byts["attend"] + byts["index"] + byts["append"]
        ix, at = mean(run["ix_in_step"]), mean(run["at_in_step"])
        rec = {"ms_per_step": ms, "steps": steps, "warmup": warmup,
               "step_breakdown_ms": {"append": mean(run["bs"]), "index": mean(run["ix"]),
                                     "attend": mean(run["at"])},
               "call_ms_in_step": {"index": ix, "attend": at},
               "cold": cold_line(wl, run["cold"], 1, None, dev),
               "algorithmic_bytes_per_step": byts,
               "gpu_launches_per_step": run["n_kernels"]}
        if not wl.prefill_new:
            # decode: every byte counted is read from HBM once (L2 flushed before each step)
            rec.update({"step_gbs": byts["total"] / (ms / 1000.0) / 1e9,
                        "step_frac_of_measured_hbm": byts["total"] / (ms / 1000.0) / 1e9 / peak,
                        "index_gbs": byts["index"] / (ix / 1000.0) / 1e9,
                        "index_frac_of_measured_hbm": byts["index"] / (ix / 1000.0) / 1e9 / peak,
                        "attend_gbs": byts["attend"] / (at / 1000.0) / 1e9,
                        "attend_frac_of_measured_hbm": byts["attend"] / (at / 1000.0) / 1e9 / peak})
        if wl.prefill_new:
            ops = index_int8_ops(wl)
            fl = attend_flops(wl)
            bf, bf_kind = _bf16_sustained()
            rec.update({"metric": "prefill tokens/s (index + attention of a causal chunk)", "unit": "tokens/s",
                        "value": wl.n_q / (ms / 1000.0),
                        "index_tensor_path": bool(lsa.lsa_index_uses_tensor_cores(st.batch, wl.H_I, wl.d_I,
                                                                                  st.budget)),
                        "index_int8_ops": ops,
                        "index_tops": ops / (ix / 1000.0) / 1e12,
                        "int8_peak_tops": int8["tops"], "int8_peak_kind": int8["kind"],
                        "index_tops_frac_of_int8_peak": (ops / (ix / 1000.0) / 1e12 / int8["tops"]
                                                         if int8["tops"] else None),
                        "attend_flops": fl, "attend_tflops": fl / (at / 1000.0) / 1e12,
                        "attend_frac_of_bf16": fl / (at / 1000.0) / 1e12 / bf, "bf16_peak_tflops": bf,
                        "bf16_peak_kind": bf_kind,
                        "attend_gather_gbs": byts["attend"] / (at / 1000.0) / 1e9,
                        "attend_unique_kv_bytes": prefill_unique_kv_bytes(wl),
                        "note": "index_tops: int8 ops of the fine-score contraction over the whole index call "
                                "(scoring + selection), so a lower bound on the tensor kernel's rate; "
                                "attend_gather_gbs counts every row's gathered K/V rows (rows repeat across the "
                                "chunk and come from L2), so it is a gather rate, not an HBM fraction"})
        elif fp8:
            rec.update({"metric": "LSA decode queries/s at 128K ctx, FP8 E4M3 KV cache", "unit": "queries/s",
                        "value": wl.n_q / (ms / 1000.0), "kv_cache": "fp8 e4m3, one scale per layer for K and V",
                        "note": "same workload as the headline with the K/V caches held as FP8 codes "
                                "(lsa_attend_fp8); attention bytes per query halve"})
        elif drafts:
            # the same step with the draft rows of a sequence attended together
            # (lsa_attend_grouped), for comparison
            grp = time_workload(wl, dev, flush, stream, steps, warmup, grouped=True)
            per_entry = wl.H_kv * 2 * wl.d * 2 * wl.G  # K and V of every kv head, every layer
            rec.update({"metric": "LSA decode queries/s, 4 draft rows per sequence", "unit": "queries/s",
                        "value": wl.n_q / (ms / 1000.0), "drafts_per_seq": wl.drafts,
                        "draft_query_share_pct": wl.draft_share,
                        "set_entries": int((st.sets >= 0).sum().item()), "union_entries": union,
                        "kv_bytes_of_the_sets": int((st.sets >= 0).sum().item()) * per_entry,
                        "kv_bytes_of_the_union": union * per_entry,
                        "grouped_attention": {"ms_per_step": grp["ms"], "value": wl.n_q / (grp["ms"] / 1000.0),
                                              "attend_ms_in_step": mean(grp["at_in_step"]),
                                              "gpu_launches_per_step": grp["n_kernels"]},
                        "note": "every row gathers its own set (lsa_attend); the draft rows of a sequence run in "
                                "one wave, so L2 serves the rows they share and HBM reads the union once "
                                "(algorithmic bytes count the union); grouped_attention is lsa_attend_grouped "
                                "(the rows of a group in one CTA over the same entry ranges)"})
            del grp
        elif wl.name == wls.CTX1M.name:
            rec.update({"metric": "LSA decode queries/s at 1M ctx", "unit": "queries/s",
                        "value": wl.n_q / (ms / 1000.0), "layers_per_index": wl.G})
        else:
            rec.update({"metric": "LSA decode queries/s, ragged batch", "unit": "queries/s",
                        "value": wl.n_q / (ms / 1000.0), "layers_per_index": wl.G, "n_seq": wl.n_seq,
                        "cached_tokens": wl.total_tokens, "min_len": min(wl.lens), "max_len": max(wl.lens)})
        out[wl.name + ("_fp8kv" if fp8 else "")] = rec
        del run, st
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lsa", choices=["lsa", "reference"])
    ap.add_argument("--workload", default=wls.BATCH128K.name)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=8.0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the 1M decode and prefill chunk measurements")
    ap.add_argument("--grouped", action="store_true",
                    help="draft-row workloads: attend through lsa_attend_grouped")
    ap.add_argument("--no-fuse-append", action="store_true",
                    help="decode steps: lsa_append then lsa_index instead of lsa_append_index")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    wl = wls.by_name(args.workload)
    if args.impl == "reference":
        return run_reference(args, wl)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
        pg = dist

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # each rank draws its own independent batch (weak scaling)
    wl_r = rank_workload(wl, rank)
    clocks = ClockSampler(local)
    run = time_workload(wl_r, dev, flush, stream, args.steps, args.warmup, pg, clocks,
                        grouped=args.grouped and wl.drafts > 1, fuse_append=not args.no_fuse_append)
    st, t = run["st"], run["t"]
    ms = max_over_ranks(run["ms"], pg, dev)
    clk = run["clocks"]
    bs_ms, ix_ms, at_ms = run["bs"], run["ix"], run["at"]
    n_kernels = run["n_kernels"]

    # ---- end to end through the public API with host buffers ----
    # the step's inputs (indexer queries and weights, queries, the appended
    # tokens' keys and K/V rows) sit in one pinned host buffer and the outputs
    # come back into another; one graph per step (LsaStep.capture_e2e): the
    # index call's inputs copied in, the queries copied on a second stream
    # while the index call runs, the attention writing the outputs into the
    # host buffer (or a copy back when the device cannot address it)
    h_in = st.in_buf.cpu().pin_memory()
    h_out = torch.empty(st.out_buf.shape, dtype=torch.uint8, pin_memory=True)
    h2d = h_in.numel()
    d2h = h_out.numel()
    st.capture_e2e(h_in, h_out)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st.replay("e2e")
        e1.record(stream)
        if i >= args.warmup:
            e2e_ms.append((e0, e1))
    torch.cuda.synchronize()
    e2e = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ms) / len(e2e_ms), pg, dev)
    if st.status_bits() != 0:
        raise RuntimeError(f"device status {st.status_bits():#x} after timing")

    value = job_rate(wl.n_q, world, ms)
    e2e_value = job_rate(wl.n_q, world, e2e)
    byts = step_bytes(wl)
    peak, peak_kind = _peaks()
    at = sum(at_ms) / len(at_ms)
    ix = sum(ix_ms) / len(ix_ms)
    bsu = sum(bs_ms) / len(bs_ms)
    at_in = max_over_ranks(sum(run["at_in_step"]) / len(run["at_in_step"]), pg, dev)
    ix_in = max_over_ranks(sum(run["ix_in_step"]) / len(run["ix_in_step"]), pg, dev)
    khash = _kernel_hash()
    roof = {"bound": "hbm", "kernel": "lsa_attend call (attend_rk_kernel split-K sparse attention + attend_merge_kernel)",
            "achieved": byts["attend"] / (at_in / 1000.0) / 1e9, "peak": peak, "unit": "GB/s",
            "frac": byts["attend"] / (at_in / 1000.0) / 1e9 / peak, "peak_kind": peak_kind,
            "traffic": _ncu_traffic(khash, wl.name),
            "bytes_per_launch": byts["attend"], "ms_per_launch": at_in,
            "timing": "CUDA events recorded inside the step graph around the lsa_attend call, mean over "
                      "one replay per timed step (L2 flushed before each)"}
    # the index call against the same roofline: its algorithmic bytes (block
    # sums of the candidate blocks, the kept blocks' keys, queries, weights,
    # the written sets; plus the append's when the call is lsa_append_index)
    # over its duration inside the step
    fused = run["fused_append"]
    ix_bytes = byts["index"] + (byts["append"] if fused else 0)
    ix_call = "lsa_append_index" if fused else "lsa_index"
    roof_index = {"bound": "hbm", "kernel": f"{ix_call} call (block selection with the HI coarse scores"
                                            f"{' and the decode append' if fused else ''}, fine scores, token "
                                            "selection with the SI assembly)",
                  "achieved": ix_bytes / (ix_in / 1000.0) / 1e9, "peak": peak, "unit": "GB/s",
                  "frac": ix_bytes / (ix_in / 1000.0) / 1e9 / peak, "peak_kind": peak_kind,
                  "traffic": _ncu_traffic(_kernel_hash(INDEX_SOURCES), wl.name, "index") if fused else None,
                  "bytes_per_launch": ix_bytes, "ms_per_launch": ix_in,
                  "timing": f"CUDA events recorded inside the step graph around the {ix_call} call, mean over "
                            "one replay per timed step (L2 flushed before each)"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8->int32 (indexer), bf16->f32 (attention)",
            "data": "synthetic (seeded SplitMix64 draws; no weights or datasets)",
            "config": {"workload": wl.name, "n_queries_per_gpu": wl.n_q, "context": max(wl.lens),
                       "layers_per_index": wl.G, "budget": {"sink": wl.sink, "window": wl.window,
                                                            "topk": wl.topk, "hi_block": wl.hi_block,
                                                            "hi_topblocks": wl.hi_topblocks},
                       "heads": {"H_I": wl.H_I, "d_I": wl.d_I, "H_q": wl.H_q, "H_kv": wl.H_kv, "d": wl.d},
                       "l2": "flushed before every timed step (2 x L2 write, outside the timed interval)",
                       "launch": ("each step replayed from one CUDA graph captured through the C ABI: "
                                  + ("lsa_append_index (the decode append, new tokens' keys and K/V rows written "
                                     "and their block sums refreshed, run by extra CTAs of the block selection; "
                                     "then the index call's kernels)" if fused else
                                     "the decode append (new tokens' keys and K/V rows written, their block sums "
                                     "refreshed), the index call")
                                  + " and the attention call on one stream, every kernel launched with "
                                  "programmatic stream serialisation; step_breakdown_ms from per-call graphs "
                                  "replayed in sequence (each with its own graph launch: lsa_append, lsa_index, "
                                  "lsa_attend); call_ms_in_step from timing events inside the step graph"
                                  + (" (its index figure includes the fused append)" if fused else "")),
                       "parallelism": f"replicas x{world} (independent batches, no collective)"},
            "step_breakdown_ms": {"append": bsu, "index": ix, "attend": at},
            "call_ms_in_step": {"index": ix_in, "attend": at_in},
            "cold": cold_line(wl, run["cold"], world, pg, dev),
            "step_gbs": byts["total"] / (ms / 1000.0) / 1e9,
            "step_frac_of_measured_hbm": byts["total"] / (ms / 1000.0) / 1e9 / peak,
            "step_frac_of_8tbs": byts["total"] / (ms / 1000.0) / 1e9 / 8000.0,
            "algorithmic_bytes_per_step": byts,
            "roofline": roof,
            "roofline_index": roof_index,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "one CUDA graph per step: the index call's inputs copied from pinned host memory, the "
                           "queries copied on a second stream while the index call runs, the attention, "
                           + ("which writes the outputs straight into pinned host memory (device-addressable "
                              "under unified addressing)" if getattr(st, "e2e_direct_out", False) else
                              "the outputs copied back to pinned host memory")
                           + "; L2 flushed before each step",
                    "ms_per_step": e2e},
            "gpu_launches": n_kernels * args.steps,
            "clocks": clk}
    if rank == 0 and not args.no_cpu_baseline:
        # the oracle on every usable host CPU (the baseline), and on one
        # thread over a bounded sample of the same queries (for reference)
        line["cpu_baseline"] = cpu_baseline_all_cores(wl, t, max_seconds=args.cpu_seconds)
        one = cpu_baseline(wl, t, max_seconds=min(5.0, args.cpu_seconds), min_seconds=min(3.0, args.cpu_seconds))
        line["cpu_baseline"]["single_thread"] = {"value": one["value"], "unit": UNIT, "cores": 1,
                                                 "sample": one["sample"]}
    if world == 1 and not args.no_secondary:
        del st, t, run
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        try:
            line["secondary"] = secondary(dev, flush, stream, min(args.steps, 10), args.warmup, peak,
                                          fuse_append=not args.no_fuse_append)
        except Exception as exc:  # the headline line still prints; the failure is reported in it
            print(f"secondary workloads failed: {exc!r}", file=sys.stderr, flush=True)
            line["secondary"] = {"error": repr(exc)}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
