"""Helpers shared by the GPU parity tests: host copies of the seeded inputs,
oracle calls on them, and the comparison rules.

Rules (fixed here, used by every parity test):
  * index sets: bit-exact;
  * attention: max |err| <= 5e-3 and relative L2 <= 1e-3 against the oracle's
    fp64 evaluation on the same bf16 values.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

ATT_MAX_ABS = 5e-3
ATT_REL_L2 = 1e-3


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy()


def oracle_sets(wl, t, hi_block=None, hi_topblocks=None, n_threads=8, rows=None):
    """Oracle index sets of the given query rows (default: all)."""
    orc = oracle.get()
    hb = wl.hi_block if hi_block is None else hi_block
    ht = wl.hi_topblocks if hi_topblocks is None else hi_topblocks
    q_idx, w, q_seq, q_len = host(t.q_idx), host(t.w), host(t.q_seq), host(t.q_len)
    if rows is not None:
        rows = np.asarray(rows)
        q_idx, w, q_seq, q_len = q_idx[rows], w[rows], q_seq[rows], q_len[rows]
    return orc.lsa_index(q_idx, host(t.k_idx), w, host(t.kv_offset), q_seq, q_len, wl.sink, wl.window, wl.topk,
                         hb, ht, n_threads=n_threads)


def oracle_attend_full(t, sets, n_threads=8):
    """Oracle attention with full host copies of K/V (small workloads)."""
    orc = oracle.get()
    return orc.lsa_attend([u16(x) for x in t.q], [u16(x) for x in t.k], [u16(x) for x in t.v], sets,
                          host(t.kv_offset), host(t.q_seq), n_threads=n_threads)


def oracle_attend_rows(t, sets, rows):
    """Oracle attention for selected rows, reading only the K/V rows each set
    names (gathered on the device by position, then renumbered 0..n-1)."""
    orc = oracle.get()
    kv_off = host(t.kv_offset)
    q_seq = host(t.q_seq)
    outs = []
    for g in range(len(t.q)):
        per = []
        for i, r in enumerate(rows):
            s = sets[i]
            valid = s[s >= 0]
            base = int(kv_off[q_seq[r]])
            idx = torch.as_tensor(valid.astype(np.int64) + base, device=t.k[g].device)
            kr = u16(t.k[g].index_select(0, idx))
            vr = u16(t.v[g].index_select(0, idx))
            local = np.full(s.shape[0], -1, np.int32)
            local[: valid.shape[0]] = np.arange(valid.shape[0], dtype=np.int32)
            per.append(orc.attend_query(u16(t.q[g][r]), kr, vr, local))
        outs.append(np.stack(per))
    return outs


def oracle_attend_rows_fp8(st, sets, rows):
    """oracle_attend_rows for a step whose K/V caches are FP8 codes
    (st.k8 / st.v8 with per-layer scales st.k_scale / st.v_scale)."""
    orc = oracle.get()
    t = st.t
    kv_off = host(t.kv_offset)
    q_seq = host(t.q_seq)
    outs = []
    for g in range(len(t.q)):
        per = []
        for i, r in enumerate(rows):
            s = sets[i]
            valid = s[s >= 0]
            base = int(kv_off[q_seq[r]])
            idx = torch.as_tensor(valid.astype(np.int64) + base, device=st.k8[g].device)
            kr = host(st.k8[g].index_select(0, idx))
            vr = host(st.v8[g].index_select(0, idx))
            local = np.full(s.shape[0], -1, np.int32)
            local[: valid.shape[0]] = np.arange(valid.shape[0], dtype=np.int32)
            per.append(orc.attend_query_fp8(u16(t.q[g][r]), kr, vr, st.k_scale[g], st.v_scale[g], local))
        outs.append(np.stack(per))
    return outs


def check_attention(got: np.ndarray, want: np.ndarray, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - want)
    max_abs = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(got - want) / den) if den > 0 else float(np.linalg.norm(got - want))
    assert max_abs <= ATT_MAX_ABS, f"{what}: max|err| {max_abs:.3e} > {ATT_MAX_ABS}"
    assert rel <= ATT_REL_L2, f"{what}: rel-L2 {rel:.3e} > {ATT_REL_L2}"
    return max_abs, rel


def check_sets(got: np.ndarray, want: np.ndarray, what=""):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        r = int(bad[0][0])
        raise AssertionError(f"{what}: index sets differ in {len(np.unique(bad[:, 0]))} rows; first row {r}: "
                             f"gpu {got[r][:16]}... oracle {want[r][:16]}... "
                             f"(first diff at col {int(bad[0][1])}: {got[r][bad[0][1]]} vs {want[r][bad[0][1]]})")


def decode_block_sums(bs: torch.Tensor, d_I: int) -> np.ndarray:
    """int8 [rows, 2*d_I] byte planes -> int64 [rows, d_I] sums (S = 256*hi + lo)."""
    a = host(bs)
    hi = a[:, :d_I].astype(np.int64)
    lo = a[:, d_I:].view(np.uint8).astype(np.int64)
    return hi * 256 + lo
