"""CPU oracle for the LSA hot path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never loads it and
shares no code with it: this module compiles ``lsa_oracle.c`` (plain C, int64
scores, fp64 attention) with the host C compiler and wraps it with ctypes and
numpy. Every function here is a thin marshalling layer; the arithmetic lives
in ``lsa_oracle.c`` and is documented there with the passages it follows.

Pins (tests/test_oracle_*.py) tie every oracle function to closed forms,
invariants and brute force that do not reuse its code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "lsa_oracle.c")
LIBRARY = os.path.join(_HERE, "liblsa_oracle.so")

_i8p = ctypes.POINTER(ctypes.c_int8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(source: str | None = None, output: str | None = None, source_text: str | None = None) -> str:
    """Compile the oracle (or a variant of its text) into a shared library.

    ``source_text`` lets the mutation tests compile a deliberately broken copy
    into a temporary file; the committed source is never modified.
    """
    output = output or LIBRARY
    src = source or SOURCE
    tmpdir = None
    if source_text is not None:
        tmpdir = tempfile.mkdtemp(prefix="lsa_oracle_")
        src = os.path.join(tmpdir, "variant.c")
        with open(src, "w") as f:
            f.write(source_text)
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-o", output, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True, capture_output=True)
    return output


def _needs_build() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    return os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)


class Oracle:
    """ctypes handle on one compiled copy of the oracle."""

    def __init__(self, path: str | None = None):
        if path is None:
            if _needs_build():
                build()
            path = LIBRARY
        self.path = path
        lib = ctypes.CDLL(path)
        lib.oracle_fine_score.restype = ctypes.c_int64
        lib.oracle_fine_score.argtypes = [_i8p, _i32p, _i8p, ctypes.c_int, ctypes.c_int]
        lib.oracle_block_sums.restype = None
        lib.oracle_block_sums.argtypes = [_i8p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _i64p]
        lib.oracle_coarse_score.restype = ctypes.c_int64
        lib.oracle_coarse_score.argtypes = [_i8p, _i32p, _i64p, ctypes.c_int, ctypes.c_int]
        lib.oracle_index_query.restype = ctypes.c_int
        lib.oracle_index_query.argtypes = [_i8p, _i32p, _i8p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, _i32p]
        lib.oracle_attend_query.restype = None
        lib.oracle_attend_query.argtypes = [_u16p, _u16p, _u16p, _i32p, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, _f64p]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_attend_query_fp8.restype = None
        lib.oracle_attend_query_fp8.argtypes = [_u16p, _u8p, _u8p, ctypes.c_double, ctypes.c_double, _i32p,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p]
        lib.oracle_lsa_index.restype = ctypes.c_int
        lib.oracle_lsa_index.argtypes = [_i8p, _i8p, _i32p, _i64p, _i32p, _i32p, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, ctypes.c_int]
        lib.oracle_lsa_attend.restype = ctypes.c_int
        lib.oracle_lsa_attend.argtypes = [ctypes.POINTER(_u16p), ctypes.POINTER(_u16p), ctypes.POINTER(_u16p),
                                          _i32p, ctypes.c_int, _i64p, _i32p, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(_f64p),
                                          ctypes.c_int]
        self.lib = lib

    # -- scalar pieces ---------------------------------------------------------
    def fine_score(self, q: np.ndarray, w: np.ndarray, k: np.ndarray) -> int:
        q = _c(q, np.int8)
        w = _c(w, np.int32)
        k = _c(k, np.int8)
        H_I, d_I = q.shape
        return int(self.lib.oracle_fine_score(_p(q, _i8p), _p(w, _i32p), _p(k, _i8p), H_I, d_I))

    def block_sums(self, k: np.ndarray, block: int) -> np.ndarray:
        k = _c(k, np.int8)
        L, d_I = k.shape
        nblk = (L + block - 1) // block
        out = np.zeros((nblk, d_I), np.int64)
        self.lib.oracle_block_sums(_p(k, _i8p), L, d_I, block, _p(out, _i64p))
        return out

    def coarse_score(self, q: np.ndarray, w: np.ndarray, S_b: np.ndarray) -> int:
        q = _c(q, np.int8)
        w = _c(w, np.int32)
        S_b = _c(S_b, np.int64)
        H_I, d_I = q.shape
        return int(self.lib.oracle_coarse_score(_p(q, _i8p), _p(w, _i32p), _p(S_b, _i64p), H_I, d_I))

    # -- one query -------------------------------------------------------------
    def index_query(self, q, w, kseq, L, sink, window, topk, hi_block=0, hi_topblocks=0) -> np.ndarray:
        q = _c(q, np.int8)
        w = _c(w, np.int32)
        kseq = _c(kseq, np.int8)
        H_I, d_I = q.shape
        assert kseq.shape[0] >= L and kseq.shape[1] == d_I
        out = np.empty(sink + window + topk, np.int32)
        n = self.lib.oracle_index_query(_p(q, _i8p), _p(w, _i32p), _p(kseq, _i8p), L, H_I, d_I, sink,
                                        window, topk, hi_block, hi_topblocks, _p(out, _i32p))
        if n < 0:
            raise ValueError("oracle_index_query rejected its arguments")
        return out

    def attend_query(self, q, kseq, vseq, idx_set) -> np.ndarray:
        """q: [H_q, d] bf16 bits (uint16); kseq/vseq: [L, H_kv, d] bf16 bits."""
        q = _c(q, np.uint16)
        kseq = _c(kseq, np.uint16)
        vseq = _c(vseq, np.uint16)
        s = _c(idx_set, np.int32)
        H_q, d = q.shape
        H_kv = kseq.shape[1]
        out = np.empty((H_q, d), np.float64)
        self.lib.oracle_attend_query(_p(q, _u16p), _p(kseq, _u16p), _p(vseq, _u16p), _p(s, _i32p),
                                     s.shape[0], H_q, H_kv, d, _p(out, _f64p))
        return out

    def e4m3_value(self, code: int) -> float:
        """The value of one FP8 E4M3 code (NaN for S.1111.111)."""
        return float(self.lib.oracle_e4m3_value(int(code) & 0xFF))

    def attend_query_fp8(self, q, kseq, vseq, k_scale, v_scale, idx_set) -> np.ndarray:
        """q: [H_q, d] bf16 bits (uint16); kseq/vseq: [L, H_kv, d] E4M3 codes (uint8);
        k = k_scale * E4M3(code), v = v_scale * E4M3(code)."""
        q = _c(q, np.uint16)
        kseq = _c(kseq, np.uint8)
        vseq = _c(vseq, np.uint8)
        s = _c(idx_set, np.int32)
        H_q, d = q.shape
        H_kv = kseq.shape[1]
        out = np.empty((H_q, d), np.float64)
        self.lib.oracle_attend_query_fp8(_p(q, _u16p), _p(kseq, _u8p), _p(vseq, _u8p), float(k_scale),
                                         float(v_scale), _p(s, _i32p), s.shape[0], H_q, H_kv, d, _p(out, _f64p))
        return out

    # -- batches ---------------------------------------------------------------
    def lsa_index(self, q_idx, k_idx, w, kv_offset, q_seq, q_len, sink, window, topk,
                  hi_block=0, hi_topblocks=0, n_threads=1) -> np.ndarray:
        q_idx = _c(q_idx, np.int8)
        k_idx = _c(k_idx, np.int8)
        w = _c(w, np.int32)
        kv_offset = _c(kv_offset, np.int64)
        q_seq = _c(q_seq, np.int32)
        q_len = _c(q_len, np.int32)
        n_q, H_I, d_I = q_idx.shape
        budget = sink + window + topk
        sets = np.empty((n_q, budget), np.int32)
        rc = self.lib.oracle_lsa_index(_p(q_idx, _i8p), _p(k_idx, _i8p), _p(w, _i32p), _p(kv_offset, _i64p),
                                       _p(q_seq, _i32p), _p(q_len, _i32p), n_q, H_I, d_I, sink, window, topk,
                                       hi_block, hi_topblocks, _p(sets, _i32p), n_threads)
        if rc != 0:
            raise ValueError("oracle_lsa_index rejected its arguments")
        return sets

    def lsa_attend(self, q_layers, k_layers, v_layers, sets, kv_offset, q_seq, n_threads=1):
        """q_layers: list of G arrays [n_q, H_q, d] (bf16 bits); k/v_layers: list of
        G arrays [T, H_kv, d]. Returns a list of G float64 arrays [n_q, H_q, d]."""
        G = len(q_layers)
        qs = [_c(x, np.uint16) for x in q_layers]
        ks = [_c(x, np.uint16) for x in k_layers]
        vs = [_c(x, np.uint16) for x in v_layers]
        sets = _c(sets, np.int32)
        kv_offset = _c(kv_offset, np.int64)
        q_seq = _c(q_seq, np.int32)
        n_q, H_q, d = qs[0].shape
        H_kv = ks[0].shape[1]
        outs = [np.empty((n_q, H_q, d), np.float64) for _ in range(G)]
        qa = (_u16p * G)(*[_p(x, _u16p) for x in qs])
        ka = (_u16p * G)(*[_p(x, _u16p) for x in ks])
        va = (_u16p * G)(*[_p(x, _u16p) for x in vs])
        oa = (_f64p * G)(*[_p(x, _f64p) for x in outs])
        rc = self.lib.oracle_lsa_attend(qa, ka, va, _p(sets, _i32p), sets.shape[1], _p(kv_offset, _i64p),
                                        _p(q_seq, _i32p), n_q, H_q, H_kv, d, G, oa, n_threads)
        if rc != 0:
            raise ValueError("oracle_lsa_attend failed")
        return outs


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _p(a: np.ndarray, ptype):
    return a.ctypes.data_as(ptype)


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from the committed source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
