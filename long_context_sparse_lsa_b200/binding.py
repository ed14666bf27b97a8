"""Python binding of liblsa.so (include/lsa.h): argument marshalling only.

Every function takes torch tensors, passes their device pointers and sizes to
the C ABI on the current CUDA stream, and raises LsaError on a non-zero
status. Every step of the hot path runs in the library's CUDA kernels; there
is no fallback. If the library is missing, loading it raises immediately.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblsa.so")

LSA_DEV_BAD_LENGTH = 0x1
LSA_DEV_BAD_SEQ = 0x2
LSA_DEV_BAD_INDEX = 0x4
LSA_DEV_BAD_WEIGHT = 0x8
LSA_DEV_TIMEOUT = 0x10
LSA_DEV_BAD_QUERY = 0x20
LSA_DEV_BAD_VALUE = 0x40

STATUS = {0: "LSA_OK", 1: "LSA_ERR_INVALID_ARG", 2: "LSA_ERR_UNSUPPORTED", 3: "LSA_ERR_CUDA",
          4: "LSA_ERR_WORKSPACE"}

EXPORTS = ["lsa_version", "lsa_last_cuda_error", "lsa_status_string", "lsa_hi_block_sums", "lsa_append",
           "lsa_index_workspace_size", "lsa_index", "lsa_attend_workspace_size", "lsa_attend", "lsa_attend_fp8",
           "lsa_merge_pairs", "lsa_score_tokens", "lsa_score_blocks", "lsa_attend_lse", "lsa_shard_sets",
           "lsa_combine", "lsa_attend_grouped_workspace_size", "lsa_attend_grouped_launches", "lsa_attend_grouped",
           "lsa_attend_si_workspace_size", "lsa_attend_si_launches", "lsa_attend_si",
           "lsa_attend_noalloc", "lsa_append_index", "lsa_append_index_launches"]

MERGE_ID_BITS = 24  # LSA_MERGE_ID_BITS


class LsaError(RuntimeError):
    def __init__(self, func: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{func} failed: {STATUS.get(status, status)}"
        if status == 3:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


class _Budget(ctypes.Structure):
    _fields_ = [("sink", ctypes.c_int32), ("window", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("hi_block", ctypes.c_int32), ("hi_topblocks", ctypes.c_int32)]


class _Batch(ctypes.Structure):
    _fields_ = [("n_seq", ctypes.c_int32), ("n_q", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("total_tokens", ctypes.c_int64),
                ("kv_offset", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p), ("blk_offset", ctypes.c_void_p),
                ("q_seq", ctypes.c_void_p), ("q_len", ctypes.c_void_p)]


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

    def c(self) -> _Budget:
        return _Budget(self.sink, self.window, self.topk, self.hi_block, self.hi_topblocks)


@dataclass
class Batch:
    """Packed-sequence batch; tensors live on the device that runs the call."""
    kv_offset: torch.Tensor   # int64 [n_seq]
    seq_lens: torch.Tensor    # int32 [n_seq]
    q_seq: torch.Tensor       # int32 [n_q]
    q_len: torch.Tensor       # int32 [n_q]
    max_len: int
    total_tokens: int
    blk_offset: torch.Tensor | None = None  # int64 [n_seq]

    def c(self) -> _Batch:
        for name, t, dt in (("kv_offset", self.kv_offset, torch.int64), ("seq_lens", self.seq_lens, torch.int32),
                            ("q_seq", self.q_seq, torch.int32), ("q_len", self.q_len, torch.int32)):
            if t.dtype != dt or not t.is_contiguous():
                raise TypeError(f"{name} must be a contiguous {dt} tensor")
        if self.blk_offset is not None and (self.blk_offset.dtype != torch.int64 or not self.blk_offset.is_contiguous()):
            raise TypeError("blk_offset must be a contiguous int64 tensor")
        return _Batch(int(self.seq_lens.numel()), int(self.q_seq.numel()), int(self.max_len), 0,
                      int(self.total_tokens), self.kv_offset.data_ptr(), self.seq_lens.data_ptr(),
                      self.blk_offset.data_ptr() if self.blk_offset is not None else None,
                      self.q_seq.data_ptr(), self.q_len.data_ptr())


_lib = None


def library_path() -> str:
    return LIB_PATH


def load_library():
    """Load liblsa.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m long_context_sparse_lsa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.lsa_version.restype = i32
    lib.lsa_version.argtypes = []
    lib.lsa_last_cuda_error.restype = i32
    lib.lsa_last_cuda_error.argtypes = []
    lib.lsa_status_string.restype = ctypes.c_char_p
    lib.lsa_status_string.argtypes = [i32]
    lib.lsa_hi_block_sums.restype = i32
    lib.lsa_hi_block_sums.argtypes = [vp, i32, i32, ctypes.POINTER(_Batch), i32, vp, i64, vp, vp]
    lib.lsa_append.restype = i32
    lib.lsa_append.argtypes = [vp, vp, i32, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                               ctypes.POINTER(vp), i32, i32, i32, vp, i64, ctypes.POINTER(_Batch), i32, vp, vp]
    lib.lsa_append_index.restype = i32
    lib.lsa_append_index.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                     i32, i32, i32, vp, vp, vp, i32, i32, i32, ctypes.POINTER(_Batch), _Budget, vp, i64,
                                     vp, vp, sz, vp, vp]
    lib.lsa_append_index_launches.restype = i32
    lib.lsa_append_index_launches.argtypes = [ctypes.POINTER(_Batch), i32, i32, _Budget, i32]
    lib.lsa_index_workspace_size.restype = sz
    lib.lsa_index_workspace_size.argtypes = [ctypes.POINTER(_Batch), i32, i32, _Budget]
    lib.lsa_index_launches.restype = i32
    lib.lsa_index_launches.argtypes = [ctypes.POINTER(_Batch), i32, i32, _Budget]
    lib.lsa_attend_launches.restype = i32
    lib.lsa_attend_launches.argtypes = [ctypes.POINTER(_Batch), i32, i32, i32, i32, i32]
    lib.lsa_index_uses_tensor_cores.restype = i32
    lib.lsa_index_uses_tensor_cores.argtypes = [ctypes.POINTER(_Batch), i32, i32, _Budget]
    lib.lsa_index.restype = i32
    lib.lsa_index.argtypes = [vp, vp, vp, i32, i32, i32, ctypes.POINTER(_Batch), _Budget, vp, i64, vp, vp, sz, vp, vp]
    lib.lsa_attend_workspace_size.restype = sz
    lib.lsa_attend_workspace_size.argtypes = [ctypes.POINTER(_Batch), i32, i32, i32, i32, i32]
    lib.lsa_attend.restype = i32
    lib.lsa_attend.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp, i32,
                               ctypes.POINTER(_Batch), i32, ctypes.POINTER(vp), vp, sz, vp, vp]
    lib.lsa_attend_fp8.restype = i32
    lib.lsa_attend_fp8.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                   ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float), i32, i32, i32, vp,
                                   i32, ctypes.POINTER(_Batch), i32, ctypes.POINTER(vp), vp, sz, vp, vp]
    lib.lsa_score_tokens.restype = i32
    lib.lsa_score_tokens.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i64, vp, i32, vp, vp, vp]
    lib.lsa_score_blocks.restype = i32
    lib.lsa_score_blocks.argtypes = [vp, vp, i32, i32, i32, i32, vp, i64, vp, vp, i32, vp, vp, vp]
    lib.lsa_merge_pairs.restype = i32
    lib.lsa_merge_pairs.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp]
    lib.lsa_attend_lse.restype = i32
    lib.lsa_attend_lse.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp, i32,
                                   ctypes.POINTER(_Batch), i32, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, sz, vp, vp]
    lib.lsa_shard_sets.restype = i32
    lib.lsa_shard_sets.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
    lib.lsa_combine.restype = i32
    lib.lsa_combine.argtypes = [vp, vp, i32, i64, i32, vp, vp, vp]
    lib.lsa_attend_grouped_workspace_size.restype = sz
    lib.lsa_attend_grouped_workspace_size.argtypes = [ctypes.POINTER(_Batch), i32, i32, i32, i32, i32, i32]
    lib.lsa_attend_grouped_launches.restype = i32
    lib.lsa_attend_grouped_launches.argtypes = [ctypes.POINTER(_Batch), i32, i32, i32, i32, i32, i32]
    lib.lsa_attend_grouped.restype = i32
    lib.lsa_attend_grouped.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp,
                                       i32, ctypes.POINTER(_Batch), i32, i32, ctypes.POINTER(vp), vp, sz, vp, vp]
    lib.lsa_attend_si_workspace_size.restype = sz
    lib.lsa_attend_si_workspace_size.argtypes = [ctypes.POINTER(_Batch), i32, i32, i32, _Budget, i32]
    lib.lsa_attend_si_launches.restype = i32
    lib.lsa_attend_si_launches.argtypes = [ctypes.POINTER(_Batch), i32, i32, i32, _Budget, i32]
    lib.lsa_attend_si.restype = i32
    lib.lsa_attend_si.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp,
                                  _Budget, ctypes.POINTER(_Batch), i32, ctypes.POINTER(vp), vp, sz, vp, vp]
    lib.lsa_attend_noalloc.restype = i32
    lib.lsa_attend_noalloc.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp,
                                       i32, ctypes.POINTER(_Batch), i32, ctypes.POINTER(vp), vp, vp]
    _lib = lib
    return lib


def _check(func: str, status: int):
    if status != 0:
        raise LsaError(func, status, load_library().lsa_last_cuda_error() if status == 3 else 0)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def lsa_version() -> int:
    return load_library().lsa_version()


def lsa_hi_block_sums(k_idx: torch.Tensor, hi_block: int, batch: Batch, block_sums: torch.Tensor,
                      n_new: int = 0, dev_status: torch.Tensor | None = None, stream=None) -> None:
    """HI block sums into ``block_sums`` (int8 [rows, 2*d_I]); n_new > 0 only
    refreshes the blocks holding each sequence's last n_new tokens."""
    lib = load_library()
    d_I = k_idx.shape[-1]
    cb = batch.c()
    st = lib.lsa_hi_block_sums(_ptr(k_idx), d_I, hi_block, ctypes.byref(cb), n_new, _ptr(block_sums),
                               block_sums.shape[0], _ptr(dev_status), _stream(stream))
    _check("lsa_hi_block_sums", st)


def lsa_index_workspace_size(batch: Batch, H_I: int, d_I: int, budget: Budget) -> int:
    cb = batch.c()
    return int(load_library().lsa_index_workspace_size(ctypes.byref(cb), H_I, d_I, budget.c()))


def lsa_index_launches(batch: Batch, H_I: int, d_I: int, budget: Budget) -> int:
    """Kernel launches lsa_index issues for this shape."""
    cb = batch.c()
    return int(load_library().lsa_index_launches(ctypes.byref(cb), H_I, d_I, budget.c()))


def lsa_attend_launches(batch: Batch, H_q: int, H_kv: int, d: int, budget: int, layers: int) -> int:
    """Kernel launches lsa_attend issues for this shape."""
    cb = batch.c()
    return int(load_library().lsa_attend_launches(ctypes.byref(cb), H_q, H_kv, d, budget, layers))


def lsa_index_uses_tensor_cores(batch: Batch, H_I: int, d_I: int, budget: Budget) -> bool:
    """True when lsa_index scores this batch as one dense tcgen05 contraction."""
    cb = batch.c()
    return bool(load_library().lsa_index_uses_tensor_cores(ctypes.byref(cb), H_I, d_I, budget.c()))


def lsa_index(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, w_max: int, batch: Batch,
              budget: Budget, index_sets: torch.Tensor, block_sums: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None, stream=None) -> None:
    """Index sets [n_q, sink+window+topk] (int32) into ``index_sets``."""
    lib = load_library()
    n_q, H_I, d_I = q_idx.shape
    cb = batch.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.lsa_index(_ptr(q_idx), _ptr(k_idx), _ptr(w), w_max, H_I, d_I, ctypes.byref(cb), budget.c(),
                       _ptr(block_sums), 0 if block_sums is None else block_sums.shape[0], _ptr(index_sets),
                       _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    _check("lsa_index", st)


def lsa_attend_workspace_size(batch: Batch, H_q: int, H_kv: int, d: int, budget: int, layers: int) -> int:
    cb = batch.c()
    return int(load_library().lsa_attend_workspace_size(ctypes.byref(cb), H_q, H_kv, d, budget, layers))


def lsa_append(k_idx_new: torch.Tensor, k_idx: torch.Tensor, k_new: list, v_new: list, k: list, v: list,
               hi_block: int, block_sums: torch.Tensor | None, batch: Batch, n_new: int,
               dev_status: torch.Tensor | None = None, stream=None) -> None:
    """Write the n_new newest tokens of every sequence (keys k_idx_new [n_seq, n_new, d_I], per-layer K/V
    rows k_new/v_new [n_seq, n_new, H_kv, d], bf16 or FP8 codes like the caches k/v) into the caches and
    refresh their blocks' sums (HI on)."""
    lib = load_library()
    G = len(k_new)
    d_I = k_idx.shape[-1]
    row_bytes = k[0].shape[1] * k[0].shape[2] * k[0].element_size() if G else 0
    arr = ctypes.c_void_p * max(G, 1)
    kn, vn, kc, vc = (arr(*[t.data_ptr() for t in x]) for x in (k_new, v_new, k, v))
    cb = batch.c()
    rows = block_sums.shape[0] if block_sums is not None else 0
    st = lib.lsa_append(_ptr(k_idx_new), _ptr(k_idx), d_I, kn, vn, kc, vc, row_bytes, G, hi_block, _ptr(block_sums),
                        rows, ctypes.byref(cb), n_new, _ptr(dev_status), _stream(stream))
    _check("lsa_append", st)


def lsa_append_index(k_idx_new: torch.Tensor, k_new: list, v_new: list, k: list, v: list, n_new: int,
                     q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, w_max: int, batch: Batch,
                     budget: Budget, index_sets: torch.Tensor, block_sums: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                     stream=None) -> None:
    """lsa_append (the n_new newest tokens' keys and K/V rows, their blocks' sums) followed by lsa_index, in one
    call; with HI on and the new tokens inside every window the append runs inside the block selection."""
    lib = load_library()
    G = len(k_new)
    n_q, H_I, d_I = q_idx.shape
    row_bytes = k[0].shape[1] * k[0].shape[2] * k[0].element_size() if G else 0
    arr = ctypes.c_void_p * max(G, 1)
    kn, vn, kc, vc = (arr(*[t.data_ptr() for t in x]) for x in (k_new, v_new, k, v))
    cb = batch.c()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rows = block_sums.shape[0] if block_sums is not None else 0
    st = lib.lsa_append_index(_ptr(k_idx_new), kn, vn, kc, vc, row_bytes, G, n_new, _ptr(q_idx), _ptr(k_idx), _ptr(w),
                              w_max, H_I, d_I, ctypes.byref(cb), budget.c(), _ptr(block_sums), rows,
                              _ptr(index_sets), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    _check("lsa_append_index", st)


def lsa_append_index_launches(batch: Batch, H_I: int, d_I: int, budget: Budget, n_new: int) -> int:
    """Kernel launches lsa_append_index issues for this shape."""
    cb = batch.c()
    return int(load_library().lsa_append_index_launches(ctypes.byref(cb), H_I, d_I, budget.c(), n_new))


def lsa_attend(q: list, k: list, v: list, index_sets: torch.Tensor, batch: Batch, out: list,
               workspace: torch.Tensor, dev_status: torch.Tensor | None = None, stream=None) -> None:
    """Sparse attention of G layers (lists of G tensors) over one index set per row."""
    lib = load_library()
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k[0].shape[1]
    arr = ctypes.c_void_p * G
    qa, ka, va, oa = (arr(*[t.data_ptr() for t in x]) for x in (q, k, v, out))
    cb = batch.c()
    st = lib.lsa_attend(qa, ka, va, H_q, H_kv, d, _ptr(index_sets), index_sets.shape[1], ctypes.byref(cb), G, oa,
                        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
                        _stream(stream))
    _check("lsa_attend", st)


def lsa_attend_grouped_workspace_size(batch: Batch, H_q: int, H_kv: int, d: int, budget: int, layers: int,
                                      group_rows: int) -> int:
    return load_library().lsa_attend_grouped_workspace_size(ctypes.byref(batch.c()), H_q, H_kv, d, budget, layers,
                                                            group_rows)


def lsa_attend_grouped_launches(batch: Batch, H_q: int, H_kv: int, d: int, budget: int, layers: int,
                                group_rows: int) -> int:
    return load_library().lsa_attend_grouped_launches(ctypes.byref(batch.c()), H_q, H_kv, d, budget, layers,
                                                      group_rows)


def lsa_attend_grouped(q: list, k: list, v: list, index_sets: torch.Tensor, batch: Batch, group_rows: int,
                       out: list, workspace: torch.Tensor, dev_status: torch.Tensor | None = None,
                       stream=None) -> None:
    """lsa_attend for rows in groups of group_rows draft rows of one sequence:
    each group's sets are gathered once as their union."""
    lib = load_library()
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k[0].shape[1]
    arr = ctypes.c_void_p * G
    qa, ka, va, oa = (arr(*[t.data_ptr() for t in x]) for x in (q, k, v, out))
    cb = batch.c()
    st = lib.lsa_attend_grouped(qa, ka, va, H_q, H_kv, d, _ptr(index_sets), index_sets.shape[1], ctypes.byref(cb),
                                G, group_rows, oa, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(dev_status), _stream(stream))
    _check("lsa_attend_grouped", st)


def lsa_attend_si_workspace_size(batch: Batch, H_q: int, H_kv: int, d: int, budget: Budget, layers: int) -> int:
    return load_library().lsa_attend_si_workspace_size(ctypes.byref(batch.c()), H_q, H_kv, d, budget.c(), layers)


def lsa_attend_si_launches(batch: Batch, H_q: int, H_kv: int, d: int, budget: Budget, layers: int) -> int:
    return load_library().lsa_attend_si_launches(ctypes.byref(batch.c()), H_q, H_kv, d, budget.c(), layers)


def lsa_attend_si(q: list, k: list, v: list, index_sets: torch.Tensor, budget: Budget, batch: Batch, out: list,
                  workspace: torch.Tensor, dev_status: torch.Tensor | None = None, stream=None) -> None:
    """lsa_attend over SI-structured sets (as lsa_index writes them): the sink
    and window runs as dense tiles, the selected entries gathered per row."""
    lib = load_library()
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k[0].shape[1]
    if index_sets.shape[1] != budget.length:
        raise ValueError("index_sets must be [n_q, sink + window + topk]")
    arr = ctypes.c_void_p * G
    qa, ka, va, oa = (arr(*[t.data_ptr() for t in x]) for x in (q, k, v, out))
    cb = batch.c()
    st = lib.lsa_attend_si(qa, ka, va, H_q, H_kv, d, _ptr(index_sets), budget.c(), ctypes.byref(cb), G, oa,
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
                           _stream(stream))
    _check("lsa_attend_si", st)


def lsa_attend_lse(q: list, k: list, v: list, index_sets: torch.Tensor, batch: Batch, out: list, lse: list,
                   workspace: torch.Tensor, dev_status: torch.Tensor | None = None, stream=None) -> None:
    """lsa_attend that also writes lse[g] (fp32 [n_q, H_q]): the log of each
    row and head's softmax denominator (-inf for an empty set)."""
    lib = load_library()
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k[0].shape[1]
    for t in lse:
        if t.dtype != torch.float32 or t.shape != (n_q, H_q) or not t.is_contiguous():
            raise TypeError("lse must hold contiguous float32 [n_q, H_q] tensors")
    arr = ctypes.c_void_p * G
    qa, ka, va, oa, la = (arr(*[t.data_ptr() for t in x]) for x in (q, k, v, out, lse))
    cb = batch.c()
    st = lib.lsa_attend_lse(qa, ka, va, H_q, H_kv, d, _ptr(index_sets), index_sets.shape[1], ctypes.byref(cb), G, oa,
                            la, _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(dev_status),
                            _stream(stream))
    _check("lsa_attend_lse", st)


def lsa_shard_sets(index_sets: torch.Tensor, lo: int, hi: int, local_sets: torch.Tensor,
                   dev_status: torch.Tensor | None = None, stream=None) -> None:
    """The entries of each row's set inside [lo, hi), as e - lo in set order,
    -1 after (int32 [n_q, budget] in and out)."""
    lib = load_library()
    if index_sets.dtype != torch.int32 or local_sets.dtype != torch.int32:
        raise TypeError("index sets must be int32")
    if local_sets.shape != index_sets.shape or not (index_sets.is_contiguous() and local_sets.is_contiguous()):
        raise TypeError("local_sets must be a contiguous tensor shaped like index_sets")
    n_q, budget = index_sets.shape
    st = lib.lsa_shard_sets(_ptr(index_sets), n_q, budget, int(lo), int(hi), _ptr(local_sets), _ptr(dev_status),
                            _stream(stream))
    _check("lsa_shard_sets", st)


def lsa_combine(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: torch.Tensor,
                lse_out: torch.Tensor | None = None, stream=None) -> None:
    """Exact log-sum-exp combination of attention partials: o_parts fp32
    [n_parts, rows..., d], lse_parts fp32 [n_parts, rows...], out fp32
    [rows..., d], lse_out fp32 [rows...] or None."""
    lib = load_library()
    for t in (o_parts, lse_parts, out) + ((lse_out,) if lse_out is not None else ()):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("lsa_combine takes contiguous float32 tensors")
    n_parts, d = o_parts.shape[0], o_parts.shape[-1]
    rows = o_parts[0].numel() // max(d, 1)
    if lse_parts.numel() != n_parts * rows or out.numel() != rows * d:
        raise ValueError("lse_parts must hold n_parts x rows values and out rows x d")
    if lse_out is not None and lse_out.numel() != rows:
        raise ValueError("lse_out must hold one value per row")
    st = lib.lsa_combine(_ptr(o_parts), _ptr(lse_parts), n_parts, rows, d, _ptr(out), _ptr(lse_out), _stream(stream))
    _check("lsa_combine", st)


def lsa_attend_fp8(q: list, k8: list, v8: list, k_scale: list, v_scale: list, index_sets: torch.Tensor,
                   batch: Batch, out: list, workspace: torch.Tensor, dev_status: torch.Tensor | None = None,
                   stream=None) -> None:
    """lsa_attend over FP8 E4M3 K/V caches (uint8 tensors [T, H_kv, d]) with per-layer scales."""
    lib = load_library()
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k8[0].shape[1]
    arr = ctypes.c_void_p * G
    qa, ka, va, oa = (arr(*[t.data_ptr() for t in x]) for x in (q, k8, v8, out))
    fa = ctypes.c_float * G
    ks, vs = fa(*[float(x) for x in k_scale]), fa(*[float(x) for x in v_scale])
    cb = batch.c()
    st = lib.lsa_attend_fp8(qa, ka, va, ks, vs, H_q, H_kv, d, _ptr(index_sets), index_sets.shape[1],
                            ctypes.byref(cb), G, oa, _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _ptr(dev_status), _stream(stream))
    _check("lsa_attend_fp8", st)


def lsa_attend_noalloc(q: list, k: list, v: list, index_sets: torch.Tensor, batch: Batch, out: list,
                       dev_status: torch.Tensor | None = None, stream=None) -> None:
    """lsa_attend without a workspace: for callers that cannot allocate device
    memory on this path; the library's fixed static scratch is used instead
    (see include/lsa.h for the size limit and the sharing rules)."""
    lib = load_library()
    G = len(q)
    n_q, H_q, d = q[0].shape
    H_kv = k[0].shape[1]
    arr = ctypes.c_void_p * G
    qa, ka, va, oa = (arr(*[t.data_ptr() for t in x]) for x in (q, k, v, out))
    cb = batch.c()
    st = lib.lsa_attend_noalloc(qa, ka, va, H_q, H_kv, d, _ptr(index_sets), index_sets.shape[1], ctypes.byref(cb),
                                G, oa, _ptr(dev_status), _stream(stream))
    _check("lsa_attend_noalloc", st)


def lsa_merge_pairs(pairs: torch.Tensor, counts: torch.Tensor, k: int, out: torch.Tensor,
                    out_values: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                    stream=None) -> None:
    """Exact top-k of each row's packed (key, id) values (include/lsa.h):
    pairs int64 [n_rows, cap] holding the uint64 bit patterns (0 = empty),
    counts int32 [n_rows], out int32 [n_rows, k] (ids ascending, -1 padded),
    out_values int64 [n_rows, k] or None (the kept entries, 0 padded)."""
    lib = load_library()
    if pairs.dtype != torch.int64 or counts.dtype != torch.int32 or out.dtype != torch.int32:
        raise TypeError("pairs must be int64, counts and out int32")
    if not (pairs.is_contiguous() and counts.is_contiguous() and out.is_contiguous()):
        raise TypeError("pairs, counts and out must be contiguous")
    n_rows, cap = pairs.shape
    if counts.shape != (n_rows,) or out.shape != (n_rows, k):
        raise ValueError("counts must be [n_rows] and out [n_rows, k]")
    if out_values is not None and (out_values.dtype != torch.int64 or out_values.shape != (n_rows, k)
                                   or not out_values.is_contiguous()):
        raise TypeError("out_values must be a contiguous int64 [n_rows, k] tensor")
    st = lib.lsa_merge_pairs(_ptr(pairs), _ptr(counts), n_rows, cap, k, _ptr(out), _ptr(out_values),
                             _ptr(dev_status), _stream(stream))
    _check("lsa_merge_pairs", st)


def lsa_score_tokens(q_idx: torch.Tensor, k_idx: torch.Tensor, w: torch.Tensor, w_max: int,
                     row_offset: torch.Tensor, positions: torch.Tensor, keys: torch.Tensor,
                     dev_status: torch.Tensor | None = None, stream=None) -> None:
    """Fine indexer keys (score + 1) of given positions: q_idx int8 [n_q, H_I,
    d_I], k_idx int8 [T, d_I], w int32 [n_q, H_I], row_offset int64 [n_q],
    positions int32 [n_q, n] (-1 empty), keys int32 [n_q, n] (uint32 bits)."""
    lib = load_library()
    n_q, H_I, d_I = q_idx.shape
    n = positions.shape[1]
    if keys.shape != (n_q, n) or keys.dtype != torch.int32 or positions.dtype != torch.int32:
        raise TypeError("positions and keys must be int32 [n_q, n]")
    st = lib.lsa_score_tokens(_ptr(q_idx), _ptr(k_idx), _ptr(w), w_max, H_I, d_I, n_q, _ptr(row_offset),
                              k_idx.shape[0], _ptr(positions), n, _ptr(keys), _ptr(dev_status), _stream(stream))
    _check("lsa_score_tokens", st)


def lsa_score_blocks(q_idx: torch.Tensor, w: torch.Tensor, w_max: int, block_sums: torch.Tensor,
                     blk_row_offset: torch.Tensor, blocks: torch.Tensor, keys: torch.Tensor,
                     dev_status: torch.Tensor | None = None, stream=None) -> None:
    """HI coarse keys (score + 1) of given blocks: block_sums int8 [rows,
    2*d_I] (byte planes), blk_row_offset int64 [n_q], blocks int32 [n_q, n]
    (-1 empty), keys int64 [n_q, n] (uint64 bits)."""
    lib = load_library()
    n_q, H_I, d_I = q_idx.shape
    n = blocks.shape[1]
    if keys.shape != (n_q, n) or keys.dtype != torch.int64 or blocks.dtype != torch.int32:
        raise TypeError("blocks must be int32 and keys int64 [n_q, n]")
    st = lib.lsa_score_blocks(_ptr(q_idx), _ptr(w), w_max, H_I, d_I, n_q, _ptr(block_sums), block_sums.shape[0],
                              _ptr(blk_row_offset), _ptr(blocks), n, _ptr(keys), _ptr(dev_status), _stream(stream))
    _check("lsa_score_blocks", st)
