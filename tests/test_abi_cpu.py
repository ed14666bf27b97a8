"""The C-ABI library on a machine without a GPU: it loads, exports every entry
point include/lsa.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest
import torch

from long_context_sparse_lsa_b200 import binding as lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("lsa_index", "lsa_attend", "lsa_hi_block_sums", "lsa_index_workspace_size",
              "lsa_attend_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = lsa.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {lsa.library_path()}").read()
    exported = set(re.findall(r" T (lsa_\w+)", out))
    assert set(declared_functions()) <= exported


def test_version_and_status_strings():
    lib = lsa.load_library()
    assert lib.lsa_version() >= 100
    assert lib.lsa_status_string(0) == b"LSA_OK"
    assert lib.lsa_status_string(4) == b"LSA_ERR_WORKSPACE"


def _batch(n_seq=1, n_q=1, max_len=100, total=100, ptr=0x1000):
    b = lsa._Batch()
    b.n_seq, b.n_q, b.max_len, b.reserved, b.total_tokens = n_seq, n_q, max_len, 0, total
    b.kv_offset = b.seq_lens = b.blk_offset = b.q_seq = b.q_len = ptr
    return b


def _budget(sink=4, window=8, topk=16, hb=0, ht=0):
    return lsa._Budget(sink, window, topk, hb, ht)


P = 0x10000  # a fake, 256-byte aligned device address: never dereferenced (validation fails first)


def _index(lib, **kw):
    args = dict(q=P, k=P, w=P, w_max=8, H_I=16, d_I=128, batch=_batch(), budget=_budget(), bs=None, rows=0,
                sets=P, ws=None, ws_bytes=0)
    args.update(kw)
    return lib.lsa_index(args["q"], args["k"], args["w"], args["w_max"], args["H_I"], args["d_I"],
                         ctypes.byref(args["batch"]), args["budget"], args["bs"], args["rows"], args["sets"],
                         args["ws"], args["ws_bytes"], None, None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(w=None), 1), (dict(sets=None), 1),
    (dict(d_I=96), 2), (dict(d_I=0), 1), (dict(H_I=0), 1), (dict(H_I=65), 2), (dict(w_max=-1), 1),
    (dict(w_max=1 << 20), 2),                       # fine scores would overflow int32
    (dict(budget=_budget(sink=-1)), 1), (dict(budget=_budget(topk=20000)), 2),
    (dict(budget=_budget(hb=64, ht=8)), 1),         # HI on without block sums
    (dict(budget=_budget(hb=512, ht=8), bs=P, rows=10), 2),
    (dict(budget=_budget(hb=64, ht=5000), bs=P, rows=10), 2),
    (dict(batch=_batch(n_seq=0)), 1), (dict(batch=_batch(max_len=0)), 1), (dict(q=P + 4), 1),
])
def test_index_rejects_before_launch(kw, want):
    lib = lsa.load_library()
    assert _index(lib, **kw) == want


def test_index_empty_batch_is_ok_without_launch():
    lib = lsa.load_library()
    assert _index(lib, batch=_batch(n_q=0)) == 0


def test_block_sums_rejects():
    lib = lsa.load_library()
    b = _batch()
    f = lib.lsa_hi_block_sums
    assert f(None, 128, 64, ctypes.byref(b), 0, P, 10, None, None) == 1
    assert f(P, 100, 64, ctypes.byref(b), 0, P, 10, None, None) == 2
    assert f(P, 128, 0, ctypes.byref(b), 0, P, 10, None, None) == 1
    assert f(P, 128, 300, ctypes.byref(b), 0, P, 10, None, None) == 2
    b.blk_offset = None
    assert f(P, 128, 64, ctypes.byref(b), 0, P, 10, None, None) == 1


def _append(lib, **kw):
    arr = (ctypes.c_void_p * 2)(P, P)
    args = dict(kin=P, kc=P, d_I=128, kn=arr, vn=arr, kcache=arr, vcache=arr, kvb=1024, layers=2, hb=64,
                bs=P, rows=10, batch=_batch(), n_new=1)
    args.update(kw)
    return lib.lsa_append(args["kin"], args["kc"], args["d_I"], args["kn"], args["vn"], args["kcache"],
                          args["vcache"], args["kvb"], args["layers"], args["hb"], args["bs"],
                          args["rows"], ctypes.byref(args["batch"]), args["n_new"], None, None)


@pytest.mark.parametrize("kw,want", [
    (dict(n_new=0), 1), (dict(kin=None), 1), (dict(kc=None), 1), (dict(kc=P + 8), 1), (dict(d_I=48), 2),
    (dict(layers=9), 2), (dict(layers=-1), 1), (dict(kvb=1000), 1), (dict(kvb=0), 1), (dict(kn=None), 1),
    (dict(hb=300), 2),
    (dict(bs=None), 1), (dict(batch=_batch(n_seq=0)), 1),
    (dict(kn=(ctypes.c_void_p * 2)(P, None)), 1),   # a null layer pointer
    (dict(vcache=(ctypes.c_void_p * 2)(P, P + 4)), 1),  # a misaligned layer pointer
])
def test_append_rejects_before_launch(kw, want):
    lib = lsa.load_library()
    assert _append(lib, **kw) == want


def _append_index(lib, **kw):
    arr = (ctypes.c_void_p * 2)(P, P)
    args = dict(kin=P, kn=arr, vn=arr, kcache=arr, vcache=arr, kvb=1024, layers=2, n_new=1, q=P, kc=P, w=P,
                w_max=8, H_I=16, d_I=128, batch=_batch(), budget=_budget(window=100, hb=64, ht=8), bs=P, rows=10,
                sets=P, ws=None, ws_bytes=0)
    args.update(kw)
    return lib.lsa_append_index(args["kin"], args["kn"], args["vn"], args["kcache"], args["vcache"], args["kvb"],
                                args["layers"], args["n_new"], args["q"], args["kc"], args["w"], args["w_max"],
                                args["H_I"], args["d_I"], ctypes.byref(args["batch"]), args["budget"], args["bs"],
                                args["rows"], args["sets"], args["ws"], args["ws_bytes"], None, None)


@pytest.mark.parametrize("kw,want", [
    (dict(n_new=0), 1), (dict(kin=None), 1), (dict(kvb=1000), 1), (dict(layers=9), 2),
    (dict(q=None), 1), (dict(sets=None), 1), (dict(d_I=96), 2), (dict(w_max=1 << 20), 2),
    (dict(bs=None), 1),                                   # HI on without block sums
    (dict(budget=_budget(sink=-1)), 1),
    (dict(ws=None, ws_bytes=0), 4),                       # fused path: the index workspace is checked first
    (dict(budget=_budget(window=10, hb=64, ht=8)), 4),    # sequential path: checked before the append's launch
    (dict(budget=_budget(hb=0, ht=0), bs=None), 4),       # HI off
])
def test_append_index_rejects_before_launch(kw, want):
    lib = lsa.load_library()
    assert _append_index(lib, **kw) == want


def test_append_index_launch_counts():
    lib = lsa.load_library()
    b = _batch(n_seq=16, n_q=16, max_len=131072, total=16 * 131072)
    fused = _budget(sink=64, window=1024, topk=2048, hb=64, ht=256)
    n_idx = lib.lsa_index_launches(ctypes.byref(b), 16, 128, fused)
    assert n_idx >= 3
    assert lib.lsa_append_index_launches(ctypes.byref(b), 16, 128, fused, 1) == n_idx
    assert lib.lsa_append_index_launches(ctypes.byref(b), 16, 128, fused, 961) == n_idx  # window == 64 + 961 - 1
    assert lib.lsa_append_index_launches(ctypes.byref(b), 16, 128, fused, 962) == n_idx + 1
    flat = _budget(sink=64, window=1024, topk=2048)
    assert lib.lsa_append_index_launches(ctypes.byref(b), 16, 128, flat, 1) == \
        lib.lsa_index_launches(ctypes.byref(b), 16, 128, flat) + 1
    assert lib.lsa_append_index_launches(ctypes.byref(b), 16, 128, fused, 0) == 0


def test_attend_fp8_rejects_before_launch():
    lib = lsa.load_library()
    b = _batch(n_q=16, max_len=131072, total=16 * 131072)
    arr = (ctypes.c_void_p * 1)(P)
    one = (ctypes.c_float * 1)(1.0)
    bad = (ctypes.c_float * 1)(float("inf"))
    f = lib.lsa_attend_fp8
    args = lambda H_q=32, ks=one, vs=one: (arr, arr, arr, ks, vs, H_q, 4, 128, P, 3136, ctypes.byref(b), 1, arr, P,
                                           1 << 30, None, None)
    assert f(*args(ks=None)) == 1
    assert f(*args(vs=None)) == 1
    assert f(*args(ks=bad)) == 1
    assert f(*args(H_q=64)) == 2  # groups of 16 query heads: bf16 caches only


def test_attend_rejects_and_sizes():
    lib = lsa.load_library()
    b = _batch(n_q=16, max_len=131072, total=16 * 131072)
    arr = (ctypes.c_void_p * 1)(P)
    f = lib.lsa_attend
    assert f(arr, arr, arr, 32, 4, 64, P, 3136, ctypes.byref(b), 1, arr, P, 1 << 30, None, None) == 2  # d != 128
    assert f(arr, arr, arr, 30, 4, 128, P, 3136, ctypes.byref(b), 1, arr, P, 1 << 30, None, None) == 1
    assert f(arr, arr, arr, 96, 4, 128, P, 3136, ctypes.byref(b), 1, arr, P, 1 << 30, None, None) == 2  # ratio 24
    assert f(arr, arr, arr, 32, 4, 128, P, 3136, ctypes.byref(b), 9, arr, P, 1 << 30, None, None) == 2  # G > 8
    assert f(arr, arr, arr, 32, 4, 128, None, 3136, ctypes.byref(b), 1, arr, P, 1 << 30, None, None) == 1
    assert f(arr, arr, arr, 32, 4, 128, P, 3136, ctypes.byref(b), 1, arr, P, 16, None, None) == 4  # workspace
    need = lib.lsa_attend_workspace_size(ctypes.byref(b), 32, 4, 128, 3136, 1)
    assert need >= 16 * 4
    need4 = lib.lsa_attend_workspace_size(ctypes.byref(b), 32, 4, 128, 3136, 4)
    assert need4 >= 4 * 16 * 4  # counters for every (layer, row)


def test_launch_counts_follow_the_shape():
    """The calls report how many kernels they launch (host fields only)."""
    import torch

    from long_context_sparse_lsa_b200 import workloads as wls

    def batch(n_seq, L, n_q=None):
        n_q = n_q or n_seq
        return lsa.Batch(torch.arange(n_seq, dtype=torch.int64) * L, torch.full((n_seq,), L, dtype=torch.int32),
                         torch.arange(n_q, dtype=torch.int32) % n_seq, torch.full((n_q,), L, dtype=torch.int32), L,
                         n_seq * L, torch.arange(n_seq, dtype=torch.int64) * ((L + 63) // 64))

    hi = lsa.Budget(64, 1024, 2048, 64, 256)
    flat = lsa.Budget(64, 1024, 2048, 0, 0)
    # 16 rows, 16 heads: coarse scores inside the block selection (3 launches)
    assert lsa.lsa_index_launches(batch(16, 131072), 16, 128, hi) == 3
    # one row: the coarse scoring kernel runs on its own (4 launches)
    assert lsa.lsa_index_launches(batch(1, 131072), 16, 128, hi) == 4
    # more than 16 indexer heads: separate coarse kernel
    assert lsa.lsa_index_launches(batch(16, 131072), 20, 128, hi) == 4
    # HI off: fine scores + token selection
    assert lsa.lsa_index_launches(batch(16, 131072), 16, 128, flat) == 2
    # attention: split over CTAs (+ merge) for few rows, one CTA per row for many
    assert lsa.lsa_attend_launches(batch(16, 131072), 32, 4, 128, 3136, 1) == 2
    assert lsa.lsa_attend_launches(batch(1, 300000, n_q=8192), 32, 4, 128, 3136, 1) == 1
    assert lsa.lsa_attend_launches(batch(16, 131072), 32, 4, 96, 3136, 1) == 0  # d != 128: unsupported


def test_binding_checks_batch_dtypes_before_any_call():
    """The binding refuses tensors of the wrong dtype or layout rather than
    passing a misread pointer across the ABI."""
    n = 3
    ok = dict(kv_offset=torch.zeros(n, dtype=torch.int64), seq_lens=torch.ones(n, dtype=torch.int32),
              q_seq=torch.arange(n, dtype=torch.int32), q_len=torch.ones(n, dtype=torch.int32))
    lsa.Batch(**ok, max_len=1, total_tokens=n).c()
    for name, bad in (("kv_offset", torch.zeros(n, dtype=torch.int32)), ("seq_lens", torch.ones(n)),
                      ("q_len", torch.ones(2 * n, dtype=torch.int32)[::2])):
        with pytest.raises(TypeError):
            lsa.Batch(**{**ok, name: bad}, max_len=1, total_tokens=n).c()
    with pytest.raises(TypeError):
        lsa.Batch(**ok, max_len=1, total_tokens=n, blk_offset=torch.zeros(n, dtype=torch.int32)).c()


def test_noalloc_refuses_shapes_beyond_its_scratch_before_launch():
    lib = lsa.load_library()
    b = _batch(n_q=4096, max_len=131072, total=4096 * 131072)
    arr = (ctypes.c_void_p * 1)(P)
    need = lib.lsa_attend_workspace_size(ctypes.byref(b), 32, 4, 128, 8192, 1)
    assert need > 8 << 20
    assert lib.lsa_attend_noalloc(arr, arr, arr, 32, 4, 128, P, 8192, ctypes.byref(b), 1, arr, None, None) == 2


def test_grouped_attention_rejects_and_counts_before_launch():
    """lsa_attend_grouped: group sizes, divisibility, GQA width and the
    budget are checked before any launch."""
    lib = lsa.load_library()
    b = _batch(n_q=16, max_len=131072, total=4 * 131072)
    arr = (ctypes.c_void_p * 1)(P)
    f = lib.lsa_attend_grouped
    args = lambda H_q=32, H_kv=4, budget=3136, D=4, ws=1 << 40: (arr, arr, arr, H_q, H_kv, 128, P, budget,
                                                                 ctypes.byref(b), 1, D, arr, P, ws, None, None)
    assert f(*args(D=3)) == 1                       # 16 rows are not groups of 3
    assert f(*args(D=16)) == 2                      # at most 8 rows per group
    assert f(*args(H_q=64)) == 2                    # GQA groups of at most 8 query heads
    assert f(*args(budget=16385)) == 2              # past LSA_MAX_BUDGET
    assert f(*args(ws=16)) == 4                     # workspace too small
    need = lib.lsa_attend_grouped_workspace_size(ctypes.byref(b), 32, 4, 128, 3136, 1, 4)
    assert need >= 16 * 32 * 128 * 4                # split partials of every (row, head)
    assert lib.lsa_attend_grouped_launches(ctypes.byref(b), 32, 4, 128, 3136, 1, 4) == 2
    assert lib.lsa_attend_grouped_launches(ctypes.byref(b), 32, 4, 128, 3136, 1, 3) == 0


def test_context_parallel_calls_reject_before_launch():
    lib = lsa.load_library()
    assert lib.lsa_shard_sets(P, 4, 100, 10, 5, P + 4096, None, None) == 1      # hi < lo
    assert lib.lsa_shard_sets(P, 4, 100, 0, 5, P, None, None) == 1              # in place
    assert lib.lsa_shard_sets(P, 4, 1 << 20, 0, 5, P + 4096, None, None) == 2   # budget too large
    assert lib.lsa_shard_sets(P, 0, 100, 0, 5, P + 4096, None, None) == 0       # nothing to do
    assert lib.lsa_combine(P, P, 0, 10, 128, P, None, None) == 1                # no parts
    assert lib.lsa_combine(P, P, 2, 10, 126, P, None, None) == 1                # d % 4
    assert lib.lsa_combine(P, P, 2, 0, 128, P, None, None) == 0                 # no rows
    b = _batch(n_q=16, max_len=131072, total=16 * 131072)
    arr = (ctypes.c_void_p * 1)(P)
    assert lib.lsa_attend_lse(arr, arr, arr, 32, 4, 128, P, 3136, ctypes.byref(b), 1, arr, None, P, 1 << 30,
                              None, None) == 1                                  # lse is required


def test_si_attention_rejects_and_counts_before_launch():
    """lsa_attend_si: one sequence, GQA groups of at most 8 heads, d = 128."""
    lib = lsa.load_library()
    arr = (ctypes.c_void_p * 1)(P)
    bud = _budget(64, 1024, 2048)
    one = _batch(n_seq=1, n_q=8192, max_len=270336, total=270336)
    two = _batch(n_seq=2, n_q=8192, max_len=270336, total=2 * 270336)
    f = lib.lsa_attend_si
    assert f(arr, arr, arr, 32, 4, 128, P, bud, ctypes.byref(two), 1, arr, P, 1 << 40, None, None) == 2
    assert f(arr, arr, arr, 64, 4, 128, P, bud, ctypes.byref(one), 1, arr, P, 1 << 40, None, None) == 2
    assert f(arr, arr, arr, 32, 4, 64, P, bud, ctypes.byref(one), 1, arr, P, 1 << 40, None, None) == 2
    assert f(arr, arr, arr, 32, 4, 128, P, _budget(-1, 8, 8), ctypes.byref(one), 1, arr, P, 1 << 40, None,
             None) == 1
    assert f(arr, arr, arr, 32, 4, 128, P, bud, ctypes.byref(one), 1, arr, P, 16, None, None) == 4
    need = lib.lsa_attend_si_workspace_size(ctypes.byref(one), 32, 4, 128, bud, 1)
    assert need >= 8192 * 32 * 4  # the gather's log-sum-exp per (row, head)
    assert lib.lsa_attend_si_launches(ctypes.byref(one), 32, 4, 128, bud, 1) == 2  # gather, dense runs
    assert lib.lsa_attend_si_launches(ctypes.byref(two), 32, 4, 128, bud, 1) == 0
