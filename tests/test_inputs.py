"""The seeded input generator: SplitMix64 on torch int64 equals the published
definition evaluated on Python integers, and the draws have the requested
ranges, shapes and layouts."""
import torch

from long_context_sparse_lsa_b200 import inputs as gen
from long_context_sparse_lsa_b200 import workloads as wls

M64 = (1 << 64) - 1


def _splitmix_reference(x):
    # Steele, Lea & Flood (2014): z += golden; z = (z ^ z>>30) * c1; z = (z ^ z>>27) * c2; z ^ z>>31
    z = (x + 0x9E3779B97F4A7C15) & M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def test_mix64_matches_definition():
    xs = [0, 1, 2, 12345, (1 << 63) - 1, 1 << 63, M64, 0xDEADBEEFCAFEBABE]
    t = torch.tensor([x - (1 << 64) if x >= (1 << 63) else x for x in xs], dtype=torch.int64)
    got = [int(v) & M64 for v in gen.mix64(t).tolist()]
    assert got == [_splitmix_reference(x) for x in xs]
    # first output of SplitMix64 seeded with 0 (the generator's own test value)
    assert _splitmix_reference(0) == 0xE220A8397B1DCDAF


def test_ranges_and_determinism():
    a = gen.uniform_int8((1000, 7), -16, 15, 3, gen.STREAM_K_IDX, "cpu")
    b = gen.uniform_int8((1000, 7), -16, 15, 3, gen.STREAM_K_IDX, "cpu")
    assert torch.equal(a, b)
    assert int(a.min()) == -16 and int(a.max()) == 15
    w = gen.uniform_weights((500,), 8, 1, gen.STREAM_W, "cpu")
    assert int(w.min()) == 1 and int(w.max()) == 8
    z = gen.normal_bf16((20000,), 0, gen.STREAM_Q, "cpu").float()
    assert abs(float(z.mean())) < 0.03 and abs(float(z.std()) - 1.0) < 0.03


def test_chunked_draw_equals_slice():
    old = gen.CHUNK
    try:
        gen.CHUNK = 1000
        a = gen.uniform_int8((5000,), -8, 7, 0, 2, "cpu")
    finally:
        gen.CHUNK = old
    b = gen.uniform_int8((5000,), -8, 7, 0, 2, "cpu")
    assert torch.equal(a, b)


def test_ragged_lengths():
    wl = wls.ragged()
    assert wl.n_seq == 64
    assert all(8192 <= L <= (1 << 20) for L in wl.lens)
    assert sum(wl.lens) <= 12 << 20


def test_layouts():
    wl = wls.small(wls.PREFILL, lens=(100,), prefill_new=10)
    off, lens, boff, q_seq, q_len, nb = wls.layout(wl, "cpu", hi_block=16)
    assert q_len.tolist() == list(range(91, 101))
    assert q_seq.tolist() == [0] * 10
    wl2 = wls.small(wls.BATCH128K, lens=(10, 33, 64), hi_block=16)
    off, lens, boff, q_seq, q_len, nb = wls.layout(wl2, "cpu")
    assert off.tolist() == [0, 10, 43] and boff.tolist() == [0, 1, 4] and nb == 8
