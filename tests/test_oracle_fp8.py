"""Pins of the oracle's FP8 KV-cache attention (CPU).

The E4M3 decode is checked against torch's independent float8_e4m3fn type on
every code and against values fixed by the format's definition; the FP8
attention is checked against the already-pinned bf16 attention on the same
values (every E4M3 value times a power of two is a bf16 exactly), and against
closed forms of its two scales.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def _codes_to_bf16_bits(codes: np.ndarray, scale: float) -> np.ndarray:
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32) * scale
    bits = vals.to(torch.bfloat16)
    assert torch.equal(bits.to(torch.float32), vals)  # exact in bf16
    return bits.view(torch.int16).numpy().view(np.uint16)


def test_e4m3_decode_matches_torch_on_every_code():
    orc = oracle.get()
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_value(c) for c in codes])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(got[~nan], want[~nan])


def test_e4m3_closed_forms():
    orc = oracle.get()
    assert orc.e4m3_value(0x00) == 0.0
    assert orc.e4m3_value(0x38) == 1.0          # exponent 7 = bias
    assert orc.e4m3_value(0xB8) == -1.0
    assert orc.e4m3_value(0x7E) == 448.0        # largest finite: 2^8 * 1.75
    assert orc.e4m3_value(0x08) == 2.0 ** -6    # smallest normal
    assert orc.e4m3_value(0x01) == 2.0 ** -9    # smallest subnormal
    assert orc.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert np.isnan(orc.e4m3_value(0x7F))


def _case(seed, L=40, H_q=8, H_kv=2, d=128):
    rng = np.random.default_rng(seed)
    q = torch.from_numpy(rng.standard_normal((H_q, d)).astype(np.float32)).to(torch.bfloat16)
    q = q.view(torch.int16).numpy().view(np.uint16)
    k = torch.from_numpy(rng.standard_normal((L, H_kv, d)).astype(np.float32)).to(torch.float8_e4m3fn)
    v = torch.from_numpy(rng.standard_normal((L, H_kv, d)).astype(np.float32)).to(torch.float8_e4m3fn)
    s = np.array([0, 3, 4, -1, 17, 18, 19, 39, -1, -1], np.int32)
    return q, k.view(torch.uint8).numpy(), v.view(torch.uint8).numpy(), s


def test_fp8_attention_equals_bf16_attention_on_the_same_values():
    orc = oracle.get()
    q, k8, v8, s = _case(1)
    for ks, vs in ((1.0, 1.0), (0.5, 2.0), (0.125, 0.25)):
        got = orc.attend_query_fp8(q, k8, v8, ks, vs, s)
        want = orc.attend_query(q, _codes_to_bf16_bits(k8, ks), _codes_to_bf16_bits(v8, vs), s)
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_fp8_attention_scales():
    orc = oracle.get()
    q, k8, v8, s = _case(2)
    base = orc.attend_query_fp8(q, k8, v8, 0.7, 1.0, s)
    # the output is linear in v_scale
    np.testing.assert_allclose(orc.attend_query_fp8(q, k8, v8, 0.7, 3.0, s), 3.0 * base, rtol=1e-13, atol=1e-13)
    # k_scale = 0: every selected row gets the same weight, the output is their V mean
    flat = orc.attend_query_fp8(q, k8, v8, 0.0, 1.0, s)
    vals = torch.from_numpy(v8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    rows = s[s >= 0]
    for h in range(q.shape[0]):
        kvh = h * k8.shape[1] // q.shape[0]
        np.testing.assert_allclose(flat[h], vals[rows, kvh].mean(axis=0), rtol=1e-13, atol=1e-13)
    # an empty set gives zeros
    assert not orc.attend_query_fp8(q, k8, v8, 1.0, 1.0, np.full(6, -1, np.int32)).any()
