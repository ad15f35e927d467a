"""Pins for the oracle's pack / unpack / quantise (bit for bit)."""
from fractions import Fraction
import itertools

import numpy as np
import pytest

from golden_io import rows


@pytest.mark.parametrize("bits", [4, 2, 8])
def test_every_byte_round_trips(orc, bits):
    per = 8 // bits
    allb = np.arange(256, dtype=np.uint8).reshape(256, 1)
    q = orc.unpack(allb, per, bits)
    assert np.array_equal(orc.pack(q, bits), allb)


@pytest.mark.parametrize("bits", [4, 2])
def test_every_code_tuple_round_trips(orc, bits):
    per = 8 // bits
    lo, hi = {4: (-8, 7), 2: (-2, 1)}[bits]
    tuples = np.array(list(itertools.product(range(lo, hi + 1), repeat=per)), np.int32)
    packed = orc.pack(tuples, bits)
    assert packed.shape == (len(tuples), 1)
    assert len(set(packed[:, 0].tolist())) == 256  # a bijection onto bytes
    assert np.array_equal(orc.unpack(packed, per, bits), tuples)


def test_int8_codes_round_trip(orc):
    q = np.arange(-128, 128, dtype=np.int32).reshape(4, 64)
    assert np.array_equal(orc.unpack(orc.pack(q, 8), 64, 8), q)


def test_pack_golden_layout(orc):
    for bits, codes, hexbytes in rows("pack_layout.txt"):
        bits = int(bits)
        q = np.array([[int(c) for c in codes.split()]], np.int32)
        want = np.array([[int(h, 16) for h in hexbytes.split()]], np.uint8)
        got = orc.pack(q, bits)
        assert np.array_equal(got, want), (bits, codes)
        assert np.array_equal(orc.unpack(want, q.shape[1], bits), q)


def test_out_of_range_code_rejected(orc):
    with pytest.raises(orc.OracleError):
        orc.pack(np.array([[8, 0]], np.int32), 4)
    with pytest.raises(orc.OracleError):
        orc.pack(np.array([[2, 0, 0, 0]], np.int32), 2)


def test_quantize_golden_rows(orc):
    for bits, vals, scale, codes in rows("quantize_rows.txt"):
        bits = int(bits)
        w = np.array([[float(v) for v in vals.split()]], np.float32)
        q, s = orc.quantize_rows(w, bits)
        assert s[0] == np.float32(float(scale)), (bits, vals)
        got = orc.unpack(q, w.shape[1], bits)[0].tolist()
        assert got == [int(c) for c in codes.split()], (bits, vals, got)


def _round_half_away_exact(v: np.float32) -> int:
    f = Fraction(float(v))
    n = int(abs(f) + Fraction(1, 2))  # floor(|v| + 1/2) in exact arithmetic
    return n if f >= 0 else -n


@pytest.mark.parametrize("bits", [4, 8, 2])
def test_quantize_random_rows_invariants(orc, bits):
    rng = np.random.default_rng(1234 + bits)
    R, C = 64, 96
    w = (rng.standard_normal((R, C)) * 0.02).astype(np.float32)
    w[3] = 0.0
    w[5, :] = np.float32(0.013)  # constant row
    q, s = orc.quantize_rows(w, bits)
    codes = orc.unpack(q, C, bits)
    qmax_div, lo, hi = {4: (7, -8, 7), 8: (127, -128, 127), 2: (1.5, -2, 1)}[bits]
    for r in range(R):
        m = np.max(np.abs(w[r]))
        if m == 0:
            assert s[r] == 0 and np.all(codes[r] == 0)
            continue
        assert s[r] == np.float32(m) / np.float32(qmax_div)
        for j in range(C):
            v = w[r, j] / s[r]  # fp32 IEEE division, as the rule states
            want = min(max(_round_half_away_exact(v), lo), hi)
            assert codes[r, j] == want
        err = np.abs(w[r].astype(np.float64) - codes[r] * np.float64(s[r]))
        assert np.all(err <= 0.5 * np.float64(s[r]) * (1 + 1e-6))
        if bits in (4, 8):
            assert np.max(np.abs(codes[r])) == int(qmax_div)  # the max element maps to +-Qmax
            assert codes[r].min() > lo  # symmetric rule never reaches the negative end
        if bits == 2:
            continue  # the int2 grid is not symmetric, so re-quantising may move codes
        # re-quantising the dequantised row gives the same codes
        wd = (codes[r] * np.float64(s[r])).astype(np.float32)[None, :]
        q2, _ = orc.quantize_rows(wd, bits)
        assert np.array_equal(orc.unpack(q2, C, bits)[0], codes[r])


def test_quantize_rejects_bad_shapes(orc):
    with pytest.raises(orc.OracleError):
        orc.quantize_rows(np.zeros((2, 3), np.float32), 4)
    with pytest.raises(orc.OracleError):
        orc.quantize_rows(np.zeros((2, 6), np.float32), 2)
    with pytest.raises(orc.OracleError):
        orc.quantize_rows(np.zeros((2, 8), np.float32), 3)


def test_dequant_is_code_times_scale(orc):
    q = np.array([[-8, -1, 0, 7]], np.int32)
    packed = orc.pack(q, 4)
    out = orc.dequant_rows(packed, np.array([0.25], np.float32), 4, 4)
    assert out.tolist() == [[-2.0, -0.25, 0.0, 1.75]]


def test_bf16_rounding(orc):
    # nearest bf16, ties to even (bf16 keeps 8 significant bits)
    cases = {1.0: 0x3F80, 1.0 + 2 ** -8: 0x3F80, 1.0 + 3 * 2 ** -8: 0x3F82,
             1.0 + 2 ** -8 + 2 ** -30: 0x3F81, -2.0: 0xC000, 0.0: 0x0000}
    for v, bits in cases.items():
        assert int(orc.double_to_bf16_bits(np.array([v]))[0]) == bits, v
    import torch
    rng = np.random.default_rng(7)
    a = (rng.standard_normal(4096) * 3).astype(np.float32)
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16_bits(a), want)
