"""Pins for the oracle's bf16 rounding, quantizers, dequant and code packing.

Each check compares the oracle with something other than itself: IEEE
bit-level rounding of float32, closed forms, an exhaustive search over the
code range, the bit layout written out by hand, or sizes printed on the pages.
"""
import json
import os

import numpy as np
import pytest

from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- bf16 rounding

def _bf16_rne_bits_of_f32(a):
    """Independent reference: RNE on the float32 bit pattern."""
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def test_round_to_bf16_matches_bit_rounding_of_float32():
    g = np.random.default_rng(1)
    v = np.concatenate([
        g.standard_normal(20000) * 0.02,
        g.standard_normal(2000) * 1e30,
        g.standard_normal(2000) * 1e-36,          # near / below the normal range
        np.ldexp(g.integers(1, 1 << 16, 2000).astype(np.float64), -149),  # float32 subnormals
    ]).astype(np.float32).astype(np.float64)
    got = Q.round_to_bf16(v)
    ref = _bf16_rne_bits_of_f32(v)
    assert np.array_equal(got, ref)


def test_round_to_bf16_ties_and_subnormals():
    # ulp of bf16 at 1.0 is 2^-7: 1 + 2^-8 ties to 1 (even), 1 + 3*2^-8 ties to 1 + 2^-6.
    assert Q.round_to_bf16(1 + 2.0 ** -8) == 1.0
    assert Q.round_to_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    # subnormal quantum 2^-133
    assert Q.round_to_bf16(2.0 ** -133) == 2.0 ** -133
    assert Q.round_to_bf16(2.0 ** -134) == 0.0
    assert Q.round_to_bf16(3 * 2.0 ** -134) == 2.0 ** -132
    assert Q.round_to_bf16(-0.0) == 0.0
    assert np.isinf(Q.round_to_bf16(3.4e38))


# ---------------------------------------------------------------- symmetric quantizer

@pytest.mark.parametrize("bits", [2, 4])
def test_exact_multiples_quantize_to_their_codes(bits):
    """w = c * 2^-m with the block's max |w| = 2^(bits-1) * 2^-m gives s = 2^-m
    and codes exactly c."""
    qmin, qmax = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    g = np.random.default_rng(bits)
    m = 9
    c = g.integers(qmin, qmax + 1, size=(5, 128))
    c[:, 0] = qmin           # force the block max |w| in both 64-blocks
    c[:, 64] = qmin
    w = c * 2.0 ** -m
    codes, s = Q.quantize_sym(w, bits, 64)
    assert np.all(s == 2.0 ** -m)
    assert np.array_equal(codes, c)


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_minimise_error_over_the_code_range(bits):
    """Brute force: each code is a nearest point of {c*s : qmin <= c <= qmax}."""
    qmin, qmax = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    w = synth.bf16_bits_to_f32(synth.normal_bf16(3, 99, bits, (16, 256), 0.02)).astype(np.float64)
    codes, s = Q.quantize_sym(w, bits, 64)
    sfull = np.repeat(s, 64, axis=1)
    cand = np.arange(qmin, qmax + 1, dtype=np.float64)
    err = np.abs(w[..., None] - cand[None, None, :] * sfull[..., None])
    best = err.min(axis=2)
    mine = np.abs(w - codes * sfull)
    assert np.all(mine <= best + 1e-18)
    # the scale is the block max |w| / 2^(bits-1) (exact: a power-of-two division of a bf16)
    amax = np.abs(w.reshape(16, 4, 64)).max(axis=2)
    assert np.array_equal(s, amax / 2 ** (bits - 1))


def test_ties_go_to_even_and_extremes_clip():
    s = 2.0 ** -6
    # INT4 block: max |w| = 8 s gives scale s; 2.5 s -> 2, 3.5 s -> 4, -0.5 s -> 0, 8 s -> clipped to 7
    w = np.zeros((1, 64))
    w[0, :5] = np.array([-8, 2.5, 3.5, -0.5, 8]) * s
    codes, sc = Q.quantize_sym(w, 4, 64)
    assert sc[0, 0] == s
    assert list(codes[0, :5]) == [-8, 2, 4, 0, 7]
    # INT2: 0.5 s -> 0, 1.5 s -> 2 -> clipped to 1, -1.5 s -> -2
    w2 = np.zeros((1, 64))
    w2[0, :4] = np.array([-2, 0.5, 1.5, -1.5]) * s
    codes2, sc2 = Q.quantize_sym(w2, 2, 64)
    assert sc2[0, 0] == s
    assert list(codes2[0, :4]) == [-2, 0, 1, -2]


def test_zero_block_and_single_nonzero():
    w = np.zeros((2, 64))
    w[1, 7] = -0.375
    codes, s = Q.quantize_sym(w, 2, 64)
    assert s[0, 0] == 0 and not codes[0].any()
    assert s[1, 0] == 0.1875 and codes[1, 7] == -2 and np.count_nonzero(codes[1]) == 1
    w[1, 7] = 0.375          # positive extreme clips to qmax
    codes, s = Q.quantize_sym(w, 4, 64)
    assert s[1, 0] == 0.375 / 8 and codes[1, 7] == 7


def test_dequant_is_code_times_scale_and_bf16_operand():
    codes = np.array([[-2, -1, 0, 1] * 16])
    s = np.array([[0.01171875]])                     # bf16-representable
    wh = Q.dequant(codes, s, 64)
    assert np.array_equal(wh[0, :4], np.array([-2, -1, 0, 1]) * 0.01171875)
    # 7 * s with an 8-bit s has 11 significant bits: the bf16 operand rounds it
    s2 = np.array([[1 + 2.0 ** -7]])                 # 8 significant bits
    op = Q.dequant_bf16_operand(np.full((1, 64), 7), s2, 64)
    assert op[0, 0] == 7 + 2.0 ** -4                 # 7 + 7*2^-7 = 7.0546875 -> 7.0625 in bf16


# ---------------------------------------------------------------- affine quantizer (scale and zero point)

@pytest.mark.parametrize("bits", [2, 4])
def test_affine_exact_grid_round_trips(bits):
    """w = z0 + s0 * u0 with both code extremes in every block gives z = z0,
    s = s0 and codes exactly u0 (all values exact in bf16)."""
    umax = (1 << bits) - 1
    g = np.random.default_rng(10 + bits)
    s0, z0 = 2.0 ** -6, -0.25
    u0 = g.integers(0, umax + 1, size=(4, 128))
    u0[:, 0] = 0
    u0[:, 1] = umax
    u0[:, 64] = umax
    u0[:, 65] = 0
    w = z0 + s0 * u0
    assert np.array_equal(Q.round_to_bf16(w), w)
    codes, s, z = Q.quantize_affine(w, bits, 64)
    assert np.all(s == s0) and np.all(z == z0)
    assert np.array_equal(codes, u0)
    assert np.array_equal(Q.dequant_affine(codes, s, z, 64), w)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("block", [64, 128])
def test_affine_codes_minimise_error_over_the_code_range(bits, block):
    """Brute force: each code is a nearest point of {s*u + z : 0 <= u < 2^bits}."""
    umax = (1 << bits) - 1
    w = synth.bf16_bits_to_f32(synth.normal_bf16(5, 98, bits, (16, 256), 0.02)).astype(np.float64)
    codes, s, z = Q.quantize_affine(w, bits, block)
    sf, zf = np.repeat(s, block, axis=1), np.repeat(z, block, axis=1)
    cand = np.arange(0, umax + 1, dtype=np.float64)
    err = np.abs(w[..., None] - (cand[None, None, :] * sf[..., None] + zf[..., None]))
    mine = np.abs(w - (codes * sf + zf))
    assert np.all(mine <= err.min(axis=2) + 1e-18)
    wb = w.reshape(16, 256 // block, block)
    assert np.array_equal(z, Q.round_to_bf16(wb.min(axis=2)))
    assert np.array_equal(s, Q.round_to_bf16((wb.max(axis=2) - wb.min(axis=2)) / umax))


def test_affine_constant_block_ties_and_clip():
    w = np.full((2, 64), 0.375)
    codes, s, z = Q.quantize_affine(w, 4, 64)
    assert np.all(s == 0) and np.all(z == 0.375) and not codes.any()
    assert np.array_equal(Q.dequant_affine(codes, s, z, 64), w)
    # INT2, min 0, max 3/64: s = 1/64; 0.5 s -> 0 and 1.5 s -> 2 (ties to even), 2.5 s -> 2
    w2 = np.zeros((1, 64))
    w2[0, :4] = np.array([0.5, 1.5, 2.5, 3.0]) / 64
    codes2, s2, z2 = Q.quantize_affine(w2, 2, 64)
    assert s2[0, 0] == 1 / 64 and z2[0, 0] == 0
    assert list(codes2[0, :4]) == [0, 2, 2, 3]


def test_affine_dequant_and_bf16_operand():
    codes = np.array([[0, 1, 2, 3] * 16], dtype=np.uint8)
    s, z = np.array([[0.01171875]]), np.array([[-0.0234375]])
    wh = Q.dequant_affine(codes, s, z, 64)
    assert np.array_equal(wh[0, :4], np.array([0, 1, 2, 3]) * 0.01171875 - 0.0234375)
    # 15 * (1 + 2^-7) + 2^-9 needs more than 8 significant bits: the operand rounds once
    op = Q.dequant_affine_bf16_operand(np.full((1, 64), 15), np.array([[1 + 2.0 ** -7]]), np.array([[2.0 ** -9]]), 64)
    assert op[0, 0] == Q.round_to_bf16(15 * (1 + 2.0 ** -7) + 2.0 ** -9) == 15.125


# ---------------------------------------------------------------- ternary quantizer

def test_ternary_closed_form():
    big, small = 5 / 128, 2.0 ** -10
    w = np.where(np.arange(64) % 2 == 0, big, small) * np.where(np.arange(64) % 3 == 0, -1, 1)
    t, s = Q.quantize_ternary(w[None, :], 64)
    # delta = 0.7 * (32*big + 32*small)/64, far above small and below big
    assert np.array_equal(t[0], (np.arange(64) % 2 == 0) * np.sign(w))
    assert s[0, 0] == big


def test_ternary_threshold_is_strict_and_empty_block_scale_zero():
    w = np.full((1, 64), 0.0)
    t, s = Q.quantize_ternary(w, 64)
    assert s[0, 0] == 0 and not t.any()
    # all |w| equal: delta = 0.7 |w| < |w| -> every weight kept, s = |w|
    w = np.full((1, 64), -0.25)
    t, s = Q.quantize_ternary(w, 64)
    assert np.all(t == -1) and s[0, 0] == 0.25


def test_ternary_zero_fraction_on_gaussian():
    """About 42% zeros for N(0, 0.02): P(|z| <= 0.7 E|z|) = erf(0.7/sqrt(pi))."""
    w = synth.bf16_bits_to_f32(synth.normal_bf16(5, 98, 0, (256, 2048), 0.02)).astype(np.float64)
    t, _ = Q.quantize_ternary(w, 64)
    from math import erf, pi, sqrt
    expect = erf(0.7 / sqrt(pi))
    frac = float(np.mean(t == 0))
    assert abs(frac - expect) < 0.02, (frac, expect)


# ---------------------------------------------------------------- packing

@pytest.mark.parametrize("bits", [2, 4])
def test_int_pack_bit_layout_every_value_every_position(bits):
    per = 32 // bits
    qmin = -(1 << (bits - 1))
    vals = np.arange(qmin, -qmin)
    for pos in range(per):
        for v in vals:
            c = np.zeros((1, per), dtype=np.int8)
            c[0, pos] = v
            word = int(Q.pack_int_codes(c, bits)[0, 0])
            assert (word >> (bits * pos)) & ((1 << bits) - 1) == v - qmin
            others = word & ~(((1 << bits) - 1) << (bits * pos))
            # every other field holds the biased code of 0
            assert all(((others >> (bits * i)) & ((1 << bits) - 1)) == -qmin for i in range(per) if i != pos)
    g = np.random.default_rng(7)
    c = g.integers(qmin, -qmin, size=(9, 256)).astype(np.int8)
    assert np.array_equal(Q.unpack_int_codes(Q.pack_int_codes(c, bits), bits), c)


def test_trit_pack_all_243_bytes_round_trip_and_examples():
    digits = np.array(np.meshgrid(*[range(3)] * 5, indexing="ij")).reshape(5, -1).T  # 243 x 5
    for d in digits:
        t = np.zeros((1, 64), dtype=np.int8)
        t[0, 60:64] = d[:4] - 1     # last byte of the block: 4 trits + padding
        t[0, 0:5] = d - 1           # first byte: 5 trits
        b = Q.pack_trits(t)
        assert int(b[0, 0]) == int(sum(d[i] * 3 ** i for i in range(5)))
        assert int(b[0, 12]) == int(sum(d[i] * 3 ** i for i in range(4)) + 1 * 81)
        assert np.array_equal(Q.unpack_trits(b, 64), t)
    t = np.zeros((1, 64), dtype=np.int8)
    t[0, :5] = [1, 0, -1, 0, 1]
    assert int(Q.pack_trits(t)[0, 0]) == 2 + 1 * 3 + 0 * 9 + 1 * 27 + 2 * 81
    t[0, :5] = -1
    assert int(Q.pack_trits(t)[0, 0]) == 0
    t[0, :5] = 1
    assert int(Q.pack_trits(t)[0, 0]) == 242


def test_format_sizes_against_the_pages():
    gold = json.load(open(os.path.join(GOLDEN, "format_sizes.json")))
    g = gold["ternary_block_bytes"]
    t = np.zeros((1, g["weights"]), dtype=np.int8)
    codes_bytes = Q.pack_trits(t).nbytes
    scale_bytes = 2 * (g["weights"] // 64)
    assert g["bf16_bytes"] == 2 * g["weights"]
    assert abs(codes_bytes + scale_bytes - g["packed_bytes_about"]) <= g["tolerance_bytes"]
    cb = gold["ternary_code_bits_per_weight"]
    assert abs(8 * Q.TERNARY_BYTES_PER_BLOCK64 / 64 - cb["about"]) <= cb["tolerance"]
    a = gold["affine_2bit_g128_effective_bits"]
    assert 2 + (16 + 16) / 128 == a["value"]
    for bits in (2, 4):
        c = np.zeros((1, 128), dtype=np.int8)
        w = Q.pack_int_codes(c, bits)
        assert w.nbytes * 8 / 128 == bits
