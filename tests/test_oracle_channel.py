"""Pins of the channel-selection oracle (oracle/channel_select.py) against
closed forms and brute force, not against the oracle's own formulas.

* The rotation: Sylvester Hadamard entries (-1)^popcount(r & i), the n = 1, 2,
  4 cases written out, and inner products preserved (what the estimate relies on).
* The sketch: rows whose rotation is ternary times a bf16 scale by
  construction come back exactly, so the estimated activation equals the
  exact one computed without any rotation.
* The score: router weight x down-column norm x |estimated activation|,
  checked by plain loops on a bank built so that every quantity is exact.
* The selection: brute-force ranking with ties.
* The layer: at a full budget it is the whole MoE layer (route + expert FFN,
  both pinned elsewhere); with no budget only the shared experts remain.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

from oracle import channel_select as C
from oracle import qmoe_oracle as Q


def _popcount(v: int) -> int:
    return bin(v).count("1")


def test_rht_small_cases_written_out():
    a, b = 0.75, -1.5
    assert np.allclose(C.rht([a], [-1.0]), [-a])
    r2 = 1.0 / math.sqrt(2.0)
    got = C.rht([a, b], [1.0, -1.0])
    assert np.allclose(got, [(a - b) * r2, (a + b) * r2], rtol=0, atol=1e-15)
    had4 = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], dtype=np.float64)
    v = np.array([0.5, -2.0, 3.0, 0.25])
    d = np.array([1.0, -1.0, -1.0, 1.0])
    assert np.allclose(C.rht(v, d), had4 @ (d * v) / 2.0, rtol=0, atol=1e-15)


@pytest.mark.parametrize("n", [8, 64, 512])
def test_rht_columns_are_sylvester_signs(n):
    # rht(e_i) with all signs +1 is column i of Had_n / sqrt(n): (-1)^popcount(r & i) / sqrt(n)
    for i in (0, 1, n // 2 - 1, n - 1):
        e = np.zeros(n)
        e[i] = 1.0
        want = np.array([(-1.0) ** _popcount(r & i) for r in range(n)]) / math.sqrt(n)
        assert np.allclose(C.rht(e, np.ones(n)), want, rtol=0, atol=1e-15)
    # a sign flip of input i flips that column
    d = np.ones(n)
    d[1] = -1.0
    e = np.zeros(n)
    e[1] = 1.0
    assert np.allclose(C.rht(e, d), -C.rht(e, np.ones(n)), rtol=0, atol=1e-15)


def test_rht_preserves_inner_products():
    rng = np.random.default_rng(3)
    n = 2048
    d = rng.choice([-1.0, 1.0], n)
    a, b = rng.standard_normal(n), rng.standard_normal(n)
    ra, rb = C.rht(a, d), C.rht(b, d)
    assert abs(ra @ rb - a @ b) < 1e-10 * (np.abs(a) @ np.abs(b))
    assert abs(np.linalg.norm(ra) - np.linalg.norm(a)) < 1e-12 * np.linalg.norm(a)


def _bf16_exact_scale(rng):
    # a positive value with at most 8 significant bits
    return float(rng.integers(128, 256)) * 2.0 ** int(rng.integers(-14, -6))


def _rotated_ternary_rows(rng, rows, n, signs, block=128, density=0.4):
    """Rows w whose rotation is s_b * t exactly (t ternary, at least one
    nonzero per block): w = d * (Had t s) / sqrt(n) by the explicit inverse."""
    t = np.where(rng.random((rows, n)) < density, rng.choice([-1, 1], (rows, n)), 0).astype(np.int8)
    t[:, ::block] = np.where(t[:, ::block] == 0, 1, t[:, ::block])   # no empty block
    s = np.array([[_bf16_exact_scale(rng) for _ in range(n // block)] for _ in range(rows)])
    r = t * np.repeat(s, block, axis=1)
    idx = np.arange(n)
    had = np.array([[(-1.0) ** _popcount(int(p & q)) for q in idx] for p in idx])
    w = (r @ had) / math.sqrt(n) * np.asarray(signs)[None, :]
    return w, t, s


def test_sketch_recovers_rows_ternary_after_rotation():
    rng = np.random.default_rng(5)
    n = 256
    d = rng.choice([-1.0, 1.0], n)
    w, t, s = _rotated_ternary_rows(rng, 6, n, d)
    tg, sg = C.sketch_rows(w, d, 128)
    assert np.array_equal(tg, t)
    assert np.array_equal(sg, s)


def test_estimated_activation_is_exact_for_exact_sketches():
    rng = np.random.default_rng(7)
    n = 256
    d = rng.choice([-1.0, 1.0], n)
    wg, _, _ = _rotated_ternary_rows(rng, 5, n, d)
    wu, _, _ = _rotated_ternary_rows(rng, 5, n, d)
    x = rng.standard_normal(n)
    sk = C.sketch_rows(wg, d) + C.sketch_rows(wu, d)
    got = C.estimated_activation(C.rht(x, d), sk)
    for j in range(5):
        g = math.fsum(wg[j, i] * x[i] for i in range(n))
        u = math.fsum(wu[j, i] * x[i] for i in range(n))
        want = g / (1.0 + math.exp(-g)) * u
        assert abs(got[j] - want) <= 1e-9 * max(1.0, abs(want))


def _exact_down_matrix(rng, H, I, bits, block):
    """W2 [H, I] whose column-wise block quantization is exact: integer codes
    times a power of two, each block holding the code -2^(bits-1)."""
    lo = -(1 << (bits - 1))
    c = rng.integers(lo, -lo, (H, I)).astype(np.float64)
    c[::block, :] = lo
    s = 2.0 ** rng.integers(-9, -5, (H // block, I)).astype(np.float64)
    return c * np.repeat(s, block, axis=0)


def test_down_columns_quantized_along_rows():
    rng = np.random.default_rng(9)
    H, I = 256, 6
    w2 = _exact_down_matrix(rng, H, I, 4, 64)
    codes, scales, w2_hat = C.quantize_down_columns(w2, 4, 64)
    assert codes.shape == (I, H) and scales.shape == (I, H // 64)
    assert np.array_equal(w2_hat, w2)


def test_scores_by_plain_loops():
    rng = np.random.default_rng(11)
    H, I, E, k, block = 128, 4, 3, 2, 64
    d = rng.choice([-1.0, 1.0], H)
    w1 = {}
    for e in range(E):
        g, _, _ = _rotated_ternary_rows(rng, I, H, d)
        u, _, _ = _rotated_ternary_rows(rng, I, H, d)
        m = np.empty((2 * I, H))
        m[0::2], m[1::2] = g, u
        w1[e] = m
    w2 = {e: _exact_down_matrix(rng, H, I, 4, block) for e in range(E)}
    bank = C.ChannelExpertBank(H, I, E, 0, block, 4, 4, lambda e: w1[e], lambda e: w2[e], d)
    T = 2
    x = rng.standard_normal((T, H))
    logits = np.array([[0.5, 2.0, -1.0], [1.0, 1.0, 0.25]], dtype=np.float32)  # token 1: a tie
    ids, w, scores = C.channel_scores(x, logits, k, bank)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        assert list(ids[t]) == order
        z = [math.exp(float(logits[t, e]) - float(logits[t, order[0]])) for e in order]
        for s, e in enumerate(order):
            ws = z[s] / sum(z)
            for j in range(I):
                g = math.fsum(w1[e][2 * j, i] * x[t, i] for i in range(H))
                u = math.fsum(w1[e][2 * j + 1, i] * x[t, i] for i in range(H))
                a = g / (1.0 + math.exp(-g)) * u
                dn = math.sqrt(math.fsum(w2[e][i, j] ** 2 for i in range(H)))
                want = ws * dn * abs(a)
                assert abs(scores[t, s * I + j] - want) <= 1e-9 * max(want, 1e-30)


def test_select_top_brute_force_with_ties():
    rng = np.random.default_rng(13)
    for n, n_keep in ((40, 7), (40, 0), (40, 40), (257, 100)):
        sc = rng.integers(0, 6, n).astype(np.float64) * 0.5   # many ties
        want = sorted(sorted(range(n), key=lambda i: (-sc[i], i))[:n_keep])
        assert list(C.select_top(sc, n_keep)) == want


def _random_bank(seed, H=256, I=32, E=4, n_shared=1, block=64, b1=2, b2=4):
    rng = np.random.default_rng(seed)
    mats1 = {e: Q.round_to_bf16(rng.standard_normal((2 * I, H)) * 0.05) for e in range(E + n_shared)}
    mats2 = {e: Q.round_to_bf16(rng.standard_normal((H, I)) * 0.05) for e in range(E + n_shared)}
    d = rng.choice([-1.0, 1.0], H)
    return C.ChannelExpertBank(H, I, E, n_shared, block, b1, b2, lambda e: mats1[e], lambda e: mats2[e], d), rng


def test_full_budget_is_the_moe_layer():
    bank, rng = _random_bank(17)
    T, k = 3, 2
    x = Q.round_to_bf16(rng.standard_normal((T, bank.H)))
    logits = rng.standard_normal((T, bank.E)).astype(np.float32)
    y, sel, _ = C.channel_forward(x, logits, k, bank, k * bank.I)
    assert np.array_equal(sel, np.tile(np.arange(k * bank.I, dtype=np.int32), (T, 1)))
    ids, w, _, _ = Q.route(logits, k)
    want = np.zeros_like(y)
    for t in range(T):
        for s in range(k):
            w1_hat, w2_hat, _, _ = bank.expert(int(ids[t, s]))
            want[t] += w[t, s] * Q.expert_ffn(x[t], w1_hat, w2_hat)[0]
        w1_hat, w2_hat, _, _ = bank.expert(bank.E)
        want[t] += Q.expert_ffn(x[t], w1_hat, w2_hat)[0]
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)


def test_no_budget_leaves_shared_experts_and_one_channel_is_the_argmax():
    bank, rng = _random_bank(19)
    T, k = 2, 2
    x = Q.round_to_bf16(rng.standard_normal((T, bank.H)))
    logits = rng.standard_normal((T, bank.E)).astype(np.float32)
    y0, sel0, scores = C.channel_forward(x, logits, k, bank, 0)
    assert sel0.shape == (T, 0)
    w1_hat, w2_hat, _, _ = bank.expert(bank.E)
    shared = np.stack([Q.expert_ffn(x[t], w1_hat, w2_hat)[0] for t in range(T)])
    assert np.allclose(y0, shared, rtol=1e-12, atol=1e-12)
    y1, sel1, _ = C.channel_forward(x, logits, k, bank, 1)
    ids, w, _, _ = Q.route(logits, k)
    for t in range(T):
        f = int(np.argmax(scores[t]))
        assert sel1[t, 0] == f
        s, j = divmod(f, bank.I)
        w1_hat, w2_hat, _, _ = bank.expert(int(ids[t, s]))
        g = math.fsum(w1_hat[2 * j, i] * x[t, i] for i in range(bank.H))
        u = math.fsum(w1_hat[2 * j + 1, i] * x[t, i] for i in range(bank.H))
        h = g / (1.0 + math.exp(-g)) * u
        assert np.allclose(y1[t] - shared[t], w[t, s] * h * w2_hat[:, j], rtol=1e-10, atol=1e-14)
