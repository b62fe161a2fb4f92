"""Pins for the oracle's routing, single linear, expert FFN and MoE layer.

Checked against exact rational brute force (fractions.Fraction), an integer
matmul, closed forms and invariants that hold for any correct implementation.
"""
from fractions import Fraction
from math import exp

import numpy as np
import pytest

from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import synth


def _bf16(shape, seed, std):
    return synth.bf16_bits_to_f32(synth.normal_bf16(seed, 77, 0, shape, std)).astype(np.float64)


# ---------------------------------------------------------------- routing

def test_route_brute_force_and_invariants():
    cfg = synth.V2LITE
    lg = synth.router_logits(cfg, 11, 37)
    k = cfg.k
    ids, w, perm, offsets = Q.route(lg, k)
    T, E = lg.shape
    for t in range(T):
        sel = list(ids[t])
        assert len(set(sel)) == k
        # every selected logit beats every unselected one (ties: lower index wins)
        for e in range(E):
            if e in sel:
                continue
            for s in sel:
                assert (lg[t, s] > lg[t, e]) or (lg[t, s] == lg[t, e] and s < e)
        # selection order = descending logit
        assert all(lg[t, sel[i]] >= lg[t, sel[i + 1]] for i in range(k - 1))
        # weights: softmax over the selected logits
        assert abs(w[t].sum() - 1) < 1e-12
        for i in range(k):
            for j in range(k):
                assert abs(w[t, i] / w[t, j] - exp(float(lg[t, sel[i]]) - float(lg[t, sel[j]]))) < 1e-9
    # perm is a permutation, sorted by expert, stable (increasing flat index within an expert)
    flat = ids.reshape(-1)
    assert sorted(perm.tolist()) == list(range(T * k))
    assert offsets[0] == 0 and offsets[-1] == T * k
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)


def test_route_ties_go_to_lower_index_and_top1_weight_one():
    lg = np.zeros((3, 8), dtype=np.float32)
    lg[1, [2, 5, 6]] = 1.0
    lg[2] = np.array([0, 3, 3, 1, 3, 0, 0, 3], dtype=np.float32)
    ids, w, _, _ = Q.route(lg, 3)
    assert ids[0].tolist() == [0, 1, 2]
    assert ids[1].tolist() == [2, 5, 6]
    assert ids[2].tolist() == [1, 2, 4]
    assert np.allclose(w[0], 1 / 3)
    ids1, w1, _, _ = Q.route(synth.router_logits(synth.TERNARY, 3, 5), 1)
    assert np.all(w1 == 1.0)


# ---------------------------------------------------------------- single linear

@pytest.mark.parametrize("bits,N,M", [(2, 1, 1), (2, 4, 3), (4, 3, 2), (4, 1, 1)])
def test_linear_exact_rational_brute_force(bits, N, M):
    """K = 64, N = 1..4: the oracle's float64 result equals the exact rational
    sum of c*s*x to within float64 rounding."""
    w = _bf16((N, 64), bits * 10 + N, 0.02)
    x = _bf16((M, 64), 100 + M, 1.0)
    codes, s = Q.quantize_sym(w, bits, 64)
    y = Q.linear(x, Q.dequant(codes, s, 64))
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(int(codes[n, k])) * Fraction(float(s[n, 0])) * Fraction(float(x[m, k]))
                        for k in range(64))
            assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 80)


@pytest.mark.parametrize("bits,N,M", [(2, 1, 1), (2, 4, 3), (4, 3, 2)])
def test_linear_affine_exact_rational_brute_force(bits, N, M):
    """K = 64, affine codes: the oracle's float64 result equals the exact
    rational sum of (s*u + z)*x to within float64 rounding."""
    w = _bf16((N, 64), bits * 10 + N + 5, 0.02)
    x = _bf16((M, 64), 200 + M, 1.0)
    codes, s, z = Q.quantize_affine(w, bits, 64)
    y = Q.linear(x, Q.dequant_affine(codes, s, z, 64))
    for m in range(M):
        for n in range(N):
            exact = sum((Fraction(int(codes[n, k])) * Fraction(float(s[n, 0])) + Fraction(float(z[n, 0])))
                        * Fraction(float(x[m, k])) for k in range(64))
            assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 80)


def test_linear_reduces_to_integer_matmul_with_unit_scale():
    g = np.random.default_rng(4)
    c = g.integers(-8, 8, size=(6, 256))
    c[:, ::64] = -8                       # max |w| = 8 in every block -> s = 1
    w = c.astype(np.float64)
    codes, s = Q.quantize_sym(w, 4, 64)
    assert np.all(s == 1.0)
    x = g.integers(-50, 50, size=(5, 256))
    y = Q.linear(x.astype(np.float64), Q.dequant(codes, s, 64))
    assert np.array_equal(y.astype(np.int64), x.astype(np.int64) @ c.T.astype(np.int64))


# ---------------------------------------------------------------- expert FFN

def test_silu_closed_form():
    assert Q.silu(0.0) == 0.0
    assert abs(Q.silu(1.0) - 1 / (1 + exp(-1))) < 1e-16
    assert abs(Q.silu(-40.0)) < 1e-15
    assert abs(Q.silu(40.0) - 40.0) < 1e-12


def test_expert_ffn_hand_example_interleaved_gate_up():
    # H = 2, I = 1: row 0 is gate, row 1 is up
    x = np.array([[1.0, 2.0]])
    w1 = np.array([[1.0, 0.0], [0.0, 1.0]])
    w2 = np.array([[1.0], [3.0]])
    h = (1 / (1 + exp(-1))) * 2.0
    assert np.allclose(Q.expert_ffn(x, w1, w2), [[h, 3 * h]], rtol=0, atol=1e-15)
    # biases: b1 shifts gate/up before SwiGLU, b2 is added after FC2
    b1 = np.array([-1.0, 0.5])           # gate 0 -> silu 0
    b2 = np.array([0.25, -0.5])
    assert np.allclose(Q.expert_ffn(x, w1, w2, b1, b2), [[0.25, -0.5]], rtol=0, atol=1e-15)
    # swapping the interleave (gate <-> up) changes the result: order matters
    assert not np.allclose(Q.expert_ffn(x, w1[::-1], w2), Q.expert_ffn(x, w1, w2))


def _bank(cfg, seed, zero_fc1=False):
    def q(fmt, wbits):
        w = synth.bf16_bits_to_f32(wbits).astype(np.float64)
        if fmt == "ternary":
            return Q.quantize_ternary(w, cfg.block)
        return Q.quantize_sym(w, 2 if fmt == "int2" else 4, cfg.block)

    def fc1(e):
        c, s = q(cfg.fc1_fmt, synth.expert_fc1(cfg, seed, e))
        return (np.zeros_like(c) if zero_fc1 else c), s

    b1 = (lambda e: synth.bf16_bits_to_f32(synth.expert_b1(cfg, seed, e)).astype(np.float64)) if cfg.bias else None
    b2 = (lambda e: synth.bf16_bits_to_f32(synth.expert_b2(cfg, seed, e)).astype(np.float64)) if cfg.bias else None
    return Q.QuantExpertBank(cfg.H, cfg.I, cfg.E, cfg.n_shared, cfg.block, fc1,
                             lambda e: q(cfg.fc2_fmt, synth.expert_fc2(cfg, seed, e)), b1, b2, cache=80)


def test_moe_batched_equals_single_token_calls():
    cfg = synth.TINY
    bank = _bank(cfg, 1)
    T = 6
    x = synth.bf16_bits_to_f32(synth.tokens(cfg.H, 1, T)).astype(np.float64)
    lg = synth.router_logits(cfg, 1, T)
    y = Q.moe_forward(x, lg, cfg.k, bank)
    for t in range(T):
        assert np.allclose(y[t], Q.moe_token(x[t], lg[t], cfg.k, bank), rtol=1e-12, atol=1e-14)


def test_moe_shared_experts_and_top1_reduce_to_single_ffn():
    import dataclasses
    cfg = dataclasses.replace(synth.V2LITE, H=128, I=64, E=8, k=1)
    bank = _bank(cfg, 2)
    x = synth.bf16_bits_to_f32(synth.tokens(cfg.H, 2, 3)).astype(np.float64)
    lg = synth.router_logits(cfg, 2, 3)
    y = Q.moe_forward(x, lg, 1, bank)
    ids, w, _, _ = Q.route(lg, 1)
    for t in range(3):
        ref = np.zeros(cfg.H)
        for e in [int(ids[t, 0]), cfg.E, cfg.E + 1]:
            w1, w2, b1, b2 = bank.weights(e)
            ref += Q.expert_ffn(x[t:t + 1], w1, w2, b1, b2)[0]
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_moe_all_zero_gate_up_codes_give_fc2_bias_only():
    import dataclasses
    cfg = dataclasses.replace(synth.PREFILL, H=128, I=64, E=8, k=2)
    bank = _bank(cfg, 3, zero_fc1=True)
    x = synth.bf16_bits_to_f32(synth.tokens(cfg.H, 3, 4)).astype(np.float64)
    lg = synth.router_logits(cfg, 3, 4)
    y = Q.moe_forward(x, lg, cfg.k, bank)
    ids, w, _, _ = Q.route(lg, cfg.k)
    for t in range(4):
        # a = b1 only -> h = silu(b1_gate) * b1_up; o = W2 h + b2
        ref = np.zeros(cfg.H)
        for s in range(cfg.k):
            w1, w2, b1, b2 = bank.weights(int(ids[t, s]))
            h = Q.silu(b1[0::2]) * b1[1::2]
            ref += w[t, s] * (w2 @ h + b2)
        assert np.allclose(y[t], ref, rtol=1e-12, atol=1e-15)
    # and without biases the output is exactly zero
    cfg0 = dataclasses.replace(cfg, bias=False)
    bank0 = _bank(cfg0, 3, zero_fc1=True)
    assert not np.any(Q.moe_forward(x, lg, cfg.k, bank0))


def test_moe_router_weights_sum_to_one_scaling():
    """If every routed expert has the same weights, the routed part equals one
    FFN (the renormalised weights sum to 1)."""
    import dataclasses
    cfg = dataclasses.replace(synth.TINY, H=128, I=64)
    base = _bank(cfg, 4)
    same = Q.QuantExpertBank(cfg.H, cfg.I, cfg.E, 0, cfg.block, lambda e: base._fc1_q(0),
                             lambda e: base._fc2_q(0))
    x = synth.bf16_bits_to_f32(synth.tokens(cfg.H, 4, 5)).astype(np.float64)
    lg = synth.router_logits(cfg, 4, 5)
    w1, w2, _, _ = same.weights(0)
    assert np.allclose(Q.moe_forward(x, lg, cfg.k, same), Q.expert_ffn(x, w1, w2), rtol=1e-12, atol=1e-15)


def test_tolerance_metrics():
    ref = np.array([1.0, -1.0, 2.0, 0.0])
    assert Q.rel_l2(ref, ref) == 0
    assert abs(Q.rel_l2(ref * 1.01, ref) - 0.01) < 1e-12
    assert abs(Q.max_err_over_rms(ref + np.array([0, 0, 0.1, 0]), ref) - 0.1 / np.sqrt(1.5)) < 1e-12
