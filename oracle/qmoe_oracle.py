"""CPU fp64 oracle for the weight-only low-bit quantized MoE expert matmul.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may call it.  It shares no code with the CUDA library.

It computes the plain definition of what the fast path computes, in float64:
quantize bf16 weights into symmetric block codes + bf16 scales, dequantize,
route tokens top-k, run each expert's FC1 (interleaved gate/up) -> SwiGLU ->
FC2 and combine with the router weights.  Sources, by page and section:

* onnxruntime PR "Enable SM80+ FP16/BF16 mixed INT2/INT4 QMoE prefill by
  default", Description and Current Scope: INT2 FC1 + INT4 FC2, symmetric
  quantization with no zero points, block 64, interleaved fused SwiGLU,
  routing + expert maps + row expansion by expert, expert bias, FC2 bias in the
  top-k weighted finalize.
* "Skip MoE channels ... top-k channel selection" explainer, section on the
  ternary sketch: three values (-1, 0, 1) plus one scale per block.
* MLX issue "2-bit quantized_matmul loses its size advantage over 4-bit at
  M >= 3", table and repro: the single quantized linear y = x W^T, group 128.
* "The QMoE sub-1-bit expert kernel is a GEMV ..." note: top-k routed tokens,
  several tokens sharing one expert.

Readings where the pages are silent:

* INT scale: s = bf16_rne(max|w| / 2^(bits-1)); codes c = clamp(rne(w/s),
  -2^(bits-1), 2^(bits-1)-1) in float64; s == 0 gives c = 0.
* Affine codes (scale and zero point per block, MLX-style): z = bf16_rne(min
  w), s = bf16_rne((max w - min w) / (2^bits - 1)), u = clamp(rne((w - z) / s),
  0, 2^bits - 1); w_hat = s * u + z.
* Ternary: delta = 0.7 * (sum|w| / block); t = sign(w) where |w| > delta
  (strict), else 0; s = bf16_rne(mean of |w| over |w| > delta), 0 if none.
  Sums run sequentially in K order in float64.
* Routing: top-k by descending fp32 logit, ties to the lower expert index,
  slot order = selection order; weights = softmax over the k selected logits
  (equal to softmax -> top-k -> renormalise); the permutation is a stable
  sort of the flat (token, slot) index by expert.
* SwiGLU: h_j = silu(g_j + b1_{2j}) * (u_j + b1_{2j+1}), silu(g) = g/(1+e^-g),
  with FC1 row 2j = gate j and row 2j+1 = up j.
* Combine: y_t = sum_s w_{t,s} (W2_e h + b2_e) + sum over shared experts
  (weight 1).

Parity status: quantizer, packing, dequant, routing, single linear and the
expert FFN are pinned by the tests under tests/test_oracle_*.py (closed forms,
exact rational brute force, exhaustive round trips, invariants).  The whole
MoE forward is pinned only through those parts and through the batching and
reduction invariants: the pages print no end-to-end values.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# bf16 helpers (own implementation; float64 values on a bf16 grid)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_to_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits; its smallest normal is 2^-126 and its
    subnormal quantum 2^-133.  Values past the largest finite bf16 become inf.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = (v != 0) & np.isfinite(v)
    _, e = np.frexp(v[nz])                       # v = m * 2^e, 0.5 <= |m| < 1
    q = np.maximum(e, -125) - 8                  # exponent of one unit in the last place
    r = np.round(np.ldexp(v[nz], -q))            # exact scaling, then half-to-even
    out[nz] = np.ldexp(r, q)
    big = np.abs(out) > np.ldexp(255.0, 127 - 7)  # > max finite bf16 (0x7F7F)
    out[big] = np.copysign(np.inf, out[big])
    out[~np.isfinite(v)] = v[~np.isfinite(v)]
    return out


# ---------------------------------------------------------------------------
# Quantizers
# ---------------------------------------------------------------------------

def quantize_sym(w, bits: int, block: int):
    """Symmetric block quantization without zero points.

    w: float64 [rows, K] holding bf16 values.  Returns (codes int8 [rows, K],
    scales float64 [rows, K // block] on the bf16 grid).
    """
    w = np.asarray(w, dtype=np.float64)
    rows, K = w.shape
    assert K % block == 0
    qmin, qmax = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    wb = w.reshape(rows, K // block, block)
    amax = np.abs(wb).max(axis=2)
    s = round_to_bf16(amax / float(1 << (bits - 1)))
    safe = np.where(s > 0, s, 1.0)
    q = np.round(wb / safe[..., None])           # half to even
    q = np.where(s[..., None] > 0, q, 0.0)
    c = np.clip(q, qmin, qmax).astype(np.int8)
    return c.reshape(rows, K), s


def quantize_affine(w, bits: int, block: int):
    """Affine (asymmetric) block quantization: one bf16 scale and one bf16 zero
    point (bias) per block, unsigned codes (MLX issue "2-bit quantized_matmul
    loses its size advantage over 4-bit at M >= 3", repro: ``mx.quantize``
    returns (wq, scales, biases); its "2.25 effective" bits per weight at
    group 128).

    Reading (the pages give no formula): z = bf16_rne(min w), s =
    bf16_rne((max w - min w) / (2^bits - 1)), u = clamp(rne((w - z) / s), 0,
    2^bits - 1) in float64; s == 0 gives u = 0.  w_hat = s * u + z.
    Returns (codes uint8 [rows, K], scales, zeros float64 [rows, K // block]).
    """
    w = np.asarray(w, dtype=np.float64)
    rows, K = w.shape
    assert K % block == 0
    umax = (1 << bits) - 1
    wb = w.reshape(rows, K // block, block)
    lo, hi = wb.min(axis=2), wb.max(axis=2)
    z = round_to_bf16(lo)
    s = round_to_bf16((hi - lo) / float(umax))
    safe = np.where(s > 0, s, 1.0)
    q = np.round((wb - z[..., None]) / safe[..., None])   # half to even
    q = np.where(s[..., None] > 0, q, 0.0)
    u = np.clip(q, 0, umax).astype(np.uint8)
    return u.reshape(rows, K), s, z


def dequant_affine(codes, scales, zeros, block: int) -> np.ndarray:
    """w_hat = s * u + z, exact in float64."""
    u = np.asarray(codes, dtype=np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), block, axis=1)
    z = np.repeat(np.asarray(zeros, dtype=np.float64), block, axis=1)
    return s * u + z


def dequant_affine_bf16_operand(codes, scales, zeros, block: int) -> np.ndarray:
    """bf16_rne(s * u + z): the affine weight operand of the bf16 tensor-core path."""
    return round_to_bf16(dequant_affine(codes, scales, zeros, block))


def quantize_ternary(w, block: int = 64):
    """Ternary {-1, 0, 1} codes with one bf16 scale per block (threshold 0.7*mean|w|)."""
    w = np.asarray(w, dtype=np.float64)
    rows, K = w.shape
    assert K % block == 0
    wb = w.reshape(rows, K // block, block)
    a = np.abs(wb)
    sum_abs = np.cumsum(a, axis=2)[..., -1]       # sequential, K order
    delta = 0.7 * (sum_abs / float(block))
    keep = a > delta[..., None]
    t = (np.sign(wb) * keep).astype(np.int8)
    cnt = keep.sum(axis=2)
    sel_sum = np.cumsum(np.where(keep, a, 0.0), axis=2)[..., -1]
    mean = np.where(cnt > 0, sel_sum / np.maximum(cnt, 1), 0.0)
    s = np.where(cnt > 0, round_to_bf16(mean), 0.0)
    return t.reshape(rows, K), s


def dequant(codes, scales, block: int) -> np.ndarray:
    """w_hat = c * s, exact in float64."""
    c = np.asarray(codes, dtype=np.float64)
    rows, K = c.shape
    s = np.repeat(np.asarray(scales, dtype=np.float64), block, axis=1)
    return c * s


def dequant_bf16_operand(codes, scales, block: int) -> np.ndarray:
    """bf16_rne(c * s): the weight operand of the bf16 tensor-core (grouped) path."""
    return round_to_bf16(dequant(codes, scales, block))


# ---------------------------------------------------------------------------
# Logical code packing (16 INT2 per u32, 8 INT4 per u32, 5 trits per byte)
# ---------------------------------------------------------------------------

def pack_int_codes(codes, bits: int) -> np.ndarray:
    """Pack signed codes [rows, K] as biased unsigned u = c + 2^(bits-1),
    32/bits codes per uint32 word, code i of a word in bits [bits*i, bits*(i+1))."""
    per = 32 // bits
    c = np.asarray(codes, dtype=np.int64)
    rows, K = c.shape
    assert K % per == 0
    u = (c + (1 << (bits - 1))).astype(np.uint64).reshape(rows, K // per, per)
    words = np.zeros((rows, K // per), dtype=np.uint64)
    for i in range(per):
        words |= u[:, :, i] << np.uint64(bits * i)
    return words.astype(np.uint32)


def unpack_int_codes(words, bits: int) -> np.ndarray:
    per = 32 // bits
    wd = np.asarray(words, dtype=np.uint64)
    rows, nw = wd.shape
    mask = np.uint64((1 << bits) - 1)
    u = np.stack([(wd >> np.uint64(bits * i)) & mask for i in range(per)], axis=2)
    return (u.astype(np.int64) - (1 << (bits - 1))).reshape(rows, nw * per).astype(np.int8)


TRITS_PER_BYTE = 5
TERNARY_BYTES_PER_BLOCK64 = 13     # 64 trits + one padding trit (t = 0)


def pack_trits(t, block: int = 64) -> np.ndarray:
    """Per row and 64-block: 13 bytes, byte j = sum_i (t[5j+i] + 1) * 3^i,
    i = 0..4; the 65th trit is padding with t = 0."""
    assert block == 64
    t = np.asarray(t, dtype=np.int64)
    rows, K = t.shape
    nb = K // 64
    d = (t + 1).reshape(rows, nb, 64)
    d = np.concatenate([d, np.ones((rows, nb, 1), dtype=np.int64)], axis=2)  # pad trit
    d = d.reshape(rows, nb, 13, 5)
    b = (d * (3 ** np.arange(5))).sum(axis=3)
    return b.reshape(rows, nb * 13).astype(np.uint8)


def unpack_trits(packed, K: int) -> np.ndarray:
    b = np.asarray(packed, dtype=np.int64)
    rows = b.shape[0]
    nb = K // 64
    b = b.reshape(rows, nb, 13)
    digits = np.stack([(b // (3 ** i)) % 3 for i in range(5)], axis=3).reshape(rows, nb, 65)
    return (digits[:, :, :64] - 1).reshape(rows, K).astype(np.int8)


# ---------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------

def route(logits, k: int):
    """Top-k routing of fp32 logits [T, E].

    Returns ids int32 [T, k], weights float64 [T, k], perm int32 [T*k]
    (flat index t*k+s of each expert-sorted position), offsets int32 [E+1].
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        order = np.argsort(-lg[t].astype(np.float64), kind="stable")  # ties: lower index first
        sel = order[:k]
        ids[t] = sel
        l = lg[t, sel].astype(np.float64)
        z = np.exp(l - l.max())
        w[t] = z / z.sum()
    flat = ids.reshape(-1)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return ids, w, perm, offsets


# ---------------------------------------------------------------------------
# Expert FFN, MoE layer, single linear
# ---------------------------------------------------------------------------

def silu(g):
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def expert_ffn(x, w1, w2, b1=None, b2=None) -> np.ndarray:
    """x [M, H]; w1 [2I, H] (row 2j gate j, row 2j+1 up j); w2 [H, I]."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    a = x @ np.asarray(w1, dtype=np.float64).T
    if b1 is not None:
        a = a + np.asarray(b1, dtype=np.float64)[None, :]
    h = silu(a[:, 0::2]) * a[:, 1::2]
    o = h @ np.asarray(w2, dtype=np.float64).T
    if b2 is not None:
        o = o + np.asarray(b2, dtype=np.float64)[None, :]
    return o


class QuantExpertBank:
    """Quantized experts, dequantized to float64 on demand (one cache entry per
    expert).  ``fc1_q(e)`` / ``fc2_q(e)`` return (codes, scales), or (codes,
    scales, zeros) for affine codes; biases may be None."""

    def __init__(self, H, I, E, n_shared, block, fc1_q, fc2_q, b1=None, b2=None, cache=8):
        self.H, self.I, self.E, self.n_shared, self.block = H, I, E, n_shared, block
        self._fc1_q, self._fc2_q, self._b1, self._b2 = fc1_q, fc2_q, b1, b2
        self._cache = {}
        self._cache_max = cache

    def _dq(self, q):
        """(codes, scales): symmetric; (codes, scales, zeros): affine."""
        return dequant(q[0], q[1], self.block) if len(q) == 2 else dequant_affine(q[0], q[1], q[2], self.block)

    def weights(self, e: int):
        if e not in self._cache:
            if len(self._cache) >= self._cache_max:
                self._cache.pop(next(iter(self._cache)))
            w1 = self._dq(self._fc1_q(e))
            w2 = self._dq(self._fc2_q(e))
            b1 = None if self._b1 is None else self._b1(e)
            b2 = None if self._b2 is None else self._b2(e)
            self._cache[e] = (w1, w2, b1, b2)
        return self._cache[e]


def moe_forward(x, logits, k: int, bank: QuantExpertBank) -> np.ndarray:
    """Whole MoE layer in float64, experts batched over the tokens they receive."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    ids, w, _, _ = route(logits, k)
    y = np.zeros((T, bank.H), dtype=np.float64)
    for e in np.unique(ids):
        tok, slot = np.nonzero(ids == e)
        w1, w2, b1, b2 = bank.weights(int(e))
        o = expert_ffn(x[tok], w1, w2, b1, b2)
        np.add.at(y, tok, w[tok, slot][:, None] * o)
    for j in range(bank.n_shared):
        w1, w2, b1, b2 = bank.weights(bank.E + j)
        y += expert_ffn(x, w1, w2, b1, b2)
    return y


def moe_token(x_t, logits_t, k: int, bank: QuantExpertBank) -> np.ndarray:
    """One token through the MoE layer (used for sampled parity and the
    batched-equals-single check)."""
    ids, w, _, _ = route(np.asarray(logits_t, dtype=np.float32)[None, :], k)
    xt = np.asarray(x_t, dtype=np.float64)[None, :]
    y = np.zeros(bank.H, dtype=np.float64)
    for s in range(k):
        w1, w2, b1, b2 = bank.weights(int(ids[0, s]))
        y += w[0, s] * expert_ffn(xt, w1, w2, b1, b2)[0]
    for j in range(bank.n_shared):
        w1, w2, b1, b2 = bank.weights(bank.E + j)
        y += expert_ffn(xt, w1, w2, b1, b2)[0]
    return y


def linear(x, w_hat) -> np.ndarray:
    """Single quantized linear: y[M, N] = x[M, K] @ w_hat[N, K]^T in float64."""
    return np.atleast_2d(np.asarray(x, dtype=np.float64)) @ np.asarray(w_hat, dtype=np.float64).T


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def max_err_over_rms(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref)) / (rms if rms > 0 else 1.0))
