"""CPU fp64 oracle for the top-k channel-selective expert read.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may call it.  It shares no code with the CUDA library.

Source: the explainer "Skip MoE channels for up to 2.69x faster MoE blocks --
top-k channel selection":

* sketch paragraph: each gate and up weight row is rotated by a randomized
  Hadamard transform, then stored as three values (-1, 0, 1) plus one scale
  per block, a 256-byte bf16 block (128 weights) becoming about 30 bytes;
* scoring paragraph: a channel's score is its router weight times the norm of
  its down column times its estimated activation; channels of different
  experts compete in one top-k; the winners are read in full and computed
  exactly;
* choosing-k paragraph: top-k fixes the number of channels read per token.

Readings where the explainer is silent (the plainest ones the rest supports):

* Rotation: v' = Had_n (d * v) / sqrt(n), Had_n the Sylvester Hadamard matrix
  (Had_1 = [1], Had_2m = [[Had_m, Had_m], [Had_m, -Had_m]]), d a vector of
  random signs given as input, n = H a power of two.  The same d rotates the
  weight rows and the token, so that w'.x' = w.x.
* The sketch is built from the bf16 weights given to the packer (the model's
  weights), with the library's ternary rule (threshold 0.7 * mean|w| per
  block, scale = bf16 of the mean |w| above it) on blocks of 128 rotated
  weights.
* Estimated activation of channel j for token x: a_j = silu(g_j) * u_j with
  g_j, u_j the sketch rows' dot products with x'; the score is
  w_{t,s} * ||W2_e[:, j]|| * |a_j| with the down matrix as stored.
* The down matrix of the channel layer is quantized column by column (blocks
  of `block` rows of W2 in each column), so that one channel is one
  contiguous read.
* The budget is n_keep channels per token over its k routed experts; ties
  are broken towards the lower flat index s * I + j.  Shared experts are read
  in full with weight 1.  No biases.
* Unselected channels contribute nothing (the explainer's low-rank estimate
  of the rest is not part of this path).

Parity status: pinned by tests/test_oracle_channel.py (closed forms of the
transform, exact recovery of sketches that are ternary by construction,
brute-force ranking with ties, and reduction to the full MoE layer at a full
budget).
"""
from __future__ import annotations

import numpy as np
import scipy.linalg

from oracle import qmoe_oracle as Q


def rht(v, signs) -> np.ndarray:
    """Randomized Hadamard transform of the last axis: Had_n (d * v) / sqrt(n)."""
    v = np.asarray(v, dtype=np.float64)
    n = v.shape[-1]
    assert n & (n - 1) == 0, "length must be a power of two"
    had = scipy.linalg.hadamard(n).astype(np.float64)
    d = np.asarray(signs, dtype=np.float64)
    return ((v * d) @ had.T) * (1.0 / np.sqrt(n))


def sketch_rows(w_rows, signs, block: int = 128):
    """Ternary sketch of weight rows [rows, H]: (trits int8 [rows, H], scales [rows, H // block])."""
    return Q.quantize_ternary(rht(w_rows, signs), block)


def quantize_down_columns(w2, bits: int, block: int):
    """Column-wise symmetric quantization of the down matrix W2 [H, I]: every
    column is cut into blocks of `block` rows.  Returns (codes int8 [I, H],
    scales [I, H // block]) in column-major order and the dequantized W2 [H, I]."""
    codes, scales = Q.quantize_sym(np.asarray(w2, dtype=np.float64).T, bits, block)
    return codes, scales, Q.dequant(codes, scales, block).T


class ChannelExpertBank:
    """Experts of the channel layer from bf16 weights: dequantized FC1 rows
    (block quantization along H, as in the full layer), column-quantized FC2,
    the gate/up sketch and the down-column norms."""

    def __init__(self, H, I, E, n_shared, block, fc1_bits, fc2_bits, w1_of, w2_of, signs, sketch_block=128):
        self.H, self.I, self.E, self.n_shared = H, I, E, n_shared
        self.block, self.fc1_bits, self.fc2_bits = block, fc1_bits, fc2_bits
        self.w1_of, self.w2_of = w1_of, w2_of            # e -> float64 [2I, H] / [H, I] on the bf16 grid
        self.signs = np.asarray(signs, dtype=np.float64)
        self.sketch_block = sketch_block
        self._cache = {}

    def expert(self, e: int):
        """(w1_hat [2I, H], w2_hat [H, I], dn [I], sketch) of expert e; the
        sketch is (gate trits, gate scales, up trits, up scales)."""
        if e not in self._cache:
            w1 = self.w1_of(e)
            c1, s1 = Q.quantize_sym(w1, self.fc1_bits, self.block)
            w1_hat = Q.dequant(c1, s1, self.block)
            _, _, w2_hat = quantize_down_columns(self.w2_of(e), self.fc2_bits, self.block)
            dn = np.sqrt((w2_hat * w2_hat).sum(axis=0))
            tg, sg = sketch_rows(w1[0::2], self.signs, self.sketch_block)
            tu, su = sketch_rows(w1[1::2], self.signs, self.sketch_block)
            self._cache[e] = (w1_hat, w2_hat, dn, (tg, sg, tu, su))
        return self._cache[e]


def estimated_activation(x_rot, sketch, sketch_block: int = 128) -> np.ndarray:
    """a_j = silu(g_j) * u_j from the sketch rows and the rotated token x' [H]."""
    tg, sg, tu, su = sketch
    g = Q.dequant(tg, sg, sketch_block) @ x_rot
    u = Q.dequant(tu, su, sketch_block) @ x_rot
    return Q.silu(g) * u


def channel_scores(x, logits, k: int, bank: ChannelExpertBank):
    """Routing plus the score of every (slot, channel) of every token.

    Returns ids [T, k], router weights [T, k] and scores float64 [T, k * I]
    (flat index s * I + j)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    ids, w, _, _ = Q.route(logits, k)
    scores = np.zeros((T, k * bank.I), dtype=np.float64)
    x_rot = rht(x, bank.signs)
    for t in range(T):
        for s in range(k):
            _, _, dn, sk = bank.expert(int(ids[t, s]))
            a = estimated_activation(x_rot[t], sk, bank.sketch_block)
            scores[t, s * bank.I:(s + 1) * bank.I] = w[t, s] * dn * np.abs(a)
    return ids, w, scores


def select_top(scores_t, n_keep: int) -> np.ndarray:
    """The n_keep best flat indices of one token (score descending, ties to the
    lower index), returned in ascending index order."""
    sc = np.asarray(scores_t, dtype=np.float64)
    order = np.lexsort((np.arange(sc.size), -sc))
    return np.sort(order[:n_keep]).astype(np.int32)


def channel_forward(x, logits, k: int, bank: ChannelExpertBank, n_keep: int):
    """The channel layer: y_t = sum over the selected (s, j) of
    w_{t,s} * h_{e,j}(x_t) * W2_e[:, j] + the shared experts in full.

    Returns (y float64 [T, H], selection int32 [T, n_keep], scores)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    ids, w, scores = channel_scores(x, logits, k, bank)
    y = np.zeros((T, bank.H), dtype=np.float64)
    sel = np.zeros((T, n_keep), dtype=np.int32)
    for t in range(T):
        sel[t] = select_top(scores[t], n_keep)
        for f in sel[t]:
            s, j = divmod(int(f), bank.I)
            w1_hat, w2_hat, _, _ = bank.expert(int(ids[t, s]))
            h = Q.silu(w1_hat[2 * j] @ x[t]) * (w1_hat[2 * j + 1] @ x[t])
            y[t] += w[t, s] * h * w2_hat[:, j]
        for sh in range(bank.n_shared):
            w1_hat, w2_hat, _, _ = bank.expert(bank.E + sh)
            y[t] += Q.expert_ffn(x[t], w1_hat, w2_hat)[0]
    return y, sel, scores
