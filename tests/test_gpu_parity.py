"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Bar: routing ids / permutation / offsets and dequantized weights bit-exact;
outputs within rel-L2 5e-3 and max |err| 3e-2 * rms(ref)."""
import numpy as np
import pytest

from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import synth

from cases import (FMTS, MAX_ERR_RMS, REL_L2, TINY_FACTORS, MoECase, bf16_dev_to_f64, block_scaled_weights,
                   oracle_quant_affine,
                   oracle_quant, small_cfg, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qm(cuda_ok):
    from skinny_gemm_top_b200 import qmoe
    qmoe.clear_status()
    yield qmoe
    assert qmoe.get_stats().device_status == 0


def _close(got, ref, what=""):
    r, m = Q.rel_l2(got, ref), Q.max_err_over_rms(got, ref)
    assert r <= REL_L2 and m <= MAX_ERR_RMS, f"{what}: rel_l2={r:.3g} max_err/rms={m:.3g}"
    return r, m


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("fmt,block,order,tiny", [
    ("int2", 64, 1, False), ("int2", 128, 0, False), ("int4", 64, 0, False), ("int4", 128, 1, False),
    ("ternary", 64, 1, False), ("ternary", 64, 0, False), ("int2", 64, 2, False), ("int4", 64, 2, False),
    ("int4", 128, 2, False), ("ternary", 64, 2, False),
    ("int2", 64, 0, True), ("int4", 128, 0, True), ("ternary", 64, 0, True), ("int4", 64, 2, True)])
def test_dequant_bit_exact(qm, fmt, block, order, tiny):
    import torch
    rows, K, n = 48, 384 if not tiny else 896, 2
    if tiny:  # blocks with tiny normal and subnormal scales
        mats = [block_scaled_weights(21 + i, rows, K, block, TINY_FACTORS) for i in range(n)]
    else:
        mats = [synth.normal_bf16(21, 60, i, (rows, K), 0.02) for i in range(n)]
    c, s = qm.pack_stack(FMTS[fmt], order, mats, block)
    dc, ds = to_dev(c), to_dev(s)
    w = qm.make_weights(FMTS[fmt], block, dc, ds, None, order)
    o32 = torch.empty((n, rows, K), dtype=torch.float32, device="cuda")
    o16 = torch.empty((n, rows, K), dtype=torch.int16, device="cuda")
    qm.dequant(w, rows, K, n, o32, o16)
    torch.cuda.synchronize()
    for i in range(n):
        codes, scales = oracle_quant(fmt, mats[i], block)
        if tiny:
            assert np.any((scales > 0) & (scales < 2.0 ** -126)), "no subnormal scale drawn"
        ref = Q.dequant(codes, scales, block)
        assert np.array_equal(o32[i].cpu().numpy().astype(np.float64), ref)
        ref16 = Q.dequant_bf16_operand(codes, scales, block)
        assert np.array_equal(Q.bf16_bits_to_f64(o16[i].cpu().numpy().view(np.uint16)), ref16)


@pytest.mark.parametrize("fmt,block,tiny", [("int2", 64, False), ("int4", 64, False), ("int2", 128, True),
                                            ("int4", 64, True), ("int4", 128, True)])
def test_grouped_operand_bit_exact_one_hot(qm, fmt, block, tiny):
    """The tcgen05 path's weight operand bf16_rne(c*s), through its own code:
    128 one-hot token rows (row m = 2^64 e_{k_m}) through qmoe_linear, which
    takes the grouped path from 48 rows on.  y[m, n] = bf16(2^64 W_op[n, k_m])
    exactly (one nonzero product, accumulated in fp32, already on the bf16
    grid), so y / 2^64 is the operand column k_m, bit for bit; the 2^64 keeps
    products and outputs of subnormal operands normal."""
    import torch
    N, K, M = 256, 1024, 128
    wb = block_scaled_weights(31, N, K, block, TINY_FACTORS) if tiny else synth.linear_weight(31, N, K)
    c, s = qm.pack(FMTS[fmt], 0, wb, block)
    dc, ds = to_dev(c), to_dev(s)
    w = qm.make_weights(FMTS[fmt], block, dc, ds)
    km = (np.arange(M) * 37 + 5) % K          # every k-step column class, every block
    x = np.zeros((M, K), dtype=np.uint16)
    x[np.arange(M), km] = synth.f32_to_bf16_bits(np.float32(2.0 ** 64))
    y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws = torch.empty(qm.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")
    qm.linear(w, N, K, to_dev(x), y, ws)
    torch.cuda.synchronize()
    st = qm.get_stats()
    assert st.last_path == qm.PATH_GROUPED
    got = bf16_dev_to_f64(y) * 2.0 ** -64
    codes, scales = oracle_quant(fmt, wb, block)
    if tiny:
        assert np.any((scales > 0) & (scales < 2.0 ** -126)), "no subnormal scale drawn"
    op = Q.dequant_bf16_operand(codes, scales, block)   # [N, K]
    assert np.array_equal(got, op[:, km].T)


# ------------------------------------------------------------------ affine codes (scale and zero point)

@pytest.mark.parametrize("fmt,block,order,tiny", [
    ("int2", 64, 1, False), ("int4", 128, 0, False), ("int4", 64, 2, False), ("int2", 128, 2, False),
    ("int2", 64, 0, True), ("int4", 128, 0, True)])
def test_dequant_affine_bit_exact(qm, fmt, block, order, tiny):
    """fp32: f32_rne(s*u + z); bf16: bf16_rne(s*u + z), one rounding each."""
    import torch
    rows, K, n = 48, 384 if not tiny else 896, 2
    if tiny:
        mats = [block_scaled_weights(41 + i, rows, K, block, TINY_FACTORS) for i in range(n)]
    else:
        mats = [synth.normal_bf16(41, 61, i, (rows, K), 0.02) for i in range(n)]
    c, s, z = qm.pack_stack_affine(FMTS[fmt], order, mats, block)
    keep = [to_dev(a) for a in (c, s, z)]  # the weight set holds raw pointers
    w = qm.make_weights(FMTS[fmt], block, keep[0], keep[1], None, order, keep[2])
    o32 = torch.empty((n, rows, K), dtype=torch.float32, device="cuda")
    o16 = torch.empty((n, rows, K), dtype=torch.int16, device="cuda")
    qm.dequant(w, rows, K, n, o32, o16)
    torch.cuda.synchronize()
    for i in range(n):
        codes, scales, zeros = oracle_quant_affine(fmt, mats[i], block)
        if tiny:
            assert np.any((scales > 0) & (scales < 2.0 ** -126)), "no subnormal scale drawn"
        exact = Q.dequant_affine(codes, scales, zeros, block)
        assert np.array_equal(o32[i].cpu().numpy(), exact.astype(np.float32))
        ref16 = Q.dequant_affine_bf16_operand(codes, scales, zeros, block)
        assert np.array_equal(Q.bf16_bits_to_f64(o16[i].cpu().numpy().view(np.uint16)), ref16)


@pytest.mark.parametrize("fmt,block,tiny", [("int2", 64, False), ("int4", 128, False), ("int4", 64, True)])
def test_grouped_operand_affine_bit_exact_one_hot(qm, fmt, block, tiny):
    """The tcgen05 path's affine operand bf16_rne(s*u + z) through qmoe_linear
    (one-hot token rows as in the symmetric test above)."""
    import torch
    N, K, M = 256, 1024, 128
    wb = block_scaled_weights(33, N, K, block, TINY_FACTORS) if tiny else synth.linear_weight(33, N, K)
    c, s, z = qm.pack_affine(FMTS[fmt], 0, wb, block)
    keep = [to_dev(a) for a in (c, s, z)]
    w = qm.make_weights(FMTS[fmt], block, keep[0], keep[1], None, 0, keep[2])
    km = (np.arange(M) * 37 + 5) % K
    x = np.zeros((M, K), dtype=np.uint16)
    x[np.arange(M), km] = synth.f32_to_bf16_bits(np.float32(2.0 ** 64))
    y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws = torch.empty(qm.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")
    qm.linear(w, N, K, to_dev(x), y, ws)
    torch.cuda.synchronize()
    assert qm.get_stats().last_path == qm.PATH_GROUPED
    got = bf16_dev_to_f64(y) * 2.0 ** -64
    codes, scales, zeros = oracle_quant_affine(fmt, wb, block)
    op = Q.dequant_affine_bf16_operand(codes, scales, zeros, block)
    assert np.array_equal(got, op[:, km].T)


@pytest.mark.parametrize("fmt,block", [("int2", 128), ("int4", 128), ("int4", 64), ("int2", 64)])
@pytest.mark.parametrize("M", [1, 5, 8, 16, 32, 64])
def test_linear_affine(qm, fmt, block, M):
    import torch
    N, K = 384, 1024
    wb = synth.linear_weight(50 + M, N, K)
    c, s, z = qm.pack_affine(FMTS[fmt], 0, wb, block)
    keep = [to_dev(a) for a in (c, s, z)]
    w = qm.make_weights(FMTS[fmt], block, keep[0], keep[1], None, 0, keep[2])
    x = synth.tokens(K, 50 + M, M)
    y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws = torch.empty(qm.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")
    qm.linear(w, N, K, to_dev(x), y, ws)
    torch.cuda.synchronize()
    codes, scales, zeros = oracle_quant_affine(fmt, wb, block)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant_affine(codes, scales, zeros, block))
    _close(bf16_dev_to_f64(y), ref, f"affine {fmt} g{block} M={M}")


@pytest.mark.parametrize("T", [1, 3, 8, 13, 40])
def test_forward_affine_layer(qm, T):
    """A MoE layer with affine codes (tiny shapes, INT2 FC1 / INT4 FC2, plus a shared expert and biases)."""
    cfg = small_cfg(synth.TINY, n_shared=1, bias=True)
    case = MoECase(cfg, seed=7, affine=True)
    x = synth.tokens(cfg.H, 7, T)
    lg = synth.router_logits(cfg, 7, T)
    y = case.run(x, lg)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"affine layer T={T}")


@pytest.mark.parametrize("f1,f2,T", [("int2", "int4", 1), ("int4", "int4", 4), ("int4", "int2", 8), ("int2", "int2", 2)])
def test_decode_affine_layer(qm, f1, f2, T):
    """Decode batches (the decode-layer kernel) with affine codes, shared experts and biases."""
    cfg = small_cfg(synth.TINY, fc1_fmt=f1, fc2_fmt=f2, n_shared=1, bias=True, E=16, k=4)
    case = MoECase(cfg, seed=8, affine=True)
    x = synth.tokens(cfg.H, 8, T)
    lg = synth.router_logits(cfg, 8, T)
    y = case.run(x, lg)
    assert qm.get_stats().last_path == qm.PATH_SMALL_M  # the decode kernel, not the grouped path
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"affine decode {f1}/{f2} T={T}")


@pytest.mark.parametrize("path,T", [("small", 13), ("small", 40), ("grouped", 13)])
def test_forward_affine_forced_paths(qm, path, T):
    """Affine layers on the small-M expert kernel (forced) and on the tcgen05 path (forced)."""
    cfg = small_cfg(synth.TINY, n_shared=1, bias=True)
    case = MoECase(cfg, seed=9, affine=True)
    x = synth.tokens(cfg.H, 9, T)
    lg = synth.router_logits(cfg, 9, T)
    y = case.run(x, lg, path=qm.PATH_SMALL_M if path == "small" else qm.PATH_GROUPED)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"affine {path} T={T}")


def test_affine_ternary_rejected(qm):
    import torch
    c, s = qm.pack(qm.TERNARY, 0, synth.linear_weight(3, 64, 128), 64)
    keep = [to_dev(c), to_dev(s), to_dev(s.copy())]
    w = qm.make_weights(qm.TERNARY, 64, keep[0], keep[1], None, 0, keep[2])
    x = to_dev(synth.tokens(128, 3, 1))
    y = torch.empty((1, 64), dtype=torch.int16, device="cuda")
    ws = torch.empty(qm.linear_workspace_size(64, 128, 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(qm.QmoeError):
        qm.linear(w, 64, 128, x, y, ws)


# ------------------------------------------------------------------ routing

def _route_case(qm, lg, k):
    import torch
    T, E = lg.shape
    d = torch.from_numpy(np.ascontiguousarray(lg)).cuda()
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    nb = qm.route_workspace_size(T, E, k)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda") if nb else None
    qm.route(d, k, ids, w, perm, off, ws)
    torch.cuda.synchronize()
    rids, rw, rperm, roff = Q.route(lg, k)
    assert np.array_equal(ids.cpu().numpy(), rids)
    assert np.array_equal(perm.cpu().numpy(), rperm)
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.allclose(w.cpu().numpy(), rw, rtol=1e-6, atol=0)
    return nb


def _tied_logits(g, T, E):
    """Few distinct values, both signs of zero: many exact ties."""
    lg = (np.round(g.standard_normal((T, E)) * 2.0) / 2.0).astype(np.float32)
    lg[:, 1::5] = -0.0
    lg[:, 3::5] = 0.0
    lg[::2, 7::9] = 0.5
    return lg


# Decode routing (T <= 8, T*k <= 64): the routing the fused decode layer kernel runs in its prologue.
@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (100, 7), (128, 8), (256, 8), (256, 1), (64, 32)])
@pytest.mark.parametrize("T", [1, 3, 8])
@pytest.mark.parametrize("tied", [False, True])
def test_route_decode_matches_oracle(qm, T, E, k, tied):
    if T * k > 64:
        pytest.skip("not a decode batch")
    g = np.random.default_rng(1000 * T + E + k)
    lg = _tied_logits(g, T, E) if tied else g.standard_normal((T, E)).astype(np.float32)
    assert _route_case(qm, lg, k) == 0  # no workspace: the decode routing ran


# General routing (two launches: per-chunk top-k and counts, stable scatter), as qmoe_forward runs it above 8 tokens.
@pytest.mark.parametrize("T,E,k", [(9, 64, 6), (37, 8, 2), (300, 128, 8), (1100, 64, 6), (4096, 128, 8),
                                   (4096, 256, 8), (129, 256, 1), (3, 64, 32)])
@pytest.mark.parametrize("tied", [False, True])
def test_route_general_matches_oracle(qm, T, E, k, tied):
    g = np.random.default_rng(7 * T + E + k)
    lg = _tied_logits(g, T, E) if tied else g.standard_normal((T, E)).astype(np.float32)
    assert _route_case(qm, lg, k) > 0  # workspace needed: the general routing ran


def test_route_rejects_small_workspace(qm):
    import torch
    T, E, k = 100, 64, 6
    lg = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    out = [torch.empty(T * k, dtype=torch.int32, device="cuda"), torch.empty(T * k, dtype=torch.float32, device="cuda"),
           torch.empty(T * k, dtype=torch.int32, device="cuda"), torch.empty(E + 1, dtype=torch.int32, device="cuda")]
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(qm.QmoeError) as e:
        qm.route(lg, k, *out, ws)
    assert e.value.status == qm.ERR_SCRATCH


# ------------------------------------------------------------------ single linear

def _linear_case(qm, fmt, block, N, K, M, seed):
    import torch
    wb = synth.linear_weight(seed, N, K)
    c, s = qm.pack(FMTS[fmt], 0, wb, block)
    dc, ds = to_dev(c), to_dev(s)
    w = qm.make_weights(FMTS[fmt], block, dc, ds)
    x = synth.tokens(K, seed, M)
    y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    ws = torch.empty(qm.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")
    qm.linear(w, N, K, to_dev(x), y, ws)
    torch.cuda.synchronize()
    return wb, x, bf16_dev_to_f64(y), (dc, ds)


@pytest.mark.parametrize("fmt,block", [("int2", 128), ("int4", 128), ("int2", 64), ("int4", 64), ("ternary", 64)])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 16, 21])
def test_linear_small_shapes(qm, fmt, block, M):
    N, K = 272, 640      # 17 tiles, 10 (or 5 ternary) k-units: ragged against 8 warps and 148 CTAs
    wb, x, y, _ = _linear_case(qm, fmt, block, N, K, M, seed=M)
    codes, scales = oracle_quant(fmt, wb, block)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant(codes, scales, block))
    _close(y, ref, f"{fmt} M={M}")


@pytest.mark.parametrize("fmt", ["int2", "int4", "ternary"])
@pytest.mark.parametrize("M", [1, 16])
def test_linear_medium_multi_tile_per_cta(qm, fmt, M):
    """Enough tiles that every CTA streams several tiles per k-unit (sub-panels of 8)."""
    N, K = 4096, 1024
    wb, x, y, _ = _linear_case(qm, fmt, 64, N, K, M, seed=11)
    codes, scales = oracle_quant(fmt, wb, 64)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant(codes, scales, 64))
    _close(y, ref, f"{fmt} M={M}")


@pytest.mark.parametrize("fmt,block", [("int2", 128), ("int4", 64)])
@pytest.mark.parametrize("M", [48, 64, 300])
def test_linear_grouped_path(qm, fmt, block, M):
    """48 rows or more with N a multiple of 128: the tcgen05 path (weights rounded
    once to bf16 there), including further 128-token chunks with a ragged tail."""
    N, K = 1024, 768
    wb, x, y, _ = _linear_case(qm, fmt, block, N, K, M, seed=40 + M)
    st = qm.get_stats()
    assert st.last_path == qm.PATH_GROUPED and st.grouped_launches == 1
    codes, scales = oracle_quant(fmt, wb, block)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant(codes, scales, block))
    _close(y, ref, f"{fmt} M={M}")


@pytest.mark.parametrize("fmt", ["int2", "int4"])
@pytest.mark.parametrize("M", [1, 8, 32])
def test_linear_full_size_sampled_rows(qm, fmt, M):
    """K=5120 -> N=17408, group 128, as benchmarked; the oracle computes 512 sampled rows."""
    N, K = 17408, 5120
    wb, x, y, _ = _linear_case(qm, fmt, 128, N, K, M, seed=7)
    rows = np.random.default_rng(0).choice(N, 512, replace=False)
    codes, scales = oracle_quant(fmt, wb[rows], 128)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant(codes, scales, 128))
    _close(y[:, rows], ref, f"{fmt} M={M}")


@pytest.mark.parametrize("fmt,block", [("int2", 128), ("int4", 64)])
@pytest.mark.parametrize("M", [1, 9, 16, 33])
def test_linear_split_along_k(qm, fmt, block, M):
    """N = 1024 (64 tiles) is split along K over the SMs; partial sums meet in the workspace.
    A second call on the same workspace must give the same result (the accumulator is cleared per call)."""
    import torch
    N, K = 1024, 2048
    wb, x, y, dev = _linear_case(qm, fmt, block, N, K, M, seed=60 + M)
    codes, scales = oracle_quant(fmt, wb, block)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant(codes, scales, block))
    _close(y, ref, f"{fmt} split M={M}")
    w = qm.make_weights(FMTS[fmt], block, dev[0], dev[1])
    ws = torch.empty(qm.linear_workspace_size(N, K, M), dtype=torch.uint8, device="cuda")
    y2 = torch.empty((M, N), dtype=torch.int16, device="cuda")
    xd = to_dev(x)
    for _ in range(2):
        qm.linear(w, N, K, xd, y2, ws)
    torch.cuda.synchronize()
    _close(bf16_dev_to_f64(y2), ref, f"{fmt} split M={M}, repeated")


@pytest.mark.parametrize("fmt", ["int2", "int4"])
@pytest.mark.parametrize("N,K,M", [(5120, 17408, 1), (5120, 17408, 6), (5120, 5120, 3)])
def test_linear_decoder_layer_shapes_sampled_rows(qm, fmt, N, K, M):
    """The decoder-layer shapes of the model-level sweep (down 17408 -> 5120, attention 5120 -> 5120), g128."""
    wb, x, y, _ = _linear_case(qm, fmt, 128, N, K, M, seed=11)
    rows = np.random.default_rng(1).choice(N, 256, replace=False)
    codes, scales = oracle_quant(fmt, wb[rows], 128)
    ref = Q.linear(Q.bf16_bits_to_f64(x), Q.dequant(codes, scales, 128))
    _close(y[:, rows], ref, f"{fmt} {N}x{K} M={M}")


# ------------------------------------------------------------------ MoE layer

@pytest.mark.parametrize("T", [1, 3, 8, 13])
def test_forward_tiny(qm, T):
    case = MoECase(synth.TINY, seed=3)
    x = synth.tokens(synth.TINY.H, 3, T)
    lg = synth.router_logits(synth.TINY, 3, T)
    y = case.run(x, lg)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, synth.TINY.k, case.bank)
    _close(y, ref, f"tiny T={T}")


def test_decode_wait_expiry_leaves_y_and_recovers(qm):
    """A bounded device wait driven to expiry: with the test hook, every CTA of
    the decode kernel waits 1 ms on a barrier nothing arrives at.  The timeout
    flag is set, y keeps its previous contents, and the next call (hook off)
    is correct."""
    import torch
    cfg = synth.TINY
    case = MoECase(cfg, seed=3)
    x_bits = synth.tokens(cfg.H, 3, 1)
    lg_np = synth.router_logits(cfg, 3, 1)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x_bits), lg_np, cfg.k, case.bank)
    layer = case.layer()
    ws = torch.empty(qm.workspace_size(layer, 1), dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    lg = torch.from_numpy(np.ascontiguousarray(lg_np, dtype=np.float32)).cuda()
    y = torch.full((1, cfg.H), 0x3F80, dtype=torch.int16, device="cuda")  # bf16 1.0 everywhere
    try:
        qm.test_set_fault(1, 1_000_000)
        qm.clear_status()
        qm.forward(layer, x, lg, y, ws)
        torch.cuda.synchronize()
        assert qm.get_stats().device_status & qm.DEVICE_TIMEOUT
        assert bool((y == 0x3F80).all()), "y was written although a CTA gave up"
    finally:
        qm.test_set_fault(0, 0)
        qm.clear_status()
    qm.forward(layer, x, lg, y, ws)
    torch.cuda.synchronize()
    assert qm.get_stats().device_status == 0
    _close(bf16_dev_to_f64(y), ref, "tiny after an expired wait")


def test_fault_hook_rejects_unknown_injection(qm):
    with pytest.raises(qm.QmoeError):
        qm.test_set_fault(2, 0)


@pytest.fixture(scope="module")
def v2lite(qm):
    return MoECase(synth.V2LITE, seed=5)


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_forward_v2lite_full_size(qm, v2lite, T):
    cfg = synth.V2LITE
    x = synth.tokens(cfg.H, 5, T)
    lg = synth.router_logits(cfg, 5, T)
    y = v2lite.run(x, lg)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, v2lite.bank)
    _close(y, ref, f"v2lite T={T}")


def test_decode_mixed_formats_and_ternary(qm):
    """Decode batches with INT2 FC1 / INT4 FC2 (tiny) and with ternary experts,
    including a segment partition where CTA groups own whole experts."""
    for cfg, T in ((synth.TINY, 5), (small_cfg(synth.TERNARY, E=16, H=512, I=768), 4)):
        case = MoECase(cfg, seed=16)
        x = synth.tokens(cfg.H, 16, T)
        lg = synth.router_logits(cfg, 16, T)
        y = case.run(x, lg)
        ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
        _close(y, ref, f"{cfg.name} decode T={T}")


@pytest.mark.parametrize("E,k,n_shared", [(100, 8, 1), (128, 4, 0), (200, 8, 2), (256, 8, 1)])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_decode_many_experts(qm, E, k, n_shared, T):
    """Decode batches (one fused launch) over 65..256 experts: the routing's
    4- and 8-experts-per-lane variants, ragged expert counts, shared experts."""
    cfg = small_cfg(synth.TINY, E=E, k=k, n_shared=n_shared, H=256, I=256, fc1_fmt="int4", fc2_fmt="int4")
    case = MoECase(cfg, seed=50 + E)
    x = synth.tokens(cfg.H, 50 + E, T)
    lg = synth.router_logits(cfg, 50 + E, T)
    y = case.run(x, lg)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"E={E} k={k} decode T={T}")


@pytest.mark.parametrize("T", [1, 5, 8])
def test_decode_routing_ties(qm, T):
    """Decode batches whose logits tie (a few distinct values, both signs of
    zero): top-k takes the lower expert index among equal logits."""
    cfg = synth.TINY
    case = MoECase(cfg, seed=17)
    x = synth.tokens(cfg.H, 17, T)
    lg = np.round(synth.router_logits(cfg, 17, T) * 2.0).astype(np.float32) / 2.0
    lg[:, 1::4] = -0.0
    lg[:, 3::4] = 0.0
    y = case.run(x, lg)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"tiny ties T={T}")


# ------------------------------------------------------------------ decode layer kernel (one launch, split along I)

PAIRS = [(a, b) for a in ("int2", "int4", "ternary") for b in ("int2", "int4", "ternary")]


@pytest.mark.parametrize("f1,f2", PAIRS)
@pytest.mark.parametrize("T", [1, 5, 8])
def test_decode_format_pairs_bias_shared(qm, f1, f2, T):
    """Every FC1/FC2 format pair on the one-launch decode kernel, with routed
    and shared experts and both biases (the FC2 bias is added once per expert
    by the block holding its first granule)."""
    cfg = small_cfg(synth.TINY, E=12, k=3, n_shared=1, H=384, I=384, fc1_fmt=f1, fc2_fmt=f2, bias=True)
    case = MoECase(cfg, seed=70 + T)
    x = synth.tokens(cfg.H, 70 + T, T)
    lg = synth.router_logits(cfg, 70 + T, T)
    y = case.run(x, lg)
    st = qm.get_stats()
    assert st.small_launches == 1 and st.grouped_launches == 0  # the one-launch decode layer
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"{f1}/{f2} T={T}")


@pytest.mark.parametrize("H,I,E,k,n_shared,T", [
    (320, 448, 64, 6, 2, 3),     # 20 output tiles over 12 warps; 28 granules per expert
    (64, 128, 4, 2, 0, 2),       # fewer output tiles than warps
    (2112, 192, 16, 4, 1, 8),    # the largest H of the decode kernel
    (256, 1024, 256, 8, 1, 8),   # 64 selected experts: many sub-panels per block
    (512, 64, 200, 1, 3, 1),     # one granule per routed expert, several shared experts
])
def test_decode_ragged_shapes(qm, H, I, E, k, n_shared, T):
    cfg = small_cfg(synth.TINY, E=E, k=k, n_shared=n_shared, H=H, I=I, fc1_fmt="int4", fc2_fmt="int4", bias=True)
    case = MoECase(cfg, seed=H + I + E)
    x = synth.tokens(cfg.H, 3, T)
    lg = synth.router_logits(cfg, 3, T)
    y = case.run(x, lg)
    assert qm.get_stats().small_launches == 1
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"H={H} I={I} E={E} k={k} T={T}")


def test_decode_wide_hidden_takes_general_path(qm):
    """H above 2112: a decode batch runs the routing / expert / combine launches."""
    cfg = small_cfg(synth.TINY, E=8, k=2, n_shared=1, H=2176, I=128, fc1_fmt="int4", fc2_fmt="int4")
    case = MoECase(cfg, seed=5)
    x = synth.tokens(cfg.H, 5, 2)
    lg = synth.router_logits(cfg, 5, 2)
    y = case.run(x, lg)
    assert qm.get_stats().small_launches == 2
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, "H=2176")


def test_decode_v2lite_with_biases(qm):
    cfg = small_cfg(synth.V2LITE, bias=True)
    case = MoECase(cfg, seed=21)
    for T in (1, 4):
        x = synth.tokens(cfg.H, 21, T)
        lg = synth.router_logits(cfg, 21, T)
        y = case.run(x, lg)
        ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
        _close(y, ref, f"v2lite+bias T={T}")


@pytest.fixture(scope="module")
def ternary_full(qm):
    """The ternary Switch-style workload at full size: d=2048, d_ff=6144, 128 experts, top-1."""
    return MoECase(synth.TERNARY, seed=4)


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_forward_ternary_full_size(qm, ternary_full, T):
    cfg = synth.TERNARY
    x = synth.tokens(cfg.H, 4, T)
    lg = synth.router_logits(cfg, 4, T)
    y = ternary_full.run(x, lg)
    pick = np.arange(T) if T <= 8 else np.random.default_rng(T).choice(T, 4, replace=False)
    ref = np.stack([Q.moe_token(Q.bf16_bits_to_f64(x[t]), lg[t], cfg.k, ternary_full.bank) for t in pick])
    _close(y[pick], ref, f"ternary full size T={T}")


@pytest.mark.parametrize("M", [1, 5, 16, 32])
def test_forward_v2lite_tokens_per_expert(qm, v2lite, M):
    """M tokens with identical router logits: every selected expert gets exactly M tokens."""
    cfg = synth.V2LITE
    x = synth.tokens(cfg.H, 6, M)
    lg = synth.shared_logit_tokens(cfg, 6, M)
    y = v2lite.run(x, lg)
    pick = np.unique(np.linspace(0, M - 1, 4).astype(int))
    ref = np.stack([Q.moe_token(Q.bf16_bits_to_f64(x[t]), lg[t], cfg.k, v2lite.bank) for t in pick])
    _close(y[pick], ref, f"v2lite M={M}")


def test_forward_ternary_reduced_experts(qm):
    cfg = small_cfg(synth.TERNARY, E=6)
    case = MoECase(cfg, seed=8)
    T = 9
    x = synth.tokens(cfg.H, 8, T)
    lg = synth.router_logits(cfg, 8, T)
    y = case.run(x, lg)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, "ternary")


def test_forward_prefill_bias_and_row_tiling(qm):
    cfg = small_cfg(synth.PREFILL, E=16, k=4, H=256, I=192)
    case = MoECase(cfg, seed=9)
    T = 70
    x = synth.tokens(cfg.H, 9, T)
    lg = synth.router_logits(cfg, 9, T)
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    y = case.run(x, lg)
    _close(y, ref, "prefill untiled")
    # a workspace that only fits ~20 tokens: explicit partial last tile
    from skinny_gemm_top_b200 import qmoe
    small_ws = qmoe.workspace_size(case.layer(), 20)
    y2 = case.run(x, lg, ws_bytes=small_ws)
    st = qmoe.get_stats()
    assert st.row_tiles > 1 and st.row_tile_tokens <= 20
    _close(y2, ref, "prefill tiled")
    y3 = case.run(x, lg, max_row_tile=32)
    assert qmoe.get_stats().row_tiles == 3
    _close(y3, ref, "prefill max_row_tile")


def test_forward_scratch_error_and_invalid_args(qm):
    import torch
    from skinny_gemm_top_b200 import qmoe
    case = MoECase(synth.TINY, seed=3)
    x = to_dev(synth.tokens(synth.TINY.H, 3, 2))
    lg = torch.from_numpy(synth.router_logits(synth.TINY, 3, 2)).cuda()
    y = torch.empty((2, synth.TINY.H), dtype=torch.int16, device="cuda")
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    need1 = qmoe.workspace_size(case.layer(), 1)  # one token row of the decode layer
    with pytest.raises(qmoe.QmoeError) as e:
        qmoe.forward(case.layer(), x, lg, y, ws, ws_bytes=need1 - 256)
    assert e.value.status == qmoe.ERR_SCRATCH
    bad = case.layer()
    bad.k = 0
    with pytest.raises(qmoe.QmoeError) as e:
        qmoe.forward(bad, x, lg, y, ws)
    assert e.value.status == qmoe.ERR_INVALID_ARG
    bad = case.layer()
    bad.E = 300
    with pytest.raises(qmoe.QmoeError) as e:
        qmoe.forward(bad, x, lg, y, ws)
    assert e.value.status == qmoe.ERR_UNSUPPORTED


# ------------------------------------------------------------------ grouped (tcgen05) path

@pytest.mark.parametrize("fc1,fc2", [("int2", "int4"), ("int4", "int4"), ("int2", "int2")])
def test_forward_grouped_forced(qm, fc1, fc2):
    """Every expert on the tcgen05 path (including experts with a single token)."""
    from skinny_gemm_top_b200 import qmoe
    cfg = small_cfg(synth.PREFILL, E=16, k=4, H=256, I=192, fc1_fmt=fc1, fc2_fmt=fc2)
    case = MoECase(cfg, seed=12)
    T = 90
    x = synth.tokens(cfg.H, 12, T)
    lg = synth.router_logits(cfg, 12, T)
    y = case.run(x, lg, path=qmoe.PATH_GROUPED)
    st = qmoe.get_stats()
    assert st.grouped_launches == 2 and st.last_path == qmoe.PATH_GROUPED
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, f"grouped {fc1}/{fc2}")


def test_forward_auto_mixes_paths(qm):
    """Zipf-skewed routing: hot experts exceed the small-M chunk and take the
    grouped path, cold ones stay on the small-M path; one token tile spans
    more than 256 tokens."""
    from skinny_gemm_top_b200 import qmoe
    cfg = small_cfg(synth.PREFILL, E=8, k=2, H=384, I=256)
    case = MoECase(cfg, seed=13)
    T = 400
    x = synth.tokens(cfg.H, 13, T)
    lg = synth.router_logits(cfg, 13, T)
    ids, _, _, _ = Q.route(lg, cfg.k)
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    assert counts.max() > 256 and counts.min() <= 32
    y = case.run(x, lg)
    st = qmoe.get_stats()
    assert st.grouped_launches == 2 and st.small_launches == 2
    ref = Q.moe_forward(Q.bf16_bits_to_f64(x), lg, cfg.k, case.bank)
    _close(y, ref, "auto")
    y2 = case.run(x, lg, path=qmoe.PATH_SMALL_M)
    assert qmoe.get_stats().grouped_launches == 0
    _close(y2, ref, "small-M forced")


@pytest.mark.slow
def test_forward_prefill_full_size_sampled(qm):
    """Prefill layer at full size: T=4096, H=2048, I=768, 128 experts top-8,
    expert biases, Zipf(1.1) router offsets, row-tiled within 256 MiB."""
    from skinny_gemm_top_b200 import qmoe
    cfg = synth.PREFILL
    case = MoECase(cfg, seed=14)
    T = 4096
    x = synth.tokens(cfg.H, 14, T)
    lg = synth.router_logits(cfg, 14, T)
    y = case.run(x, lg, ws_bytes=256 << 20)
    st = qmoe.get_stats()
    assert st.row_tiles >= 2 and st.grouped_launches >= 2
    pick = np.random.default_rng(1).choice(T, 6, replace=False)
    ref = np.stack([Q.moe_token(Q.bf16_bits_to_f64(x[t]), lg[t], cfg.k, case.bank) for t in pick])
    _close(y[pick], ref, "prefill full size")
