"""CPU tests of the C-ABI library: it loads, exports every declared symbol, and
its host packer agrees bit for bit with the oracle's quantizer."""
import os
import re

import numpy as np
import pytest

from oracle import qmoe_oracle as Q
from skinny_gemm_top_b200 import qmoe, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "qmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qmoe_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 12
    lib = qmoe.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(qmoe.EXPORTS), set(names) ^ set(qmoe.EXPORTS)


def test_status_strings():
    assert qmoe.status_str(qmoe.OK) == "ok"
    assert "workspace" in qmoe.status_str(qmoe.ERR_SCRATCH)


def _oracle_q(fmt, w_bits, block):
    w = Q.bf16_bits_to_f64(w_bits)
    if fmt == qmoe.TERNARY:
        return Q.quantize_ternary(w, block)
    return Q.quantize_sym(w, fmt, block)


@pytest.mark.parametrize("fmt,block,order", [
    (qmoe.INT2, 64, qmoe.ROWS_GATE_UP), (qmoe.INT4, 64, qmoe.ROWS_PLAIN), (qmoe.INT2, 128, qmoe.ROWS_PLAIN),
    (qmoe.INT4, 128, qmoe.ROWS_PLAIN), (qmoe.TERNARY, 64, qmoe.ROWS_GATE_UP), (qmoe.TERNARY, 64, qmoe.ROWS_PLAIN),
    (qmoe.INT2, 64, qmoe.ROWS_KSPLIT), (qmoe.INT4, 64, qmoe.ROWS_KSPLIT), (qmoe.INT4, 128, qmoe.ROWS_KSPLIT),
    (qmoe.TERNARY, 64, qmoe.ROWS_KSPLIT)])
def test_pack_matches_oracle_quantizer(fmt, block, order):
    rows, K = 48, 256
    w = synth.normal_bf16(9, 50, fmt * 10 + block, (rows, K), 0.02)
    codes, scales = qmoe.pack(fmt, order, w, block)
    cb, sb = qmoe.pack_size(fmt, rows, K, block)
    assert codes.nbytes == cb and scales.nbytes == sb
    c, s = qmoe.unpack_host(fmt, order, codes, scales, rows, K, block)
    oc, os_ = _oracle_q(fmt, w, block)
    assert np.array_equal(c, oc)
    assert np.array_equal(Q.bf16_bits_to_f64(s), os_)


@pytest.mark.parametrize("fmt,block,order", [
    (qmoe.INT2, 64, qmoe.ROWS_GATE_UP), (qmoe.INT4, 64, qmoe.ROWS_PLAIN), (qmoe.INT2, 128, qmoe.ROWS_PLAIN),
    (qmoe.INT4, 128, qmoe.ROWS_KSPLIT), (qmoe.INT2, 64, qmoe.ROWS_KSPLIT)])
def test_pack_affine_matches_oracle_quantizer(fmt, block, order):
    rows, K = 48, 256
    w = synth.normal_bf16(9, 51, fmt * 10 + block, (rows, K), 0.02)
    codes, scales, zeros = qmoe.pack_affine(fmt, order, w, block)
    cb, sb = qmoe.pack_size(fmt, rows, K, block)
    assert codes.nbytes == cb and scales.nbytes == sb and zeros.nbytes == sb
    c, s = qmoe.unpack_host(fmt, order, codes, scales, rows, K, block)
    _, z = qmoe.unpack_host(fmt, order, codes, zeros, rows, K, block)
    ou, os_, oz = Q.quantize_affine(Q.bf16_bits_to_f64(w), fmt, block)
    assert np.array_equal(c.astype(np.int64) + (1 << (fmt - 1)), ou.astype(np.int64))
    assert np.array_equal(Q.bf16_bits_to_f64(s), os_)
    assert np.array_equal(Q.bf16_bits_to_f64(z), oz)


def test_pack_affine_rejects_ternary():
    w = synth.normal_bf16(9, 52, 0, (16, 128), 0.02)
    with pytest.raises(qmoe.QmoeError):
        qmoe.pack_affine(qmoe.TERNARY, qmoe.ROWS_PLAIN, w, 64)


@pytest.mark.parametrize("fmt,block", [(qmoe.INT2, 64), (qmoe.INT4, 128), (qmoe.TERNARY, 64)])
def test_pack_matches_oracle_quantizer_tiny_and_subnormal(fmt, block):
    """Blocks scaled down to tiny normal and subnormal bf16 values: both
    quantizers give the same codes and scales (subnormal scales included)."""
    from cases import TINY_FACTORS, block_scaled_weights
    rows, K = 32, 896
    w = block_scaled_weights(5, rows, K, block, TINY_FACTORS)
    codes, scales = qmoe.pack(fmt, qmoe.ROWS_PLAIN, w, block)
    c, s = qmoe.unpack_host(fmt, qmoe.ROWS_PLAIN, codes, scales, rows, K, block)
    oc, os_ = _oracle_q(fmt, w, block)
    assert np.any((os_ > 0) & (os_ < 2.0 ** -126))
    assert np.array_equal(c, oc)
    assert np.array_equal(Q.bf16_bits_to_f64(s), os_)


def test_pack_sizes_are_the_format_densities():
    assert qmoe.pack_size(qmoe.INT2, 16, 5120, 128) == (16 * 5120 // 4, 16 * 40 * 2)
    assert qmoe.pack_size(qmoe.INT4, 16, 5120, 128) == (16 * 5120 // 2, 16 * 40 * 2)
    assert qmoe.pack_size(qmoe.TERNARY, 16, 2048, 64) == (16 * 2048 * 13 // 64, 16 * 32 * 2)


def test_pack_every_code_at_every_position():
    """Weights that quantize to known codes (exact multiples of a power-of-two
    scale) come back through the physical layout unchanged at every position."""
    rows, K = 32, 128
    g = np.random.default_rng(3)
    for fmt in (qmoe.INT2, qmoe.INT4):
        qmin, qmax = -(1 << (fmt - 1)), (1 << (fmt - 1)) - 1
        c = g.integers(qmin, qmax + 1, size=(rows, K))
        c[:, 0] = qmin
        c[:, 64] = qmin
        w = synth.f32_to_bf16_bits((c * 2.0 ** -7).astype(np.float32))
        for order in (qmoe.ROWS_PLAIN, qmoe.ROWS_GATE_UP, qmoe.ROWS_KSPLIT):
            codes, scales = qmoe.pack(fmt, order, w, 64)
            cc, ss = qmoe.unpack_host(fmt, order, codes, scales, rows, K, 64)
            assert np.array_equal(cc, c)
            assert np.all(Q.bf16_bits_to_f64(ss) == 2.0 ** -7)
    t = g.integers(-1, 2, size=(rows, K))
    w = synth.f32_to_bf16_bits((t * 0.25).astype(np.float32))
    codes, scales = qmoe.pack(qmoe.TERNARY, qmoe.ROWS_PLAIN, w, 64)
    cc, _ = qmoe.unpack_host(qmoe.TERNARY, qmoe.ROWS_PLAIN, codes, scales, rows, K, 64)
    assert np.array_equal(cc, t)


@pytest.mark.parametrize("args,status", [
    ((qmoe.INT2, 0, 15, 64, 64), qmoe.ERR_INVALID_ARG),      # rows % 16
    ((qmoe.INT2, 0, 16, 96, 64), qmoe.ERR_INVALID_ARG),      # K % 64
    ((qmoe.INT2, 0, 16, 64, 32), qmoe.ERR_UNSUPPORTED),      # block
    ((qmoe.TERNARY, 0, 16, 64, 64), qmoe.ERR_UNSUPPORTED),   # ternary needs K % 128
    ((7, 0, 16, 64, 64), qmoe.ERR_INVALID_ARG),              # format
    ((qmoe.INT4, 3, 16, 64, 64), qmoe.ERR_INVALID_ARG),      # row order
])
def test_pack_rejects_bad_arguments(args, status):
    fmt, order, rows, K, block = args
    w = np.zeros((max(rows, 1), K), dtype=np.uint16)
    codes = np.zeros(1 << 16, dtype=np.uint8)
    st = qmoe.lib().qmoe_pack(fmt, order, w.ctypes.data, rows, K, block, codes.ctypes.data, codes.ctypes.data)
    assert st == status


def test_fault_hook_validates_host_side():
    """The fault-injection hook only sets host state: no GPU needed."""
    from skinny_gemm_top_b200 import qmoe
    with pytest.raises(qmoe.QmoeError):
        qmoe.test_set_fault(5, 0)
    qmoe.test_set_fault(0, 0)


# ---------------------------------------------------------------- channel layer packing

def _codes_of(buf: np.ndarray, n: int, bits: int) -> np.ndarray:
    """Signed codes of a little-endian bit-packed row (stored c + 2^(bits-1))."""
    words = np.frombuffer(np.ascontiguousarray(buf).tobytes(), dtype="<u4")
    per = 32 // bits
    i = np.arange(n)
    u = (words[i // per] >> ((i % per) * bits).astype(np.uint32)) & ((1 << bits) - 1)
    return u.astype(np.int64) - (1 << (bits - 1))


@pytest.mark.parametrize("f1,f2,block,H,I", [(4, 4, 128, 512, 12), (2, 4, 64, 1024, 5), (2, 2, 128, 512, 3),
                                             (4, 4, 64, 2048, 3)])
def test_chan_pack_matches_oracle(f1, f2, block, H, I):
    from oracle import channel_select as CS
    w1 = synth.normal_bf16(21, 70, 0, (2 * I, H), 0.02)
    w2 = synth.normal_bf16(21, 71, 0, (H, I), 0.02)
    d = synth.rht_signs(21, H)
    R, SK = qmoe.chan_sizes(f1, f2, H, block)
    assert R % 16 == 0 and SK % 16 == 0
    rec, sk, dn = qmoe.chan_pack(f1, f2, w1, w2, block, d)
    w1d, w2d = Q.bf16_bits_to_f64(w1), Q.bf16_bits_to_f64(w2)
    cg, sg = Q.quantize_sym(w1d[0::2], f1, block)
    cu, su = Q.quantize_sym(w1d[1::2], f1, block)
    cd, sd, w2_hat = CS.quantize_down_columns(w2d, f2, block)
    tg, stg = CS.sketch_rows(w1d[0::2], d)
    tu, stu = CS.sketch_rows(w1d[1::2], d)
    SB, rb1, rb2 = H // block, H * f1 // 8, H * f2 // 8
    for j in range(I):
        r = rec[j * R:(j + 1) * R]
        assert np.array_equal(_codes_of(r[:rb1], H, f1), cg[j])
        assert np.array_equal(_codes_of(r[rb1:2 * rb1], H, f1), cu[j])
        assert np.array_equal(_codes_of(r[2 * rb1:2 * rb1 + rb2], H, f2), cd[j])
        sc = Q.bf16_bits_to_f64(np.frombuffer(r[2 * rb1 + rb2:2 * rb1 + rb2 + 6 * SB].tobytes(), dtype="<u2"))
        assert np.array_equal(sc, np.concatenate([sg[j], su[j], sd[j]]))
        assert not r[2 * rb1 + rb2 + 6 * SB:].any()
        s = sk[j * SK:(j + 1) * SK]
        assert np.array_equal(_codes_of(s[:H // 4], H, 2), tg[j])
        assert np.array_equal(_codes_of(s[H // 4:H // 2], H, 2), tu[j])
        ss = Q.bf16_bits_to_f64(np.frombuffer(s[H // 2:H // 2 + 4 * (H // 128)].tobytes(), dtype="<u2"))
        assert np.array_equal(ss, np.concatenate([stg[j], stu[j]]))
    want_dn = np.sqrt((w2_hat * w2_hat).sum(axis=0))
    assert np.allclose(dn, want_dn, rtol=1e-7, atol=0)


def test_chan_pack_without_sketch_and_bad_arguments():
    H, I = 512, 4
    w1 = synth.normal_bf16(3, 70, 1, (2 * I, H), 0.02)
    w2 = synth.normal_bf16(3, 71, 1, (H, I), 0.02)
    rec, sk, dn = qmoe.chan_pack(4, 4, w1, w2, 64, None, sketch=False)
    assert sk is None and dn is None and rec.size == I * qmoe.chan_sizes(4, 4, H, 64)[0]
    for args, st in (((3, 4, 512, 64), qmoe.ERR_INVALID_ARG), ((4, 4, 768, 64), qmoe.ERR_UNSUPPORTED),
                     ((4, 4, 256, 64), qmoe.ERR_UNSUPPORTED), ((4, 4, 4096, 64), qmoe.ERR_UNSUPPORTED),
                     ((4, 4, 512, 32), qmoe.ERR_UNSUPPORTED)):
        with pytest.raises(qmoe.QmoeError) as ei:
            qmoe.chan_sizes(*args)
        assert ei.value.status == st
    bad = np.ones(H, dtype=np.float32)
    bad[5] = 0.5
    with pytest.raises(qmoe.QmoeError) as ei:
        qmoe.chan_pack(4, 4, w1, w2, 64, bad)
    assert ei.value.status == qmoe.ERR_INVALID_ARG


def test_chan_workspace_size_validates_on_the_host():
    """qmoe_chan_workspace_size runs on the host: shapes and limits are checked without a device."""
    H, I, E, k = 2048, 1408, 64, 6
    # fake, 16-byte aligned device addresses: the size query never dereferences them
    layer = qmoe.make_chan_layer(H, I, E, k, 2, qmoe.INT4, qmoe.INT4, 128, None, None, None, None)
    layer.records = layer.sketch = layer.dn = layer.signs = 0x10000
    n = qmoe.chan_workspace_size(layer, 1, 1521)
    R, _ = qmoe.chan_sizes(qmoe.INT4, qmoe.INT4, H, 128)
    assert n >= 1 * k * I * 4 + 1521 * 4 + 4096 * 4 + H * 4 and n % 256 == 0
    assert qmoe.chan_workspace_size(layer, 8, 1521) > n
    for T, nk in ((0, 10), (9, 10), (1, k * I + 1), (1, -1)):
        with pytest.raises(qmoe.QmoeError) as ei:
            qmoe.chan_workspace_size(layer, T, nk)
        assert ei.value.status == qmoe.ERR_INVALID_ARG
    bad = qmoe.make_chan_layer(H, I, E, 9, 2, qmoe.INT4, qmoe.INT4, 128, None, None, None, None)  # k > 8
    bad.records = bad.sketch = bad.dn = bad.signs = 0x10000
    with pytest.raises(qmoe.QmoeError):
        qmoe.chan_workspace_size(bad, 1, 10)
    big = qmoe.make_chan_layer(H, 8192, E, k, 2, qmoe.INT4, qmoe.INT4, 128, None, None, None, None)  # k * I > 32768
    big.records = big.sketch = big.dn = big.signs = 0x10000
    with pytest.raises(qmoe.QmoeError) as ei:
        qmoe.chan_workspace_size(big, 1, 10)
    assert ei.value.status == qmoe.ERR_UNSUPPORTED
    unaligned = qmoe.make_chan_layer(H, I, E, k, 2, qmoe.INT4, qmoe.INT4, 128, None, None, None, None)
    unaligned.records, unaligned.sketch, unaligned.dn, unaligned.signs = 0x10008, 0x10000, 0x10000, 0x10000
    with pytest.raises(qmoe.QmoeError) as ei:
        qmoe.chan_workspace_size(unaligned, 1, 10)
    assert ei.value.status == qmoe.ERR_INVALID_ARG
