"""ctypes binding of the qmoe C ABI (``include/qmoe.h``).

Argument marshalling only: every step of the path runs in ``libqmoe.so``.
Device arguments are torch CUDA tensors (their ``data_ptr()`` is passed),
host arguments are numpy arrays.  A missing library raises at import time;
there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqmoe.so")

INT2, TERNARY, INT4 = 2, 3, 4
FMT = {"int2": INT2, "int4": INT4, "ternary": TERNARY}
ROWS_PLAIN, ROWS_GATE_UP, ROWS_KSPLIT = 0, 1, 2
PATH_AUTO, PATH_SMALL_M, PATH_GROUPED = 0, 1, 2
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_SCRATCH, ERR_CUDA, ERR_TIMEOUT, ERR_STATIC_SCRATCH = range(7)
STATIC_SCRATCH_BYTES = 8 << 20  # QMOE_STATIC_SCRATCH_BYTES


class QmoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} ({status})")


class Weights(C.Structure):
    _fields_ = [("fmt", C.c_int), ("block", C.c_int), ("row_order", C.c_int), ("codes", C.c_void_p),
                ("scales", C.c_void_p), ("bias", C.c_void_p), ("zeros", C.c_void_p)]


class Layer(C.Structure):
    _fields_ = [("H", C.c_int), ("I", C.c_int), ("E", C.c_int), ("k", C.c_int), ("n_shared", C.c_int),
                ("fc1", Weights), ("fc2", Weights), ("path", C.c_int), ("max_row_tile", C.c_int)]


class ChanLayer(C.Structure):
    _fields_ = [("H", C.c_int), ("I", C.c_int), ("E", C.c_int), ("k", C.c_int), ("n_shared", C.c_int),
                ("fmt1", C.c_int), ("fmt2", C.c_int), ("block", C.c_int), ("records", C.c_void_p),
                ("sketch", C.c_void_p), ("dn", C.c_void_p), ("signs", C.c_void_p)]


class Stats(C.Structure):
    _fields_ = [("last_path", C.c_int), ("row_tiles", C.c_int), ("row_tile_tokens", C.c_int),
                ("small_launches", C.c_int), ("grouped_launches", C.c_int), ("device_status", C.c_uint32)]


EXPORTS = {
    "qmoe_pack_size": [C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)],
    "qmoe_pack": [C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p],
    "qmoe_pack_affine": [C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                         C.c_void_p],
    "qmoe_unpack_host": [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                         C.c_void_p],
    "qmoe_dequant": [C.POINTER(Weights), C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p],
    "qmoe_route_workspace_size": [C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t)],
    "qmoe_route": [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                   C.c_void_p, C.c_size_t, C.c_void_p],
    "qmoe_workspace_size": [C.POINTER(Layer), C.c_int, C.POINTER(C.c_size_t)],
    "qmoe_forward": [C.POINTER(Layer), C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_size_t,
                     C.c_void_p],
    "qmoe_forward_static": [C.POINTER(Layer), C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p],
    "qmoe_linear_workspace_size": [C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t)],
    "qmoe_linear": [C.POINTER(Weights), C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                    C.c_size_t, C.c_void_p],
    "qmoe_get_stats": [C.POINTER(Stats)],
    "qmoe_clear_status": [],
    "qmoe_test_set_fault": [C.c_int, C.c_ulonglong],
    "qmoe_status_str": [C.c_int],
    "qmoe_trace_start": [C.c_int],
    "qmoe_trace_stop": [],
    "qmoe_trace_read": [C.c_int, C.POINTER(C.c_int), C.c_void_p, C.c_void_p],
    "qmoe_kernel_name": [C.c_int],
    "qmoe_chan_sizes": [C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)],
    "qmoe_chan_pack": [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                       C.c_void_p, C.c_void_p, C.c_void_p],
    "qmoe_chan_workspace_size": [C.POINTER(ChanLayer), C.c_int, C.c_int, C.POINTER(C.c_size_t)],
    "qmoe_chan_forward": [C.POINTER(ChanLayer), C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p],
}

if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m skinny_gemm_top_b200.build`")
_lib = C.CDLL(_LIB_PATH)
for _name, _args in EXPORTS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = C.c_char_p if _name in ("qmoe_status_str", "qmoe_kernel_name") else C.c_int


def lib() -> C.CDLL:
    return _lib


def lib_path() -> str:
    return _LIB_PATH


def status_str(status: int) -> str:
    return _lib.qmoe_status_str(int(status)).decode()


def _check(status: int, where: str):
    if status != OK:
        raise QmoeError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ---------------------------------------------------------------- host packing

def pack_size(fmt: int, rows: int, K: int, block: int):
    cb, sb = C.c_size_t(), C.c_size_t()
    _check(_lib.qmoe_pack_size(fmt, rows, K, block, C.byref(cb), C.byref(sb)), "qmoe_pack_size")
    return cb.value, sb.value


def pack(fmt: int, row_order: int, w_bits: np.ndarray, block: int):
    """Quantize + pack one bf16 matrix (uint16 bits [rows, K]) -> (codes u8, scales u8)."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    rows, K = w.shape
    cb, sb = pack_size(fmt, rows, K, block)
    codes = np.empty(cb, dtype=np.uint8)
    scales = np.empty(sb, dtype=np.uint8)
    _check(_lib.qmoe_pack(fmt, row_order, _ptr(w), rows, K, block, _ptr(codes), _ptr(scales)), "qmoe_pack")
    return codes, scales


def pack_affine(fmt: int, row_order: int, w_bits: np.ndarray, block: int):
    """Affine quantize + pack one bf16 matrix -> (codes u8, scales u8, zeros u8)."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    rows, K = w.shape
    cb, sb = pack_size(fmt, rows, K, block)
    codes = np.empty(cb, dtype=np.uint8)
    scales = np.empty(sb, dtype=np.uint8)
    zeros = np.empty(sb, dtype=np.uint8)
    _check(_lib.qmoe_pack_affine(fmt, row_order, _ptr(w), rows, K, block, _ptr(codes), _ptr(scales), _ptr(zeros)),
           "qmoe_pack_affine")
    return codes, scales, zeros


def pack_stack_affine(fmt: int, row_order: int, mats, block: int):
    """pack_affine for matrices back to back."""
    cs, ss, zs = [], [], []
    for m in mats:
        c, s, z = pack_affine(fmt, row_order, m, block)
        cs.append(c)
        ss.append(s)
        zs.append(z)
    return np.concatenate(cs), np.concatenate(ss), np.concatenate(zs)


def pack_stack(fmt: int, row_order: int, mats, block: int):
    """Pack matrices back to back (matrix e at e * codes_bytes)."""
    cs, ss = [], []
    for m in mats:
        c, s = pack(fmt, row_order, m, block)
        cs.append(c)
        ss.append(s)
    return np.concatenate(cs), np.concatenate(ss)


def unpack_host(fmt: int, row_order: int, codes: np.ndarray, scales: np.ndarray, rows: int, K: int, block: int):
    c = np.empty((rows, K), dtype=np.int8)
    s = np.empty((rows, K // block), dtype=np.uint16)
    _check(_lib.qmoe_unpack_host(fmt, row_order, _ptr(np.ascontiguousarray(codes)),
                                 _ptr(np.ascontiguousarray(scales)), rows, K, block, _ptr(c), _ptr(s)),
           "qmoe_unpack_host")
    return c, s


def chan_sizes(fmt1: int, fmt2: int, H: int, block: int):
    """(record_bytes, sketch_bytes) of the channel layer."""
    r, k = C.c_size_t(), C.c_size_t()
    _check(_lib.qmoe_chan_sizes(fmt1, fmt2, H, block, C.byref(r), C.byref(k)), "qmoe_chan_sizes")
    return r.value, k.value


def chan_pack(fmt1: int, fmt2: int, w1_bits: np.ndarray, w2_bits: np.ndarray, block: int, signs=None,
              sketch: bool = True):
    """Channel records of one expert (w1 [2I, H], w2 [H, I] bf16 bits) -> (records u8 [I * R],
    sketch u8 [I * SK] or None, dn float32 [I] or None)."""
    w1 = np.ascontiguousarray(w1_bits, dtype=np.uint16)
    w2 = np.ascontiguousarray(w2_bits, dtype=np.uint16)
    two_i, H = w1.shape
    I = two_i // 2
    R, SK = chan_sizes(fmt1, fmt2, H, block)
    rec = np.empty(I * R, dtype=np.uint8)
    sk = np.empty(I * SK, dtype=np.uint8) if sketch else None
    dn = np.empty(I, dtype=np.float32) if sketch else None
    sg = None if signs is None else np.ascontiguousarray(signs, dtype=np.float32)
    _check(_lib.qmoe_chan_pack(fmt1, fmt2, H, I, block, _ptr(w1), _ptr(w2), _ptr(sg), _ptr(rec), _ptr(sk), _ptr(dn)),
           "qmoe_chan_pack")
    return rec, sk, dn


# ---------------------------------------------------------------- device entry points

def make_weights(fmt: int, block: int, codes, scales, bias=None, row_order: int = ROWS_PLAIN, zeros=None) -> Weights:
    """Device weight set; row_order is the one the codes were packed with
    (GATE_UP for a layer's FC1, KSPLIT for its FC2, PLAIN for a single linear);
    zeros for affine codes (pack_affine)."""
    return Weights(fmt, block, row_order, _ptr(codes), _ptr(scales), _ptr(bias), _ptr(zeros))


def make_layer(H, I, E, k, n_shared, fc1: Weights, fc2: Weights, path=PATH_AUTO, max_row_tile=0) -> Layer:
    return Layer(H, I, E, k, n_shared, fc1, fc2, path, max_row_tile)


def dequant(w: Weights, rows: int, K: int, n_mats: int, out_f32=None, out_bf16=None, stream=None):
    _check(_lib.qmoe_dequant(C.byref(w), rows, K, n_mats, _ptr(out_f32), _ptr(out_bf16), _stream(stream)),
           "qmoe_dequant")


def route_workspace_size(T: int, E: int, k: int) -> int:
    b = C.c_size_t()
    _check(_lib.qmoe_route_workspace_size(T, E, k, C.byref(b)), "qmoe_route_workspace_size")
    return b.value


def route(logits, k: int, ids, weights, perm, offsets, ws=None, ws_bytes: int | None = None, stream=None):
    T, E = logits.shape
    nbytes = (0 if ws is None else ws.numel() * ws.element_size()) if ws_bytes is None else ws_bytes
    _check(_lib.qmoe_route(_ptr(logits), T, E, k, _ptr(ids), _ptr(weights), _ptr(perm), _ptr(offsets), _ptr(ws),
                           nbytes, _stream(stream)), "qmoe_route")


def workspace_size(layer: Layer, T: int) -> int:
    b = C.c_size_t()
    _check(_lib.qmoe_workspace_size(C.byref(layer), T, C.byref(b)), "qmoe_workspace_size")
    return b.value


def forward(layer: Layer, x, logits, y, ws, ws_bytes: int | None = None, stream=None):
    T = x.shape[0]
    nbytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.qmoe_forward(C.byref(layer), _ptr(x), _ptr(logits), T, _ptr(y), _ptr(ws), nbytes,
                             _stream(stream)), "qmoe_forward")


def forward_static(layer: Layer, x, logits, y, stream=None):
    """qmoe_forward with the library's fixed device scratch (no workspace, no allocation)."""
    _check(_lib.qmoe_forward_static(C.byref(layer), _ptr(x), _ptr(logits), x.shape[0], _ptr(y), _stream(stream)),
           "qmoe_forward_static")


def linear_workspace_size(N: int, K: int, M: int) -> int:
    b = C.c_size_t()
    _check(_lib.qmoe_linear_workspace_size(N, K, M, C.byref(b)), "qmoe_linear_workspace_size")
    return b.value


def linear(w: Weights, N: int, K: int, x, y, ws, ws_bytes: int | None = None, stream=None):
    M = x.shape[0]
    nbytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.qmoe_linear(C.byref(w), N, K, _ptr(x), M, _ptr(y), _ptr(ws), nbytes, _stream(stream)),
           "qmoe_linear")


def make_chan_layer(H, I, E, k, n_shared, fmt1, fmt2, block, records, sketch, dn, signs) -> ChanLayer:
    return ChanLayer(H, I, E, k, n_shared, fmt1, fmt2, block, _ptr(records), _ptr(sketch), _ptr(dn), _ptr(signs))


def chan_workspace_size(layer: ChanLayer, T: int, n_keep: int) -> int:
    b = C.c_size_t()
    _check(_lib.qmoe_chan_workspace_size(C.byref(layer), T, n_keep, C.byref(b)), "qmoe_chan_workspace_size")
    return b.value


def chan_forward(layer: ChanLayer, x, logits, n_keep: int, y, ws, sel=None, scores=None, ws_bytes: int | None = None,
                 stream=None):
    T = x.shape[0]
    nbytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    _check(_lib.qmoe_chan_forward(C.byref(layer), _ptr(x), _ptr(logits), T, n_keep, _ptr(y), _ptr(sel), _ptr(scores),
                                  _ptr(ws), nbytes, _stream(stream)), "qmoe_chan_forward")


def get_stats() -> Stats:
    s = Stats()
    _check(_lib.qmoe_get_stats(C.byref(s)), "qmoe_get_stats")
    return s


def clear_status():
    _check(_lib.qmoe_clear_status(), "qmoe_clear_status")


DEVICE_TIMEOUT, DEVICE_BAD_SEGMENT = 1, 2


def test_set_fault(inject: int, wait_limit_ns: int = 0):
    """Test hook: fault injection for the decode-layer kernel (qmoe.h)."""
    _check(_lib.qmoe_test_set_fault(inject, wait_limit_ns), "qmoe_test_set_fault")


# ---------------------------------------------------------------- tracing

def trace_start(cap: int):
    _check(_lib.qmoe_trace_start(cap), "qmoe_trace_start")


def trace_stop():
    _check(_lib.qmoe_trace_stop(), "qmoe_trace_stop")


def trace_read(cap: int = 1 << 16):
    """[(kernel name, ms)] of the recorded launches (synchronizes the device)."""
    n = C.c_int()
    ids = np.zeros(cap, dtype=np.int32)
    ms = np.zeros(cap, dtype=np.float32)
    _check(_lib.qmoe_trace_read(cap, C.byref(n), _ptr(ids), _ptr(ms)), "qmoe_trace_read")
    m = min(cap, n.value)
    return [(_lib.qmoe_kernel_name(int(i)).decode(), float(t)) for i, t in zip(ids[:m], ms[:m])]
