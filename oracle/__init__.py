"""CPU oracle for the per-layer NF4 pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  It wraps the plain-C oracle in ``aqnf4_oracle.c`` (built by
``oracle/build.py``) with numpy-facing helpers.  It shares no code with the CUDA path.

Weights are passed as numpy ``uint16`` bit patterns plus a dtype code
(``F16 = 0``, ``BF16 = 1``), so both 16-bit formats travel the same way.
"""
import ctypes

import numpy as np

from . import build as _build

F16 = 0
BF16 = 1

_lib = None


def load():
    """Build (if stale) and load the oracle library."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    lib.oracle_default_pmax.restype = ctypes.c_double
    lib.oracle_codebook.argtypes = [ctypes.c_double, P, P]
    lib.oracle_codebook.restype = ctypes.c_int
    lib.oracle_quantize.argtypes = [P, ctypes.c_int, i64, P, P, P, P, P]
    lib.oracle_quantize.restype = None
    lib.oracle_layer_error.argtypes = [P, ctypes.c_int, i64, P, P, P, P, P]
    lib.oracle_layer_error.restype = None
    lib.oracle_layer_error_dq.argtypes = [P, ctypes.c_int, i64, P, P, P, P, P]
    lib.oracle_layer_error_dq.restype = ctypes.c_int
    lib.oracle_select_blocks.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, i64,
                                         ctypes.c_int, P, P, P]
    lib.oracle_select_blocks.restype = ctypes.c_int
    lib.oracle_nf4_linear.argtypes = [P, ctypes.c_int, i64, i64, P, P, P, i64, ctypes.c_int,
                                      P, P, P]
    lib.oracle_nf4_linear.restype = ctypes.c_int
    lib.oracle_double_quant.argtypes = [P, i64, P, P, P]
    lib.oracle_double_quant.restype = None
    lib.oracle_dequantize.argtypes = [P, P, P, P, i64, ctypes.c_int, P, P]
    lib.oracle_dequantize.restype = None
    lib.oracle_double_quant_centered.argtypes = [P, i64, P, P, P, P]
    lib.oracle_double_quant_centered.restype = None
    lib.oracle_dequantize_centered.argtypes = [P, P, P, P, i64, ctypes.c_int, P, P]
    lib.oracle_dequantize_centered.restype = None
    lib.oracle_layer_error_dqc.argtypes = [P, ctypes.c_int, i64, P, P, P, P, P]
    lib.oracle_layer_error_dqc.restype = ctypes.c_int
    lib.oracle_cost_bytes.argtypes = [i64]
    lib.oracle_cost_bytes.restype = i64
    lib.oracle_select_topk.argtypes = [P, P, ctypes.c_int, i64, ctypes.c_int, P, P]
    lib.oracle_select_topk.restype = ctypes.c_int
    lib.oracle_f32_to_dtype_bits.argtypes = [ctypes.c_float, ctypes.c_int]
    lib.oracle_f32_to_dtype_bits.restype = ctypes.c_uint16
    lib.oracle_dtype_bits_to_f32.argtypes = [ctypes.c_uint16, ctypes.c_int]
    lib.oracle_dtype_bits_to_f32.restype = ctypes.c_float
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_pmax() -> float:
    return load().oracle_default_pmax()


def codebook(p_max: float = None):
    """(levels float32[16], midpoints float32[15]) of the NF4 codebook."""
    lib = load()
    if p_max is None:
        p_max = lib.oracle_default_pmax()
    levels = np.zeros(16, np.float32)
    mids = np.zeros(15, np.float32)
    if lib.oracle_codebook(p_max, _ptr(levels), _ptr(mids)) != 0:
        raise ValueError("p_max must lie in (1/2, 1)")
    return levels, mids


def _as_bits(w):
    w = np.ascontiguousarray(w)
    if w.dtype == np.float16:
        return w.view(np.uint16)
    if w.dtype != np.uint16:
        raise TypeError("weights must be float16 or uint16 bit patterns")
    return w


def quantize(w, dtype, book=None):
    """Blockwise NF4: returns (packed uint8[ceil(n/2)], absmax float32[ceil(n/64)], nonfinite)."""
    w = _as_bits(w).reshape(-1)
    n = w.size
    levels, mids = book if book is not None else codebook()
    packed = np.zeros((n + 1) // 2, np.uint8)
    absmax = np.zeros((n + 63) // 64, np.float32)
    flag = np.zeros(1, np.int32)
    load().oracle_quantize(_ptr(w), dtype, n, _ptr(levels), _ptr(mids), _ptr(packed),
                           _ptr(absmax), _ptr(flag))
    return packed, absmax, bool(flag[0])


def layer_error(w, dtype, book=None):
    """(sq_err, sq_w, rel_err) of one layer."""
    w = _as_bits(w).reshape(-1)
    levels, mids = book if book is not None else codebook()
    se = np.zeros(1, np.float64)
    sw = np.zeros(1, np.float64)
    rel = np.zeros(1, np.float32)
    load().oracle_layer_error(_ptr(w), dtype, w.size, _ptr(levels), _ptr(mids), _ptr(se),
                              _ptr(sw), _ptr(rel))
    return float(se[0]), float(sw[0]), float(rel[0])


def layer_error_dq(w, dtype, book=None):
    """(sq_err, sq_w, rel_err) of one layer reconstructed from double-quantized constants."""
    w = _as_bits(w).reshape(-1)
    levels, mids = book if book is not None else codebook()
    se = np.zeros(1, np.float64)
    sw = np.zeros(1, np.float64)
    rel = np.zeros(1, np.float32)
    if load().oracle_layer_error_dq(_ptr(w), dtype, w.size, _ptr(levels), _ptr(mids), _ptr(se),
                                    _ptr(sw), _ptr(rel)) != 0:
        raise MemoryError("oracle_layer_error_dq")
    return float(se[0]), float(sw[0]), float(rel[0])


def double_quant(absmax):
    """8-bit / 256-block double quantization: (codes8 uint8[nb], scales float32[ceil(nb/256)], nonfinite)."""
    absmax = np.ascontiguousarray(absmax, np.float32).reshape(-1)
    nb = absmax.size
    codes8 = np.zeros(nb, np.uint8)
    scales = np.zeros((nb + 255) // 256, np.float32)
    flag = np.zeros(1, np.int32)
    load().oracle_double_quant(_ptr(absmax), nb, _ptr(codes8), _ptr(scales), _ptr(flag))
    return codes8, scales, bool(flag[0])


def dequantize(packed, n, out_dtype, codes8=None, scales=None, absmax=None, book=None):
    """NF4 -> 16-bit bit patterns (uint16[n]); DQ constants if codes8 is given, else absmax."""
    levels, _ = book if book is not None else codebook()
    packed = np.ascontiguousarray(packed, np.uint8)
    out = np.zeros(n, np.uint16)
    if codes8 is not None:
        codes8 = np.ascontiguousarray(codes8, np.uint8)
        scales = np.ascontiguousarray(scales, np.float32)
    else:
        absmax = np.ascontiguousarray(absmax, np.float32)
    load().oracle_dequantize(_ptr(packed), _ptr(codes8), _ptr(scales), _ptr(absmax), n,
                             out_dtype, _ptr(levels), _ptr(out))
    return out


def cost_bytes(n: int) -> int:
    return int(load().oracle_cost_bytes(n))


def select_topk(rel_err, cost, budget: int, k_cap: int = -1):
    """Kept layer indices in rank order (list of int)."""
    e = np.ascontiguousarray(rel_err, np.float32)
    c = np.ascontiguousarray(cost, np.int64)
    L = e.size
    sel = np.zeros(max(L, 1), np.int32)
    k = np.zeros(1, np.int32)
    if load().oracle_select_topk(_ptr(e), _ptr(c), L, int(budget), int(k_cap), _ptr(sel),
                                 _ptr(k)) != 0:
        raise ValueError("invalid selection arguments")
    return [int(i) for i in sel[: k[0]]]


def nf4_linear(x_bits, x_dtype, packed, codes8, scales, N: int, w_dtype, book=None):
    """(y float64[M, N], yabs float64[M, N]) of y = x w_hat^T for x (M x K 16-bit bit patterns)
    and the N x K layer stored as packed codes + codes8 + scales."""
    levels, _ = book if book is not None else codebook()
    x = np.ascontiguousarray(x_bits, np.uint16)
    M, K = x.shape
    y = np.zeros((M, N), np.float64)
    yabs = np.zeros((M, N), np.float64)
    if load().oracle_nf4_linear(_ptr(x), x_dtype, M, K, _ptr(np.ascontiguousarray(packed, np.uint8)),
                                _ptr(np.ascontiguousarray(codes8, np.uint8)),
                                _ptr(np.ascontiguousarray(scales, np.float32)), N, w_dtype,
                                _ptr(levels), _ptr(y), _ptr(yabs)) != 0:
        raise MemoryError("oracle_nf4_linear")
    return y, yabs


BLOCKS_BY_DEPTH = 0
BLOCKS_BY_ERROR = 1


def select_blocks(sq_err, sq_w, block_of, cost, num_blocks: int, budget: int, order: int):
    """(ranking list[int], block scores float32[B], kept k) of the block-level selection."""
    se = np.ascontiguousarray(sq_err, np.float64)
    sw = np.ascontiguousarray(sq_w, np.float64)
    bo = np.ascontiguousarray(block_of, np.int32)
    c = np.ascontiguousarray(cost, np.int64)
    rank = np.zeros(max(num_blocks, 1), np.int32)
    err = np.zeros(max(num_blocks, 1), np.float32)
    k = np.zeros(1, np.int32)
    if load().oracle_select_blocks(_ptr(se), _ptr(sw), _ptr(bo), _ptr(c), se.size, num_blocks,
                                   int(budget), int(order), _ptr(rank), _ptr(err),
                                   _ptr(k)) != 0:
        raise ValueError("invalid block selection arguments")
    return [int(i) for i in rank[:num_blocks]], err[:num_blocks].copy(), int(k[0])


def f32_to_dtype_bits(values, dtype):
    lib = load()
    v = np.asarray(values, np.float32).reshape(-1)
    return np.array([lib.oracle_f32_to_dtype_bits(float(x), dtype) for x in v], np.uint16)


def dtype_bits_to_f32(bits, dtype):
    lib = load()
    b = np.asarray(bits, np.uint16).reshape(-1)
    return np.array([lib.oracle_dtype_bits_to_f32(int(x), dtype) for x in b], np.float32)


__all__ = ["F16", "BF16", "load", "default_pmax", "codebook", "quantize", "layer_error",
           "layer_error_dq", "select_blocks", "nf4_linear", "BLOCKS_BY_DEPTH", "BLOCKS_BY_ERROR",
           "double_quant", "dequantize", "cost_bytes", "select_topk", "f32_to_dtype_bits",
           "dtype_bits_to_f32"]



def double_quant_centered(absmax):
    """(codes8 uint8[nb], scales float32[nd], means float32[nd], nonfinite) of the mean-centred
    8-bit double quantization of the binary32 block constants."""
    a = np.ascontiguousarray(absmax, np.float32)
    nb = a.size
    nd = (nb + 255) // 256
    codes8 = np.zeros(nb, np.uint8)
    scales = np.zeros(nd, np.float32)
    means = np.zeros(nd, np.float32)
    bad = ctypes.c_int(0)
    load().oracle_double_quant_centered(_ptr(a), nb, _ptr(codes8), _ptr(scales), _ptr(means),
                                        ctypes.byref(bad))
    return codes8, scales, means, bool(bad.value)


def dequantize_centered(packed, n: int, out_dtype, codes8, scales, means, book=None):
    """uint16[n] 16-bit bit patterns of the NF4 tensor rebuilt from mean-centred DQ storage."""
    levels, _ = book if book is not None else codebook()
    out = np.zeros(n, np.uint16)
    load().oracle_dequantize_centered(_ptr(np.ascontiguousarray(packed, np.uint8)),
                                      _ptr(np.ascontiguousarray(codes8, np.uint8)),
                                      _ptr(np.ascontiguousarray(scales, np.float32)),
                                      _ptr(np.ascontiguousarray(means, np.float32)), n,
                                      out_dtype, _ptr(levels), _ptr(out))
    return out


def layer_error_dqc(w, dtype, book=None):
    """(sq_err, sq_w, rel_err) of one layer stored in NF4 with mean-centred DQ."""
    w = _as_bits(w).reshape(-1)
    levels, mids = book if book is not None else codebook()
    se = np.zeros(1, np.float64)
    sw = np.zeros(1, np.float64)
    rel = np.zeros(1, np.float32)
    if load().oracle_layer_error_dqc(_ptr(w), dtype, w.size, _ptr(levels), _ptr(mids), _ptr(se),
                                     _ptr(sw), _ptr(rel)) != 0:
        raise MemoryError("oracle_layer_error_dqc")
    return float(se[0]), float(sw[0]), float(rel[0])
