"""Python binding of libaqnf4 (ctypes): argument marshalling only.

Every function named ``aqnf4_*`` here calls the C entry point of the same name; tensors
are passed by ``data_ptr()``, streams by their CUDA handle.  Every step of the NF4 pass
runs in the library's CUDA kernels: there is no fallback of any kind, and loading fails
loudly when the library has not been built (``python -m quantized_lora_setup_b200.build``).

The helpers below the raw bindings (``quantize``, ``score_layers`` ...) only allocate the
output tensors with torch and then call the bindings.
"""
import ctypes
import os
from typing import List, Optional, Sequence

import torch

from .build import LIB

AQNF4_OK = 0
AQNF4_ERR_INVALID_ARG = 1
AQNF4_ERR_ALIGNMENT = 2
AQNF4_ERR_DTYPE = 3
AQNF4_ERR_NONFINITE = 4
AQNF4_ERR_CUDA = 5
AQNF4_ERR_TIMEOUT = 6
AQNF4_ERR_WORKSPACE = 7

AQNF4_F16 = 0
AQNF4_BF16 = 1
AQNF4_SCORE_DQ_ABSMAX = 1  # aqnf4_layer.flags
AQNF4_SCORE_DQ_CENTERED = 2
AQNF4_BLOCKS_BY_DEPTH = 0  # aqnf4_select_blocks orders
AQNF4_BLOCKS_BY_ERROR = 1

_DT_CODE = {torch.float16: AQNF4_F16, torch.bfloat16: AQNF4_BF16}
_CODE_DT = {AQNF4_F16: torch.float16, AQNF4_BF16: torch.bfloat16}

BLOCK = 64
DQ_BLOCK = 256


class Aqnf4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class aqnf4_layer(ctypes.Structure):
    """Mirror of the C struct aqnf4_layer (see include/aqnf4.h)."""

    _fields_ = [
        ("w", ctypes.c_void_p),
        ("numel", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("flags", ctypes.c_int32),
        ("packed", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("codes8", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
    ]


_lib = None


def library() -> ctypes.CDLL:
    """Load libaqnf4.so (raises if it was never built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise ImportError(
            f"libaqnf4.so is missing ({LIB}); build it with "
            "`python -m quantized_lora_setup_b200.build`")
    lib = ctypes.CDLL(LIB)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    st = ctypes.c_int
    lib.aqnf4_status_string.argtypes = [st]
    lib.aqnf4_status_string.restype = ctypes.c_char_p
    lib.aqnf4_codebook.argtypes = [ctypes.c_double, P, P]
    lib.aqnf4_codebook.restype = st
    lib.aqnf4_quantize.argtypes = [P, i32, i64, P, P, P, P]
    lib.aqnf4_quantize.restype = st
    lib.aqnf4_double_quant.argtypes = [P, i64, P, P, P, P]
    lib.aqnf4_double_quant.restype = st
    lib.aqnf4_dequantize.argtypes = [P, P, P, P, i64, i32, P, P]
    lib.aqnf4_dequantize.restype = st
    lib.aqnf4_double_quant_centered.argtypes = [P, i64, P, P, P, P, P]
    lib.aqnf4_double_quant_centered.restype = st
    lib.aqnf4_dequantize_centered.argtypes = [P, P, P, P, i64, i32, P, P]
    lib.aqnf4_dequantize_centered.restype = st
    lib.aqnf4_workspace_size.argtypes = [P, i32]
    lib.aqnf4_workspace_size.restype = ctypes.c_size_t
    lib.aqnf4_layer_error.argtypes = [P, i32, P, ctypes.c_size_t, P, P, P, P, P]
    lib.aqnf4_layer_error.restype = st
    lib.aqnf4_layer_error_noalloc.argtypes = [P, i32, P, P, P, P, P]
    lib.aqnf4_layer_error_noalloc.restype = st
    lib.aqnf4_select_topk.argtypes = [P, P, i32, i64, i32, P, P, P]
    lib.aqnf4_select_topk.restype = st
    lib.aqnf4_selftest_wait_timeout.argtypes = [i64, P, P, P]
    lib.aqnf4_selftest_wait_timeout.restype = st
    lib.aqnf4_selftest_division.argtypes = [P, P, i64, P, P]
    lib.aqnf4_selftest_division.restype = st
    lib.aqnf4_nf4_linear.argtypes = [P, i32, i64, i64, P, P, P, i64, P, i32, P, P]
    lib.aqnf4_nf4_linear.restype = st
    lib.aqnf4_nf4_linear_splits.argtypes = [i64, i64, i64]
    lib.aqnf4_nf4_linear_splits.restype = i32
    lib.aqnf4_select_blocks.argtypes = [P, P, P, P, i32, i32, i64, i32, P, P, P, P, P]
    lib.aqnf4_select_blocks.restype = st
    lib.aqnf4_slot_tables.argtypes = [P, P, P]
    lib.aqnf4_slot_tables.restype = st
    lib.aqnf4_cost_bytes.argtypes = [i64]
    lib.aqnf4_cost_bytes.restype = i64
    lib.aqnf4_launch_count.argtypes = []
    lib.aqnf4_launch_count.restype = ctypes.c_uint64
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return library().aqnf4_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != AQNF4_OK:
        raise Aqnf4Error(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _req(t: Optional[torch.Tensor], name: str, dtypes, min_numel: int = 0,
         optional: bool = False) -> None:
    """Checks the C ABI cannot make on bare pointers, done before any launch: a CUDA tensor,
    contiguous, of an accepted dtype (None: any; the library checks 16-bit formats itself)
    and holding at least min_numel elements.  Raises ValueError."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name}: required")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {min_numel} needed")


def _storage_sizes(n: int):
    """(packed bytes, blocks, DQ scales) of n weights."""
    nb = (n + BLOCK - 1) // BLOCK
    return (n + 1) // 2, nb, (nb + DQ_BLOCK - 1) // DQ_BLOCK


def dtype_code(dtype: torch.dtype) -> int:
    try:
        return _DT_CODE[dtype]
    except KeyError:
        raise Aqnf4Error(AQNF4_ERR_DTYPE, "dtype") from None


# ---------------------------------------------------------------- raw bindings


def aqnf4_codebook(p_max: float = 0.0):
    """(levels float32[16], mids float32[15]) as numpy arrays, from the library."""
    import numpy as np
    levels = np.zeros(16, np.float32)
    mids = np.zeros(15, np.float32)
    _check(library().aqnf4_codebook(p_max, levels.ctypes.data_as(ctypes.c_void_p),
                                    mids.ctypes.data_as(ctypes.c_void_p)), "aqnf4_codebook")
    return levels, mids


def aqnf4_quantize(w: torch.Tensor, packed: Optional[torch.Tensor], absmax: Optional[torch.Tensor],
                   dev_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    npk, nb, _ = _storage_sizes(w.numel())
    _req(w, "w", None)
    _req(packed, "packed", (torch.uint8,), npk, optional=True)
    _req(absmax, "absmax", (torch.float32,), nb, optional=True)
    _req(dev_flag, "dev_flag", (torch.int32,), 1, optional=True)
    _check(library().aqnf4_quantize(_ptr(w), dtype_code(w.dtype), w.numel(), _ptr(packed),
                                    _ptr(absmax), _ptr(dev_flag), _stream(stream)),
           "aqnf4_quantize")


def aqnf4_double_quant(absmax: torch.Tensor, codes8: torch.Tensor, scales: torch.Tensor,
                       dev_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    nb = absmax.numel()
    _req(absmax, "absmax", (torch.float32,))
    _req(codes8, "codes8", (torch.uint8,), nb)
    _req(scales, "scales", (torch.float32,), (nb + DQ_BLOCK - 1) // DQ_BLOCK)
    _req(dev_flag, "dev_flag", (torch.int32,), 1, optional=True)
    _check(library().aqnf4_double_quant(_ptr(absmax), absmax.numel(), _ptr(codes8), _ptr(scales),
                                        _ptr(dev_flag), _stream(stream)), "aqnf4_double_quant")


def aqnf4_dequantize(packed: torch.Tensor, codes8: Optional[torch.Tensor],
                     scales: Optional[torch.Tensor], absmax: Optional[torch.Tensor], n: int,
                     out: torch.Tensor, stream=None) -> None:
    npk, nb, nsc = _storage_sizes(n)
    _req(packed, "packed", (torch.uint8,), npk)
    _req(codes8, "codes8", (torch.uint8,), nb, optional=True)
    _req(scales, "scales", (torch.float32,), nsc, optional=True)
    _req(absmax, "absmax", (torch.float32,), nb, optional=True)
    _req(out, "out", None, n)
    _check(library().aqnf4_dequantize(_ptr(packed), _ptr(codes8), _ptr(scales), _ptr(absmax), n,
                                      dtype_code(out.dtype), _ptr(out), _stream(stream)),
           "aqnf4_dequantize")


def aqnf4_double_quant_centered(absmax: torch.Tensor, codes8: torch.Tensor,
                                scales: torch.Tensor, means: torch.Tensor,
                                dev_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    nb = absmax.numel()
    nd = (nb + DQ_BLOCK - 1) // DQ_BLOCK
    _req(absmax, "absmax", (torch.float32,))
    _req(codes8, "codes8", (torch.uint8,), nb)
    _req(scales, "scales", (torch.float32,), nd)
    _req(means, "means", (torch.float32,), nd)
    _req(dev_flag, "dev_flag", (torch.int32,), 1, optional=True)
    _check(library().aqnf4_double_quant_centered(_ptr(absmax), nb, _ptr(codes8), _ptr(scales),
                                                 _ptr(means), _ptr(dev_flag), _stream(stream)),
           "aqnf4_double_quant_centered")


def aqnf4_dequantize_centered(packed: torch.Tensor, codes8: torch.Tensor, scales: torch.Tensor,
                              means: torch.Tensor, n: int, out: torch.Tensor,
                              stream=None) -> None:
    npk, nb, nsc = _storage_sizes(n)
    _req(packed, "packed", (torch.uint8,), npk)
    _req(codes8, "codes8", (torch.uint8,), nb)
    _req(scales, "scales", (torch.float32,), nsc)
    _req(means, "means", (torch.float32,), nsc)
    _req(out, "out", None, n)
    _check(library().aqnf4_dequantize_centered(_ptr(packed), _ptr(codes8), _ptr(scales),
                                               _ptr(means), n, dtype_code(out.dtype), _ptr(out),
                                               _stream(stream)), "aqnf4_dequantize_centered")


def make_layers(layers: Sequence[dict]):
    """ctypes array of aqnf4_layer from dicts with keys w, packed, absmax, codes8, scales
    and optionally flags (AQNF4_SCORE_* bits)."""
    arr = (aqnf4_layer * len(layers))()
    for i, d in enumerate(layers):
        w = d["w"]
        _req(w, f"layers[{i}].w", None)
        npk, nb, nsc = _storage_sizes(w.numel())
        for key, dt, need in (("packed", torch.uint8, npk), ("absmax", torch.float32, nb),
                              ("codes8", torch.uint8, nb), ("scales", torch.float32, nsc)):
            _req(d.get(key), f"layers[{i}].{key}", (dt,), need, optional=True)
        arr[i].w = w.data_ptr()
        arr[i].numel = w.numel()
        arr[i].dtype = dtype_code(w.dtype)
        arr[i].flags = int(d.get("flags", 0))
        for key in ("packed", "absmax", "codes8", "scales"):
            t = d.get(key)
            setattr(arr[i], key, None if t is None else t.data_ptr())
    return arr


def aqnf4_workspace_size(layers) -> int:
    arr = layers if isinstance(layers, ctypes.Array) else make_layers(layers)
    return int(library().aqnf4_workspace_size(arr, len(arr)))


def _check_outputs(L, sq_err, sq_w, rel_err, dev_flag):
    _req(sq_err, "sq_err", (torch.float64,), L, optional=True)
    _req(sq_w, "sq_w", (torch.float64,), L, optional=True)
    _req(rel_err, "rel_err", (torch.float32,), L, optional=True)
    _req(dev_flag, "dev_flag", (torch.int32,), 1, optional=True)


def aqnf4_layer_error(layers, workspace: torch.Tensor, sq_err: Optional[torch.Tensor],
                      sq_w: Optional[torch.Tensor], rel_err: Optional[torch.Tensor],
                      dev_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    arr = layers if isinstance(layers, ctypes.Array) else make_layers(layers)
    _req(workspace, "workspace", None)
    _check_outputs(len(arr), sq_err, sq_w, rel_err, dev_flag)
    nbytes = workspace.numel() * workspace.element_size()
    _check(library().aqnf4_layer_error(arr, len(arr), _ptr(workspace), nbytes, _ptr(sq_err),
                                       _ptr(sq_w), _ptr(rel_err), _ptr(dev_flag),
                                       _stream(stream)), "aqnf4_layer_error")


def aqnf4_layer_error_noalloc(layers, sq_err: Optional[torch.Tensor],
                              sq_w: Optional[torch.Tensor], rel_err: Optional[torch.Tensor],
                              dev_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """aqnf4_layer_error with the library's built-in scratch instead of a workspace."""
    arr = layers if isinstance(layers, ctypes.Array) else make_layers(layers)
    _check_outputs(len(arr), sq_err, sq_w, rel_err, dev_flag)
    _check(library().aqnf4_layer_error_noalloc(arr, len(arr), _ptr(sq_err), _ptr(sq_w),
                                               _ptr(rel_err), _ptr(dev_flag), _stream(stream)),
           "aqnf4_layer_error_noalloc")


def aqnf4_select_topk(rel_err: torch.Tensor, cost_bytes: torch.Tensor, budget_bytes: int,
                      k_cap: int, sel_idx: torch.Tensor, k_out: torch.Tensor,
                      stream=None) -> None:
    L = rel_err.numel()
    _req(rel_err, "rel_err", (torch.float32,))
    _req(cost_bytes, "cost_bytes", (torch.int64,), L)
    _req(sel_idx, "sel_idx", (torch.int32,), L)
    _req(k_out, "k_out", (torch.int32,), 1)
    _check(library().aqnf4_select_topk(_ptr(rel_err), _ptr(cost_bytes), rel_err.numel(),
                                       int(budget_bytes), int(k_cap), _ptr(sel_idx), _ptr(k_out),
                                       _stream(stream)), "aqnf4_select_topk")


def aqnf4_selftest_wait_timeout(timeout_ns: int, dev_flag: torch.Tensor,
                                waited_ns: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(library().aqnf4_selftest_wait_timeout(int(timeout_ns), _ptr(dev_flag), _ptr(waited_ns),
                                                 _stream(stream)), "aqnf4_selftest_wait_timeout")


def aqnf4_selftest_division(a: torch.Tensor, s: torch.Tensor, out: torch.Tensor,
                            stream=None) -> None:
    """out[i] = (short reciprocal of a[i], __frcp_rn(a[i]), short quotient a[i]/s[i],
    __fdiv_rn(a[i], s[i])); out is float32 (n, 4)."""
    n = a.numel()
    _req(a, "a", (torch.float32,))
    _req(s, "s", (torch.float32,), n)
    _req(out, "out", (torch.float32,), 4 * n)
    _check(library().aqnf4_selftest_division(_ptr(a), _ptr(s), n, _ptr(out), _stream(stream)),
           "aqnf4_selftest_division")


def aqnf4_nf4_linear(x: torch.Tensor, packed: torch.Tensor, codes8: torch.Tensor,
                     scales: torch.Tensor, N: int, y: torch.Tensor,
                     dev_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """y (M x N) = x (M x K) w_hat^T for the N x K layer stored as packed + codes8 + scales;
    y may be float32 or x's dtype."""
    if x.dim() != 2:
        raise ValueError("x must be M x K")
    M, K = x.shape
    out_f32 = 1 if y.dtype == torch.float32 else 0
    if not out_f32 and y.dtype != x.dtype:
        raise ValueError("y must be float32 or x's dtype")
    npk, nb, nsc = _storage_sizes(N * K)
    _req(x, "x", None)
    _req(packed, "packed", (torch.uint8,), npk)
    _req(codes8, "codes8", (torch.uint8,), nb)
    _req(scales, "scales", (torch.float32,), nsc)
    _req(y, "y", None, M * N)
    _req(dev_flag, "dev_flag", (torch.int32,), 1, optional=True)
    _check(library().aqnf4_nf4_linear(_ptr(x), dtype_code(x.dtype), M, K, _ptr(packed),
                                      _ptr(codes8), _ptr(scales), N, _ptr(y), out_f32,
                                      _ptr(dev_flag), _stream(stream)), "aqnf4_nf4_linear")


def aqnf4_nf4_linear_splits(M: int, N: int, K: int) -> int:
    return int(library().aqnf4_nf4_linear_splits(M, N, K))


def aqnf4_select_blocks(sq_err: torch.Tensor, sq_w: torch.Tensor, block_of: torch.Tensor,
                        cost_bytes: torch.Tensor, num_blocks: int, budget_bytes: int, order: int,
                        block_rank: torch.Tensor, block_err: Optional[torch.Tensor],
                        k_out: torch.Tensor, stream=None,
                        dev_flag: Optional[torch.Tensor] = None) -> None:
    L = sq_err.numel()
    _req(sq_err, "sq_err", (torch.float64,))
    _req(sq_w, "sq_w", (torch.float64,), L)
    _req(block_of, "block_of", (torch.int32,), L)
    _req(cost_bytes, "cost_bytes", (torch.int64,), L)
    _req(block_rank, "block_rank", (torch.int32,), num_blocks)
    _req(block_err, "block_err", (torch.float32,), num_blocks, optional=True)
    _req(k_out, "k_out", (torch.int32,), 1)
    _req(dev_flag, "dev_flag", (torch.int32,), 1, optional=True)
    _check(library().aqnf4_select_blocks(_ptr(sq_err), _ptr(sq_w), _ptr(block_of),
                                         _ptr(cost_bytes), sq_err.numel(), num_blocks,
                                         budget_bytes, order, _ptr(block_rank), _ptr(block_err),
                                         _ptr(k_out), _ptr(dev_flag), _stream(stream)),
           "aqnf4_select_blocks")


def aqnf4_slot_tables():
    """(curve float32[2], slot_mid float32[32], slot_level float32[32]) of the fused pass."""
    import numpy as np
    curve = np.zeros(2, np.float32)
    slot_mid = np.zeros(32, np.float32)
    slot_level = np.zeros(32, np.float32)
    _check(library().aqnf4_slot_tables(curve.ctypes.data_as(ctypes.c_void_p),
                                       slot_mid.ctypes.data_as(ctypes.c_void_p),
                                       slot_level.ctypes.data_as(ctypes.c_void_p)),
           "aqnf4_slot_tables")
    return curve, slot_mid, slot_level


def aqnf4_cost_bytes(n: int) -> int:
    return int(library().aqnf4_cost_bytes(n))


def aqnf4_launch_count() -> int:
    return int(library().aqnf4_launch_count())


# ---------------------------------------------------------------- allocating helpers


def nblocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def nscales(n: int) -> int:
    return (nblocks(n) + DQ_BLOCK - 1) // DQ_BLOCK


def quantize(w: torch.Tensor, stream=None):
    """NF4-quantize one tensor: returns (packed uint8[ceil(n/2)], absmax float32[ceil(n/64)])."""
    n = w.numel()
    packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device=w.device)
    absmax = torch.empty(nblocks(n), dtype=torch.float32, device=w.device)
    aqnf4_quantize(w, packed, absmax, None, stream)
    return packed, absmax


def double_quant(absmax: torch.Tensor, stream=None):
    nb = absmax.numel()
    codes8 = torch.empty(nb, dtype=torch.uint8, device=absmax.device)
    scales = torch.empty((nb + DQ_BLOCK - 1) // DQ_BLOCK, dtype=torch.float32, device=absmax.device)
    aqnf4_double_quant(absmax, codes8, scales, None, stream)
    return codes8, scales


def double_quant_centered(absmax: torch.Tensor, stream=None):
    """(codes8, scales, means) of the mean-centred double quantization."""
    nb = absmax.numel()
    nd = (nb + DQ_BLOCK - 1) // DQ_BLOCK
    codes8 = torch.empty(nb, dtype=torch.uint8, device=absmax.device)
    scales = torch.empty(nd, dtype=torch.float32, device=absmax.device)
    means = torch.empty(nd, dtype=torch.float32, device=absmax.device)
    aqnf4_double_quant_centered(absmax, codes8, scales, means, None, stream)
    return codes8, scales, means


def dequantize(packed: torch.Tensor, n: int, dtype: torch.dtype = torch.bfloat16,
               codes8=None, scales=None, absmax=None, stream=None) -> torch.Tensor:
    out = torch.empty(n, dtype=dtype, device=packed.device)
    aqnf4_dequantize(packed, codes8, scales, absmax, n, out, stream)
    return out


class NF4Storage:
    """Device buffers of one layer's NF4 storage (packed nibbles + double-quantized absmax)."""

    def __init__(self, n: int, device, with_absmax: bool = False):
        self.n = n
        self.packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device=device)
        self.codes8 = torch.empty(nblocks(n), dtype=torch.uint8, device=device)
        self.scales = torch.empty(nscales(n), dtype=torch.float32, device=device)
        self.absmax = (torch.empty(nblocks(n), dtype=torch.float32, device=device)
                       if with_absmax else None)


def score_layers(weights: List[torch.Tensor], storages: Optional[List[NF4Storage]] = None,
                 stream=None, dq_score=False):
    """Run the fused quantize+score pass: returns (sq_err f64[L], sq_w f64[L], rel_err f32[L]).
    dq_score: score against the double-quantized constants -- True or "absmax" for the
    plain 8-bit DQ (AQNF4_SCORE_DQ_ABSMAX), "centered" for mean-centred DQ
    (AQNF4_SCORE_DQ_CENTERED)."""
    dev = weights[0].device
    L = len(weights)
    flags = {False: 0, None: 0, True: AQNF4_SCORE_DQ_ABSMAX, "absmax": AQNF4_SCORE_DQ_ABSMAX,
             "centered": AQNF4_SCORE_DQ_CENTERED}[dq_score]
    descs = []
    for i, w in enumerate(weights):
        d = {"w": w, "flags": flags}
        if storages is not None:
            s = storages[i]
            d.update(packed=s.packed, codes8=s.codes8, scales=s.scales, absmax=s.absmax)
        descs.append(d)
    arr = make_layers(descs)
    ws = torch.empty(max(aqnf4_workspace_size(arr), 256), dtype=torch.uint8, device=dev)
    sq_err = torch.empty(L, dtype=torch.float64, device=dev)
    sq_w = torch.empty(L, dtype=torch.float64, device=dev)
    rel = torch.empty(L, dtype=torch.float32, device=dev)
    aqnf4_layer_error(arr, ws, sq_err, sq_w, rel, None, stream)
    return sq_err, sq_w, rel


def select_topk(rel_err: torch.Tensor, cost_bytes: torch.Tensor, budget_bytes: int,
                k_cap: int = -1, stream=None):
    """Returns (ranking int32[L] on the device, k int32[1] on the device)."""
    L = rel_err.numel()
    sel = torch.empty(L, dtype=torch.int32, device=rel_err.device)
    k = torch.empty(1, dtype=torch.int32, device=rel_err.device)
    aqnf4_select_topk(rel_err, cost_bytes, budget_bytes, k_cap, sel, k, stream)
    return sel, k
