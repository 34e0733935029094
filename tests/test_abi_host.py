"""The C-ABI library on the host (no GPU): it loads, exports every declared symbol, its
host-only functions agree with the oracle, and argument checks fail before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
from quantized_lora_setup_b200 import aqnf4
from quantized_lora_setup_b200.build import INCLUDE, build

HEADER = os.path.join(INCLUDE, "aqnf4.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return aqnf4.library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"AQNF4_API\s+[\w\s\*]+?\b(aqnf4_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for required in ("aqnf4_codebook", "aqnf4_quantize", "aqnf4_double_quant",
                     "aqnf4_dequantize", "aqnf4_layer_error", "aqnf4_select_topk",
                     "aqnf4_workspace_size", "aqnf4_cost_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name


def test_library_codebook_matches_oracle_bit_for_bit(lib):
    lv, md = aqnf4.aqnf4_codebook()
    olv, omd = oracle.codebook()
    assert np.array_equal(lv.view(np.uint32), olv.view(np.uint32))
    assert np.array_equal(md.view(np.uint32), omd.view(np.uint32))
    for pm in (0.9, 0.99, 0.75):
        lv, md = aqnf4.aqnf4_codebook(pm)
        olv, omd = oracle.codebook(pm)
        assert np.array_equal(lv, olv) and np.array_equal(md, omd)
    with pytest.raises(aqnf4.Aqnf4Error):
        aqnf4.aqnf4_codebook(1.5)


def test_cost_bytes_matches_oracle(lib):
    for n in (1, 2, 63, 64, 65, 16383, 16384, 16385, 4096 * 11008, 5120 * 13824):
        assert aqnf4.aqnf4_cost_bytes(n) == oracle.cost_bytes(n)
    assert aqnf4.aqnf4_cost_bytes(0) == -1


class FakeTensor:
    """Just enough of a tensor for the binding's marshalling (never dereferenced)."""

    def __init__(self, addr, numel, dtype=None, itemsize=1):
        self._addr, self._numel, self.dtype, self._itemsize = addr, numel, dtype, itemsize

    def data_ptr(self):
        return self._addr

    def numel(self):
        return self._numel

    def element_size(self):
        return self._itemsize


def layer(addr=0x10000, numel=100, dtype=aqnf4.AQNF4_BF16, **kw):
    d = aqnf4.aqnf4_layer()
    d.w, d.numel, d.dtype, d.flags = addr, numel, dtype, kw.get("flags", 0)
    d.packed = kw.get("packed")
    d.absmax = kw.get("absmax")
    d.codes8 = kw.get("codes8")
    d.scales = kw.get("scales")
    return d


def test_workspace_size(lib):
    arr = (aqnf4.aqnf4_layer * 3)(layer(numel=1), layer(numel=16384), layer(numel=16385))
    assert lib.aqnf4_workspace_size(arr, 3) == 256  # 4 tiles x 16 B, rounded up to 256
    big = (aqnf4.aqnf4_layer * 1)(layer(numel=16384 * 100))
    assert lib.aqnf4_workspace_size(big, 1) == 1792
    assert lib.aqnf4_workspace_size(arr, 0) == 0
    assert lib.aqnf4_workspace_size(None, 3) == 0


def test_argument_checks_return_before_any_launch(lib):
    V = ctypes.c_void_p
    before = lib.aqnf4_launch_count()
    # quantize
    assert lib.aqnf4_quantize(None, 1, 100, V(0x10000), V(0x20000), None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_quantize(V(0x10000), 1, 0, None, None, None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_quantize(V(0x10000), 7, 10, None, None, None, None) == aqnf4.AQNF4_ERR_DTYPE
    assert lib.aqnf4_quantize(V(0x10008), 1, 10, None, None, None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    assert lib.aqnf4_quantize(V(0x10000), 1, 10, V(0x20004), None, None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # double quant
    assert lib.aqnf4_double_quant(None, 10, V(0x100), V(0x200), None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_double_quant(V(0x102), 10, V(0x100), V(0x200), None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # dequantize: codes8 requires scales, plain needs absmax
    assert lib.aqnf4_dequantize(V(0x100), V(0x200), None, None, 10, 1, V(0x300), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_dequantize(V(0x100), None, None, None, 10, 1, V(0x300), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_dequantize(V(0x100), None, None, V(0x400), 10, 5, V(0x300), None) == aqnf4.AQNF4_ERR_DTYPE
    assert lib.aqnf4_dequantize(V(0x100), None, None, V(0x400), 10, 1, V(0x308), None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # layer error
    one = (aqnf4.aqnf4_layer * 1)(layer())
    ws = V(0x100000)
    assert lib.aqnf4_layer_error(one, 0, ws, 4096, None, None, None, None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    for flags in (3, 4, -1):  # unknown bits, or both score flags at once
        bad = (aqnf4.aqnf4_layer * 1)(layer(flags=flags))
        assert lib.aqnf4_layer_error(bad, 1, ws, 4096, None, None, None, None, None) == \
            aqnf4.AQNF4_ERR_INVALID_ARG
    bad = (aqnf4.aqnf4_layer * 1)(layer(codes8=0x5000))
    assert lib.aqnf4_layer_error(bad, 1, ws, 4096, None, None, None, None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    bad = (aqnf4.aqnf4_layer * 1)(layer(dtype=9))
    assert lib.aqnf4_layer_error(bad, 1, ws, 4096, None, None, None, None, None) == aqnf4.AQNF4_ERR_DTYPE
    bad = (aqnf4.aqnf4_layer * 1)(layer(addr=0x10002))
    assert lib.aqnf4_layer_error(bad, 1, ws, 4096, None, None, None, None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    assert lib.aqnf4_layer_error(one, 1, None, 4096, None, None, None, None, None) == aqnf4.AQNF4_ERR_WORKSPACE
    assert lib.aqnf4_layer_error(one, 1, V(0x100010), 4096, None, None, None, None, None) == aqnf4.AQNF4_ERR_WORKSPACE
    assert lib.aqnf4_layer_error(one, 1, ws, 8, None, None, None, None, None) == aqnf4.AQNF4_ERR_WORKSPACE
    assert lib.aqnf4_layer_error(one, 1, ws, 4096, V(0x104), None, None, None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # select
    assert lib.aqnf4_select_topk(V(0x100), V(0x200), 5, -1, -1, V(0x300), V(0x400), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_select_topk(V(0x100), V(0x200), 0, 10, -1, V(0x300), V(0x400), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_select_topk(V(0x100), V(0x204), 5, 10, -1, V(0x300), V(0x400), None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # block selection
    args = [V(0x100), V(0x200), V(0x300), V(0x400), 5, 3, 10, aqnf4.AQNF4_BLOCKS_BY_DEPTH,
            V(0x500), None, V(0x600), None, None]
    for i, bad_value in ((0, None), (4, 0), (5, 0), (5, 2049), (6, -1), (7, 2), (10, None)):
        a = list(args)
        a[i] = bad_value
        assert lib.aqnf4_select_blocks(*a) == aqnf4.AQNF4_ERR_INVALID_ARG, (i, bad_value)
    a = list(args)
    a[0] = V(0x104)
    assert lib.aqnf4_select_blocks(*a) == aqnf4.AQNF4_ERR_ALIGNMENT
    a = list(args)
    a[11] = V(0x702)  # dev_flag not 4-byte aligned
    assert lib.aqnf4_select_blocks(*a) == aqnf4.AQNF4_ERR_ALIGNMENT
    # bounded-wait diagnostic
    assert lib.aqnf4_selftest_wait_timeout(0, V(0x100), None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_selftest_wait_timeout(3_000_000_000, V(0x100), None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_selftest_wait_timeout(1000, None, None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_selftest_wait_timeout(1000, V(0x102), None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # fused GEMM: row tiles beyond the grid's y limit are rejected up front
    gemm = [V(0x100), aqnf4.AQNF4_BF16, 65535 * 256, 64, V(0x200), V(0x300), V(0x400), 256,
            V(0x500), 0, None, None]
    big = list(gemm)
    big[2] = 65535 * 256 + 1
    assert lib.aqnf4_nf4_linear(*big) == aqnf4.AQNF4_ERR_INVALID_ARG
    # mean-centred DQ and its dequantization
    assert lib.aqnf4_double_quant_centered(V(0x100), 0, V(0x200), V(0x300), V(0x400), None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_double_quant_centered(V(0x100), 10, V(0x200), V(0x300), None, None, None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_double_quant_centered(V(0x100), 10, V(0x200), V(0x300), V(0x402), None, None) == aqnf4.AQNF4_ERR_ALIGNMENT
    assert lib.aqnf4_dequantize_centered(V(0x100), V(0x200), V(0x300), None, 64, 1, V(0x500), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_dequantize_centered(V(0x100), V(0x200), V(0x300), V(0x400), 64, 7, V(0x500), None) == aqnf4.AQNF4_ERR_DTYPE
    assert lib.aqnf4_dequantize_centered(V(0x108), V(0x200), V(0x300), V(0x400), 64, 1, V(0x500), None) == aqnf4.AQNF4_ERR_ALIGNMENT
    # division diagnostic
    assert lib.aqnf4_selftest_division(V(0x100), V(0x200), 0, V(0x300), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_selftest_division(None, V(0x200), 4, V(0x300), None) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert lib.aqnf4_selftest_division(V(0x100), V(0x200), 4, V(0x308), None) == aqnf4.AQNF4_ERR_ALIGNMENT
    assert lib.aqnf4_launch_count() == before


def test_status_strings(lib):
    for code in range(8):
        assert aqnf4.status_string(code)
    assert aqnf4.status_string(99) == "unknown status"


def test_binding_names_match_the_header():
    for name in declared_functions():
        if name in ("aqnf4_status_string",):
            continue
        assert callable(getattr(aqnf4, name)), name


class _FakeCuda:
    """Stands in for a CUDA tensor in the binding's argument checks (no device needed)."""

    def __init__(self, n, dtype, contiguous=True):
        self.is_cuda, self.dtype, self._n, self._c = True, dtype, n, contiguous

    def numel(self):
        return self._n

    def is_contiguous(self):
        return self._c


def test_binding_argument_checks():
    req = aqnf4._req
    req(None, "x", None, optional=True)
    req(_FakeCuda(10, torch.uint8), "x", (torch.uint8,), 10)
    for bad, msg in ((_FakeCuda(9, torch.uint8), "at least 10"),
                     (_FakeCuda(10, torch.int8), "dtype"),
                     (_FakeCuda(10, torch.uint8, contiguous=False), "contiguous"),
                     (torch.zeros(10, dtype=torch.uint8), "CUDA")):
        with pytest.raises(ValueError, match=msg):
            req(bad, "x", (torch.uint8,), 10)
    with pytest.raises(ValueError, match="required"):
        req(None, "x", None)
    # storage sizes of n weights: packed bytes, 64-element blocks, 256-block DQ scales
    assert aqnf4._storage_sizes(1) == (1, 1, 1)
    assert aqnf4._storage_sizes(16384) == (8192, 256, 1)
    assert aqnf4._storage_sizes(16385) == (8193, 257, 2)


def test_wrappers_reject_host_tensors_before_any_launch():
    before = aqnf4.library().aqnf4_launch_count()
    w = torch.zeros(128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        aqnf4.aqnf4_quantize(w, None, None)
    with pytest.raises(ValueError, match="CUDA"):
        aqnf4.aqnf4_dequantize(torch.zeros(64, dtype=torch.uint8), None, None,
                               torch.zeros(2, dtype=torch.float32), 128,
                               torch.zeros(128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="M x K"):
        aqnf4.aqnf4_nf4_linear(torch.zeros(64, dtype=torch.bfloat16), None, None, None, 1,
                               torch.zeros(1, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        aqnf4.make_layers([{"w": w}])
    assert aqnf4.library().aqnf4_launch_count() == before


def test_header_is_plain_c_and_links(lib, tmp_path):
    """The header compiles as strict C11 and a C program links against the library: the
    codebook, cost closed form and early argument checks it prints match the oracle."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(aqnf4.LIB)
    exe = str(tmp_path / "abi_consumer")
    src = os.path.join(os.path.dirname(__file__), "abi_consumer.c")
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", INCLUDE,
                    src, "-o", exe, "-L", lib_dir, "-laqnf4", f"-Wl,-rpath,{lib_dir}"],
                   check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    rows = [line.split() for line in out.splitlines()]
    levels, mids = oracle.codebook()
    got_l = [float.fromhex(r[2]) for r in rows if r[0] == "level"]
    got_m = [float.fromhex(r[2]) for r in rows if r[0] == "mid"]
    assert np.array_equal(np.float32(got_l), np.asarray(levels, np.float32))
    assert np.array_equal(np.float32(got_m), np.asarray(mids, np.float32))
    for r in rows:
        if r[0] == "cost":
            assert int(r[2]) == oracle.cost_bytes(int(r[1]))
    kv = {r[0]: r[1] for r in rows if len(r) == 2}
    assert int(kv["layer_error_null_w"]) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert int(kv["dequantize_null"]) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert int(kv["nf4_linear_bad_k"]) == aqnf4.AQNF4_ERR_INVALID_ARG
    assert int(kv["nf4_linear_splits_bad_k"]) == 0
    assert int(kv["launches"]) == 0
    assert out.splitlines()[-1] == "status " + aqnf4.status_string(aqnf4.AQNF4_ERR_ALIGNMENT)
