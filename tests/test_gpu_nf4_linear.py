"""The fused NF4-dequant GEMM (aqnf4_nf4_linear) against the oracle's binary64 product.

The layer's storage comes from the oracle (quantize + double quantization), so the kernel
is checked independently of the library's own quantizer.  Bound: the kernel sums products
that are exact in binary32 (16-bit times 16-bit), so any summation order stays within
K * 2^-23 * sum |x w_hat| of the binary64 result; a 16-bit output adds its own rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_lora_setup_b200 import aqnf4, synth


DT = {torch.float16: oracle.F16, torch.bfloat16: oracle.BF16}


def _case(M, N, K, dt, seed):
    rng = np.random.default_rng(seed)
    w = torch.from_numpy((rng.standard_normal((N, K)) * 0.02).astype(np.float32)).to(dt)
    packed, absmax, _ = oracle.quantize(synth.bits_u16(w), DT[dt])
    codes8, scales, _ = oracle.double_quant(absmax)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(dt)
    return x, packed, codes8, scales


def _run(cuda, x, packed, codes8, scales, N, out_dtype):
    M, K = x.shape
    y = torch.full((M, N), float("nan"), dtype=out_dtype, device=cuda)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    aqnf4.aqnf4_nf4_linear(x.to(cuda), torch.from_numpy(packed).to(cuda),
                           torch.from_numpy(codes8).to(cuda), torch.from_numpy(scales).to(cuda),
                           N, y, flag)
    torch.cuda.synchronize()
    assert flag.item() == 0
    return y.double().cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (1, 1, 64), (200, 300, 256),
                                   (256, 384, 4096), (130, 129, 192), (64, 100, 128),
                                   (70, 260, 320), (600, 300, 256), (520, 1000, 512),
                                   (1024, 512, 960), (300, 1001, 448), (257, 256, 64),
                                   (300, 512, 192), (513, 384, 320)])
def test_nf4_linear_matches_oracle(cuda, dt, M, N, K):
    """Shapes with one CTA per tile, with split K, and with two row tiles per CTA pair
    (several row tiles and no split: 600, 520 and 1024 rows; an odd count of row tiles
    leaves the last pair's second CTA without rows; 1, 3 or 5 steps of K leave some of
    the pair's four dequantizing groups without a step)."""
    x, packed, codes8, scales = _case(M, N, K, dt, seed=M + N + K)
    ref, rabs = oracle.nf4_linear(synth.bits_u16(x).reshape(M, K), DT[dt], packed, codes8,
                                  scales, N, DT[dt])
    bound = K * 2.0 ** -23 * rabs + 1e-30
    y32 = _run(cuda, x, packed, codes8, scales, N, torch.float32)
    assert np.all(np.abs(y32 - ref) <= bound)
    y16 = _run(cuda, x, packed, codes8, scales, N, dt)
    ulp = 2.0 ** -8 if dt == torch.bfloat16 else 2.0 ** -11
    assert np.all(np.abs(y16 - ref) <= bound + ulp * (np.abs(ref) + bound) + 6e-8)


@pytest.mark.gpu
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K,S", [(128, 11008, 4096, 3), (16, 1024, 2048, 4),
                                     (300, 512, 8192, 8), (7, 1023, 2048, 4),
                                     (300, 6400, 1024, 2), (128, 5376, 3584, 7),
                                     (200, 10240, 2048, 3)])
def test_nf4_linear_split_k_matches_oracle(cuda, dt, M, N, K, S):
    """Few output tiles: K is split over the S CTAs of a cluster, which add their partials
    on chip in split order (16-byte stores when N is a multiple of 4, one output at a time
    otherwise: 7 x 1023; two row tiles, the second ragged: 300 x ...; both 128-row halves of
    one tile: 200 x 10240)."""
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert aqnf4.aqnf4_nf4_linear_splits(M, N, K) == S
    assert aqnf4.aqnf4_nf4_linear_splits(M, N, K) > 1
    x, packed, codes8, scales = _case(M, N, K, dt, seed=K + M)
    ref, rabs = oracle.nf4_linear(synth.bits_u16(x).reshape(M, K), DT[dt], packed, codes8,
                                  scales, N, DT[dt])
    bound = K * 2.0 ** -23 * rabs + 1e-30
    y1 = _run(cuda, x, packed, codes8, scales, N, torch.float32)
    y2 = _run(cuda, x, packed, codes8, scales, N, torch.float32)
    assert np.all(np.abs(y1 - ref) <= bound)
    assert np.array_equal(y1, y2)  # the partial sums are added in a fixed order
    y16 = _run(cuda, x, packed, codes8, scales, N, dt)
    ulp = 2.0 ** -8 if dt == torch.bfloat16 else 2.0 ** -11
    assert np.all(np.abs(y16 - ref) <= bound + ulp * (np.abs(ref) + bound) + 6e-8)


@pytest.mark.gpu
def test_nf4_linear_full_mlp_shape_sampled_rows(cuda):
    """The 7B MLP up-projection at 4096 tokens (11008 x 4096, bf16; CTA pairs with two-CTA
    MMAs), as the bench times it: rows of y from several row tiles, from both CTAs of a pair
    and from both 128-row halves of a tile, against the oracle's product of those rows."""
    M, N, K = 4096, 11008, 4096
    x, packed, codes8, scales = _case(M, N, K, torch.bfloat16, seed=11)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    aqnf4.aqnf4_nf4_linear(x.to(cuda), torch.from_numpy(packed).to(cuda),
                           torch.from_numpy(codes8).to(cuda), torch.from_numpy(scales).to(cuda),
                           N, y, flag)
    torch.cuda.synchronize()
    assert flag.item() == 0
    rows = np.array([0, 127, 128, 255, 256, 511, 1100, 2047, 2048, 3071, 4000, 4095])
    ref, rabs = oracle.nf4_linear(synth.bits_u16(x[rows]).reshape(len(rows), K), oracle.BF16,
                                  packed, codes8, scales, N, oracle.BF16)
    got = y[torch.from_numpy(rows).to(cuda)].double().cpu().numpy()
    assert np.all(np.abs(got - ref) <= K * 2.0 ** -23 * rabs + 1e-30)


@pytest.mark.gpu
def test_nf4_linear_uses_the_library_storage(cuda):
    """Storage written by the fused scoring pass (bit-equal to the oracle's) gives the same y."""
    M, N, K = 64, 256, 512
    rng = np.random.default_rng(9)
    w = torch.from_numpy((rng.standard_normal((N, K)) * 0.02).astype(np.float32)).to(torch.bfloat16)
    x, packed, codes8, scales = _case(M, N, K, torch.bfloat16, seed=9)
    packed, absmax, _ = oracle.quantize(synth.bits_u16(w), oracle.BF16)
    codes8, scales, _ = oracle.double_quant(absmax)
    st = aqnf4.NF4Storage(N * K, cuda)
    aqnf4.score_layers([w.reshape(-1).to(cuda)], [st])
    torch.cuda.synchronize()
    assert np.array_equal(st.packed.cpu().numpy(), packed)
    assert np.array_equal(st.codes8.cpu().numpy(), codes8)
    y_oracle_storage = _run(cuda, x, packed, codes8, scales, N, torch.float32)
    y_lib_storage = _run(cuda, x, st.packed.cpu().numpy(), st.codes8.cpu().numpy(),
                         st.scales.cpu().numpy(), N, torch.float32)
    np.testing.assert_array_equal(y_lib_storage, y_oracle_storage)


def test_nf4_linear_rejects_bad_shapes():
    lib = aqnf4.library()
    V = __import__("ctypes").c_void_p
    before = lib.aqnf4_launch_count()
    args = [V(0x1000), aqnf4.AQNF4_BF16, 4, 64, V(0x2000), V(0x3000), V(0x4000), 8, V(0x5000),
            1, None, None]
    for i, bad in ((3, 0), (3, 96), (3, 63), (2, 0), (7, 0), (0, None), (8, None)):
        a = list(args)
        a[i] = bad
        assert lib.aqnf4_nf4_linear(*a) == aqnf4.AQNF4_ERR_INVALID_ARG, (i, bad)
    a = list(args)
    a[1] = 7
    assert lib.aqnf4_nf4_linear(*a) == aqnf4.AQNF4_ERR_DTYPE
    a = list(args)
    a[0] = V(0x1008)
    assert lib.aqnf4_nf4_linear(*a) == aqnf4.AQNF4_ERR_ALIGNMENT
    for out_f32, y in ((1, 0x5004), (0, 0x5002)):  # y must allow 16-byte vector stores
        a = list(args)
        a[8], a[9] = V(y), out_f32
        assert lib.aqnf4_nf4_linear(*a) == aqnf4.AQNF4_ERR_ALIGNMENT, (out_f32, y)
    assert lib.aqnf4_launch_count() == before
    assert aqnf4.aqnf4_nf4_linear_splits(4, 8, 96) == 0


def test_split_k_counts():
    """The split rule on a 148-SM part (what the library assumes without a device):
    enough splits for one wave, at least 8 steps of 64 each, at most 8 (one cluster), none
    when the tiles fill it."""
    if torch.cuda.is_available() and torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("counts below are for 148 SMs")
    # 11008 x 4096 layer, 128 tokens: 43 output tiles -> 148 // 43 = 3 splits
    assert aqnf4.aqnf4_nf4_linear_splits(128, 11008, 4096) == 3
    # 16 tokens, 1024 outputs, K 2048: 4 tiles -> 37, capped by 32 steps / 8 = 4
    assert aqnf4.aqnf4_nf4_linear_splits(16, 1024, 2048) == 4
    # 4 tiles, K 8192: 37, capped at 8 CTAs per cluster
    assert aqnf4.aqnf4_nf4_linear_splits(300, 512, 8192) == 8
    # K = 512: 8 steps cannot be split into two halves of >= 8 steps
    assert aqnf4.aqnf4_nf4_linear_splits(16, 1024, 512) == 1
    # 4096 tokens x 11008: 16 x 43 = 688 tiles fill the GPU: no split
    assert aqnf4.aqnf4_nf4_linear_splits(4096, 11008, 4096) == 1
    # not a valid shape
    assert aqnf4.aqnf4_nf4_linear_splits(16, 1024, 100) == 0
