"""The synthetic workloads have the recipe's shapes and sizes (no GPU): layer counts,
element and byte totals, formats, budgets, the mix of value distributions, and seeded
determinism of the host generator."""
import numpy as np
import torch

from quantized_lora_setup_b200 import synth

GIB = 1 << 30


def test_tiny():
    wl = synth.tiny(0)
    assert len(wl.layers) == 28 and wl.numel == 3_162_112 and wl.weight_bytes == 6_324_224
    assert {l.dtype for l in wl.layers} == {torch.float16}
    assert sum(l.dist == "t" for l in wl.layers) == 2 and wl.k_cap == 2
    assert {(l.rows, l.cols) for l in wl.layers} == {(256, 256), (688, 256), (256, 688)}


def test_1p4b():
    wl = synth.model_1p4b(0)
    assert len(wl.layers) == 96 and wl.numel == 1_207_959_552
    assert {l.dtype for l in wl.layers} == {torch.float16}
    assert sum(l.dist == "t" for l in wl.layers) == 10
    assert all(0.01 <= l.sigma <= 0.04 for l in wl.layers)
    assert wl.budgets == (int(0.2 * GIB),)


def test_7b():
    wl = synth.model_7b(0)
    assert len(wl.layers) == 224 and wl.numel == 6_476_005_376
    assert wl.weight_bytes == 12_952_010_752
    assert {l.dtype for l in wl.layers} == {torch.bfloat16}
    assert wl.budgets == (GIB,)
    for l in wl.layers:
        b = int(l.name.split(".")[0][3:])
        assert abs(l.sigma - (0.01 + 0.02 * b / 31)) < 1e-12
        assert len(l.outlier_cols) == max(1, round(0.001 * l.cols)) and l.outlier_factor == 20
    assert synth.block_index(wl) == [b for b in range(32) for _ in range(7)]


def test_14b():
    wl = synth.model_14b(0)
    assert len(wl.layers) == 280 and wl.numel == 11_010_048_000
    assert {l.dtype for l in wl.layers} == {torch.bfloat16}
    assert wl.budgets == (int(0.2 * GIB), GIB, 4 * GIB)
    kinds = [l.dist for l in wl.layers]
    assert 0.3 < kinds.count("t") / len(kinds) < 0.7  # a fair coin per layer


def test_dequant_shapes_span_the_range():
    assert synth.DEQUANT_SHAPES[0] == (4096, 4096) and synth.DEQUANT_SHAPES[-1] == (28672, 8192)


def test_host_generator_is_seeded():
    wl = synth.tiny(0)
    a = synth.layer_host(wl.layers[3], wl.seed, 3)
    b = synth.layer_host(wl.layers[3], wl.seed, 3)
    c = synth.layer_host(wl.layers[3], wl.seed + 1, 3)
    assert torch.equal(a, b) and not torch.equal(a, c)
    x = a.float().numpy()
    assert abs(x.std() - 0.02) < 0.002 and abs(x.mean()) < 0.002
