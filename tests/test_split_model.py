"""The split model (top-K layers in 16 bits, the rest NF4 + DQ) and its memory report.

CPU: the byte accounting against the oracle's cost model.  GPU: materialize() against the
oracle -- the kept set, every NF4 layer's dequantized weights bit for bit, the kept layers
untouched, and the report's extra bytes equal to the kept layers' cost, within budget.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_lora_setup_b200 import aqnf4, split_model, synth

DT = {torch.float16: oracle.F16, torch.bfloat16: oracle.BF16}


def test_nf4_storage_bytes_closed_form():
    for n in (1, 2, 63, 64, 65, 16383, 16384, 16385, 4096 * 11008, 5120 * 13824):
        nb = -(-n // 64)
        expect = -(-n // 2) + nb + 4 * -(-nb // 256)
        assert split_model.nf4_storage_bytes(n) == expect
        assert split_model.nf4_storage_bytes(n) == 2 * n - oracle.cost_bytes(n)
        assert split_model.nf4_bytes(aqnf4.NF4Storage(n, "cpu")) == expect


def test_memory_report_accounting_on_host_tensors():
    """A hand-built split model: extra bytes = the kept layers' cost exactly."""
    sizes = [(256, 256), (688, 256), (7, 13), (1, 1)]
    layers = []
    kept = [1, 2]
    for i, shape in enumerate(sizes):
        n = shape[0] * shape[1]
        if i in kept:
            w = torch.zeros(shape, dtype=torch.bfloat16)
            layers.append(split_model.SplitLayer(i, "fp16", shape, w.dtype, 0.1, w, None))
        else:
            layers.append(split_model.SplitLayer(i, "nf4", shape, torch.bfloat16, 0.1, None,
                                                 aqnf4.NF4Storage(n, "cpu")))
    cost = sum(oracle.cost_bytes(sizes[i][0] * sizes[i][1]) for i in kept)
    for budget, ok in ((cost, True), (cost - 1, False)):
        rep = split_model.SplitModel(layers, [1, 2, 0, 3], kept, budget).memory_report()
        assert rep["extra_bytes"] == cost
        assert rep["total_bytes"] == rep["all_nf4_bytes"] + cost
        assert rep["within_budget"] is ok
        assert rep["fp16_layers"] == 2 and rep["layers"] == 4


def _oracle_model(weights):
    rel, dq = [], []
    for w in weights:
        b = synth.bits_u16(w.cpu())
        rel.append(oracle.layer_error(b, DT[w.dtype])[2])
        packed, absmax, _ = oracle.quantize(b, DT[w.dtype])
        codes8, scales, _ = oracle.double_quant(absmax)
        dq.append(oracle.dequantize(packed, b.size, DT[w.dtype], codes8=codes8, scales=scales))
    return np.array(rel, np.float32), dq


@pytest.mark.gpu
@pytest.mark.parametrize("budget_frac", [0.0, 0.3, 1.0])
def test_materialize_tiny_model(cuda, budget_frac):
    wl = synth.tiny(0)
    weights = [synth.layer_host(s, wl.seed, i).to(cuda) for i, s in enumerate(wl.layers)]
    cost = [aqnf4.aqnf4_cost_bytes(w.numel()) for w in weights]
    budget = int(budget_frac * sum(cost))
    model = split_model.materialize(weights, budget)
    rel, dq = _oracle_model(weights)
    assert model.kept == oracle.select_topk(rel, cost, budget)
    for i, L in enumerate(model.layers):
        w16 = model.weight(i)
        assert tuple(w16.shape) == tuple(weights[i].shape)
        if i in model.kept:
            assert L.kind == "fp16" and w16.data_ptr() == weights[i].data_ptr()
        else:
            assert L.kind == "nf4"
            got = synth.bits_u16(w16.cpu())
            assert np.array_equal(got, dq[i]), i
    rep = model.memory_report()
    assert rep["extra_bytes"] == sum(cost[i] for i in model.kept)
    assert rep["within_budget"] and rep["extra_bytes"] <= budget


@pytest.mark.gpu
def test_materialize_ranks_by_dq_score_when_asked(cuda):
    wl = synth.tiny(1)
    weights = [synth.layer_host(s, wl.seed, i).to(cuda) for i, s in enumerate(wl.layers)]
    cost = [aqnf4.aqnf4_cost_bytes(w.numel()) for w in weights]
    budget = sum(cost) // 4
    model = split_model.materialize(weights, budget, dq_score=True)
    rel = np.array([oracle.layer_error_dq(synth.bits_u16(w.cpu()), DT[w.dtype])[2]
                    for w in weights], np.float32)
    assert model.kept == oracle.select_topk(rel, cost, budget)
    np.testing.assert_allclose([L.rel_err for L in model.layers], rel, rtol=1e-5)


@pytest.mark.gpu
def test_split_model_linear_matches_oracle(cuda):
    """y = x w^T through the split model: the kept layer by cuBLAS on its 16-bit weights, an
    NF4 layer by the fused tensor-core GEMM; both within the binary32 accumulation bound of
    the oracle's binary64 product of what the layer holds."""
    rng = np.random.default_rng(41)
    shapes = [(256, 512), (384, 256), (130, 192)]
    weights = [torch.from_numpy((rng.standard_normal(sh) * 0.02).astype(np.float32))
               .to(torch.bfloat16).to(cuda) for sh in shapes]
    cost = [aqnf4.aqnf4_cost_bytes(w.numel()) for w in weights]
    # the largest layer's cost: the first-ranked layer always fits, not all of them can
    model = split_model.materialize(weights, budget_bytes=max(cost))
    kinds = {L.kind for L in model.layers}
    assert kinds == {"fp16", "nf4"}
    M = 96
    for i, w in enumerate(weights):
        N, K = shapes[i]
        x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
        y = model.linear(i, x.to(cuda), out_dtype=torch.float32).double().cpu().numpy()
        if model.layers[i].kind == "fp16":
            w64 = w.double().cpu().numpy()
        else:
            w64 = model.weight(i).double().cpu().numpy()
            packed, absmax, _ = oracle.quantize(synth.bits_u16(w.cpu()), oracle.BF16)
            codes8, scales, _ = oracle.double_quant(absmax)
            ref, _ = oracle.nf4_linear(synth.bits_u16(x).reshape(M, K), oracle.BF16, packed,
                                       codes8, scales, N, oracle.BF16)
            x64 = x.double().numpy()
            assert np.allclose(x64 @ w64.T, ref, rtol=0, atol=1e-12)  # weight(i) is w_hat
        x64 = x.double().numpy()
        ref = x64 @ w64.T
        bound = K * 2.0 ** -23 * (np.abs(x64) @ np.abs(w64).T) + 1e-30
        assert np.all(np.abs(y - ref) <= bound), i


@pytest.mark.gpu
def test_split_model_linear_dequantize_path_matches_oracle(cuda):
    """The branch that multiplies dequantized weights: an NF4 layer whose K (100, 72) is not a
    multiple of 64, so NF4 blocks cross rows, and an x in the other 16-bit format on a layer
    the fused GEMM could take.  Each result is within the binary32 accumulation bound of the
    oracle's binary64 product of x (in the layer's format) with the oracle's w_hat."""
    rng = np.random.default_rng(43)
    shapes = [(160, 100), (96, 72), (128, 128)]
    weights = [torch.from_numpy((rng.standard_normal(sh) * 0.02).astype(np.float32))
               .to(torch.bfloat16).to(cuda) for sh in shapes]
    model = split_model.materialize(weights, budget_bytes=0)  # every layer stays NF4
    assert all(L.kind == "nf4" for L in model.layers)
    M = 40
    cases = [(0, torch.bfloat16), (1, torch.bfloat16), (2, torch.float16), (2, torch.bfloat16)]
    for i, x_dtype in cases:
        N, K = shapes[i]
        want = "fused-nf4" if (K % 64 == 0 and x_dtype == torch.bfloat16) else \
            "dequantize+cublas"
        assert model.linear_path(i, x_dtype) == want, (i, x_dtype)
        x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(x_dtype)
        y = model.linear(i, x.to(cuda), out_dtype=torch.float32).double().cpu().numpy()
        xl = x.to(torch.bfloat16)  # x as the product sees it: in the layer's format
        packed, absmax, _ = oracle.quantize(synth.bits_u16(weights[i].cpu()), oracle.BF16)
        codes8, scales, _ = oracle.double_quant(absmax)
        ref, rabs = oracle.nf4_linear(synth.bits_u16(xl).reshape(M, K), oracle.BF16, packed,
                                      codes8, scales, N, oracle.BF16)
        bound = K * 2.0 ** -23 * rabs + 1e-30
        assert np.all(np.abs(y - ref) <= bound), (i, x_dtype)
