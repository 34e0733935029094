"""aqnf4_layer_error_noalloc: the scoring pass for callers that cannot provide device memory.

Some callers only receive device pointers from a host framework and have no allocator at
the call site (or run where new device allocations are not allowed), so they cannot hand
over the workspace aqnf4_layer_error needs.  The no-allocation entry point keeps that
scratch in the library itself.  This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from quantized_lora_setup_b200 import aqnf4, synth

RTOL = 1e-5  # the tolerance the parity tests use for the error sums


def _layers(dev):
    wl = synth.tiny(2)
    weights = [synth.layer_host(s, wl.seed, i).to(dev) for i, s in enumerate(wl.layers)]
    weights += [synth.random_bits_host(n, seed=n, dtype=torch.bfloat16).to(dev)
                for n in (1, 65, 16385, 3 * 16384 + 17)]
    return weights


def _run(weights, dev, noalloc: bool):
    stor = [aqnf4.NF4Storage(w.numel(), dev) for w in weights]
    descs = aqnf4.make_layers([{"w": w, "packed": s.packed, "codes8": s.codes8,
                                "scales": s.scales} for w, s in zip(weights, stor)])
    L = len(weights)
    se = torch.empty(L, dtype=torch.float64, device=dev)
    sw = torch.empty(L, dtype=torch.float64, device=dev)
    rel = torch.empty(L, dtype=torch.float32, device=dev)
    if noalloc:
        aqnf4.aqnf4_layer_error_noalloc(descs, se, sw, rel)
    else:
        ws = torch.empty(max(256, aqnf4.aqnf4_workspace_size(descs)), dtype=torch.uint8, device=dev)
        aqnf4.aqnf4_layer_error(descs, ws, se, sw, rel)
    torch.cuda.synchronize()
    return stor, se.cpu().numpy(), sw.cpu().numpy(), rel.cpu().numpy()


@pytest.mark.gpu
def test_noalloc_matches_workspace_version_twice(cuda):
    weights = _layers(cuda)
    ref_stor, ref_se, ref_sw, ref_rel = _run(weights, cuda, noalloc=False)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        stor, se, sw, rel = _run(weights, cuda, noalloc=True)
        np.testing.assert_allclose(se, ref_se, rtol=RTOL, atol=0)
        np.testing.assert_allclose(sw, ref_sw, rtol=RTOL, atol=0)
        np.testing.assert_allclose(rel, ref_rel, rtol=RTOL, atol=0)
        for a, b in zip(stor, ref_stor):
            assert torch.equal(a.packed, b.packed)
            assert torch.equal(a.codes8, b.codes8)
            assert torch.equal(a.scales, b.scales)


def test_noalloc_rejects_requests_above_its_scratch():
    """More than 2^19 tiles of 16384 elements is refused before anything is launched."""
    lib = aqnf4.library()
    d = aqnf4.aqnf4_layer()
    d.w, d.numel, d.dtype, d.flags = 0x10000, (1 << 19) * 16384 + 1, aqnf4.AQNF4_BF16, 0
    arr = (aqnf4.aqnf4_layer * 1)(d)
    before = lib.aqnf4_launch_count()
    st = lib.aqnf4_layer_error_noalloc(arr, 1, None, None, None, None, None)
    assert st == aqnf4.AQNF4_ERR_WORKSPACE
    assert lib.aqnf4_launch_count() == before
    assert lib.aqnf4_layer_error_noalloc(None, 1, None, None, None, None, None) == \
        aqnf4.AQNF4_ERR_INVALID_ARG
