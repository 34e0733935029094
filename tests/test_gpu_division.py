"""The fused pass's short reciprocal and quotient against CUDA's correctly rounded ones.

The host replay (tests/division_check.c) proves the short forms for every 16-bit input under
the documented 1-ulp bound of the hardware reciprocal approximation; this test runs them on
the GPU beside __frcp_rn and __fdiv_rn, for every 16-bit value in the fast range and a large
sample of pairs, in both formats.
"""
import numpy as np
import pytest
import torch

from quantized_lora_setup_b200 import aqnf4

pytestmark = pytest.mark.gpu


def _values(fmt):
    """Every finite non-negative value of a 16-bit format, as float32, ascending."""
    bits = np.arange(0x8000, dtype=np.uint16)
    x = bits.view(np.float16).astype(np.float32) if fmt == "f16" else \
        (bits.astype(np.uint32) << 16).view(np.float32)
    return x[np.isfinite(x)]


def _run(a, s):
    dev = torch.device("cuda:0")
    ta = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)
    ts = torch.from_numpy(np.ascontiguousarray(s, np.float32)).to(dev)
    out = torch.empty(a.size, 4, dtype=torch.float32, device=dev)
    aqnf4.aqnf4_selftest_division(ta, ts, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("fmt", ["bf16", "f16"])
def test_short_reciprocal_matches_frcp_rn(fmt):
    v = _values(fmt)
    a = v[(v >= 2.0 ** -40) & (v <= 2.0 ** 40)]
    o = _run(a, np.ones_like(a))
    assert np.array_equal(o[:, 0].view(np.uint32), o[:, 1].view(np.uint32))
    assert np.array_equal(o[:, 1], (np.float32(1) / a).astype(np.float32))


@pytest.mark.parametrize("fmt", ["bf16", "f16"])
def test_short_quotient_matches_fdiv_rn(fmt):
    v = _values(fmt)
    fast = v[(v >= 2.0 ** -40) & (v <= 2.0 ** 40)]
    rng = np.random.default_rng(11)
    s = np.repeat(fast, 256)
    # a <= s: a random fraction of the values below each s (index-uniform, so every binade
    # and the tiny and subnormal values appear), plus a = s and a = 0 for every s
    hi = np.searchsorted(v, s, side="right")
    a = v[(rng.random(s.size) * hi).astype(np.int64)]
    a = np.concatenate([a, fast, np.zeros_like(fast)])
    s = np.concatenate([s, fast, fast])
    o = _run(a, s)
    q, ref = o[:, 2], o[:, 3]
    assert np.array_equal(ref, (a / s).astype(np.float32))
    big = ref >= 2.0 ** -30
    assert np.array_equal(q[big].view(np.uint32), ref[big].view(np.uint32))
    code = np.rint((q * np.float32(255)).astype(np.float32))
    code_ref = np.rint((ref * np.float32(255)).astype(np.float32))
    assert np.array_equal(code, code_ref)
