"""GPU parity: every libaqnf4 entry point against the CPU oracle on the same seeded bytes.

Bit-exact: NF4 codes / packed bytes, absmax, DQ bytes and scales, dequantized values,
the selected layer set.  Floating point: per-layer sq_err, sq_w and rel_err within a
relative 1e-5.  That bound follows from the kernel's arithmetic: each thread sums at most
64 squares in binary32 (relative error <= 64 u, u = 2^-24), a warp adds 32 such partial
sums in binary32 (<= 5 u more) and everything above that is binary64, so the relative
error of a sum of non-negative terms stays below 70 u ~ 4.2e-6; the square root halves it
for rel_err.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_lora_setup_b200 import aqnf4, synth

pytestmark = pytest.mark.gpu
RTOL = 1e-5

DT = {torch.float16: oracle.F16, torch.bfloat16: oracle.BF16}


def bits(t):
    return synth.bits_u16(t)


def u32(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def same_float_bits(got, ref):
    g, r = np.asarray(got, np.float32), np.asarray(ref, np.float32)
    return np.all((u32(g) == u32(r)) | (np.isnan(g) & np.isnan(r)))


SIZES = [1, 2, 3, 7, 8, 9, 15, 16, 17, 63, 64, 65, 127, 128, 1000, 16383, 16384, 16385,
         3 * 16384 + 17, 100003, 262145]


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("n", SIZES)
def test_quantize_ragged_sizes(cuda, dt, n):
    w = synth.random_bits_host(n, seed=n, dtype=dt)
    packed, absmax = aqnf4.quantize(w.to(cuda))
    op, oa, _ = oracle.quantize(bits(w), DT[dt])
    assert np.array_equal(packed.cpu().numpy(), op)
    assert same_float_bits(absmax.cpu().numpy(), oa)


def _all_values_blocks(dt, a):
    """Every finite value of dt with |x| <= a, 63 per block, each block led by +a."""
    allb = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(dt)
    v = allb.float()
    keep = torch.isfinite(v) & (v.abs() <= a)
    vals = allb[keep]
    nblk = (vals.numel() + 62) // 63
    pad = torch.zeros(nblk * 63 - vals.numel(), dtype=dt)
    body = torch.cat([vals, pad]).reshape(nblk, 63)
    lead = torch.full((nblk, 1), a, dtype=torch.float32).to(dt)
    return torch.cat([lead, body], dim=1).reshape(-1)


@pytest.mark.parametrize("dt,a", [
    (torch.bfloat16, 1.0), (torch.bfloat16, 0.02), (torch.bfloat16, 3.0e38),
    (torch.bfloat16, 1e-30), (torch.bfloat16, 2.0 ** -128), (torch.bfloat16, 2.0 ** -126),
    (torch.float16, 1.0), (torch.float16, 65504.0), (torch.float16, 1e-3), (torch.float16, 3e-7)])
def test_quantize_every_value_of_the_format(cuda, dt, a):
    """All 16-bit values against one block maximum: covers every midpoint neighbourhood."""
    w = _all_values_blocks(dt, a)
    packed, absmax = aqnf4.quantize(w.to(cuda))
    op, oa, _ = oracle.quantize(bits(w), DT[dt])
    assert np.array_equal(packed.cpu().numpy(), op)
    assert same_float_bits(absmax.cpu().numpy(), oa)
    se, sw, rel = aqnf4.score_layers([w.to(cuda)])
    ose, osw, orel = oracle.layer_error(bits(w), DT[dt])
    assert se.item() == pytest.approx(ose, rel=RTOL)
    assert sw.item() == pytest.approx(osw, rel=RTOL)
    assert rel.item() == pytest.approx(orel, rel=RTOL)


def test_quantize_special_blocks(cuda):
    rng = np.random.default_rng(0)
    blocks = []
    blocks.append(np.zeros(64))                       # zero block -> code 7
    blocks.append(-np.zeros(64))                      # negative zeros
    z = np.zeros(64); z[17] = -0.5; blocks.append(z)  # single value, negative maximum
    blocks.append(rng.standard_normal(64) * 1e-39)    # subnormal absmax (bf16)
    blocks.append(-np.abs(rng.standard_normal(64)))   # all negative
    blocks.append(np.full(64, 0.25))                  # constant block
    blocks.append(rng.standard_normal(64) * 5e37)     # near the top of the range
    w = torch.from_numpy(np.concatenate(blocks).astype(np.float32)).to(torch.bfloat16)
    packed, absmax = aqnf4.quantize(w.to(cuda))
    op, oa, _ = oracle.quantize(bits(w), oracle.BF16)
    assert np.array_equal(packed.cpu().numpy(), op)
    assert same_float_bits(absmax.cpu().numpy(), oa)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_nonfinite_input_sets_the_flag(cuda, dt):
    w = synth.random_bits_host(64 * 40, seed=3, dtype=dt)
    w[5] = float("nan")
    w[64 * 7 + 3] = float("inf")
    w[64 * 9] = float("-inf")
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    n = w.numel()
    packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device=cuda)
    absmax = torch.empty(aqnf4.nblocks(n), dtype=torch.float32, device=cuda)
    aqnf4.aqnf4_quantize(w.to(cuda), packed, absmax, flag)
    assert flag.item() == aqnf4.AQNF4_ERR_NONFINITE
    op, oa, onf = oracle.quantize(bits(w), DT[dt])
    assert onf
    assert np.array_equal(packed.cpu().numpy(), op)
    assert same_float_bits(absmax.cpu().numpy(), oa)
    flag.zero_()
    clean = synth.random_bits_host(64 * 40, seed=4, dtype=dt)
    rel = torch.empty(2, device=cuda)
    aqnf4.aqnf4_layer_error([{"w": clean.to(cuda)}, {"w": w.to(cuda)}],
                            torch.empty(4096, dtype=torch.uint8, device=cuda), None, None, rel,
                            flag)
    assert flag.item() == aqnf4.AQNF4_ERR_NONFINITE
    assert math.isnan(rel[1].item()) and not math.isnan(rel[0].item())


def _run_layers(cuda, weights, with_absmax=True):
    stor = [aqnf4.NF4Storage(w.numel(), cuda, with_absmax=with_absmax) for w in weights]
    se, sw, rel = aqnf4.score_layers([w.to(cuda) for w in weights], stor)
    torch.cuda.synchronize()
    return stor, se.cpu().numpy(), sw.cpu().numpy(), rel.cpu().numpy()


def _check_layer(w, st, se, sw, rel):
    dt = DT[w.dtype]
    b = bits(w)
    op, oa, _ = oracle.quantize(b, dt)
    oc, osc, _ = oracle.double_quant(oa)
    ose, osw, orel = oracle.layer_error(b, dt)
    assert np.array_equal(st.packed.cpu().numpy(), op)
    if st.absmax is not None:
        assert same_float_bits(st.absmax.cpu().numpy(), oa)
    assert np.array_equal(st.codes8.cpu().numpy(), oc)
    assert same_float_bits(st.scales.cpu().numpy(), osc)
    assert se == pytest.approx(ose, rel=RTOL, abs=0)
    assert sw == pytest.approx(osw, rel=RTOL, abs=0)
    assert rel == pytest.approx(orel, rel=RTOL, abs=0)
    return orel


def _selection_agrees(gpu_rel, ora_rel, cost, budget, k_cap, gpu_sel):
    """Selected set bit-exact; near-ties at the cut are checked on the oracle's scores."""
    ref = oracle.select_topk(ora_rel, cost, budget, k_cap)
    if sorted(gpu_sel) == sorted(ref):
        return True
    # tie-ambiguous only if the GPU scores at the cut are within 2e-5 of each other
    order = oracle.select_topk(gpu_rel, cost, 1 << 62, -1)
    k = len(gpu_sel)
    if 0 < k < len(order):
        a, b = gpu_rel[order[k - 1]], gpu_rel[order[k]]
        if abs(a - b) <= 2e-5 * max(abs(a), abs(b)):
            return True
    return False


def test_tiny_model_end_to_end(cuda):
    wl = synth.tiny(0)
    weights = [synth.layer_host(s, wl.seed, i) for i, s in enumerate(wl.layers)]
    stor, se, sw, rel = _run_layers(cuda, weights)
    orel = [_check_layer(w, st, se[i], sw[i], rel[i]) for i, (w, st) in enumerate(zip(weights, stor))]
    cost = np.array([aqnf4.aqnf4_cost_bytes(s.numel) for s in wl.layers], np.int64)
    sel, k = aqnf4.select_topk(torch.from_numpy(rel).to(cuda), torch.from_numpy(cost).to(cuda),
                               wl.budgets[0], wl.k_cap)
    kk = k.item()
    got = sel.cpu().numpy()[:kk].tolist()
    assert kk == 2
    assert got == oracle.select_topk(rel, cost, wl.budgets[0], wl.k_cap)
    assert _selection_agrees(rel, orel, cost, wl.budgets[0], wl.k_cap, got)
    assert sorted(got) == sorted(i for i, s in enumerate(wl.layers) if s.dist == "t")


def test_mixed_dtypes_ragged_layers(cuda):
    sizes = [1, 65, 16383, 16385, 50000, 7, 100003, 64, 32768 + 1]
    weights = [synth.random_bits_host(n, seed=100 + i,
                                      dtype=torch.float16 if i % 3 == 0 else torch.bfloat16)
               for i, n in enumerate(sizes)]
    weights[4] = weights[4] * 0  # an all-zero layer: rel_err 0
    stor, se, sw, rel = _run_layers(cuda, weights)
    for i, (w, st) in enumerate(zip(weights, stor)):
        _check_layer(w, st, se[i], sw[i], rel[i])
    assert rel[4] == 0.0


def test_more_layers_than_one_launch_holds(cuda):
    weights = [synth.random_bits_host(64 * (1 + i % 5) + i % 3, seed=i, dtype=torch.bfloat16)
               for i in range(400)]
    stor, se, sw, rel = _run_layers(cuda, weights, with_absmax=False)
    for i in (0, 1, 383, 384, 385, 399):
        _check_layer(weights[i], stor[i], se[i], sw[i], rel[i])


def test_repeat_calls_are_bit_identical(cuda):
    wl = synth.tiny(1)
    weights = [synth.layer_host(s, wl.seed, i) for i, s in enumerate(wl.layers)]
    a = _run_layers(cuda, weights)
    b = _run_layers(cuda, weights)
    for x, y in zip(a[1:], b[1:]):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))
    for s1, s2 in zip(a[0], b[0]):
        assert torch.equal(s1.packed, s2.packed) and torch.equal(s1.codes8, s2.codes8)


def test_double_quant_standalone_and_fused_agree(cuda):
    rng = np.random.default_rng(5)
    for nb in (1, 255, 256, 257, 1000, 4096 + 3):
        a = np.abs(rng.standard_normal(nb)).astype(np.float32) * 0.03
        if nb > 300:
            a[256:512] = 0.0  # a zero DQ block
        codes8, scales = aqnf4.double_quant(torch.from_numpy(a).to(cuda))
        oc, osc, _ = oracle.double_quant(a)
        assert np.array_equal(codes8.cpu().numpy(), oc)
        assert same_float_bits(scales.cpu().numpy(), osc)
    # the fused pass's DQ equals the standalone one on its own absmax
    w = synth.random_bits_host(16384 * 3 + 999, seed=9, dtype=torch.bfloat16).to(cuda)
    st = aqnf4.NF4Storage(w.numel(), cuda, with_absmax=True)
    aqnf4.score_layers([w], [st])
    c2, s2 = aqnf4.double_quant(st.absmax)
    assert torch.equal(c2, st.codes8) and torch.equal(s2, st.scales)


def test_double_quant_nonfinite_flag(cuda):
    a = np.ones(600, np.float32)
    a[300] = np.nan
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    codes8 = torch.empty(600, dtype=torch.uint8, device=cuda)
    scales = torch.empty(3, dtype=torch.float32, device=cuda)
    aqnf4.aqnf4_double_quant(torch.from_numpy(a).to(cuda), codes8, scales, flag)
    assert flag.item() == aqnf4.AQNF4_ERR_NONFINITE
    oc, osc, _ = oracle.double_quant(a)
    assert np.array_equal(codes8.cpu().numpy(), oc)
    assert same_float_bits(scales.cpu().numpy(), osc)


def test_double_quant_centered_matches_oracle(cuda):
    """Mean-centred DQ (an option from outside the pages): codes, h and mean bit-exact on
    ragged sizes, wide and narrow value ranges, a constant block, a zero block, subnormal
    and huge constants mixed with ordinary ones."""
    rng = np.random.default_rng(15)
    cases = []
    for nb in (1, 2, 255, 256, 257, 1000, 4096 + 3, 30000):
        a = np.abs(rng.standard_normal(nb)).astype(np.float32) * 0.03
        if nb > 600:
            a[256:512] = np.float32(0.0125)   # a constant block: h = 0, codes 128
            a[512:520] = 0.0                  # zeros inside a block
        cases.append(a)
    wide = np.abs(rng.standard_normal(2048)).astype(np.float32) * \
        np.exp2(rng.integers(-30, 30, 2048)).astype(np.float32)
    wide[:5] = [1e-40, 3e-39, 2.0 ** -140, 1e30, 0.0]  # subnormal, tiny and huge constants
    cases.append(wide)
    for a in cases:
        codes8, scales, means = aqnf4.double_quant_centered(torch.from_numpy(a).to(cuda))
        oc, osc, omu, _ = oracle.double_quant_centered(a)
        assert np.array_equal(codes8.cpu().numpy(), oc), a.size
        assert same_float_bits(scales.cpu().numpy(), osc), a.size
        assert same_float_bits(means.cpu().numpy(), omu), a.size


def test_double_quant_centered_nonfinite_flag(cuda):
    a = np.full(600, 0.5, np.float32)
    a[300] = np.nan
    a[10] = np.inf
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    nd = 3
    codes8 = torch.empty(600, dtype=torch.uint8, device=cuda)
    scales = torch.empty(nd, dtype=torch.float32, device=cuda)
    means = torch.empty(nd, dtype=torch.float32, device=cuda)
    aqnf4.aqnf4_double_quant_centered(torch.from_numpy(a).to(cuda), codes8, scales, means, flag)
    assert flag.item() == aqnf4.AQNF4_ERR_NONFINITE
    oc, osc, omu, onf = oracle.double_quant_centered(a)
    assert onf
    assert np.array_equal(codes8.cpu().numpy(), oc)
    assert same_float_bits(scales.cpu().numpy(), osc)
    assert same_float_bits(means.cpu().numpy(), omu)


@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n", [1, 9, 64, 65, 16384 + 3, 200001])
def test_dequantize_centered_matches_oracle(cuda, out_dt, n):
    w = synth.random_bits_host(n, seed=n + 17, dtype=torch.bfloat16)
    op, oa, _ = oracle.quantize(bits(w), oracle.BF16)
    oc, osc, omu, _ = oracle.double_quant_centered(oa)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(cuda)
    out = torch.empty(n, dtype=out_dt, device=cuda)
    aqnf4.aqnf4_dequantize_centered(dev(op), dev(oc), dev(osc), dev(omu), n, out)
    ref = oracle.dequantize_centered(op, n, DT[out_dt], oc, osc, omu)
    assert np.array_equal(bits(out.cpu()), ref)


@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n", [1, 2, 7, 8, 9, 63, 64, 65, 1023, 16384 + 3, 200001])
def test_dequantize_matches_oracle(cuda, out_dt, n):
    w = synth.random_bits_host(n, seed=n + 7, dtype=torch.bfloat16)
    op, oa, _ = oracle.quantize(bits(w), oracle.BF16)
    oc, osc, _ = oracle.double_quant(oa)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(cuda)
    got = aqnf4.dequantize(dev(op), n, out_dt, codes8=dev(oc), scales=dev(osc))
    ref = oracle.dequantize(op, n, DT[out_dt], codes8=oc, scales=osc)
    assert np.array_equal(bits(got.cpu()), ref)
    got2 = aqnf4.dequantize(dev(op), n, out_dt, absmax=dev(oa))
    ref2 = oracle.dequantize(op, n, DT[out_dt], absmax=oa)
    assert np.array_equal(bits(got2.cpu()), ref2)


@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n", [9, 65, 1023, 16384 + 3, 200001])
def test_dequantize_16_byte_aligned_output(cuda, out_dt, n):
    """An output that is 16- but not 32-byte aligned takes the 16-byte-store path (an
    aligned one the 32-byte-store path, above); both, plain and mean-centred, equal the
    oracle bit for bit, and the 16 bytes in front of the output stay untouched."""
    w = synth.random_bits_host(n, seed=n + 23, dtype=torch.bfloat16)
    op, oa, _ = oracle.quantize(bits(w), oracle.BF16)
    oc, osc, _ = oracle.double_quant(oa)
    cc, csc, cmu, _ = oracle.double_quant_centered(oa)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(cuda)
    buf = torch.full((n + 8,), 7, dtype=out_dt, device=cuda)  # 256-byte aligned allocation
    out = buf[8:]  # 16 bytes in: aligned to 16 bytes, not to 32
    assert out.data_ptr() % 32 == 16
    aqnf4.aqnf4_dequantize(dev(op), dev(oc), dev(osc), None, n, out)
    assert np.array_equal(bits(out.cpu()), oracle.dequantize(op, n, DT[out_dt], codes8=oc,
                                                            scales=osc))
    aqnf4.aqnf4_dequantize_centered(dev(op), dev(cc), dev(csc), dev(cmu), n, out)
    assert np.array_equal(bits(out.cpu()), oracle.dequantize_centered(op, n, DT[out_dt], cc,
                                                                     csc, cmu))
    assert torch.equal(buf[:8].cpu(), torch.full((8,), 7, dtype=out_dt))


@pytest.mark.parametrize("seed", range(8))
def test_select_topk_matches_oracle(cuda, seed):
    rng = np.random.default_rng(seed)
    L = int(rng.choice([1, 2, 5, 28, 280, 1100, 2500]))
    e = rng.uniform(0, 1, L).astype(np.float32)
    e[rng.uniform(size=L) < 0.2] = 0.5  # ties
    e[rng.uniform(size=L) < 0.05] = np.nan
    cost = rng.integers(1, 1 << 30, L).astype(np.int64)
    if seed % 3 == 0:
        cost[rng.integers(0, L)] = -5  # a layer cheaper in 16 bits than in NF4
    budget = int(rng.integers(0, int(cost[cost > 0].sum()) + 1))
    k_cap = int(rng.choice([-1, 0, 1, 3, L]))
    sel, k = aqnf4.select_topk(torch.from_numpy(e).to(cuda), torch.from_numpy(cost).to(cuda),
                               budget, k_cap)
    ref = oracle.select_topk(e, cost, budget, k_cap)
    got = sel.cpu().numpy()
    assert got[: k.item()].tolist() == ref
    full = oracle.select_topk(e, np.zeros(L, np.int64), 0, -1)
    assert got.tolist() == full  # the whole ranking is returned


def test_bounded_wait_gives_up_and_reports(cuda):
    """A wait on an mbarrier nothing completes ends with AQNF4_ERR_TIMEOUT, not a hang, and the
    context keeps working afterwards."""
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    waited = torch.zeros(1, dtype=torch.int64, device=cuda)
    aqnf4.aqnf4_selftest_wait_timeout(20_000_000, flag, waited)  # 20 ms
    torch.cuda.synchronize()
    assert flag.item() == aqnf4.AQNF4_ERR_TIMEOUT
    assert 20_000_000 <= waited.item() < 2_000_000_000
    # the device is still usable: a normal call right after succeeds and is correct
    w = synth.random_bits_host(1000, seed=5, dtype=torch.bfloat16)
    packed, _ = aqnf4.quantize(w.to(cuda))
    assert np.array_equal(packed.cpu().numpy(), oracle.quantize(bits(w), oracle.BF16)[0])


def _midpoint_tie_blocks(dt):
    """Blocks whose elements normalise exactly onto a codebook midpoint or one ulp beside it.

    For every 16-bit block maximum a and every target m (each midpoint and its binary32
    neighbours), the 16-bit values next to m * a are tried; those with fl(x * fl(1/a)) == m
    are kept.  A block is [a, its ties..., zeros], so its absmax is a.  These are the inputs
    where the code is decided by a comparison with no slack at all ("QLoRA", "How It Works":
    the nearest level, with ties going to the lower one).  binary16 has about 150 such
    elements; bfloat16 has none (with 8-bit significands x * fl(1/a) never lands on these
    binary32 midpoints; the closest are about 11 ulps away), so only binary16 is tested.
    """
    levels, mids = oracle.codebook()
    targets = np.concatenate([mids, np.nextafter(mids, np.float32(2)),
                              np.nextafter(mids, np.float32(-2))]).astype(np.float32)
    h = np.arange(0x8000, dtype=np.int64)
    av = torch.from_numpy(h.astype(np.int16)).view(dt).float().numpy()
    keep = np.isfinite(av) & (av >= 2.0 ** -126)
    h, av = h[keep], av[keep]
    r = (np.float32(1) / av).astype(np.float32)
    est = (targets[None, :] * av[:, None]).astype(np.float32)          # (A, T)
    est16 = torch.from_numpy(est).to(dt).view(torch.int16).numpy().astype(np.int64)
    blocks = []
    for d in (-1, 0, 1):
        cand = est16 + np.where(est16 >= 0, d, -d)                      # magnitude neighbours
        cand16 = (cand & 0xFFFF).astype(np.uint16).view(np.int16)
        xv = torch.from_numpy(cand16).view(dt).float().numpy()
        v = (xv * r[:, None]).astype(np.float32)
        hit = (v == targets[None, :]) & (np.abs(xv) <= av[:, None])
        for ai in np.nonzero(hit.any(1))[0]:
            xs = xv[ai][hit[ai]]
            blocks.append((av[ai], xs))
    w = []
    for a, xs in blocks:
        for s in range(0, len(xs), 63):
            body = np.zeros(63, np.float32)
            part = xs[s:s + 63]
            body[:len(part)] = part
            w.append(np.concatenate([[a], body]))
    return torch.from_numpy(np.concatenate(w).astype(np.float32)).to(dt)


def test_quantize_exact_midpoint_ties(cuda):
    dt = torch.float16
    w = _midpoint_tie_blocks(dt)
    assert w.numel() >= 64 * 200
    packed, absmax = aqnf4.quantize(w.to(cuda))
    op, oa, _ = oracle.quantize(bits(w), DT[dt])
    assert np.array_equal(packed.cpu().numpy(), op)
    assert same_float_bits(absmax.cpu().numpy(), oa)
    stor = aqnf4.NF4Storage(w.numel(), cuda)
    se, sw, rel = aqnf4.score_layers([w.to(cuda)], [stor])
    assert np.array_equal(stor.packed.cpu().numpy(), op)
    ose, osw, orel = oracle.layer_error(bits(w), DT[dt])
    assert se.item() == pytest.approx(ose, rel=RTOL)
    assert rel.item() == pytest.approx(orel, rel=RTOL)


# ------------------------------------------------- score against the DQ constants


def _dq_case_layers():
    """Ragged random layers of both formats plus one with special blocks inside a DQ block:
    zeros, a block far below the DQ block's maximum (its constant double-quantizes to 0),
    a subnormal maximum and a huge one."""
    rng = np.random.default_rng(31)
    out = []
    for n, dt in ((1, torch.bfloat16), (65, torch.float16), (16385, torch.bfloat16),
                  (3 * 16384 + 17, torch.float16), (100003, torch.bfloat16)):
        sig = np.repeat(rng.uniform(0.002, 0.05, n // 64 + 1), 64)[:n]
        out.append(torch.from_numpy((rng.standard_normal(n) * sig).astype(np.float32)).to(dt))
    blocks = [rng.standard_normal(64) * 0.02 for _ in range(300)]
    blocks[3] = np.zeros(64)
    blocks[4] = rng.standard_normal(64) * 1e-6           # code8 0: rebuilt from a' = 0
    blocks[5] = rng.standard_normal(64) * 1e-39          # subnormal absmax (generic path)
    blocks[6] = rng.standard_normal(64) * 3e20           # above 2^40 (generic path)
    blocks[7] = rng.standard_normal(64) * 2e-4           # small non-zero code8
    out.append(torch.from_numpy(np.concatenate(blocks).astype(np.float32)).to(torch.bfloat16))
    return out


def test_dq_score_matches_oracle_and_keeps_the_storage(cuda):
    ws = _dq_case_layers()
    dev = [w.to(cuda) for w in ws]
    plain_st = [aqnf4.NF4Storage(w.numel(), cuda) for w in dev]
    dq_st = [aqnf4.NF4Storage(w.numel(), cuda) for w in dev]
    _, _, _ = aqnf4.score_layers(dev, plain_st)
    se, sw, rel = aqnf4.score_layers(dev, dq_st, dq_score=True)
    torch.cuda.synchronize()
    for i, w in enumerate(ws):
        ose, osw, orel = oracle.layer_error_dq(bits(w), DT[w.dtype])
        assert se[i].item() == pytest.approx(ose, rel=RTOL), i
        assert sw[i].item() == pytest.approx(osw, rel=RTOL), i
        assert rel[i].item() == pytest.approx(orel, rel=RTOL), i
        for name in ("packed", "codes8", "scales"):  # the flag changes only the score
            assert torch.equal(getattr(dq_st[i], name), getattr(plain_st[i], name)), (i, name)


def test_centered_dq_score_matches_oracle_and_keeps_the_storage(cuda):
    """The score against mean-centred DQ constants (a format from outside the pages) within
    1e-5 of the oracle's, on ragged layers with zero, tiny and huge blocks; the stored
    outputs stay the plain format's."""
    ws = _dq_case_layers()
    dev = [w.to(cuda) for w in ws]
    plain_st = [aqnf4.NF4Storage(w.numel(), cuda) for w in dev]
    dq_st = [aqnf4.NF4Storage(w.numel(), cuda) for w in dev]
    aqnf4.score_layers(dev, plain_st)
    se, sw, rel = aqnf4.score_layers(dev, dq_st, dq_score="centered")
    torch.cuda.synchronize()
    for i, w in enumerate(ws):
        ose, osw, orel = oracle.layer_error_dqc(bits(w), DT[w.dtype])
        assert se[i].item() == pytest.approx(ose, rel=RTOL), i
        assert sw[i].item() == pytest.approx(osw, rel=RTOL), i
        assert rel[i].item() == pytest.approx(orel, rel=RTOL), i
        for name in ("packed", "codes8", "scales"):
            assert torch.equal(getattr(dq_st[i], name), getattr(plain_st[i], name)), (i, name)


@pytest.mark.parametrize("extreme", ["smallest", "largest"])
def test_centered_dq_score_h_at_either_extreme(cuda, extreme):
    """h = max |a - mu| comes from the tile's smallest constant (255 blocks near 1, one zero
    block: mu near 1) or from its largest (255 blocks near 1, one block of 1000)."""
    rng = np.random.default_rng(41 if extreme == "smallest" else 42)
    w = rng.uniform(-1.0, 1.0, size=(256, 64)).astype(np.float32)
    w[:, 0] = 1.0  # every block's absmax is 1 ...
    if extreme == "smallest":
        w[77] = 0.0  # ... but one zero block
    else:
        w[77] *= 1000.0  # ... but one huge block
    for dt in (torch.bfloat16, torch.float16):
        x = torch.from_numpy(w.reshape(-1)).to(dt)
        st = [aqnf4.NF4Storage(x.numel(), cuda)]
        se, sw, rel = aqnf4.score_layers([x.to(cuda)], st, dq_score="centered")
        torch.cuda.synchronize()
        ose, osw, orel = oracle.layer_error_dqc(bits(x), DT[dt])
        assert se[0].item() == pytest.approx(ose, rel=RTOL)
        assert sw[0].item() == pytest.approx(osw, rel=RTOL)
        assert rel[0].item() == pytest.approx(orel, rel=RTOL)


def test_three_scores_in_one_call(cuda):
    """Flags are per layer: plain, DQ-absmax and centred scores mixed in one launch."""
    ws = _dq_case_layers()
    dev = [w.to(cuda) for w in ws]
    modes = [0, aqnf4.AQNF4_SCORE_DQ_ABSMAX, aqnf4.AQNF4_SCORE_DQ_CENTERED]
    refs = [oracle.layer_error, oracle.layer_error_dq, oracle.layer_error_dqc]
    descs = aqnf4.make_layers([{"w": w, "flags": modes[i % 3]} for i, w in enumerate(dev)])
    L = len(dev)
    wsp = torch.empty(max(256, aqnf4.aqnf4_workspace_size(descs)), dtype=torch.uint8, device=cuda)
    se = torch.empty(L, dtype=torch.float64, device=cuda)
    rel = torch.empty(L, dtype=torch.float32, device=cuda)
    aqnf4.aqnf4_layer_error(descs, wsp, se, None, rel)
    torch.cuda.synchronize()
    for i, w in enumerate(ws):
        ose, _, orel = refs[i % 3](bits(w), DT[w.dtype])
        assert se[i].item() == pytest.approx(ose, rel=RTOL), i
        assert rel[i].item() == pytest.approx(orel, rel=RTOL), i


def test_dq_and_plain_scores_in_one_call(cuda):
    """Flags are per layer: alternating layers in one launch each get their own score."""
    ws = _dq_case_layers()
    dev = [w.to(cuda) for w in ws]
    descs = aqnf4.make_layers([{"w": w, "flags": aqnf4.AQNF4_SCORE_DQ_ABSMAX if i % 2 else 0}
                               for i, w in enumerate(dev)])
    L = len(dev)
    wsp = torch.empty(max(256, aqnf4.aqnf4_workspace_size(descs)), dtype=torch.uint8, device=cuda)
    se = torch.empty(L, dtype=torch.float64, device=cuda)
    sw = torch.empty(L, dtype=torch.float64, device=cuda)
    rel = torch.empty(L, dtype=torch.float32, device=cuda)
    aqnf4.aqnf4_layer_error(descs, wsp, se, sw, rel)
    torch.cuda.synchronize()
    for i, w in enumerate(ws):
        ref = oracle.layer_error_dq if i % 2 else oracle.layer_error
        ose, _, orel = ref(bits(w), DT[w.dtype])
        assert se[i].item() == pytest.approx(ose, rel=RTOL), i
        assert rel[i].item() == pytest.approx(orel, rel=RTOL), i


def test_dq_score_nonfinite_tile_is_nan(cuda):
    """An infinite weight makes its DQ block's scale infinite, so every constant of that
    block rebuilds as NaN: the score is NaN (as in the oracle) and the flag is set."""
    rng = np.random.default_rng(32)
    z = rng.standard_normal(64 * 300) * 0.02
    z[64 * 10 + 3] = np.inf
    w = torch.from_numpy(z.astype(np.float32)).to(torch.bfloat16)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    descs = aqnf4.make_layers([{"w": w.to(cuda), "flags": aqnf4.AQNF4_SCORE_DQ_ABSMAX}])
    wsp = torch.empty(256, dtype=torch.uint8, device=cuda)
    rel = torch.empty(1, dtype=torch.float32, device=cuda)
    aqnf4.aqnf4_layer_error(descs, wsp, None, None, rel, flag)
    torch.cuda.synchronize()
    assert math.isnan(oracle.layer_error_dq(bits(w), oracle.BF16)[2])
    assert math.isnan(rel.item())
    assert flag.item() == aqnf4.AQNF4_ERR_NONFINITE


# ------------------------------------------------------------ block-level selection


def _block_case(rng, L, B):
    block_of = np.sort(rng.integers(0, B, L)).astype(np.int32)
    sw = rng.uniform(0.5, 40.0, L)
    se = rng.uniform(0.002, 0.05, L) * sw
    cost = rng.integers(1, 1 << 30, L).astype(np.int64)
    return se, sw, block_of, cost


@pytest.mark.parametrize("order", [aqnf4.AQNF4_BLOCKS_BY_DEPTH, aqnf4.AQNF4_BLOCKS_BY_ERROR])
@pytest.mark.parametrize("seed,L,B", [(0, 7, 3), (1, 224, 32), (2, 280, 40), (3, 3000, 1500),
                                      (4, 5, 2048)])
def test_select_blocks_matches_oracle(cuda, order, seed, L, B):
    rng = np.random.default_rng(seed)
    se, sw, block_of, cost = _block_case(rng, L, B)
    if L > 10:
        se[L // 3] = np.nan                          # a non-finite layer ranks its block last
        se[L // 2] = se[L // 2 + 1] = 0.0            # equal scores
        sw[L // 2] = sw[L // 2 + 1] = 1.0
    total = int(cost.sum())
    d = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(cuda)
    for budget in (0, total // 7, total // 2, total):
        rank = torch.empty(B, dtype=torch.int32, device=cuda)
        err = torch.empty(B, dtype=torch.float32, device=cuda)
        k = torch.empty(1, dtype=torch.int32, device=cuda)
        aqnf4.aqnf4_select_blocks(d(se, torch.float64), d(sw, torch.float64),
                                  d(block_of, torch.int32), d(cost, torch.int64), B, budget,
                                  order, rank, err, k)
        orank, oerr, ok = oracle.select_blocks(se, sw, block_of, cost, B, budget, order)
        assert same_float_bits(err.cpu().numpy(), oerr)
        assert rank.cpu().tolist() == orank
        assert k.item() == ok


def test_select_blocks_on_scored_model(cuda):
    """The 7B-shaped model's real scores, grouped by transformer block."""
    wl = synth.workload("7b")
    weights = [synth.layer_device(s, wl.seed, i, cuda) for i, s in enumerate(wl.layers)]
    se, sw, _ = aqnf4.score_layers(weights)
    del weights
    block_of = torch.tensor(synth.block_index(wl), dtype=torch.int32, device=cuda)
    cost = torch.tensor([aqnf4.aqnf4_cost_bytes(s.numel) for s in wl.layers], dtype=torch.int64,
                        device=cuda)
    B = int(block_of.max().item()) + 1
    for order in (aqnf4.AQNF4_BLOCKS_BY_DEPTH, aqnf4.AQNF4_BLOCKS_BY_ERROR):
        rank = torch.empty(B, dtype=torch.int32, device=cuda)
        k = torch.empty(1, dtype=torch.int32, device=cuda)
        aqnf4.aqnf4_select_blocks(se, sw, block_of, cost, B, wl.budgets[0], order, rank, None, k)
        orank, _, ok = oracle.select_blocks(se.cpu().numpy(), sw.cpu().numpy(),
                                            block_of.cpu().numpy(), cost.cpu().numpy(), B,
                                            wl.budgets[0], order)
        assert rank.cpu().tolist() == orank and k.item() == ok


def test_select_blocks_reports_a_bad_block_index(cuda):
    se = torch.ones(4, dtype=torch.float64, device=cuda)
    block_of = torch.tensor([0, 1, 5, 1], dtype=torch.int32, device=cuda)
    cost = torch.ones(4, dtype=torch.int64, device=cuda)
    rank = torch.empty(2, dtype=torch.int32, device=cuda)
    k = torch.empty(1, dtype=torch.int32, device=cuda)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda)
    aqnf4.aqnf4_select_blocks(se, se, block_of, cost, 2, 10, aqnf4.AQNF4_BLOCKS_BY_DEPTH, rank,
                              None, k, dev_flag=flag)
    assert k.item() == -1
    assert flag.item() == aqnf4.AQNF4_ERR_INVALID_ARG
    # a valid call leaves the flag word alone
    flag.zero_()
    block_of = torch.tensor([0, 1, 1, 1], dtype=torch.int32, device=cuda)
    aqnf4.aqnf4_select_blocks(se, se, block_of, cost, 2, 10, aqnf4.AQNF4_BLOCKS_BY_DEPTH, rank,
                              None, k, dev_flag=flag)
    assert k.item() == 2 and flag.item() == 0
