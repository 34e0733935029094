"""Pins of the CPU oracle to facts fixed outside it (no GPU).

Each test checks the oracle against something it does not share code with: numbers the
pages state (tests/golden/pages_facts.json), library routines (scipy / statistics normal
quantiles, numpy and torch 16-bit rounding), closed forms, invariants (monotonicity,
power-of-two scale invariance, exact round trip), and brute force on small inputs
(nearest level by exhaustive search, selection over all subsets).  The last tests plant
mistakes in the oracle's inputs and check that the pins catch them.
"""
import itertools
import json
import math
import os
from statistics import NormalDist

import numpy as np
import pytest
import torch
from scipy.special import ndtri
from scipy.stats import norm

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")
with open(GOLDEN) as _f:
    FACTS = json.load(_f)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def codes_of(packed: np.ndarray, n: int) -> np.ndarray:
    c = np.stack([packed >> 4, packed & 15], axis=1).reshape(-1)
    return c[:n].astype(np.int64)


# ------------------------------------------------------------------ codebook


def test_codebook_shape_and_anchors(book):
    levels, mids = book
    assert levels.size == FACTS["nf4_values"]["value"] == 16
    assert levels[0] == -1.0 and levels[15] == 1.0
    assert levels[7] == 0.0 and not np.signbit(levels[7])
    assert np.all(np.diff(levels.astype(np.float64)) > 0)
    # 7 negative levels, exact zero, 8 positive (asymmetric so that 0 and both ends exist)
    assert (levels < 0).sum() == 7 and (levels > 0).sum() == 8
    assert np.all((mids > levels[:-1]) & (mids < levels[1:]))


def test_codebook_against_library_quantiles(book):
    """Normal quantiles recomputed with scipy's ndtri and with statistics.NormalDist."""
    levels, mids = book
    pm = oracle.default_pmax()
    assert pm == pytest.approx(1 - 0.5 * (1 / 32 + 1 / 30), abs=0)
    pos = [ndtri(pm - k * (pm - 0.5) / 8) for k in range(8)]
    neg = [-ndtri(pm - k * (pm - 0.5) / 7) for k in range(7)]
    ref = np.array(sorted(pos + neg + [0.0])) / ndtri(pm)
    assert np.array_equal(levels, ref.astype(np.float32))
    nd = NormalDist()
    ref2 = np.array(sorted([nd.inv_cdf(pm - k * (pm - 0.5) / 8) for k in range(8)]
                           + [-nd.inv_cdf(pm - k * (pm - 0.5) / 7) for k in range(7)] + [0.0]))
    ref2 /= nd.inv_cdf(pm)
    assert np.max(np.abs(levels.astype(np.float64) - ref2)) < 2 ** -24
    mref = ((levels[:-1].astype(np.float64) + levels[1:].astype(np.float64)) / 2).astype(np.float32)
    assert np.array_equal(mids, mref)


def test_codebook_equal_probability_spacing(book):
    """Each half's levels sit at evenly spaced normal probabilities ("equal share")."""
    levels, _ = book
    z = ndtri(oracle.default_pmax())
    p = norm.cdf(levels.astype(np.float64) * z)
    assert np.allclose(np.diff(p[:8]), np.diff(p[:8]).mean(), rtol=0, atol=1e-7)
    assert np.allclose(np.diff(p[7:]), np.diff(p[7:]).mean(), rtol=0, atol=1e-7)
    assert p[0] == pytest.approx(1 - oracle.default_pmax(), abs=1e-7)
    assert p[15] == pytest.approx(oracle.default_pmax(), abs=1e-7)


def test_codebook_histogram_roughly_flat(book):
    """Normal samples at the codebook's own scale land nearly evenly on the 16 values."""
    _, mids = book
    z = ndtri(oracle.default_pmax())
    x = np.random.default_rng(0).standard_normal(400_000) / z
    h = np.bincount(np.searchsorted(mids.astype(np.float64), x, side="left"), minlength=16)
    r = h / h.mean()
    assert r.min() > 0.8 and r.max() < 1.2, r


def test_codebook_rejects_bad_pmax():
    for bad in (0.5, 1.0, 0.2, 1.5):
        with pytest.raises(ValueError):
            oracle.codebook(bad)


# ---------------------------------------------------------------- conversions


def test_dtype_decode_all_bit_patterns():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f16 = oracle.dtype_bits_to_f32(allbits, oracle.F16)
    ref16 = allbits.view(np.float16).astype(np.float32)
    same = (f16.view(np.uint32) == ref16.view(np.uint32)) | (np.isnan(f16) & np.isnan(ref16))
    assert same.all()
    bf = oracle.dtype_bits_to_f32(allbits, oracle.BF16)
    refb = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).float().numpy()
    same = (bf.view(np.uint32) == refb.view(np.uint32)) | (np.isnan(bf) & np.isnan(refb))
    assert same.all()


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_dtype_rounding_matches_libraries(dtype):
    rng = np.random.default_rng(1)
    parts = [rng.standard_normal(20000).astype(np.float32) * s for s in (1e-8, 1e-5, 0.02, 3, 7e4)]
    # ties and their neighbours: halfway points between adjacent 16-bit values
    base = rng.standard_normal(4000).astype(np.float32)
    if dtype == oracle.F16:
        lo = base.astype(np.float16).astype(np.float32)
    else:
        lo = torch.from_numpy(base).to(torch.bfloat16).float().numpy()
    hi = np.nextafter(lo, np.float32(np.inf) * np.sign(lo + 1e-30))
    parts += [lo, (lo.astype(np.float64) + 2.0 ** -30).astype(np.float32), hi]
    if dtype == oracle.BF16:
        parts.append(np.array([3.3e38, -3.39e38, 1e-39, -2e-40, 0.0, -0.0], np.float32))
    else:
        parts.append(np.array([65519.0, 65520.0, -70000.0, 6e-8, 3e-8, 2.9e-8, -0.0], np.float32))
    x = np.concatenate(parts)
    got = oracle.f32_to_dtype_bits(x, dtype)
    if dtype == oracle.F16:
        with np.errstate(over="ignore"):
            ref = x.astype(np.float16).view(np.uint16)
    else:
        ref = bits_of(torch.from_numpy(x).to(torch.bfloat16))
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- quantize


def _nearest_level_bruteforce(v64: np.ndarray, levels: np.ndarray) -> np.ndarray:
    d = np.abs(v64[:, None] - levels.astype(np.float64)[None, :])
    return np.argmin(d, axis=1)  # argmin takes the first (lower) index on ties


def _normalized(x32: np.ndarray, a: float) -> np.ndarray:
    r = np.float32(1.0) / np.float32(a)
    return (x32 * r).astype(np.float32)


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_codes_equal_nearest_level_bruteforce(book, dtype):
    levels, mids = book
    rng = np.random.default_rng(7)
    tdt = torch.float16 if dtype == oracle.F16 else torch.bfloat16
    w = torch.from_numpy(
        np.concatenate([rng.standard_normal(64 * 300), rng.standard_t(3, 64 * 200),
                        rng.uniform(-1, 1, 64 * 100)]).astype(np.float32) * 0.02).to(tdt)
    bits = bits_of(w)
    packed, absmax, nonfinite = oracle.quantize(bits, dtype)
    assert not nonfinite
    codes = codes_of(packed, bits.size)
    x = w.float().numpy()
    # the oracle's absmax is the plain max |x| per block
    assert np.array_equal(absmax, np.abs(x).reshape(-1, 64).max(axis=1))
    v = np.concatenate([_normalized(xb, a) for xb, a in zip(x.reshape(-1, 64), absmax)])
    brute = _nearest_level_bruteforce(v.astype(np.float64), levels)
    diff = codes != brute
    # the midpoint rule and exhaustive search may only differ within 1 ulp of a midpoint
    if diff.any():
        vv = v[diff]
        gap = np.min(np.abs(vv[:, None].astype(np.float64) - mids.astype(np.float64)[None, :]), axis=1)
        assert np.all(gap <= np.spacing(np.abs(vv)) * 1.0), (vv, gap)
    assert diff.sum() <= 2


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_round_trip_on_scaled_levels(book, dtype):
    """Weights equal to dtype(level * a), with a present, come back exactly: error 0."""
    levels, _ = book
    rng = np.random.default_rng(3)
    tdt = torch.float16 if dtype == oracle.F16 else torch.bfloat16
    nblk = 64
    codes = rng.integers(0, 16, size=(nblk, 64))
    codes[:, 5] = rng.choice([0, 15], size=nblk)  # absmax element (|level| = 1)
    a = torch.from_numpy(rng.uniform(0.001, 0.5, nblk).astype(np.float32)).to(tdt).float().numpy()
    prod = (levels[codes] * a[:, None]).astype(np.float32)
    w = torch.from_numpy(prod.reshape(-1)).to(tdt)
    bits = bits_of(w)
    packed, absmax, _ = oracle.quantize(bits, dtype)
    assert np.array_equal(absmax, a)
    assert np.array_equal(codes_of(packed, bits.size), codes.reshape(-1))
    # the packed layout: even element in the high nibble
    c = codes.reshape(-1)
    assert np.array_equal(packed, ((c[0::2] << 4) | c[1::2]).astype(np.uint8))
    se, sw, rel = oracle.layer_error(bits, dtype)
    assert se == 0.0 and rel == 0.0 and sw > 0
    back = oracle.dequantize(packed, bits.size, dtype, absmax=absmax)
    assert np.array_equal(back, bits)


def test_zero_block_and_ragged_tail(book):
    w = np.zeros(65, np.float16)
    w[64] = 0.5
    packed, absmax, _ = oracle.quantize(w, oracle.F16)
    assert packed.size == 33 and absmax.size == 2
    assert np.all(packed[:32] == 0x77)
    assert absmax[0] == 0.0 and absmax[1] == 0.5
    assert packed[32] == 0xF0  # code 15 in the high nibble, low nibble left 0
    se, sw, rel = oracle.layer_error(np.zeros(100, np.float16), oracle.F16)
    assert (se, sw, rel) == (0.0, 0.0, 0.0)


def test_codes_monotone_in_x(book):
    rng = np.random.default_rng(11)
    x = np.sort(rng.standard_normal((50, 64)).astype(np.float16), axis=1)
    packed, _, _ = oracle.quantize(x.reshape(-1), oracle.F16)
    c = codes_of(packed, x.size).reshape(50, 64)
    assert np.all(np.diff(c, axis=1) >= 0)


@pytest.mark.parametrize("k", [-9, -1, 3, 20])
def test_power_of_two_scale_invariance(k):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(64 * 40) * 0.02).astype(np.float32)
    w = torch.from_numpy(x).to(torch.bfloat16)
    ws = (w.float() * 2.0 ** k).to(torch.bfloat16)  # exact: power of two, no range issue
    assert torch.equal(ws.float() / 2.0 ** k, w.float())
    p1, a1, _ = oracle.quantize(bits_of(w), oracle.BF16)
    p2, a2, _ = oracle.quantize(bits_of(ws), oracle.BF16)
    assert np.array_equal(p1, p2)
    assert np.array_equal(a2, (a1 * 2.0 ** k).astype(np.float32))
    r1 = oracle.layer_error(bits_of(w), oracle.BF16)[2]
    r2 = oracle.layer_error(bits_of(ws), oracle.BF16)[2]
    assert r1 == r2


def test_subnormal_absmax_block_is_scale_invariant():
    """A bf16 block below the fp32 normal range codes like the same block scaled by 2^100."""
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(64 * 8) * 1e-39).astype(np.float32)
    w = torch.from_numpy(x).to(torch.bfloat16)
    big = (w.double() * 2.0 ** 100).to(torch.bfloat16)
    assert torch.equal((big.double() / 2.0 ** 100).to(torch.bfloat16), w)
    p1, a1, _ = oracle.quantize(bits_of(w), oracle.BF16)
    p2, _, _ = oracle.quantize(bits_of(big), oracle.BF16)
    assert np.all(a1 < 2.0 ** -126)
    assert np.array_equal(p1, p2)


def test_nonfinite_inputs_flagged():
    w = np.zeros(200, np.float16)
    w[3] = np.nan
    w[100] = np.inf
    packed, absmax, nonfinite = oracle.quantize(w, oracle.F16)
    assert nonfinite and np.isnan(absmax[0]) and np.isinf(absmax[1])
    assert math.isnan(oracle.layer_error(w, oracle.F16)[2])


# ---------------------------------------------------------------- score


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_layer_error_matches_bruteforce_reconstruction(book, dtype):
    levels, _ = book
    rng = np.random.default_rng(21)
    tdt = torch.float16 if dtype == oracle.F16 else torch.bfloat16
    n = 64 * 97 + 13
    w = torch.from_numpy((rng.standard_t(4, n) * 0.01).astype(np.float32)).to(tdt)
    bits = bits_of(w)
    x = w.double().numpy()
    nb = (n + 63) // 64
    se = 0.0
    for b in range(nb):
        xb = w.float().numpy()[64 * b: 64 * b + 64]
        a = np.float32(np.abs(xb).max())
        v = _normalized(xb, a)
        c = _nearest_level_bruteforce(v.astype(np.float64), levels)
        what = torch.from_numpy((levels[c] * a).astype(np.float32)).to(tdt).double().numpy()
        se += float(np.sum((x[64 * b: 64 * b + 64] - what) ** 2))
    o_se, o_sw, o_rel = oracle.layer_error(bits, dtype)
    assert o_sw == pytest.approx(float(np.sum(x * x)), rel=1e-13)
    assert o_se == pytest.approx(se, rel=1e-12)
    assert o_rel == pytest.approx(math.sqrt(se / float(np.sum(x * x))), rel=1e-6)


def test_heavy_tailed_layers_rank_first_on_tiny():
    from quantized_lora_setup_b200 import synth
    wl = synth.tiny(0)
    rel, cost = [], []
    for i, spec in enumerate(wl.layers):
        w = synth.layer_host(spec, wl.seed, i)
        rel.append(oracle.layer_error(bits_of(w), oracle.F16)[2])
        cost.append(oracle.cost_bytes(spec.numel))
    heavy = sorted(i for i, s in enumerate(wl.layers) if s.dist == "t")
    sel = oracle.select_topk(rel, cost, wl.budgets[0], wl.k_cap)
    assert sorted(sel) == heavy
    normal = [r for i, r in enumerate(rel) if i not in heavy]
    assert min(rel[i] for i in heavy) > 1.05 * max(normal)


def _expected_normal_block_error(levels, mids, block=64):
    """Limit of the relative NF4 error of a large layer of i.i.d. N(0, 1) weights in blocks
    of `block`, by fp64 quadrature (no sampling, no quantizer).  Given the block absmax a,
    the block holds one element at +-a (coded exactly) and block - 1 elements ~ N(0, 1)
    truncated to (-a, a).  On the cell (a m_(j-1), a m_j] every x goes to c = a q_j, and
    the integral of (x - c)^2 phi(x) over [l, h] has the closed form
    (Phi(h) - Phi(l)) + l phi(l) - h phi(h) - 2c (phi(l) - phi(h)) + c^2 (Phi(h) - Phi(l)).
    a has density block * 2 phi(a) (2 Phi(a) - 1)^(block - 1).  The layer's error tends to
    sqrt((block - 1) / block * E_a[g(a)]) with g(a) the conditional mean square error."""
    from scipy.integrate import quad
    q = np.asarray(levels, np.float64)
    edges = np.concatenate([[-1.0], np.asarray(mids, np.float64), [1.0]])

    def g(a):
        lo, hi = a * edges[:-1], a * edges[1:]
        c = a * q
        P = norm.cdf(hi) - norm.cdf(lo)
        m2 = P + lo * norm.pdf(lo) - hi * norm.pdf(hi)
        m1 = norm.pdf(lo) - norm.pdf(hi)
        return float(np.sum(m2 - 2 * c * m1 + c * c * P)) / (2 * norm.cdf(a) - 1)

    def dens(a):
        return block * 2 * norm.pdf(a) * (2 * norm.cdf(a) - 1) ** (block - 1)

    mass = quad(dens, 0, 12, limit=400, points=[2, 3])[0]
    eg = quad(lambda a: g(a) * dens(a), 0, 12, limit=400, points=[2, 3])[0]
    assert abs(mass - 1) < 1e-9
    return math.sqrt((block - 1) / block * eg)


def test_expected_error_of_normal_blocks(book):
    """The oracle's score of a 2^22-element N(0, 1) layer (binary16, rounding negligible)
    against the quadrature limit: within 0.2 % (the sampling spread over seeds is about
    0.03 %).  One wrong level moves the limit by 23 %."""
    levels, mids = book
    e_inf = _expected_normal_block_error(levels, mids)
    assert 0.05 < e_inf < 0.2
    x = np.random.default_rng(2024).standard_normal(1 << 22).astype(np.float16)
    e = oracle.layer_error(x.view(np.uint16), oracle.F16)[2]
    assert abs(e / e_inf - 1) < 2e-3, (e, e_inf)
    # the limit is the same for every block size only if the quantizer ignores it: blocks
    # of 256 share their absmax over more elements and must give a larger error
    assert _expected_normal_block_error(levels, mids, 256) > 1.05 * e_inf


# ---------------------------------------------------------------- double quantization


def test_dq_saving_matches_page_figure():
    n = 64 * 256 * 10
    absmax = np.random.default_rng(0).uniform(0, 1, n // 64).astype(np.float32)
    codes8, scales, _ = oracle.double_quant(absmax)
    bits_dq = (codes8.nbytes + scales.nbytes) * 8 / n
    bits_plain = absmax.nbytes * 8 / n
    saving = bits_plain - bits_dq
    assert saving == 0.5 - (8 / 64 + 32 / (64 * 256)) == 0.373046875
    fact = FACTS["dq_saving_bits_per_param"]
    assert round(saving, fact["decimals"]) == fact["value"]


def test_dq_special_cases():
    s = np.float32(0.37)
    a = np.array([s] * 256 + [0.0, s / 2, s] + [0.0] * 253 + [0.0] * 10, np.float32)
    codes8, scales, nf = oracle.double_quant(a)
    assert not nf
    assert np.all(codes8[:256] == 255) and scales[0] == s
    assert list(codes8[256:259]) == [0, 128, 255]  # 127.5 rounds to the even 128
    assert scales[2] == 0.0 and np.all(codes8[512:] == 0)
    back = oracle.dequantize(np.zeros(128, np.uint8), 256, oracle.F16, codes8=codes8[:4],
                             scales=scales[:1])
    assert back.size == 256
    a2 = np.array([1.0, np.nan], np.float32)
    _, sc2, nf2 = oracle.double_quant(a2)
    assert nf2 and np.isnan(sc2[0])


def test_dq_codes_equal_bruteforce_nearest():
    rng = np.random.default_rng(4)
    a = np.abs(rng.standard_normal(256 * 37 + 5)).astype(np.float32) * 0.05
    codes8, scales, _ = oracle.double_quant(a)
    for d in range(scales.size):
        blk = a[256 * d: 256 * d + 256].astype(np.float64)
        s = float(scales[d])
        assert s == blk.max()
        grid = np.arange(256) / 255.0 * s
        brute = np.argmin(np.abs(blk[:, None] - grid[None, :]), axis=1)
        got = codes8[256 * d: 256 * d + blk.size]
        diff = got != brute
        assert diff.sum() <= 1  # only within one rounding of a half-way point
        if diff.any():
            frac = blk[diff] / s * 255
            assert np.all(np.abs(frac - np.floor(frac) - 0.5) < 1e-5)


def test_dqc_saving_matches_page_figure():
    """Mean-centred DQ stores 8-bit codes plus two binary32 numbers per 256 constants:
    8/64 + 64/(64*256) bits per weight, 0.37109375 less than binary32 constants -- the pages'
    0.37 bits as well ("QLoRA", How It Works)."""
    n = 64 * 256 * 10
    absmax = np.random.default_rng(0).uniform(0, 1, n // 64).astype(np.float32)
    codes8, scales, means, _ = oracle.double_quant_centered(absmax)
    bits = (codes8.nbytes + scales.nbytes + means.nbytes) * 8 / n
    saving = absmax.nbytes * 8 / n - bits
    assert saving == 0.5 - (8 / 64 + 64 / (64 * 256)) == 0.37109375
    fact = FACTS["dq_saving_bits_per_param"]
    assert round(saving, fact["decimals"]) == fact["value"]


def test_dqc_mean_is_the_exact_mean():
    """For 16-bit constants a few binades apart the binary64 tree sum is exact, so the mean
    is the exact rational mean rounded to binary64, then to binary32 (also for a short
    last block)."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    for nb in (256 * 3, 256 * 2 + 37):
        a = torch.from_numpy(np.abs(rng.standard_normal(nb) * 0.03).astype(np.float32)) \
            .to(torch.bfloat16).float().numpy()
        _, _, means, _ = oracle.double_quant_centered(a)
        for d in range(means.size):
            blk = a[256 * d: 256 * d + 256]
            exact = sum(Fraction(float(v)) for v in blk) / blk.size
            assert means[d] == np.float32(float(exact)), d


def test_dqc_codes_equal_bruteforce_nearest():
    """Each code is the nearest of the 255 rebuildable offsets fl(fl(q/127) h), q in
    [-127, 127], to a - mu, except within one rounding of a half-way point."""
    rng = np.random.default_rng(6)
    a = np.abs(rng.standard_normal(256 * 29 + 11)).astype(np.float32) * 0.05
    codes8, scales, means, _ = oracle.double_quant_centered(a)
    q = np.arange(-127, 128)
    for d in range(scales.size):
        blk = a[256 * d: 256 * d + 256]
        h, mu = scales[d], means[d]
        c = (blk - mu).astype(np.float32).astype(np.float64)
        assert h == np.abs(c).max()
        grid = ((q.astype(np.float32) / np.float32(127)) * h).astype(np.float64)
        brute = q[np.argmin(np.abs(c[:, None] - grid[None, :]), axis=1)]
        got = codes8[256 * d: 256 * d + blk.size].astype(np.int64) - 128
        diff = got != brute
        assert diff.sum() <= 2
        if diff.any():
            t = c[diff] / h * 127
            assert np.all(np.abs(t - np.floor(t) - 0.5) < 1e-4)


def test_dqc_special_blocks():
    """A block of one repeated value rebuilds it exactly (h = 0, codes 128); a block of two
    values symmetric about their mean codes to the ends 1 and 255 and rebuilds both
    exactly; a non-finite constant is flagged."""
    v = np.float32(0.0375)
    codes8, scales, means, nf = oracle.double_quant_centered(np.full(256, v, np.float32))
    assert not nf and scales[0] == 0 and means[0] == v and np.all(codes8 == 128)
    lo, hi = np.float32(0.25), np.float32(0.75)
    a = np.array([lo, hi] * 128, np.float32)
    codes8, scales, means, _ = oracle.double_quant_centered(a)
    assert means[0] == 0.5 and scales[0] == 0.25
    assert list(codes8[:2]) == [1, 255]
    rebuilt = (((codes8.astype(np.int32) - 128).astype(np.float32) / np.float32(127))
               * scales[0] + means[0]).astype(np.float32)
    assert np.array_equal(rebuilt, a)
    _, _, _, nf = oracle.double_quant_centered(np.array([1.0, np.inf], np.float32))
    assert nf


def test_dqc_rebuilt_constants_are_closer_for_clustered_constants(book):
    """Centring on the mean spends the 8-bit code on [mu - h, mu + h] instead of [0, s]: for
    the absmax values of normal 64-blocks (mean about 2.4 sigma, spread about as wide) the
    code's step is about 3/4 of the plain code's, so the rebuilt constants land closer on
    average, each within h/254 plus rounding."""
    rng = np.random.default_rng(7)
    w = torch.from_numpy((rng.standard_normal(64 * 256 * 8) * 0.02).astype(np.float32)) \
        .to(torch.bfloat16)
    _, absmax, _ = oracle.quantize(bits_of(w), oracle.BF16)
    c8, sc, mu, _ = oracle.double_quant_centered(absmax)
    rc = (((c8.astype(np.int32) - 128).astype(np.float32) / np.float32(127))
          * np.repeat(sc, 256) + np.repeat(mu, 256)).astype(np.float32)
    p8, ps, _ = oracle.double_quant(absmax)
    rp = ((p8.astype(np.float32) / np.float32(255)) * np.repeat(ps, 256)).astype(np.float32)
    err_c = np.abs(rc.astype(np.float64) - absmax)
    err_p = np.abs(rp.astype(np.float64) - absmax)
    assert err_c.mean() < 0.85 * err_p.mean()
    assert np.all(err_c <= np.repeat(sc, 256) / 254 * (1 + 1e-5) + 4e-7 * absmax)


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_dqc_layer_error_is_the_error_of_the_dequantized_model(book, dtype):
    """The layer error against mean-centred DQ constants equals the error of what the
    centred dequantization rebuilds, summed here in numpy (3 DQ blocks, ragged tail)."""
    rng = np.random.default_rng(23)
    n = 64 * 700 + 13
    tdt = torch.float16 if dtype == oracle.F16 else torch.bfloat16
    z = rng.standard_normal(n) * np.repeat(rng.uniform(0.005, 0.05, n // 64 + 1), 64)[:n]
    w = torch.from_numpy(z.astype(np.float32)).to(tdt)
    bits = bits_of(w)
    packed, absmax, _ = oracle.quantize(bits, dtype)
    codes8, scales, means, _ = oracle.double_quant_centered(absmax)
    deq = oracle.dequantize_centered(packed, n, dtype, codes8, scales, means)
    deq = torch.from_numpy(deq.view(np.int16)).view(tdt).double().numpy()
    x = w.double().numpy()
    se, sw, rel = oracle.layer_error_dqc(bits, dtype)
    assert se == pytest.approx(float(np.sum((x - deq) ** 2)), rel=1e-12)
    assert sw == oracle.layer_error(bits, dtype)[1]
    assert rel == pytest.approx(math.sqrt(se / sw), rel=1e-6)
    assert se != oracle.layer_error_dq(bits, dtype)[0]


def test_dequant_with_exact_dq_equals_plain_absmax(book):
    """Constants that double-quantize exactly (code 255) dequantize like the raw absmax."""
    rng = np.random.default_rng(8)
    w = torch.from_numpy((rng.standard_normal(256 * 64) * 0.02).astype(np.float32)).to(torch.bfloat16)
    bits = bits_of(w)
    packed, absmax, _ = oracle.quantize(bits, oracle.BF16)
    flat = np.full_like(absmax, absmax.max())
    codes8, scales, _ = oracle.double_quant(flat)
    assert np.all(codes8 == 255)
    d1 = oracle.dequantize(packed, bits.size, oracle.BF16, codes8=codes8, scales=scales)
    d2 = oracle.dequantize(packed, bits.size, oracle.BF16, absmax=flat)
    assert np.array_equal(d1, d2)


def test_dequant_reconstructs_layer_error(book):
    """The error the score reports is the error of the dequantized weights."""
    rng = np.random.default_rng(12)
    n = 64 * 33 + 7
    w = torch.from_numpy((rng.standard_normal(n) * 0.03).astype(np.float32)).to(torch.float16)
    bits = bits_of(w)
    packed, absmax, _ = oracle.quantize(bits, oracle.F16)
    deq = oracle.dequantize(packed, n, oracle.F16, absmax=absmax).view(np.float16).astype(np.float64)
    x = w.double().numpy()
    se, sw, _ = oracle.layer_error(bits, oracle.F16)
    assert se == pytest.approx(float(np.sum((x - deq) ** 2)), rel=1e-12)


@pytest.mark.parametrize("dtype", [oracle.F16, oracle.BF16])
def test_dq_layer_error_is_the_error_of_the_dequantized_model(book, dtype):
    """The DQ-absmax score equals the error of what aqnf4_dequantize rebuilds from
    packed codes + codes8 + scales (3 DQ blocks, ragged tail), summed here in numpy."""
    rng = np.random.default_rng(21)
    n = 64 * 700 + 13
    tdt = torch.float16 if dtype == oracle.F16 else torch.bfloat16
    z = rng.standard_normal(n) * np.repeat(rng.uniform(0.005, 0.05, n // 64 + 1), 64)[:n]
    w = torch.from_numpy(z.astype(np.float32)).to(tdt)
    bits = bits_of(w)
    packed, absmax, _ = oracle.quantize(bits, dtype)
    codes8, scales, _ = oracle.double_quant(absmax)
    deq = oracle.dequantize(packed, n, dtype, codes8=codes8, scales=scales)
    deq = torch.from_numpy(deq.view(np.int16)).view(tdt).double().numpy()
    x = w.double().numpy()
    se, sw, rel = oracle.layer_error_dq(bits, dtype)
    assert se == pytest.approx(float(np.sum((x - deq) ** 2)), rel=1e-12)
    assert sw == oracle.layer_error(bits, dtype)[1]
    assert rel == pytest.approx(math.sqrt(se / sw), rel=1e-6)
    # and it is not the plain score: the DQ constants differ from the binary32 absmax
    assert se != oracle.layer_error(bits, dtype)[0]


def test_dq_layer_error_equals_plain_when_constants_survive(book):
    """Every block holding the same maximum A: code8 = 255 and a' = A, so both scores agree."""
    rng = np.random.default_rng(22)
    z = rng.uniform(-0.9, 0.9, (600, 64)).astype(np.float32) * 0.05
    z[:, 5] = 0.05
    w = torch.from_numpy(z.reshape(-1)).to(torch.bfloat16)
    bits = bits_of(w)
    assert oracle.layer_error_dq(bits, oracle.BF16) == oracle.layer_error(bits, oracle.BF16)


def test_dq_layer_error_of_a_block_coded_to_zero(book):
    """A block whose constant is below s/510 double-quantizes to 0, so a' = 0, w_hat = 0
    and the block adds exactly its sum of squares to the error."""
    rng = np.random.default_rng(23)
    big = rng.uniform(-1.0, 1.0, 64).astype(np.float32)
    big[0] = 1.0
    small = (rng.uniform(-1.0, 1.0, 64) * 1e-3).astype(np.float32)
    wb = torch.from_numpy(big).to(torch.bfloat16)
    ws = torch.from_numpy(small).to(torch.bfloat16)
    bits = np.concatenate([bits_of(wb), bits_of(ws)])
    _, absmax, _ = oracle.quantize(bits, oracle.BF16)
    codes8, _, _ = oracle.double_quant(absmax)
    assert codes8.tolist() == [255, 0]
    se, sw, _ = oracle.layer_error_dq(bits, oracle.BF16)
    se_big = oracle.layer_error(bits_of(wb), oracle.BF16)[0]
    xs = ws.double().numpy()
    assert se == se_big + float(np.sum(xs * xs))


# ---------------------------------------------------------------- selection


def _bruteforce_select(e, cost, budget, k_cap):
    L = len(e)

    def before(j, i):
        if math.isnan(e[j]) != math.isnan(e[i]):
            return math.isnan(e[i])
        if not math.isnan(e[j]) and e[j] != e[i]:
            return e[j] > e[i]
        return j < i

    best = ()
    for r in range(L + 1):
        for S in itertools.combinations(range(L), r):
            s = set(S)
            if k_cap >= 0 and len(s) > k_cap:
                continue
            if sum(cost[i] for i in s) > budget:
                continue
            closed = all(not before(j, i) for i in s for j in range(L) if j not in s)
            if closed and len(s) > len(best):
                best = S
    return sorted(best)


@pytest.mark.parametrize("seed", range(6))
def test_select_equals_bruteforce_over_subsets(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 11))
    e = rng.choice([0.05, 0.1, 0.1, 0.2, 0.3, float("nan")], size=L).astype(np.float32)
    e = np.where(rng.uniform(size=L) < 0.5, rng.uniform(0, 1, L).astype(np.float32), e)
    cost = rng.integers(1, 100, L)
    budget = int(rng.integers(0, 300))
    k_cap = int(rng.choice([-1, 0, 1, 2, 5]))
    got = oracle.select_topk(e, cost, budget, k_cap)
    assert sorted(got) == _bruteforce_select(list(map(float, e)), list(cost), budget, k_cap)


def test_select_rules():
    e = [0.3, 0.5, 0.5, float("nan"), 0.1]
    assert oracle.select_topk(e, [1] * 5, 100) == [1, 2, 0, 4, 3]  # ties by index, NaN last
    assert oracle.select_topk(e, [1] * 5, 100, k_cap=2) == [1, 2]
    assert oracle.select_topk(e, [1] * 5, 0) == []
    # walking the ranking stops at the first layer that does not fit
    assert oracle.select_topk([0.9, 0.8, 0.7], [5, 10, -8], 8) == [0]
    with pytest.raises(ValueError):
        oracle.select_topk(e, [1] * 5, -1)


# ------------------------------------------------ linear layer on NF4 weights


def _nf4_layer(rng, N, K, sigma=0.02, tdt=torch.bfloat16):
    w = torch.from_numpy((rng.standard_normal((N, K)) * sigma).astype(np.float32)).to(tdt)
    b = bits_of(w)
    dt = oracle.BF16 if tdt == torch.bfloat16 else oracle.F16
    packed, absmax, _ = oracle.quantize(b, dt)
    codes8, scales, _ = oracle.double_quant(absmax)
    return packed, codes8, scales


@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (5, 7, 128), (33, 20, 320)])
def test_nf4_linear_equals_blas_on_dequantized_weights(M, N, K):
    """y = x w_hat^T against numpy's BLAS product of the oracle's dequantized weights."""
    rng = np.random.default_rng(M * 1000 + N)
    packed, codes8, scales = _nf4_layer(rng, N, K)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    y, yabs = oracle.nf4_linear(bits_of(x).reshape(M, K), oracle.BF16, packed, codes8, scales,
                                N, oracle.BF16)
    wq = oracle.dequantize(packed, N * K, oracle.BF16, codes8=codes8, scales=scales)
    w64 = torch.from_numpy(wq.view(np.int16)).view(torch.bfloat16).double().numpy().reshape(N, K)
    x64 = x.double().numpy()
    ref = x64 @ w64.T
    assert np.all(np.abs(y - ref) <= 1e-12 * np.maximum(yabs, 1e-300))
    assert np.allclose(yabs, np.abs(x64) @ np.abs(w64).T, rtol=1e-12, atol=0)
    assert np.all(yabs >= np.abs(y))


def test_nf4_linear_exact_on_representable_weights():
    """Weights NF4 + DQ store exactly -- bf16(level * 0.5), every block holding the maximum
    0.5 so that code8 = 255 and a' = 0.5 -- and small integer activations: w_hat = w and the
    product is exact in binary64."""
    levels, _ = oracle.codebook()
    rng = np.random.default_rng(3)
    N, K, M = 6, 128, 4
    codes = rng.integers(0, 16, (N, K))
    codes[:, 0] = 15                                   # every block's maximum is 0.5
    wb = torch.from_numpy((levels[codes] * np.float32(0.5)).astype(np.float32)).to(torch.bfloat16)
    w = wb.float().numpy()
    packed, absmax, _ = oracle.quantize(bits_of(wb), oracle.BF16)
    codes8, scales, _ = oracle.double_quant(absmax)
    assert np.all(codes8 == 255)
    x = rng.integers(-3, 4, (M, K)).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    y, _ = oracle.nf4_linear(bits_of(xb).reshape(M, K), oracle.BF16, packed, codes8, scales, N,
                             oracle.BF16)
    assert np.array_equal(y, x.astype(np.float64) @ w.astype(np.float64).T)


# ------------------------------------------------------ block-level selection


@pytest.mark.parametrize("seed", range(4))
def test_blocks_of_one_layer_select_like_layers(seed):
    """With one layer per block, ranking blocks by error is the layer selection itself."""
    rng = np.random.default_rng(seed)
    L = 12
    sw = rng.uniform(0.5, 50.0, L)
    rel = rng.uniform(0.05, 0.2, L).astype(np.float32)
    rel[3] = rel[7]                                   # a tie: lower index first
    se = (rel.astype(np.float64) ** 2) * sw
    # the block score rounds sqrt(se/sw) to binary32: use exactly what the layers report
    rel = np.sqrt(se / sw).astype(np.float32)
    cost = rng.integers(1, 100, L)
    for budget in (0, 50, 200, 400, 10 ** 6):
        rank, err, k = oracle.select_blocks(se, sw, np.arange(L), cost, L, budget,
                                            oracle.BLOCKS_BY_ERROR)
        assert np.array_equal(err.view(np.uint32), rel.view(np.uint32))
        assert rank[:k] == oracle.select_topk(rel, cost, budget)


def test_block_score_closed_forms():
    """A block whose layers share one relative error e scores e; in general the block score
    lies between its layers' smallest and largest relative errors."""
    rng = np.random.default_rng(5)
    block_of = np.repeat(np.arange(4), 7)
    sw = rng.uniform(1.0, 30.0, block_of.size)
    rel = rng.uniform(0.05, 0.2, block_of.size)
    rel[block_of == 2] = 0.125                        # exact in binary and in its square
    se = rel ** 2 * sw
    _, err, _ = oracle.select_blocks(se, sw, block_of, np.ones(block_of.size), 4, 0,
                                     oracle.BLOCKS_BY_ERROR)
    assert err[2] == np.float32(0.125)
    for b in range(4):
        r = rel[block_of == b]
        assert r.min() * (1 - 1e-6) <= err[b] <= r.max() * (1 + 1e-6)


def test_blocks_by_depth_keep_the_top_that_fits():
    """By depth, the kept blocks are the last k blocks for the largest k whose summed cost
    fits (brute force over k); a block with no layers costs nothing."""
    rng = np.random.default_rng(6)
    B = 9
    block_of = np.sort(rng.integers(0, B, 40))
    block_of[block_of == 4] = 5                       # block 4 has no layers
    cost = rng.integers(1, 50, block_of.size)
    se = rng.uniform(0, 1, block_of.size)
    sw = rng.uniform(1, 2, block_of.size)
    bcost = np.array([cost[block_of == b].sum() for b in range(B)])
    for budget in range(0, int(bcost.sum()) + 5, 7):
        rank, _, k = oracle.select_blocks(se, sw, block_of, cost, B, budget,
                                          oracle.BLOCKS_BY_DEPTH)
        assert rank == list(range(B - 1, -1, -1))
        best = 0
        for kk in range(B + 1):
            if bcost[B - kk:].sum() <= budget:
                best = kk
            else:
                break
        assert k == best


def test_block_selection_nan_last_and_argument_checks():
    se = np.array([0.1, np.nan, 0.4, 0.2])
    sw = np.ones(4)
    rank, err, k = oracle.select_blocks(se, sw, [0, 1, 2, 3], [1, 1, 1, 1], 4, 10,
                                        oracle.BLOCKS_BY_ERROR)
    assert rank == [2, 3, 0, 1] and k == 4 and np.isnan(err[1])
    with pytest.raises(ValueError):
        oracle.select_blocks(se, sw, [0, 1, 2, 4], [1, 1, 1, 1], 4, 10, oracle.BLOCKS_BY_ERROR)
    with pytest.raises(ValueError):
        oracle.select_blocks(se, sw, [0, 1, 2, 3], [1, 1, 1, 1], 4, -1, oracle.BLOCKS_BY_DEPTH)


def test_cost_bytes_closed_form():
    for n in (1, 7, 64, 65, 4096 * 4096, 11008 * 4096, 16385):
        nb = -(-n // 64)
        assert oracle.cost_bytes(n) == 2 * n - (-(-n // 2) + nb + 4 * -(-nb // 256))
    # the 0.2 GiB quality-setting budget keeps a few 4096x4096 layers
    per = oracle.cost_bytes(4096 * 4096)
    assert int(FACTS["quality_setting_extra_memory_gib"]["value"] * 2 ** 30) // per == 8


# ---------------------------------------------------------------- planted mistakes


def test_pins_catch_a_reversed_codebook(book):
    levels, mids = book
    wrong = (-levels[::-1].copy(), -mids[::-1].copy())  # a plausible sign slip
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, size=(8, 64))
    codes[:, 0] = 15
    a = np.float32(0.25)
    w = torch.from_numpy((levels[codes] * a).astype(np.float32).reshape(-1)).to(torch.float16)
    se, _, _ = oracle.layer_error(bits_of(w), oracle.F16, book=wrong)
    assert se > 0  # the round-trip pin would fail


def test_pins_catch_thresholds_off_by_one_index(book):
    levels, mids = book
    wrong = (levels, levels[1:].copy())  # thresholds at q[j+1] instead of the midpoints
    rng = np.random.default_rng(7)
    w = torch.from_numpy((rng.standard_normal(64 * 50) * 0.02).astype(np.float32)).to(torch.float16)
    bits = bits_of(w)
    p_ok, a_ok, _ = oracle.quantize(bits, oracle.F16)
    p_bad, _, _ = oracle.quantize(bits, oracle.F16, book=wrong)
    x = w.float().numpy()
    v = np.concatenate([_normalized(xb, a) for xb, a in zip(x.reshape(-1, 64), a_ok)])
    brute = _nearest_level_bruteforce(v.astype(np.float64), levels)
    assert np.array_equal(codes_of(p_ok, bits.size), brute)
    assert not np.array_equal(codes_of(p_bad, bits.size), brute)
