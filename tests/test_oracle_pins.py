"""Pins for the CPU oracle: values and properties fixed by the pages and by arithmetic,
independent of the oracle's own code.

  * golden fixtures derived by hand (tests/golden/*.txt) for the packing order and for one
    hand-quantized group at every width (Per-group(128) article, sec. 3.1, 3.3, 3.4);
  * exact rational evaluation of the IEEE fp32 quantizer (correct rounding of every
    operation, ties to even), including constructed exact ties;
  * invariants: pack/unpack round trip, |w - deq| <= step/2 (+ rounding), codes in
    [1, 2^b - 1] (the clamp never binds), the all-zero group;
  * the uniform-noise model step^2/12 and SNR rising with bits, per-group beating
    per-channel on outlier-laden weights (sec. 3.1 comparison table, sec. 4.2);
  * the fp64 linear layer against numpy's dgemm and against exact rational sums.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import twin
from bit_weight_quantization_wq_b200 import synth

from conftest import GOLDEN

BITS = (3, 4, 5, 6, 7)


# ----------------------------------------------------------------------- exact helpers

def _round_int_half_even(m: Fraction) -> int:
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 != 0):
        fl += 1
    return fl


def f32_round(x: Fraction) -> Fraction:
    """Correctly rounded (nearest, ties to even) binary32 value of an exact rational."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                    # subnormal range shares the smallest exponent
    ulp = Fraction(2) ** (e - 23)
    return sign * _round_int_half_even(a / ulp) * ulp


F101 = f32_round(Fraction(101, 100))    # 1.01 as an fp32 constant


def exact_quantize_group(w_vals, bits):
    """Step and codes of one group from the sec. 3.1 formulas, every fp32 operation
    evaluated exactly and then correctly rounded."""
    amax = max(abs(Fraction(float(v))) for v in w_vals)
    s = f32_round(amax * F101)
    step = f32_round(2 * s / ((1 << bits) - 1))
    q_max = ((1 << bits) - 1) // 2
    codes = []
    for v in w_vals:
        if step == 0:
            q = 0
        else:
            q = _round_int_half_even(f32_round(Fraction(float(v)) / step))
            q = max(-q_max, min(q_max, q))
        codes.append(q + (1 << (bits - 1)))
    return step, codes


def bf16(values):
    return synth.f32_to_bf16_bits(np.asarray(values, np.float32))


def _parse(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([p.strip() for p in line.split("|")])
    return rows


# ----------------------------------------------------------------------- golden pins

def test_bit_order_golden():
    rows = _parse(os.path.join(GOLDEN, "bit_order.txt"))
    assert len(rows) == 10
    for bits_s, codes_s, bytes_s in rows:
        bits = int(bits_s)
        codes = np.array([[int(c) for c in codes_s.split()]], np.uint8)
        expect = np.array([[int(b, 16) for b in bytes_s.split()]], np.uint8)
        got = oracle.pack(codes, bits)
        assert got.tolist() == expect.tolist(), (bits, codes_s)
        assert oracle.unpack(expect, codes.shape[1], bits).tolist() == codes.tolist()
        assert twin.pack(codes, bits).tolist() == expect.tolist()


def test_hand_group_golden():
    rows = _parse(os.path.join(GOLDEN, "hand_group.txt"))
    weights = [float(v) for v in rows[0][1].split()]
    assert rows[0][0] == "weights"
    group = np.zeros((1, 128), np.uint16)
    group[0, :8] = bf16(weights)
    # every listed weight is exactly representable in bf16
    assert synth.bf16_bits_to_f32(group[0, :8]).tolist() == weights
    for bits_s, codes_s, head_s, zeros_s in rows[1:]:
        bits = int(bits_s)
        codes, scales = oracle.quantize(group, bits)
        assert codes[0, :8].tolist() == [int(c) for c in codes_s.split()]
        assert (codes[0, 8:] == (1 << (bits - 1))).all()
        assert scales[0, 0] == pytest.approx(1.01 / ((1 << bits) - 1), rel=1e-6)
        packed = oracle.pack(codes, bits)[0]
        assert packed.size == 16 * bits                       # 128 codes -> 16*b bytes
        head = [int(b, 16) for b in head_s.split()]
        zeros = [int(b, 16) for b in zeros_s.split()]
        assert packed[:bits].tolist() == head
        assert packed[bits:].tolist() == zeros * 15


def test_packed_sizes_match_table():
    # 3 bit: 8 -> 3 bytes, 4: 2 -> 1, 5: 8 -> 5, 6: 4 -> 3, 7: 8 -> 7
    table = {3: (8, 3), 4: (2, 1), 5: (8, 5), 6: (4, 3), 7: (8, 7)}
    for bits, (n_w, n_b) in table.items():
        codes = np.zeros((3, 128), np.uint8)
        assert oracle.pack(codes, bits).shape == (3, 128 * n_b // n_w)


# ----------------------------------------------------------------------- exact IEEE pins

def _random_groups(rng, n_groups):
    out = []
    for i in range(n_groups):
        kind = i % 4
        if kind == 0:
            w = rng.standard_normal(128) * 0.02
        elif kind == 1:
            w = rng.standard_normal(128) * 0.015
            w[rng.integers(128)] = rng.choice([-1, 1]) * rng.uniform(0.2, 0.5)
        elif kind == 2:
            w = rng.uniform(-1, 1, 128) * 10.0 ** rng.uniform(-6, 3)
        else:
            w = rng.standard_normal(128) * 1e-3
            w[:64] = 0
        out.append(bf16(w))
    return np.stack(out)


@pytest.mark.parametrize("bits", BITS)
def test_exact_ieee_quantizer(bits):
    rng = np.random.default_rng(7 + bits)
    W = _random_groups(rng, 24)                     # 24 rows, one group each
    codes, scales = oracle.quantize(W, bits)
    for n in range(W.shape[0]):
        vals = synth.bf16_bits_to_f32(W[n])
        step, expect = exact_quantize_group(vals, bits)
        assert Fraction(float(scales[n, 0])) == step
        assert codes[n].tolist() == expect


@pytest.mark.parametrize("bits", BITS)
def test_round_half_even_on_exact_ties(bits):
    """Find groups [abs_max, w, 0, ...] whose fp32 quotient w/step is exactly k + 1/2, confirm
    each tie with exact rationals, and check that the oracle rounds it to the even neighbour.

    The search itself uses numpy fp32 only to propose candidates; every candidate is then
    decided by the exact evaluation."""
    exps = np.arange(-20, 8)
    mant = np.arange(128, 256)
    amax = (mant[None, :] / 128.0 * 2.0 ** exps[:, None]).astype(np.float32).ravel()
    levels = np.float32((1 << bits) - 1)
    step = (np.float32(2.0) * (amax * np.float32(1.01))) / levels
    q_max = ((1 << bits) - 1) // 2
    cases = []
    for t in np.arange(q_max) + 0.5:
        v = synth.bf16_bits_to_f32(bf16(np.float32(t) * step))
        hit = ((v / step) == np.float32(t)) & (v < amax) & (v > 0)
        cases += [(float(a), float(w)) for a, w in zip(amax[hit], v[hit])]
        if len(cases) >= 48:
            break
    assert len(cases) >= 4, "too few exact ties found; widen the search"
    W = np.zeros((len(cases), 128), np.uint16)
    for i, (a, w) in enumerate(cases):
        W[i, 0], W[i, 1] = bf16([a])[0], bf16([w])[0]
    codes, _ = oracle.quantize(W, bits)
    n_ties = 0
    for i, (a, w) in enumerate(cases):
        step_x, expect = exact_quantize_group([a, w], bits)
        r = f32_round(Fraction(w) / step_x)
        if (r - Fraction(1, 2)).denominator != 1:
            continue                                   # not an exact tie after all
        n_ties += 1
        lo = int(r - Fraction(1, 2))
        even = lo if lo % 2 == 0 else lo + 1
        assert expect[1] == even + (1 << (bits - 1))
        assert codes[i, 1] == expect[1], (a, w, r)
    assert n_ties >= 4


# ----------------------------------------------------------------------- invariants

@pytest.mark.parametrize("bits", BITS)
def test_pack_unpack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(9, 384)).astype(np.uint8)
    packed = oracle.pack(codes, bits)
    assert packed.shape == (9, 384 * bits // 8)
    assert (oracle.unpack(packed, 384, bits) == codes).all()
    assert (twin.unpack(packed, 384, bits) == codes).all()


@pytest.mark.parametrize("bits", BITS)
def test_error_bound_and_code_range(bits):
    rng = np.random.default_rng(100 + bits)
    W = np.concatenate([_random_groups(rng, 32).reshape(8, 512),
                        synth.weight(rng, 8, 512, 0.02)], axis=0)
    codes, scales = oracle.quantize(W, bits)
    deq = oracle.dequant(codes, scales, bits)
    w = synth.bf16_bits_to_f32(W).astype(np.float64)
    step = np.repeat(scales.astype(np.float64), 128, axis=1)
    err = np.abs(w - deq)
    bound = step / 2 + (np.abs(w) + np.abs(deq)) * 2.0 ** -24
    assert (err <= bound).all()
    # the clamp never binds: |w|/step < 2^(b-1) - 1 + 1/2, so codes stay in [1, 2^b - 1]
    nz = step > 0
    assert (np.abs(w[nz]) / step[nz]).max() < (1 << (bits - 1)) - 0.5
    assert codes.min() >= 1 and codes.max() <= (1 << bits) - 1


@pytest.mark.parametrize("bits", BITS)
def test_clamp_never_binds_for_any_bf16_abs_max(bits):
    """Sec. 3.1 clamps q to +-(2^(b-1) - 1). For every finite bf16 abs_max, the largest
    quotient of the group, RN(abs_max / step) with the page's fp32 step, stays below
    2^(b-1) - 1/2, so round() never reaches the clamp (|w| <= abs_max and RN is monotone).
    numpy's float32 multiply and divide are IEEE correctly rounded."""
    a = synth.bf16_bits_to_f32(np.arange(1, 0x7F80, dtype=np.uint16))
    with np.errstate(over="ignore"):
        s = a * np.float32(1.01)
        step = (np.float32(2.0) * s) / np.float32((1 << bits) - 1)
        r = a / step
    assert np.isfinite(a).all() and r.dtype == np.float32
    assert np.nanmax(r) < (1 << (bits - 1)) - 0.5
    # and the oracle agrees: groups whose abs_max is each of these values keep codes in range
    W = np.zeros((len(a) // 8, 128), np.uint16)
    W[:, 0] = np.arange(1, 0x7F80, dtype=np.uint16)[: len(W) * 8 : 8]
    W[:, 1] = W[:, 0] | 0x8000
    codes, _ = oracle.quantize(W, bits)
    assert codes.min() >= 1 and codes.max() <= (1 << bits) - 1


@pytest.mark.parametrize("bits", BITS)
def test_all_zero_group(bits):
    W = np.zeros((2, 256), np.uint16)
    W[1, 128:] = bf16(np.linspace(-1, 1, 128))
    codes, scales = oracle.quantize(W, bits)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
    assert (codes[0] == 1 << (bits - 1)).all() and (codes[1, :128] == 1 << (bits - 1)).all()
    deq = oracle.dequant(codes, scales, bits)
    assert (deq[0] == 0).all()


def test_uniform_noise_model_and_snr_rise():
    """For Gaussian weights the rounding error is ~U(-step/2, step/2): MSE ~ mean(step^2)/12.
    SNR must rise with bits, by ~6 dB per bit once the noise is uniform."""
    rng = np.random.default_rng(5)
    W = synth.f32_to_bf16_bits(rng.standard_normal((256, 2048)).astype(np.float32) * 0.02)
    w = synth.bf16_bits_to_f32(W).astype(np.float64)
    snr = {}
    for bits in BITS:
        codes, scales = oracle.quantize(W, bits)
        deq = oracle.dequant(codes, scales, bits)
        mse = np.mean((w - deq) ** 2)
        model = np.mean(scales.astype(np.float64) ** 2) / 12
        if bits >= 4:
            assert 0.9 < mse / model < 1.1, (bits, mse / model)
        snr[bits] = oracle.snr_db(w, deq)
    for b in BITS[:-1]:
        assert snr[b + 1] > snr[b]
        if b >= 4:
            assert 5.5 < snr[b + 1] - snr[b] < 6.5
    # closed form with E[abs_max] of 128 Gaussians ~ 2.9 sigma gives ~19 dB at 4 bits
    assert 17.5 < snr[4] < 20.5


def test_per_group_beats_per_channel_on_outliers():
    """Sec. 3.1 / sec. 4.2: per-group(128) scales beat one scale per output channel."""
    rng = np.random.default_rng(11)
    W = synth.weight(rng, 512, 2048, 0.02)
    w = synth.bf16_bits_to_f32(W)
    c_g, s_g = oracle.quantize(W, 4, 128)
    c_c, s_c = oracle.quantize(W, 4, 2048)
    snr_g = oracle.snr_db(w, oracle.dequant(c_g, s_g, 4, 128))
    snr_c = oracle.snr_db(w, oracle.dequant(c_c, s_c, 4, 2048))
    assert snr_g > snr_c + 3.0, (snr_g, snr_c)


@pytest.mark.parametrize("bits", BITS)
def test_twin_matches_c_oracle(bits):
    rng = np.random.default_rng(200 + bits)
    W = np.concatenate([synth.weight(rng, 24, 1024, 0.015),
                        _random_groups(rng, 64).reshape(8, 1024)], axis=0)
    W[3, 256:384] = 0
    c1, s1 = oracle.quantize(W, bits)
    c2, s2 = twin.quantize(W, bits)
    assert (c1 == c2).all()
    assert (s1.view(np.uint32) == s2.view(np.uint32)).all()
    p1 = oracle.pack(c1, bits)
    assert (p1 == twin.pack(c2, bits)).all()
    assert (oracle.dequant(c1, s1, bits) == twin.dequant(c2, s2, bits)).all()


# ----------------------------------------------------------------------- linear layer

def _linear_inputs(rng, M, N, K, r):
    W = synth.weight(rng, N, K, 0.02)
    codes, scales = oracle.quantize(W, 4)
    deq = oracle.dequant(codes, scales, 4)
    x = synth.activations(rng, M, K)
    L1 = synth.f32_to_bf16_bits(rng.standard_normal((K, r)).astype(np.float32) * 0.1) if r else None
    L2 = synth.f32_to_bf16_bits(rng.standard_normal((r, N)).astype(np.float32) * 0.1) if r else None
    b = synth.bias(rng, N)
    return x, deq, L1, L2, b


def test_linear_reduces_to_dgemm():
    rng = np.random.default_rng(3)
    x, deq, _, _, _ = _linear_inputs(rng, 16, 96, 256, 0)
    y = oracle.linear_rows(x, deq)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ deq.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_linear_lowrank_and_bias_match_dgemm():
    rng = np.random.default_rng(4)
    x, deq, L1, L2, b = _linear_inputs(rng, 8, 64, 384, 32)
    y = oracle.linear_rows(x, deq, L1, L2, b)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = (xf @ deq.astype(np.float64).T
           + (xf @ synth.bf16_bits_to_f32(L1).astype(np.float64)) @ synth.bf16_bits_to_f32(L2).astype(np.float64)
           + synth.bf16_bits_to_f32(b).astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-11)
    # a row subset gives the same rows
    rows = np.array([7, 0, 3])
    np.testing.assert_array_equal(oracle.linear_rows(x, deq, L1, L2, b, rows), y[rows])


def test_linear_exact_tiny():
    """Exact rational sums on a tiny case: the fp64 oracle is within fp64 rounding."""
    rng = np.random.default_rng(8)
    M, N, K, r = 2, 3, 128, 2
    x, deq, L1, L2, b = _linear_inputs(rng, M, N, K, r)
    y = oracle.linear_rows(x, deq, L1, L2, b)
    F = lambda v: Fraction(float(v))
    xf, l1f, l2f, bf = (synth.bf16_bits_to_f32(a) for a in (x, L1, L2, b))
    for m in range(M):
        t = [sum(F(xf[m, k]) * F(l1f[k, j]) for k in range(K)) for j in range(r)]
        for n in range(N):
            terms = [F(xf[m, k]) * F(deq[n, k]) for k in range(K)]
            terms += [t[j] * F(l2f[j, n]) for j in range(r)] + [F(bf[n])]
            exact = sum(terms)
            mag = sum(abs(v) for v in terms)
            assert abs(Fraction(y[m, n]) - exact) <= mag * Fraction(K + 8, 2 ** 52)


def test_linear_error_excludes_only_the_output_rounding():
    """The max-error bar of the linear-layer tolerance counts error beyond the bf16 output's
    correct rounding: the correctly rounded fp64 result passes with zero excess even where
    an element is 12x the rms, and a one-ulp mistake on that element does not."""
    from bit_weight_quantization_wq_b200 import synth
    from helpers import linear_error
    rng = np.random.default_rng(3)
    y_ref = rng.standard_normal(4096)
    y_ref[17] = 12.0 * np.sqrt(np.mean(y_ref ** 2)) + 0.013
    y_bits = synth.f32_to_bf16_bits(y_ref.astype(np.float32))
    rel, mx = linear_error(y_bits, y_ref)
    assert mx == 0.0 and rel < 3e-3
    bumped = y_bits.copy()
    bumped[17] += 1                                    # one bf16 ulp off at the largest element
    assert linear_error(bumped, y_ref)[1] > 0.0
