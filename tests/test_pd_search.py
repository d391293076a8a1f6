"""Per-tensor bit-width search (Per-group(128) article, sec. 3.2): the library's host routine
against the numpy oracle (same random starts, so the same widths), the oracle pinned against
brute force on small tables, and the error table's oracle pinned against exact arithmetic.
No GPU."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import pd
from bit_weight_quantization_wq_b200 import _binding as B
from bit_weight_quantization_wq_b200 import synth
from conftest import GOLDEN

BITS = [3, 4, 5, 6, 7]


@pytest.fixture(scope="module")
def L():
    from bit_weight_quantization_wq_b200 import build
    build.build()
    return B.lib()


def _table(rng, T, spread=1.0):
    """Log-linear error model: MSE_i(b) = s_i 4^-b (1 + noise), s_i log-normal."""
    s = np.exp(rng.normal(0.0, spread, T))
    n = rng.choice([5120 * 5120, 13824 * 5120], T, p=[0.8, 0.2]).astype(np.int64)
    mse = s[:, None] * 4.0 ** (-np.array(BITS, float)[None, :]) * np.exp(rng.normal(0.0, 0.1, (T, len(BITS))))
    return mse, n


@pytest.mark.parametrize("seed,T,target", [(0, 40, 5.0), (1, 120, 4.0), (2, 525, 5.0), (3, 60, 3.5)])
def test_library_matches_oracle(L, seed, T, target):
    rng = np.random.default_rng(seed)
    mse, n = _table(rng, T)
    t0 = rng.standard_normal((4, T)) * 0.5
    b_o, tot_o, bpw_o, r_o = pd.pd_search(mse, n, BITS, target, 500, 4, t0)
    b_l, tot_l, bpw_l, r_l = B.wq_pd_search(mse, n, BITS, target, t0)
    assert np.array_equal(b_o, b_l) and r_o == r_l
    assert tot_l == pytest.approx(tot_o, rel=1e-12) and bpw_l == pytest.approx(bpw_o, rel=1e-12)


def _brute_force(mse, n, target):
    best = None
    for combo in itertools.product(range(len(BITS)), repeat=len(n)):
        idx = np.array(combo)
        bpw = np.sum(n * np.array(BITS)[idx]) / n.sum()
        if bpw > target + 1e-12:
            continue
        tot = np.sum(n * mse[np.arange(len(n)), idx]) / n.sum()
        if best is None or tot < best[0]:
            best = (tot, idx)
    return best


def test_oracle_on_a_hand_table():
    """Four equal-size tensors, errors falling 4x per bit, sensitivities 100 : 1 : 1 : 0.01
    at a 5.0 budget. By enumeration of all 625 allocations the optimum is 7, 5, 5, 3 bits,
    12x less error than uniform 5 bits. The relaxation does not promise the optimum (the
    page notes that its restarts do not guarantee it); it meets the budget, gives the most
    sensitive tensor the most bits, and lands within 4x of the optimum and more than 3x below
    uniform."""
    s = np.array([100.0, 1.0, 1.0, 0.01])
    mse = s[:, None] * 4.0 ** (-np.array(BITS, float)[None, :])
    n = np.full(4, 1 << 20, np.int64)
    opt_tot, opt_idx = _brute_force(mse, n, 5.0)
    assert list(np.array(BITS)[opt_idx]) == [7, 5, 5, 3]
    uniform = float(np.mean(mse[:, 2]))
    assert uniform / opt_tot > 12
    rng = np.random.default_rng(7)
    widths, tot, bpw, _ = pd.pd_search(mse, n, BITS, 5.0, 500, 15, rng.standard_normal((15, 4)) * 0.5)
    assert bpw <= 5.0 + 1e-12
    assert widths[0] == widths.max() and widths[0] > 5
    assert tot <= 4.0 * opt_tot and tot < uniform / 3.0


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_oracle_near_brute_force_on_small_random_tables(seed):
    """Six tensors of random sizes and sensitivities: the search meets the budget (within the
    0.05 BPW slack) and its error is within 2x of the enumerated optimum."""
    rng = np.random.default_rng(seed)
    mse, _ = _table(rng, 6, spread=1.5)
    n = rng.integers(1 << 18, 1 << 22, 6)
    opt_tot, _ = _brute_force(mse, n, 5.0)
    widths, tot, bpw, _ = pd.pd_search(mse, n, BITS, 5.0, 500, 15, rng.standard_normal((15, 6)) * 0.5)
    assert bpw <= 5.05 and tot <= 2.0 * opt_tot


def test_search_beats_uniform_on_diverse_weights():
    """An error table measured by the oracle on 24 synthetic weights whose scales and outlier
    rates differ tensor to tensor: at a 5.0 budget the search's allocation meets the budget and
    has less total error than giving every tensor 5 bits."""
    rng = np.random.default_rng(21)
    rows, n = [], []
    for i in range(24):
        sigma = float(np.exp(rng.uniform(np.log(0.003), np.log(0.08))))
        W = synth.weight(rng, 64, 512, sigma, outlier_frac=float(rng.choice([0.0, 1e-3, 1e-2])))
        e = pd.quant_error(W)
        rows.append(e[:5] / W.size)
        n.append(W.size)
    mse, n = np.array(rows), np.array(n, np.int64)
    uniform = float(np.sum(n * mse[:, 2]) / n.sum())
    widths, tot, bpw, _ = pd.pd_search(mse, n, BITS, 5.0, 500, 15, rng.standard_normal((15, 24)) * 0.5)
    assert bpw <= 5.05 and tot < uniform


def test_error_table_oracle_against_exact_arithmetic():
    """The hand-worked group of the golden fixture (8 weights, then zeros): each width's sum of
    squared errors equals the exact rational sum of (w - fl32(q * step))^2 over the hand codes,
    with the step as the oracle stores it (pinned elsewhere against exact evaluation)."""
    lines = [l for l in open(f"{GOLDEN}/hand_group.txt") if l.strip() and not l.startswith("#")]
    weights = [float(v) for v in lines[0].split("|")[1].split()]
    W = np.zeros((1, 128), np.uint16)
    W[0, :8] = synth.f32_to_bf16_bits(np.array(weights, np.float32))
    err = pd.quant_error(W)
    for line in lines[1:]:
        b_str, codes_str = line.split("|")[:2]
        b = int(b_str)
        codes = [int(v) for v in codes_str.split()]
        _, scales = oracle.quantize(W, b)
        step = np.float32(scales[0, 0])
        exact = Fraction(0)
        for wv, c in zip(weights, codes):
            deq = np.float32(np.float32(c - (1 << (b - 1))) * step)      # one fp32 rounding
            exact += (Fraction(wv) - Fraction(float(deq))) ** 2
        exact += Fraction(0)   # the 120 zero weights dequantize to q = 0: no error
        assert err[b - 3] == pytest.approx(float(exact), rel=1e-15, abs=0.0), b
    assert err[5] == pytest.approx(sum(w * w for w in weights), rel=1e-15)


def test_pd_search_argument_checks(L):
    import ctypes
    ok = np.zeros((2, 5)) + 1e-6
    n = np.array([10, 10], np.int64)
    t0 = np.zeros((1, 2))
    with pytest.raises(B.WQError):
        B.wq_pd_search(ok, n, [3, 4, 4, 6, 7], 5.0, t0)             # widths not increasing
    with pytest.raises(B.WQError):
        B.wq_pd_search(ok, n, BITS, 8.0, t0)                       # target outside the widths
    with pytest.raises(B.WQError):
        B.wq_pd_search(ok * np.nan, n, BITS, 5.0, t0)              # not a finite table
    with pytest.raises(B.WQError):
        B.wq_pd_search(ok, np.array([10, 0], np.int64), BITS, 5.0, t0)
    assert L.wq_pd_search(None, None, 2, None, 5, 5.0, 10, 1, None, None, None) == B.WQ_ERR_INVALID_ARG
