"""Oracle of the per-tensor bit-width search and of its error table (test infrastructure only).

Per-group(128) mixed-precision article, sec. 3.2 ("PD-Guided Mixed Precision Bit
Allocation"): choose one width b_i per tensor to minimize sum_i ||W_i - Q_{b_i}(W_i)||_F^2
subject to sum_i n_i b_i / sum_i n_i = target BPW, by a primal-dual relaxation: one
continuous parameter per tensor mapped to a continuous width through a sigmoid, a soft
assignment of that width to the candidate widths with a softmax at an annealed temperature,
the table's errors averaged under that assignment, the budget enforced by a Lagrange term plus
a quadratic penalty, iterated from several random starts; the result is rounded and the best
start kept.

The page leaves these steps open; the readings taken here (and by the library) are:
  * dist(b, c) = |b - c|;
  * the table entries are per-weight MSEs, divided by one reference value (the weight-averaged
    MSE of the uniform allocation at the candidate nearest the target) so that the data term is
    O(1) next to the page's Lagrange start 0.5 and penalty weight 1e4 -- a constant factor, so
    the minimizer of the constrained problem is unchanged;
  * "gradient descent" on the parameters is Adam (lr 0.05, betas 0.9 / 0.999, eps 1e-8); the
    multiplier takes plain gradient ascent steps of 0.05 (primal descent, dual ascent);
  * rounding takes the nearest candidate (the lower one on a tie); "pick best" keeps the start
    with the smallest total error among those whose rounded BPW is at most target + 0.05 (the
    page's own run lands at 5.05 for a 5.0 target), else the one with the smallest BPW; ties
    go to the earlier start.
The random starts (randn * 0.5 per tensor and start) are inputs, so the library and this
oracle run from the same numbers.
"""
import numpy as np

from . import dequant, quantize

ADAM_LR, ADAM_B1, ADAM_B2, ADAM_EPS = 0.05, 0.9, 0.999, 1e-8
DUAL_LR = 0.05
LAGRANGE0 = 0.5
PENALTY = 1e4
BPW_SLACK = 0.05


def quant_error(W_bits, widths=(3, 4, 5, 6, 7), group=128):
    """Error table row of one weight: [sum (w - deq_b)^2 for each width b] + [sum w^2], fp64,
    with deq_b = dequant(quantize(W, b)) of the oracle (sec. 3.1 and 3.4)."""
    w = (np.asarray(W_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    out = []
    for b in widths:
        codes, scales = quantize(W_bits, b, group)
        e = w - dequant(codes, scales, b, group).astype(np.float64)
        out.append(float(np.sum(e * e)))
    out.append(float(np.sum(w * w)))
    return np.array(out)


def nearest_candidate(b_cont, bits):
    """Index of the candidate width nearest each continuous width (lower one on a tie)."""
    d = np.abs(np.asarray(b_cont, np.float64)[:, None] - np.asarray(bits, np.float64)[None, :])
    return np.argmin(d, axis=1)


def pd_search(mse_table, n_params, bits, target_bpw, n_iters, n_restarts, t_init):
    """The search of sec. 3.2. mse_table (T, B) per-weight MSE of tensor i at width bits[j];
    n_params (T,); bits (B,) increasing; t_init (n_restarts, T) the random starts.
    Returns (chosen widths (T,), total MSE of the choice, its BPW, index of the kept start)."""
    mse = np.asarray(mse_table, np.float64)
    n = np.asarray(n_params, np.float64)
    c = np.asarray(bits, np.float64)
    T = mse.shape[0]
    total = n.sum()
    b_min, b_max = c[0], c[-1]
    ref_col = int(nearest_candidate([target_bpw], c)[0])
    ref = float(np.sum(n * mse[:, ref_col]) / total)
    m = mse / ref
    best = None
    for r in range(n_restarts):
        t = np.array(t_init[r], np.float64)
        lagrange = LAGRANGE0
        m1 = np.zeros(T)
        m2 = np.zeros(T)
        for it in range(n_iters):
            sig = 1.0 / (1.0 + np.exp(-t))
            bit_cont = sig * (b_max - b_min) + b_min
            temp = max(2.0 * (1.0 - it / n_iters), 0.05)
            # soft assignment of each continuous width to the candidate widths
            dist = np.abs(bit_cont[:, None] - c[None, :])
            z = -dist / temp
            z = z - z.max(axis=1, keepdims=True)
            wts = np.exp(z)
            wts = wts / wts.sum(axis=1, keepdims=True)
            smooth = (wts * m).sum(axis=1)
            bpw = float(np.sum(bit_cont * n) / total)
            gap = bpw - target_bpw
            # d loss / d bit_cont: the smoothed error, the Lagrange term and the penalty
            dz = -np.sign(bit_cont[:, None] - c[None, :]) / temp
            d_smooth = (m * wts * (dz - (wts * dz).sum(axis=1, keepdims=True))).sum(axis=1)
            g_b = n / total * (d_smooth + lagrange + 2.0 * PENALTY * gap)
            g_t = g_b * sig * (1.0 - sig) * (b_max - b_min)
            # primal: Adam step on t; dual: ascent on the multiplier
            k = it + 1
            m1 = ADAM_B1 * m1 + (1.0 - ADAM_B1) * g_t
            m2 = ADAM_B2 * m2 + (1.0 - ADAM_B2) * g_t * g_t
            t = t - ADAM_LR * (m1 / (1.0 - ADAM_B1 ** k)) / (np.sqrt(m2 / (1.0 - ADAM_B2 ** k)) + ADAM_EPS)
            lagrange = lagrange + DUAL_LR * gap
        sig = 1.0 / (1.0 + np.exp(-t))
        idx = nearest_candidate(sig * (b_max - b_min) + b_min, c)
        tot = float(np.sum(n * mse[np.arange(T), idx]) / total)
        bp = float(np.sum(n * c[idx]) / total)
        feasible = bp <= target_bpw + BPW_SLACK
        if best is None:
            best = (idx, tot, bp, r, feasible)
        else:
            _, btot, bbp, _, bfeas = best
            if (feasible and (not bfeas or tot < btot)) or (not feasible and not bfeas and bp < bbp):
                best = (idx, tot, bp, r, feasible)
    idx, tot, bp, r, _ = best
    return c[idx].astype(np.int64), tot, bp, r
