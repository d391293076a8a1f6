// pd_search.h -- per-tensor bit-width search (host code).
//
// Per-group(128) mixed-precision article, sec. 3.2 ("PD-Guided Mixed Precision Bit
// Allocation"): minimize sum_i ||W_i - Q_{b_i}(W_i)||_F^2 over one width b_i per tensor,
// subject to sum_i n_i b_i / sum_i n_i = target BPW. The relaxation: one continuous parameter
// t_i per tensor, b_i = sigmoid(t_i) (b_max - b_min) + b_min; a softmax over -|b_i - c_j| / T
// assigns b_i softly to the candidate widths c_j at a temperature annealed from 2 to 0.05;
// the tensor's error is the table's errors averaged under that assignment; the loss adds a
// Lagrange term lambda (BPW - target) and a penalty 1e4 (BPW - target)^2. The parameters take
// Adam steps (lr 0.05) down the loss, the multiplier plain ascent steps (0.05) from 0.5;
// after the iterations each width is rounded to the nearest candidate, and of all the random
// starts the one with the smallest total error within target + 0.05 BPW is kept.
// The table's per-weight MSEs are divided by one reference value (the uniform allocation's
// error at the candidate nearest the target), a constant factor that leaves the minimizer of
// the constrained problem unchanged but puts the data term on the scale of the page's
// constants. The random starts are the caller's input, so the search is deterministic.
#pragma once

#include <cmath>
#include <vector>

namespace wq {

struct PdResult {
    double total_mse, bpw;
    int restart;
};

inline int pd_nearest(double b, const int *bits, int n_bits) {
    int best = 0;
    double bd = std::fabs(b - bits[0]);
    for (int j = 1; j < n_bits; ++j) {
        const double d = std::fabs(b - bits[j]);
        if (d < bd) { bd = d; best = j; }
    }
    return best;
}

// mse: n x n_bits per-weight MSE (row-major); t_init: n_restarts x n random starts.
inline PdResult pd_search_host(const double *mse, const int64_t *n_params, int n, const int *bits, int n_bits,
                               double target, int n_iters, int n_restarts, const double *t_init, int *bits_out) {
    constexpr double kLr = 0.05, kB1 = 0.9, kB2 = 0.999, kEps = 1e-8, kDualLr = 0.05, kLambda0 = 0.5;
    constexpr double kPenalty = 1e4, kSlack = 0.05;
    double total = 0.0;
    for (int i = 0; i < n; ++i) total += (double)n_params[i];
    const double b_min = bits[0], b_max = bits[n_bits - 1];
    const int ref_col = pd_nearest(target, bits, n_bits);
    double ref = 0.0;
    for (int i = 0; i < n; ++i) ref += (double)n_params[i] * mse[(size_t)i * n_bits + ref_col];
    ref /= total;
    std::vector<double> m((size_t)n * n_bits), t(n), m1(n), m2(n), sig(n), bc(n), w(n_bits), dz(n_bits);
    for (size_t k = 0; k < m.size(); ++k) m[k] = mse[k] / ref;
    std::vector<int> idx(n), best_idx(n);
    PdResult best{0.0, 0.0, -1};
    bool best_feasible = false;
    for (int r = 0; r < n_restarts; ++r) {
        for (int i = 0; i < n; ++i) { t[i] = t_init[(size_t)r * n + i]; m1[i] = m2[i] = 0.0; }
        double lagrange = kLambda0;
        for (int it = 0; it < n_iters; ++it) {
            const double temp = std::fmax(2.0 * (1.0 - (double)it / n_iters), 0.05);
            double bpw = 0.0;
            for (int i = 0; i < n; ++i) {
                sig[i] = 1.0 / (1.0 + std::exp(-t[i]));
                bc[i] = sig[i] * (b_max - b_min) + b_min;
                bpw += bc[i] * (double)n_params[i];
            }
            bpw /= total;
            const double gap = bpw - target;
            const int k = it + 1;
            const double c1 = 1.0 - std::pow(kB1, k), c2 = 1.0 - std::pow(kB2, k);
            for (int i = 0; i < n; ++i) {
                // soft assignment and the derivative of the smoothed error
                double zmax = -INFINITY;
                for (int j = 0; j < n_bits; ++j) zmax = std::fmax(zmax, -std::fabs(bc[i] - bits[j]) / temp);
                double sum = 0.0;
                for (int j = 0; j < n_bits; ++j) { w[j] = std::exp(-std::fabs(bc[i] - bits[j]) / temp - zmax); sum += w[j]; }
                double a = 0.0;
                for (int j = 0; j < n_bits; ++j) {
                    w[j] /= sum;
                    const double d = bc[i] - bits[j];
                    dz[j] = -((d > 0.0) - (d < 0.0)) / temp;
                    a += w[j] * dz[j];
                }
                double d_smooth = 0.0;
                for (int j = 0; j < n_bits; ++j) d_smooth += m[(size_t)i * n_bits + j] * w[j] * (dz[j] - a);
                const double g_b = (double)n_params[i] / total * (d_smooth + lagrange + 2.0 * kPenalty * gap);
                const double g_t = g_b * sig[i] * (1.0 - sig[i]) * (b_max - b_min);
                m1[i] = kB1 * m1[i] + (1.0 - kB1) * g_t;
                m2[i] = kB2 * m2[i] + (1.0 - kB2) * g_t * g_t;
                t[i] = t[i] - kLr * (m1[i] / c1) / (std::sqrt(m2[i] / c2) + kEps);
            }
            lagrange = lagrange + kDualLr * gap;
        }
        double tot = 0.0, bp = 0.0;
        for (int i = 0; i < n; ++i) {
            const double s = 1.0 / (1.0 + std::exp(-t[i]));
            idx[i] = pd_nearest(s * (b_max - b_min) + b_min, bits, n_bits);
            tot += (double)n_params[i] * mse[(size_t)i * n_bits + idx[i]];
            bp += (double)n_params[i] * bits[idx[i]];
        }
        tot /= total;
        bp /= total;
        const bool feasible = bp <= target + kSlack;
        const bool take = best.restart < 0 || (feasible && (!best_feasible || tot < best.total_mse)) ||
                          (!feasible && !best_feasible && bp < best.bpw);
        if (take) {
            best = PdResult{tot, bp, r};
            best_feasible = feasible;
            best_idx = idx;
        }
    }
    for (int i = 0; i < n; ++i) bits_out[i] = bits[best_idx[i]];
    return best;
}

}  // namespace wq
