// Offline calibration, host code: stepq_lifetime_weight and
// stepq_allocate_bits (lifetime-aware bit allocation, below) and
// stepq_impact_weights (the plan's row-impact weights from the scores that
// the row-impact kernel accumulates: w = sqrt(mean squared weighting factor)).
//
// hyper.ai summary of the paper, section "Method" (the Lifetime-Aware Bit
// Allocation paragraph): per state unit, the reconstruction distortion at
// each candidate width and the mean log retention of its gates; an error
// left in the state decays by the retention at every update, so the weight
// of a unit's distortion is how long that error lives; under an average bit
// budget the widths minimise the lifetime-weighted distortion, and the units
// of highest risk stay in FP16 as sparse pivots.  The rcap.io post
// ("Temporal") places this, and the pivot choice, offline.
//
// Forms the pages leave open, as taken here: lifetime weight
// sum_{j>=0} exp(j ell) = 1 / (1 - exp(ell)) with ell the mean log gate;
// pivots = largest weight * distortion at the budget width; the widths of
// the rest are the exact minimum under the budget (a multiple-choice
// knapsack over 2-bit upgrades, solved by a recurrence over the units).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <numeric>
#include <vector>

#include "stepq_internal.cuh"

namespace {

constexpr int kWidths[3] = {4, 6, 8};
constexpr size_t kMaxTable = size_t(1) << 31;  // bytes of the choice table

int invalid(const char *msg) { return stepq::set_error(STEPQ_ERR_INVALID, msg); }

}  // namespace

extern "C" int stepq_lifetime_weight(int64_t n_units, int64_t n_steps, int32_t gates_per_unit,
                                     const float *gate, double *weight) {
    stepq::set_error(STEPQ_OK, "");
    if (n_units <= 0 || n_steps <= 0 || gates_per_unit <= 0)
        return invalid("n_units, n_steps and gates_per_unit must be positive");
    if (!gate || !weight) return invalid("gate and weight must not be NULL");
    if (n_units > (int64_t(1) << 40) / n_steps / gates_per_unit) return invalid("gate array too large");
    const int64_t total = n_units * n_steps * gates_per_unit;
    for (int64_t i = 0; i < total; ++i)
        if (!(gate[i] > 0.0f && gate[i] < 1.0f)) return invalid("every gate must lie in (0, 1)");
    const double count = double(n_steps) * double(gates_per_unit);
    for (int64_t u = 0; u < n_units; ++u) {
        double acc = 0.0;  // sum of log g over steps (outer) and the unit's gates (inner)
        for (int64_t t = 0; t < n_steps; ++t) {
            const float *g = gate + (t * n_units + u) * gates_per_unit;
            for (int32_t r = 0; r < gates_per_unit; ++r) acc += std::log(double(g[r]));
        }
        const double ell = acc / count;  // mean log retention, < 0
        weight[u] = 1.0 / (1.0 - std::exp(ell));
    }
    return STEPQ_OK;
}

extern "C" int stepq_impact_weights(int64_t n_rows, int64_t count, const double *score_sum, float *w) {
    stepq::set_error(STEPQ_OK, "");
    if (n_rows <= 0 || count <= 0) return invalid("n_rows and count must be positive");
    if (!score_sum || !w) return invalid("score_sum and w must not be NULL");
    for (int64_t i = 0; i < n_rows; ++i)
        if (!(std::isfinite(score_sum[i]) && score_sum[i] > 0.0))
            return invalid("every score sum must be finite and > 0 (a row that never reaches the readout)");
    for (int64_t i = 0; i < n_rows; ++i) w[i] = float(std::sqrt(score_sum[i] / double(count)));
    return STEPQ_OK;
}

extern "C" int stepq_allocate_bits(int64_t n_units, const double *weight, const double *dist,
                                   int32_t budget_bits, int64_t n_pivots, uint8_t *bits) {
    stepq::set_error(STEPQ_OK, "");
    if (n_units <= 0) return invalid("n_units must be positive");
    if (!weight || !dist || !bits) return invalid("weight, dist and bits must not be NULL");
    if (budget_bits != 4 && budget_bits != 6 && budget_bits != 8)
        return invalid("budget_bits must be 4, 6 or 8");
    if (n_pivots < 0 || n_pivots > n_units) return invalid("n_pivots outside [0, n_units]");
    for (int64_t u = 0; u < n_units; ++u) {
        if (!(std::isfinite(weight[u]) && weight[u] > 0.0)) return invalid("weights must be finite and > 0");
        for (int o = 0; o < 3; ++o)
            if (!(std::isfinite(dist[u * 3 + o]) && dist[u * 3 + o] >= 0.0))
                return invalid("distortions must be finite and >= 0");
    }
    const int col = (budget_bits - 4) / 2;
    const int64_t N = n_units - n_pivots;
    const int64_t K = N * (budget_bits - 4) / 2;  // 2-bit upgrades the budget allows
    if (N > 0 && size_t(N) * size_t(K + 1) > kMaxTable) return invalid("too many units for the choice table");

    // pivots: largest risk weight * distortion at the budget width, ties to
    // the lower index
    std::vector<int64_t> order(n_units);
    std::iota(order.begin(), order.end(), int64_t(0));
    std::vector<double> risk(n_units);
    for (int64_t u = 0; u < n_units; ++u) risk[u] = weight[u] * dist[u * 3 + col];
    std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
        return risk[a] > risk[b] || (risk[a] == risk[b] && a < b);
    });
    std::vector<uint8_t> is_pivot(n_units, 0);
    for (int64_t t = 0; t < n_pivots; ++t) is_pivot[order[t]] = 1;
    std::vector<int64_t> rest;
    rest.reserve(N);
    for (int64_t u = 0; u < n_units; ++u)
        if (!is_pivot[u]) rest.push_back(u);

    // V_t(k) = min over o <= min(k, 2) of c_t(o) + V_{t+1}(k - o), V_N = 0;
    // strict < over o = 0, 1, 2 keeps the smaller width on equal sums
    std::vector<uint8_t> choice(size_t(N) * size_t(K + 1));
    std::vector<double> nxt(K + 1, 0.0), cur(K + 1);
    for (int64_t t = N - 1; t >= 0; --t) {
        const int64_t u = rest[t];
        const double c0 = weight[u] * dist[u * 3 + 0];
        const double c1 = weight[u] * dist[u * 3 + 1];
        const double c2 = weight[u] * dist[u * 3 + 2];
        uint8_t *ch = choice.data() + size_t(t) * size_t(K + 1);
        for (int64_t k = 0; k <= K; ++k) {
            double best = c0 + nxt[k];
            uint8_t pick = 0;
            if (k >= 1) {
                const double v = c1 + nxt[k - 1];
                if (v < best) { best = v; pick = 1; }
            }
            if (k >= 2) {
                const double v = c2 + nxt[k - 2];
                if (v < best) { best = v; pick = 2; }
            }
            cur[k] = best;
            ch[k] = pick;
        }
        std::swap(cur, nxt);
    }
    for (int64_t u = 0; u < n_units; ++u) bits[u] = 16;
    int64_t k = K;
    for (int64_t t = 0; t < N; ++t) {
        const int o = choice[size_t(t) * size_t(K + 1) + size_t(k)];
        bits[rest[t]] = uint8_t(kWidths[o]);
        k -= o;
    }
    return STEPQ_OK;
}
