// stepq_alloc.cpp -- lifetime-aware bit allocation (host, run offline).
//
// STEPQuant summary, "Method" (second paragraph) and the ONTLE blog post: for each unit,
// estimate the reconstruction distortion at the candidate widths and the memory lifetime
// from the mean log retention; error retention after j updates decays exponentially,
// which gives a lifetime weight; under an average bit budget choose the widths that
// minimise the lifetime-weighted distortion.
//   rho_u = 2^(-1/half_life_u),  w_u = sum_j rho_u^j = 1 / (1 - rho_u),
//   minimise sum_u w_u D_u(b_u)  s.t.  sum_u b_u <= floor(N * avg_bits).
// Solved exactly by dynamic programming over the number of bits spent so far.
//
// FP16 pivots (same paragraph: the highest-risk units are kept in FP16 as sparse
// pivots): the n_pivots units with the largest lifetime-weighted distortion at the widest
// candidate width become width 16, outside the budget; the others are allocated as above
// with the budget floor((N - n_pivots) * avg_bits).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <numeric>
#include <vector>

#include "stepq.h"

namespace {

double lifetime_weight(double half_life) { return -1.0 / std::expm1(-std::log(2.0) / half_life); }  // 1 / (1 - 2^(-1/h))

int check_args(const double *half_life, const double *distortion, int32_t N, const uint8_t *cand, int32_t C,
               double avg_bits, const uint8_t *bits_out)
{
    if (!half_life || !cand || !bits_out || N <= 0 || C <= 0 || C > 3) return STEPQ_INVALID_ARG;
    if (!std::isfinite(avg_bits) || avg_bits <= 0.0) return STEPQ_INVALID_ARG;
    for (int c = 0; c < C; ++c) {
        if (cand[c] != 4 && cand[c] != 6 && cand[c] != 8) return STEPQ_INVALID_ARG;
        for (int d = 0; d < c; ++d)
            if (cand[d] == cand[c]) return STEPQ_INVALID_ARG;
    }
    for (int u = 0; u < N; ++u)
        if (!std::isfinite(half_life[u]) || half_life[u] <= 0.0) return STEPQ_INVALID_ARG;
    if (distortion)
        for (long long e = 0; e < (long long)N * C; ++e)
            if (!std::isfinite(distortion[e]) || distortion[e] < 0.0) return STEPQ_INVALID_ARG;
    return STEPQ_OK;
}

// The exact DP over the units listed in `units` (indices into half_life / distortion).
int allocate_dp(const double *half_life, const double *distortion, const std::vector<int> &units,
                const uint8_t *cand, int32_t C, double avg_bits, uint8_t *bits_out)
{
    const int N = int(units.size());
    if (N == 0) return STEPQ_OK;

    const long long budget = (long long)std::floor(double(N) * avg_bits + 1e-9);
    if (budget < 0 || budget > (1LL << 24)) return STEPQ_INVALID_ARG;
    const int B = int(budget);
    // candidates visited in ascending width (ties keep the narrower width)
    std::vector<int> order(C);
    for (int c = 0; c < C; ++c) order[c] = c;
    for (int a = 0; a < C; ++a)
        for (int b = a + 1; b < C; ++b)
            if (cand[order[b]] < cand[order[a]]) std::swap(order[a], order[b]);

    const double INF = std::numeric_limits<double>::infinity();
    std::vector<double> best(B + 1, INF), next(B + 1);
    std::vector<int8_t> choice(size_t(N) * (B + 1), -1);   // candidate index taken by unit u at total s
    best[0] = 0.0;
    for (int u = 0; u < N; ++u) {
        const double w = lifetime_weight(half_life[units[u]]);
        std::fill(next.begin(), next.end(), INF);
        for (int s = 0; s <= B; ++s) {
            if (best[s] == INF) continue;
            for (int oi = 0; oi < C; ++oi) {
                const int c = order[oi];
                const int s2 = s + cand[c];
                if (s2 > B) continue;
                const double D = distortion ? distortion[(long long)units[u] * C + c] : std::ldexp(1.0, -2 * cand[c]);
                const double v = best[s] + w * D;
                if (v < next[s2]) {
                    next[s2] = v;
                    choice[size_t(u) * (B + 1) + s2] = int8_t(c);
                }
            }
        }
        best.swap(next);
    }
    int s_best = -1;
    for (int s = 0; s <= B; ++s)
        if (best[s] < INF && (s_best < 0 || best[s] < best[s_best])) s_best = s;
    if (s_best < 0) return STEPQ_INVALID_ARG;       // no assignment fits the budget
    for (int u = N - 1, s = s_best; u >= 0; --u) {
        const int c = choice[size_t(u) * (B + 1) + s];
        bits_out[units[u]] = cand[c];
        s -= cand[c];
    }
    return STEPQ_OK;
}

}  // namespace

extern "C" int stepq_allocate_bits(const double *half_life, const double *distortion, int32_t N,
                                   const uint8_t *cand, int32_t C, double avg_bits, uint8_t *bits_out)
{
    const int st = check_args(half_life, distortion, N, cand, C, avg_bits, bits_out);
    if (st != STEPQ_OK) return st;
    std::vector<int> units(N);
    std::iota(units.begin(), units.end(), 0);
    return allocate_dp(half_life, distortion, units, cand, C, avg_bits, bits_out);
}

extern "C" int stepq_allocate_bits_pivots(const double *half_life, const double *distortion, int32_t N,
                                          const uint8_t *cand, int32_t C, double avg_bits, int32_t n_pivots,
                                          uint8_t *bits_out)
{
    const int st = check_args(half_life, distortion, N, cand, C, avg_bits, bits_out);
    if (st != STEPQ_OK) return st;
    if (n_pivots < 0 || n_pivots > N) return STEPQ_INVALID_ARG;
    int top = 0;
    for (int c = 1; c < C; ++c)
        if (cand[c] > cand[top]) top = c;
    std::vector<double> risk(N);
    for (int u = 0; u < N; ++u)
        risk[u] = lifetime_weight(half_life[u]) *
                  (distortion ? distortion[(long long)u * C + top] : std::ldexp(1.0, -2 * cand[top]));
    std::vector<int> byrisk(N);
    std::iota(byrisk.begin(), byrisk.end(), 0);
    std::stable_sort(byrisk.begin(), byrisk.end(), [&](int x, int y) { return risk[x] > risk[y]; });
    std::vector<char> pivot(N, 0);
    for (int k = 0; k < n_pivots; ++k) pivot[byrisk[k]] = 1;
    std::vector<int> rest;
    for (int u = 0; u < N; ++u) {
        if (pivot[u])
            bits_out[u] = 16;
        else
            rest.push_back(u);
    }
    return allocate_dp(half_life, distortion, rest, cand, C, avg_bits, bits_out);
}
