// select.cpp -- GlowQ-S selective restore (host).
//
// GlowQ pages, papernotes.org summary, key design 4: units are ranked by the
// normalised error ratio g_ner(u) = ||E_u||_F^2 / ||W_u||_F^2 and only the
// top-k are restored; when the signal is weak the ranking falls back to the
// layer order.  The pages do not define "weak"; this library takes it to mean
// a NaN score or all scores within a relative spread of 1e-6.
#include <algorithm>
#include <cmath>
#include <numeric>
#include <vector>

#include "glowq.h"

extern "C" glowq_status glowq_select_restore(const double* err_fro2, const double* w_fro2,
                                             const int32_t* layer_idx, const int32_t* kind, int32_t n_units,
                                             int32_t k, uint8_t* restore_mask, int32_t* order,
                                             int32_t* used_fallback) {
    if (n_units < 0 || k < 0 || k > n_units) return GLOWQ_ERR_ARG;
    if (n_units > 0 && (!err_fro2 || !w_fro2 || !layer_idx || !kind || !restore_mask)) return GLOWQ_ERR_ARG;
    std::vector<double> score((size_t)n_units);
    bool any_nan = false;
    double hi = -INFINITY, lo = INFINITY;
    for (int32_t u = 0; u < n_units; ++u) {
        score[u] = err_fro2[u] / w_fro2[u];
        if (std::isnan(score[u])) {
            any_nan = true;
        } else {
            hi = std::max(hi, score[u]);
            lo = std::min(lo, score[u]);
        }
    }
    const bool weak = any_nan || n_units == 0 || (hi - lo) <= 1e-6 * std::max(std::fabs(hi), 1e-300);
    std::vector<int32_t> idx((size_t)n_units);
    std::iota(idx.begin(), idx.end(), 0);
    auto layer_key = [&](int32_t a, int32_t b) {
        if (layer_idx[a] != layer_idx[b]) return layer_idx[a] < layer_idx[b];
        if (kind[a] != kind[b]) return kind[a] < kind[b];
        return a < b;
    };
    if (weak) {
        std::sort(idx.begin(), idx.end(), layer_key);
    } else {
        std::sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
            if (score[a] != score[b]) return score[a] > score[b];
            return layer_key(a, b);
        });
    }
    for (int32_t u = 0; u < n_units; ++u) restore_mask[u] = 0;
    for (int32_t i = 0; i < k; ++i) restore_mask[idx[i]] = 1;
    if (order)
        for (int32_t i = 0; i < n_units; ++i) order[i] = idx[i];
    if (used_fallback) *used_fallback = weak ? 1 : 0;
    return GLOWQ_OK;
}
