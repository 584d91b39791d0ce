// select.cpp -- GlowQ-S selective restore (host).
//
// GlowQ pages, papernotes.org summary, key design 4: units are ranked by an
// importance score and only the top-k are restored; the pages name two scores,
// the covariance-aligned GSVD energy capture g_ec(u) = sum_{j<=r}
// sigma_j(M_u)^2 / ||M_u||_F^2 and the normalised error ratio g_ner(u) =
// ||E_u||_F^2 / ||W_u||_F^2, and fall back to the layer order when the signal
// is weak.  The pages do not define "weak"; this library takes it to mean a
// NaN score or all scores within a relative spread of 1e-6.  They do not say
// how the two scores combine either: a call ranks by one score, g_ner computed
// here from the error norms (glowq_select_restore) or any score the caller
// computed, such as g_ec from the offline solve (glowq_select_restore_scores).
#include <algorithm>
#include <cmath>
#include <numeric>
#include <vector>

#include "glowq.h"

namespace {

// Descending score, exact ties by ascending (layer, kind, index); the plain
// layer order when the signal is weak (a NaN score, or all scores within a
// relative spread of 1e-6 of the largest magnitude).
glowq_status rank_units(const double* score, const int32_t* layer_idx, const int32_t* kind, int32_t n_units,
                        int32_t k, uint8_t* restore_mask, int32_t* order, int32_t* used_fallback) {
    bool any_nan = false;
    double hi = -INFINITY, lo = INFINITY;
    for (int32_t u = 0; u < n_units; ++u) {
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

}  // namespace

extern "C" glowq_status glowq_select_restore(const double* err_fro2, const double* w_fro2,
                                             const int32_t* layer_idx, const int32_t* kind, int32_t n_units,
                                             int32_t k, uint8_t* restore_mask, int32_t* order,
                                             int32_t* used_fallback) {
    if (n_units < 0 || k < 0 || k > n_units) return GLOWQ_ERR_ARG;
    if (n_units > 0 && (!err_fro2 || !w_fro2 || !layer_idx || !kind || !restore_mask)) return GLOWQ_ERR_ARG;
    std::vector<double> score((size_t)n_units);
    for (int32_t u = 0; u < n_units; ++u) score[u] = err_fro2[u] / w_fro2[u];
    return rank_units(score.data(), layer_idx, kind, n_units, k, restore_mask, order, used_fallback);
}

extern "C" glowq_status glowq_select_restore_scores(const double* score, const int32_t* layer_idx,
                                                    const int32_t* kind, int32_t n_units, int32_t k,
                                                    uint8_t* restore_mask, int32_t* order,
                                                    int32_t* used_fallback) {
    if (n_units < 0 || k < 0 || k > n_units) return GLOWQ_ERR_ARG;
    if (n_units > 0 && (!score || !layer_idx || !kind || !restore_mask)) return GLOWQ_ERR_ARG;
    return rank_units(score, layer_idx, kind, n_units, k, restore_mask, order, used_fallback);
}
