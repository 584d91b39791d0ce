"""Pins for the oracle's GlowQ-S selective restore.

Pages: papernotes.org GlowQ summary, key design 4 (score g_ner(u) =
||E_u||_F^2 / ||W_u||_F^2, activate only the top-k units, fall back to layer
order when the signal is weak) and the efficiency paragraph (about 50% of the
groups restored).  Pins: brute-force sorting of hand-built tables with ties,
NaNs and flat scores.
"""
import numpy as np

import oracle


def _brute(e, w, layer, kind, k):
    sc = [ei / wi for ei, wi in zip(e, w)]
    weak = any(np.isnan(sc)) or (max(sc) - min(sc)) <= 1e-6 * max(abs(max(sc)), 1e-300)
    if weak:
        order = sorted(range(len(e)), key=lambda u: (layer[u], kind[u], u))
    else:
        order = sorted(range(len(e)), key=lambda u: (-sc[u], layer[u], kind[u], u))
    mask = np.zeros(len(e), np.uint8)
    mask[order[:k]] = 1
    return mask, np.array(order), weak


def test_top_k_by_ratio_with_ties():
    e = [4.0, 1.0, 3.0, 2.0, 3.0, 0.5]
    w = [2.0, 1.0, 1.0, 2.0, 1.0, 1.0]       # scores 2, 1, 3, 1, 3, 0.5
    layer = [0, 0, 1, 1, 0, 2]
    kind = [0, 1, 0, 1, 1, 0]
    mask, order, score, weak = oracle.select_restore(e, w, layer, kind, 3)
    bm, bo, bw = _brute(e, w, layer, kind, 3)
    assert not weak and not bw
    assert np.array_equal(order, bo) and np.array_equal(mask, bm)
    assert list(order[:3]) == [4, 2, 0]      # tie 3.0: layer 0 before layer 1
    assert np.allclose(score, np.array(e) / np.array(w))


def test_weak_signal_falls_back_to_layer_order():
    n = 8
    e = [1.0] * n
    w = [2.0] * n
    layer = [3, 1, 2, 0, 1, 0, 3, 2]
    kind = [0, 1, 0, 1, 0, 0, 1, 1]
    mask, order, _, weak = oracle.select_restore(e, w, layer, kind, 4)
    bm, bo, bw = _brute(e, w, layer, kind, 4)
    assert weak and bw
    assert np.array_equal(order, bo) and np.array_equal(mask, bm)


def test_nan_score_falls_back():
    e = [1.0, 2.0, 3.0]
    w = [1.0, 0.0 * np.nan, 1.0]
    mask, order, _, weak = oracle.select_restore(e, w, [2, 1, 0], [0, 0, 0], 1)
    assert weak and list(order) == [2, 1, 0] and list(mask) == [0, 0, 1]


def test_random_tables_against_brute_force():
    g = np.random.default_rng(0)
    for trial in range(50):
        n = int(g.integers(1, 40))
        e = list(np.round(g.random(n) * 5, 1))
        w = list(np.round(g.random(n) * 5 + 0.1, 1))
        layer = list(g.integers(0, 10, n))
        kind = list(g.integers(0, 4, n))
        k = int(g.integers(0, n + 1))
        mask, order, _, weak = oracle.select_restore(e, w, layer, kind, k)
        bm, bo, bw = _brute(e, w, layer, kind, k)
        assert weak == bw
        assert np.array_equal(order, bo) and np.array_equal(mask, bm)
        assert mask.sum() == k


def _brute_scores(sc, layer, kind, k):
    weak = any(np.isnan(sc)) or (max(sc) - min(sc)) <= 1e-6 * max(abs(max(sc)), 1e-300)
    if weak:
        order = sorted(range(len(sc)), key=lambda u: (layer[u], kind[u], u))
    else:
        order = sorted(range(len(sc)), key=lambda u: (-sc[u], layer[u], kind[u], u))
    mask = np.zeros(len(sc), np.uint8)
    mask[order[:k]] = 1
    return mask, np.array(order), weak


def test_select_by_score_against_brute_force_and_ratio_path():
    """Ranking by an arbitrary score (e.g. g_ec) follows the same rule, and on
    score = err / w it is exactly the g_ner selection."""
    g = np.random.default_rng(3)
    for trial in range(50):
        n = int(g.integers(1, 40))
        sc = list(np.round(g.random(n) * 2, 2 if trial % 2 else 6))
        if trial % 9 == 4:
            sc = [0.5] * n                                       # flat: layer order
        layer = list(g.integers(0, 10, n))
        kind = list(g.integers(0, 4, n))
        k = int(g.integers(0, n + 1))
        mask, order, weak = oracle.select_by_score(sc, layer, kind, k)
        bm, bo, bw = _brute_scores(sc, layer, kind, k)
        assert weak == bw
        assert np.array_equal(order, bo) and np.array_equal(mask, bm)
        e = np.array(sc) * 3.0
        w = np.full(n, 3.0)
        m2, o2, _, w2 = oracle.select_restore(e, w, layer, kind, k)
        m3, o3, w3 = oracle.select_by_score(e / w, layer, kind, k)
        assert np.array_equal(o2, o3) and np.array_equal(m2, m3) and w2 == w3
