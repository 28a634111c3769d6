"""The seeded input recipe (CPU): token distributions, weight statistics and the
regenerate-a-subset property that the stored oracle outputs rely on."""
from dataclasses import replace

import numpy as np
import pytest

from workloads import TINY, SMALL, WORKLOADS, make_tokens, make_weights, make_weight
from workloads.generate import weight_shapes

Z300 = WORKLOADS["300m-12+12-b512"]


def _ranks(tokens: np.ndarray, V: int) -> np.ndarray:
    """Map token ids back to their Zipf ranks (1-based) through the seeded permutation."""
    perm = np.random.default_rng([3, V]).permutation(V)
    inv = np.empty(V, np.int64)
    inv[perm] = np.arange(V)
    return inv[tokens] + 1


def test_zipf_tokens_follow_the_power_law():
    wl = Z300
    V, s = wl.model.V, wl.zipf_s
    tok = make_tokens(wl, seqs=range(128))                       # 131072 draws
    r = _ranks(tok.ravel(), V)
    n = r.size
    p = np.arange(1, V + 1, dtype=np.float64) ** -s
    p /= p.sum()                                                 # P(rank r) = r^-s / H(V, s)
    counts = np.bincount(r, minlength=V + 1)[1:]
    for k in range(1, 11):                                       # the head: within 5 sigma each
        sigma = np.sqrt(n * p[k - 1] * (1 - p[k - 1]))
        assert abs(counts[k - 1] - n * p[k - 1]) <= 5 * sigma, k
    ks = np.arange(1, 51)
    slope = np.polyfit(np.log(ks), np.log(counts[:50]), 1)[0]
    assert slope == pytest.approx(-s, abs=0.06)


def test_uniform_tokens_cover_the_vocabulary_evenly():
    wl = TINY
    V = wl.model.V
    tok = make_tokens(wl.with_batch(64, wl.T)).ravel()
    counts = np.bincount(tok, minlength=V)
    expected = tok.size / V
    chi2 = ((counts - expected) ** 2 / expected).sum()
    assert chi2 < V + 6 * np.sqrt(2 * V)                         # chi-square, V-1 dof, ~6 sigma


def test_markov_rows_are_concentrated_like_dirichlet_point_one():
    """The small workload's recipe on a 4-token vocabulary, where every order-2 context recurs:
    Dirichlet(0.1) rows put most of their mass on one token (top share ~0.85 on average), while
    rows near uniform would give ~0.3."""
    wl = replace(SMALL, model=replace(SMALL.model, V=4), T=4096)
    tok = make_tokens(wl, seqs=range(4))
    follow: dict[tuple[int, int], list[int]] = {}
    for seq in tok:
        for t in range(2, len(seq)):
            follow.setdefault((int(seq[t - 2]), int(seq[t - 1])), []).append(int(seq[t]))
    tops = [np.bincount(v, minlength=4).max() / len(v) for v in follow.values() if len(v) >= 50]
    assert len(tops) >= 4
    assert np.mean(tops) > 0.6


@pytest.mark.parametrize("name", ["tiny-f32", "small-bf16", "300m-12+12-b512"])
def test_a_subset_of_sequences_regenerates_identically(name):
    wl = WORKLOADS[name]
    sub = [0, 3, 5] if wl.B > 5 else [0, wl.B - 1]
    whole = make_tokens(wl.with_batch(max(sub) + 1, wl.T))
    np.testing.assert_array_equal(make_tokens(wl, seqs=sub), whole[sub])
    np.testing.assert_array_equal(make_tokens(wl, seqs=sub), make_tokens(wl, seqs=sub))


def test_weight_statistics_and_per_tensor_streams():
    m = SMALL.model
    w = make_weights(m)
    assert set(w) == set(weight_shapes(m))
    for name, a in w.items():
        assert a.shape == weight_shapes(m)[name] and a.dtype == np.float32
        if name.endswith("_norm"):
            assert np.all(a == 1.0)
        elif name == "merge_bias":
            assert np.all(a == 0.0)
        elif a.size >= 4096:
            assert abs(float(a.std()) - 0.02) < 0.002 and abs(float(a.mean())) < 0.002, name
    # one tensor regenerated alone equals the one in the full dict; another seed differs
    np.testing.assert_array_equal(make_weight(m, "layers.2.w_up"), w["layers.2.w_up"])
    assert not np.array_equal(make_weight(m, "layers.2.w_up", seed=1), w["layers.2.w_up"])
    assert not np.array_equal(w["layers.0.wq"], w["layers.0.wk"])
