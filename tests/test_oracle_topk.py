"""Pins for the oracle's top-k region selection (step A3).

[P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: a radix-style top-k keeps the best
512 regions per query and always includes the query's own region; §第二招 (sparse_config
table): at most 512 regions per query.  Fixed reading: own region + the k-1 best
eligible regions (r < own) by (score desc, index asc); output ascending, count =
min(k, own + 1), padding -1.
"""
import numpy as np
import pytest

import oracle

G = 4


def brute(scores, q_pos, k):
    """Python's sorted() on (-score, index): an independent evaluation."""
    nq = scores.shape[0]
    out = []
    for i in range(nq):
        own = q_pos[i] // 8
        row = []
        for g in range(G):
            order = sorted(range(own), key=lambda r: (-float(scores[i, g, r]), r))
            row.append(sorted(order[: k - 1] + [own]))
        out.append(row)
    return out


def check(scores, q_pos, k):
    idx, cnt = oracle.topk_regions(scores, q_pos, k)
    ref = brute(scores, q_pos, k)
    for i in range(len(q_pos)):
        own = q_pos[i] // 8
        for g in range(G):
            c = int(cnt[i, g])
            assert c == min(k, own + 1)
            assert list(idx[i, g, :c]) == ref[i][g]
            assert np.all(idx[i, g, c:] == -1)
            assert own in idx[i, g, :c]
            assert np.all(idx[i, g, :c] <= own)
    return idx, cnt


@pytest.mark.parametrize("k", [1, 2, 7, 16, 64])
def test_brute_force_random(k):
    rng = np.random.default_rng(k)
    nq, ld = 5, 300
    s = rng.standard_normal((nq, G, ld)).astype(np.float32)
    q_pos = [0, 7, 8, 800, 8 * 300 - 1 + 1]
    check(s, q_pos, k)


def test_brute_force_heavy_ties():
    rng = np.random.default_rng(11)
    s = rng.integers(0, 4, (3, G, 500)).astype(np.float32)     # four distinct values only
    check(s, [4000, 2001, 999], 50)


def test_all_zero_scores_pick_the_lowest_indices():
    s = np.zeros((1, G, 100), np.float32)
    idx, cnt = check(s, [8 * 100 + 3], 11)
    for g in range(G):
        assert list(idx[0, g, :11]) == list(range(10)) + [100]


def test_signed_zero_ties_with_zero():
    s = np.zeros((1, G, 6), np.float32)
    s[0, :, 1] = -0.0
    s[0, :, 4] = -0.0
    idx, _ = oracle.topk_regions(s, [48], 4)
    assert list(idx[0, 0, :4]) == [0, 1, 2, 6]


def test_own_region_is_forced_even_with_the_worst_score():
    s = np.ones((1, G, 20), np.float32)
    s[0, :, 12] = -1e30                      # a low score at the own index is never looked at
    idx, cnt = check(s, [12 * 8 + 5], 3)
    assert list(idx[0, 0, :3]) == [0, 1, 12]


def test_scores_at_or_beyond_the_own_region_are_ignored():
    s = np.zeros((1, G, 30), np.float32)
    s[0, :, 10:] = 1e9
    idx, _ = oracle.topk_regions(s, [10 * 8], 4)
    assert list(idx[0, 0, :4]) == [0, 1, 2, 10]


def test_count_is_k_when_enough_regions():
    rng = np.random.default_rng(5)
    s = rng.random((1, G, 4096)).astype(np.float32)
    idx, cnt = check(s, [4096 * 8 - 1], 512)
    assert np.all(cnt == 512)


def test_k_at_least_region_count_selects_everything():
    rng = np.random.default_rng(6)
    s = rng.random((1, G, 40)).astype(np.float32)
    idx, cnt = check(s, [39 * 8 + 2], 512)
    assert np.all(cnt == 40)
    assert list(idx[0, 2, :40]) == list(range(40))


def test_property_random_small_rows():
    """Random tiny cases (hypothesis): rows of up to 40 regions drawn from a handful of values
    (with -0.0 beside +0.0), any query position inside the row, any k: the oracle equals the
    sort-based brute force."""
    hypothesis = pytest.importorskip("hypothesis")
    st = hypothesis.strategies

    @hypothesis.settings(max_examples=150, deadline=None, derandomize=True)
    @hypothesis.given(st.integers(1, 40), st.integers(1, 45), st.data())
    def run(ld, k, data):
        vals = st.sampled_from([0.0, -0.0, 0.5, 1.0, 1.0 + 2.0 ** -23, 3.0])
        s = np.array(data.draw(st.lists(vals, min_size=G * ld, max_size=G * ld)), dtype=np.float32)
        s = s.reshape(1, G, ld)
        pos = data.draw(st.integers(0, 8 * ld - 1))
        check(s, [pos], k)

    run()
