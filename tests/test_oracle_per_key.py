"""Pins for the oracle's brute-force per-key indexer (the comparison baseline
that LSA's bucket retrieval replaces) and its recall measure.

The per-key indexer scores every long-range-available key of a query and
reads the best R of them.  Pinned by: a pure-Python re-derivation (tuples
sorted by the standard library, sums in plain Python floats) on tiny inputs,
closed forms where the ranking is known in advance, explicit ties, the budget
edges, and agreement with the bucket selection when the budget covers every
key."""
import numpy as np
import pytest

import oracle
import synth


def _py_select(lat, q, pos, R, W, S):
    """The definition written out with Python floats and sorted()."""
    n_s = min(S, pos + 1)
    w0 = max(pos - W + 1, n_s)
    cand = []
    for t in range(S, pos - W + 1):
        s = 0.0
        for d in range(len(q)):
            s += float(lat[t][d]) * float(q[d])      # binary64, ascending dimension
        cand.append((-s, t))
    taken = sorted(t for _, t in sorted(cand)[:R])
    return list(range(n_s)) + taken + list(range(w0, pos + 1))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_pure_python_definition(seed):
    rng = np.random.default_rng(seed)
    T = 160
    lat = rng.standard_normal((T, 16)).astype(np.float32)
    qs = rng.standard_normal((40, 16)).astype(np.float32)
    pos = rng.integers(0, T, 40)
    for R, W, S in [(10, 8, 4), (0, 8, 4), (1, 1, 0), (500, 3, 2), (7, 0, 0)]:
        idx, cnt = oracle.select_per_key(lat, qs, pos, R, W, S)
        for i in range(len(pos)):
            want = _py_select(lat, qs[i], int(pos[i]), R, W, S)
            assert cnt[i] == len(want)
            assert idx[i, :cnt[i]].tolist() == want
            assert np.all(idx[i, cnt[i]:] == -1)


def test_closed_form_ranking():
    # key t has score t + 1 against the all-ones query: the best R available
    # keys are the R latest positions before the window
    T, dl = 256, 64
    lat = np.zeros((T, dl), np.float32)
    for t in range(T):
        lat[t, t % dl] = t + 1
    q = np.ones((1, dl), np.float32)
    R, W, S, pos = 20, 16, 4, 200
    idx, cnt = oracle.select_per_key(lat, q, np.array([pos]), R, W, S)
    hi = pos - W
    assert idx[0, :cnt[0]].tolist() == (list(range(S)) + list(range(hi - R + 1, hi + 1)) +
                                        list(range(pos - W + 1, pos + 1)))


def test_ties_go_to_the_lowest_positions():
    T = 100
    lat = np.ones((T, 8), np.float32)                 # every key scores the same
    q = np.ones((1, 8), np.float32)
    idx, cnt = oracle.select_per_key(lat, q, np.array([90]), 5, 10, 4)
    assert idx[0, 4:9].tolist() == [4, 5, 6, 7, 8]


def test_budget_edges_and_invariants():
    rng = np.random.default_rng(3)
    T = 300
    lat = rng.standard_normal((T, 64)).astype(np.float32)
    qs = rng.standard_normal((30, 64)).astype(np.float32)
    pos = np.arange(0, T, 10)
    W, S = 12, 4
    for R in (0, 1, 7, 64, 10 ** 6):
        idx, cnt = oracle.select_per_key(lat, qs, pos, R, W, S)
        for i, p in enumerate(pos):
            row = idx[i, :cnt[i]]
            avail = max(0, p - W - S + 1)
            n_s = min(S, p + 1)
            n_w = p + 1 - max(p - W + 1, n_s)
            assert cnt[i] == n_s + min(R, avail) + n_w
            assert len(set(row.tolist())) == cnt[i]          # no duplicates
            assert row.max() <= p and row.min() >= 0         # causal
            lr = row[n_s:cnt[i] - n_w]
            assert np.all((lr >= S) & (lr <= p - W))
            if 0 < len(lr) < avail:                          # every taken key beats every other
                sc = oracle.per_key_scores(lat[S:p - W + 1], qs[i])
                taken = np.isin(np.arange(S, p - W + 1), lr)
                assert sc[taken].min() >= sc[~taken].max()


def test_full_budget_reads_what_the_bucket_selection_reads():
    # with a budget covering every available key both indexers read the same set
    w = synth.workload("tiny", T=2048, nq=64, B=1, Hq=4, Hkv=1, d=64, M=16, p=4, G=32, k=4, L=3,
                       R=10 ** 6, W=16, S=4, dtype="f32")
    inp = synth.prefill_inputs(w, 4, "cpu")
    lat = inp["latent_K"][0].numpy()
    idx_b = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
    idx_b.extend(lat, 0, w.T)
    q = inp["latent_Q"][0].numpy()
    pos = inp["positions"][0].numpy()
    bi, bc, _, _ = oracle.select(idx_b, q, pos, w.R, w.W, w.S)
    ki, kc = oracle.select_per_key(lat, q, pos, w.R, w.W, w.S)
    for i in range(len(pos)):
        assert sorted(bi[i, :bc[i]].tolist()) == ki[i, :kc[i]].tolist()
    assert np.all(oracle.recall(bi, bc, ki, kc, pos, w.S, w.W) == 1.0)


def test_recall_counts_long_range_keys_only():
    ref = np.array([[0, 1, 10, 20, 30, 95, 96, -1]], np.int32)
    sel = np.array([[0, 1, 10, 30, 50, 95, 96, -1]], np.int32)
    r = oracle.recall(sel, np.array([7]), ref, np.array([7]), np.array([96]), 2, 2)
    assert r[0] == pytest.approx(2 / 3)                      # 10 and 30 of {10, 20, 30}


def test_hand_worked_cases():
    # tests/golden/per_key_hand.json: rows worked by hand from the definition
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "per_key_hand.json")))
    lat = np.array(g["latent_K"], np.float32)
    for c in g["cases"]:
        s_max = c["R"] + c["W"] + c["S"]
        idx, cnt = oracle.select_per_key(lat, np.array([c["q"]], np.float32), np.array([c["pos"]]),
                                         c["R"], c["W"], c["S"], s_max=s_max)
        assert idx[0, :cnt[0]].tolist() == c["row"], c["derivation"]
        assert np.all(idx[0, cnt[0]:] == -1)
