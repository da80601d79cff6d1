"""Pins for the oracle's retrieval: ranking, greedy budget fill, sinks and window.

The main pin is an independent brute force of the selection in its key-sort
form: the long-range keys are the first R of all available keys sorted by
(rank of their bucket, position).  Whole buckets taken while they fit and the
next one truncated in ascending position is exactly that prefix, so any
dropped term, wrong comparison or off-by-one in the oracle's greedy loop shows
up as a difference."""
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _brute_select(idx, q, pos, R, W, S):
    """Key-sort restatement: returns (sinks, long-range keys in take order, window)."""
    nb = idx.n_buckets
    s = idx.cent_rt[:nb].astype(np.float64) @ q.astype(np.float64)
    order = np.lexsort((np.arange(nb), -s))          # score desc, then lowest id
    rank = np.empty(nb, np.int64)
    rank[order] = np.arange(nb)
    # bucket of every indexed key
    key_bucket = {}
    off, mem = idx.csr()
    for g in range(nb):
        for j in mem[off[g]:off[g + 1]]:
            for r in range(idx.p):
                key_bucket[int(j) * idx.p + r] = g
    j0 = idx.n_blocks * idx.G
    for o, g in enumerate(idx.open_bucket):
        if g >= 0:
            for r in range(idx.p):
                key_bucket[(j0 + o) * idx.p + r] = int(g)
    avail = [t for t in range(S, pos - W + 1) if t in key_bucket]
    avail.sort(key=lambda t: (rank[key_bucket[t]], t))
    lr = avail[:R]
    sinks = list(range(0, min(S, pos + 1)))
    window = list(range(max(pos - W + 1, min(S, pos + 1)), pos + 1))
    return sinks, lr, window


def _index(w, seed=0, rt_bf16=False, t_build=None):
    inp = synth.prefill_inputs(w, seed, "cpu")
    lat = inp["latent_K"][0].float().numpy()
    idx = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=rt_bf16)
    idx.extend(lat, 0, t_build if t_build is not None else w.T)
    return inp, lat, idx


@pytest.fixture(scope="module")
def small():
    # Small blocks so that buckets are small and truncation happens often.
    w = synth.workload("tiny", T=2048, nq=64, G=32, k=4, R=100, W=16, S=3, M=16)
    inp, lat, idx = _index(w)
    return w, inp, idx


def test_select_matches_key_sort_brute_force(small):
    w, inp, idx = small
    rng = np.random.default_rng(5)
    pos = np.concatenate([np.arange(0, 40), rng.integers(40, w.T, 200), [w.T - 1]])
    lq = inp["latent_Q"][0].numpy()
    qs = lq[rng.integers(0, lq.shape[0], len(pos))]
    out, cnt, _, nlr = oracle.select(idx, qs, pos, w.R, w.W, w.S)
    for i, p in enumerate(pos):
        sinks, lr, window = _brute_select(idx, qs[i], int(p), w.R, w.W, w.S)
        want = sinks + lr + window
        got = out[i, :cnt[i]].tolist()
        assert got == want, (i, int(p))
        assert nlr[i] == len(lr)
        assert np.all(out[i, cnt[i]:] == -1)


@pytest.mark.parametrize("R", [0, 1, 7, 64, 100000])
def test_select_budget_edges(small, R):
    w, inp, idx = small
    pos = np.array([0, 1, 2, 3, 18, 19, 20, 500, 1500, w.T - 1])
    qs = inp["latent_Q"][0].numpy()[: len(pos)]
    out, cnt, _, nlr = oracle.select(idx, qs, pos, R, w.W, w.S, s_max=w.T + 8)
    for i, p in enumerate(pos):
        p = int(p)
        n_s = min(w.S, p + 1)
        n_w = p + 1 - max(p - w.W + 1, n_s)
        n_lr = min(R, max(0, p - w.W + 1 - w.S))
        assert cnt[i] == n_s + n_lr + n_w and nlr[i] == n_lr
        sel = out[i, :cnt[i]]
        assert len(np.unique(sel)) == len(sel)              # no duplicates
        assert sel.min() >= 0 and sel.max() <= p             # causal
        assert sel[:n_s].tolist() == list(range(n_s))        # sinks first
        assert sel[cnt[i] - n_w:].tolist() == list(range(p + 1 - n_w, p + 1))  # window last
        lr = sel[n_s:n_s + n_lr]
        assert np.all((lr >= w.S) & (lr <= p - w.W))         # long-range outside both
        if R >= p + 1:
            assert sorted(sel.tolist()) == list(range(p + 1))  # budget covers everything


def test_select_read_budget_golden():
    cases = json.load(open(os.path.join(GOLDEN, "read_budget.json")))["cases"]
    # A cheap index (latent dim 2) over a full 10M context, so that the pages'
    # own positions can be used; the count formula does not depend on dl.
    rng = np.random.default_rng(6)
    T = 10485760
    lat = rng.standard_normal((T, 2)).astype(np.float32)
    idx = oracle.Index(T, 4, 1024, 16, 1, rt_bf16=False, dl=2)
    idx.extend(lat, 0, T)
    for c in cases:
        q = rng.standard_normal((1, 2)).astype(np.float32)
        out, cnt, _, nlr = oracle.select(idx, q, np.array([c["pos"]]), c["R"], c["W"], c["S"],
                                         s_max=c["R"] + c["W"] + c["S"])
        assert cnt[0] == c["count"] and nlr[0] == c["n_lr"], c["note"]


def test_select_truncation_is_ascending_prefix_of_one_bucket(small):
    w, inp, idx = small
    qs = inp["latent_Q"][0].numpy()[:32]
    pos = np.full(32, w.T - 1)
    out, cnt, _, nlr = oracle.select(idx, qs, pos, w.R, w.W, w.S)
    off, mem = idx.csr()
    kb = np.empty(len(mem) * idx.p, np.int64)          # bucket of every indexed key
    for g in range(idx.n_buckets):
        for j in mem[off[g]:off[g + 1]]:
            kb[j * idx.p:(j + 1) * idx.p] = g
    for i in range(32):
        lr = out[i, w.S:w.S + nlr[i]]
        b = kb[lr]
        # buckets appear as contiguous runs; within a run positions ascend
        runs = np.flatnonzero(np.diff(b)) + 1
        seen = set()
        for seg in np.split(np.arange(len(lr)), runs):
            g = int(b[seg[0]])
            assert g not in seen
            seen.add(g)
            assert np.all(np.diff(lr[seg]) > 0)
        # only the last run may be a strict subset of its bucket's available keys
        for seg in np.split(np.arange(len(lr)), runs)[:-1]:
            g = int(b[seg[0]])
            avail = [t for j in mem[off[g]:off[g + 1]] for t in range(j * idx.p, (j + 1) * idx.p)
                     if w.S <= t <= w.T - 1 - w.W]
            assert lr[seg].tolist() == avail


def test_select_scores_use_retrieval_copy():
    # With rt_bf16 the ranking uses the bf16-rounded centroids: rebuilding the
    # brute force from cent (unrounded) may differ, from cent_rt must not.
    w = synth.workload("tiny", T=2048, nq=32, G=32, k=4, R=60, W=16, S=3, M=16)
    inp, lat, idx = _index(w, seed=1, rt_bf16=True)
    assert not np.array_equal(idx.cent, idx.cent_rt)
    qs = inp["latent_Q"][0].numpy()
    pos = np.full(len(qs), w.T - 1)
    out, cnt, _, _ = oracle.select(idx, qs, pos, w.R, w.W, w.S)
    for i in range(len(qs)):
        s, lr, win = _brute_select(idx, qs[i], w.T - 1, w.R, w.W, w.S)
        assert out[i, :cnt[i]].tolist() == s + lr + win


def test_select_margin_flags_near_ties():
    # Two buckets whose centroids tie for a query must report margin 0 when
    # they sit at the cut, and the set must then follow the lowest id.
    w = synth.workload("tiny", T=2048, nq=8, G=32, k=4, R=20, W=16, S=3, M=16)
    inp, lat, idx = _index(w, seed=2)
    nb = idx.n_buckets
    idx.cent_rt[: nb] = idx.cent_rt[0]          # every bucket scores the same
    q = inp["latent_Q"][0].numpy()[:1]
    out, cnt, mg, nlr = oracle.select(idx, q, np.array([w.T - 1]), w.R, w.W, w.S)
    assert mg[0] == 0.0
    s, lr, win = _brute_select(idx, q[0], w.T - 1, w.R, w.W, w.S)
    assert out[0, :cnt[0]].tolist() == s + lr + win
