"""Pins of the oracle's D-LSA Tree (two-level index and the walk down it).

Reading ("Prefrontal's Latent Sparse Attention speeds up one attention layer
72x at 10M tokens ...", section "What it changes": clusters are grouped into a
hierarchy, a query scores a few clusters at each level and walks down;
"Latent Sparse Attention: un indice gerarchico per contesti lunghi", paragraph
on Flat vs Tree: the tree computes less, a wrong branch can leave keys out):
level 2 clusters the buckets' centroids into super-buckets; a query keeps its
best `branches` super-buckets and ranks and fills only their buckets.

Each pin would fail on a plausible mistake in the oracle:
  * walking every branch reproduces Flat bit for bit (a dropped bucket, a
    wrong bucket order or a fill difference shows);
  * an independent restatement in Python floats (super scores, branch choice,
    key-sort fill) agrees on small inputs (a wrong tie rule, branch count,
    sign or index shows);
  * a hand-built index with two far-apart topics: one branch reads only the
    query's topic, two branches fall through to the other when the first runs
    out;
  * level 2 is a proper clustering of the buckets: CSR bijection, ascending
    members, each super-centroid the normalised binary64 mean of its members.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _index(w, seed, rt_bf16, t_end=None):
    inp = synth.prefill_inputs(w, seed, "cpu")
    lat = inp["latent_K"][0].float().numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=rt_bf16)
    orc.extend(lat, 0, t_end or w.T)
    return inp, orc


@pytest.mark.parametrize("rt_bf16,t_end", [(False, None), (True, None), (False, 8192 - 500)])
def test_every_branch_is_flat(rt_bf16, t_end):
    w = synth.workload("tiny", T=8192, nq=96, dtype="bf16" if rt_bf16 else "f32")
    inp, orc = _index(w, 3, rt_bf16, t_end)
    tree = oracle.Tree(orc, 5, 3)
    end = t_end or w.T
    pos = np.linspace(w.W + 10, end - 1, w.nq).astype(np.int64)
    q = inp["latent_Q"][0].float().numpy()
    a, ac = oracle.tree_select(orc, tree, q, pos, tree.n_super, w.R, w.W, w.S)
    b, bc, _, _ = oracle.select(orc, q, pos, w.R, w.W, w.S)
    assert np.array_equal(ac, bc) and np.array_equal(a, b)


def _py_dot(a, b):
    s = 0.0
    for x, y in zip(a.tolist(), b.tolist()):
        s += float(x) * float(y)          # exact products, binary64 sum in order
    return s


def _brute_tree(orc, tree, q, pos, branches, R, W, S):
    """The walk restated with Python floats and sorted(): branch choice, the
    chosen buckets' available keys, long-range = first R of them sorted by
    (bucket rank, position)."""
    sup = sorted(range(tree.n_super), key=lambda h: (-_py_dot(q, tree.sup_rt[h]), h))[:branches]
    buckets = [int(g) for h in sup for g in tree.members[tree.offsets[h]:tree.offsets[h + 1]]]
    ranked = sorted(buckets, key=lambda g: (-_py_dot(q, orc.cent_rt[g]), g))
    keys = []
    for r, g in enumerate(ranked):
        for x in range(orc.offsets[g], orc.offsets[g + 1]):
            j = int(orc.members[x])
            for t in range(j * orc.p, j * orc.p + orc.p):
                if S <= t <= pos - W:
                    keys.append((r, t))
    keys.sort()
    n_s = min(S, pos + 1)
    w0 = max(pos - W + 1, n_s)
    return list(range(n_s)) + [t for _, t in keys[:R]] + list(range(w0, pos + 1))


@pytest.mark.parametrize("branches", [1, 2, 3])
def test_walk_matches_an_independent_restatement(branches):
    w = synth.workload("tiny", T=4096, nq=24, G=32, k=4, R=150, W=40, S=3, M=24)
    inp, orc = _index(w, 5, False)
    tree = oracle.Tree(orc, 6, 2)
    rng = np.random.default_rng(5)
    pos = rng.integers(0, w.T, size=w.nq)
    pos[:3] = [0, w.W, w.T - 1]
    q = inp["latent_Q"][0].float().numpy()
    a, ac = oracle.tree_select(orc, tree, q, pos, branches, w.R, w.W, w.S)
    for i in range(w.nq):
        ref = _brute_tree(orc, tree, q[i], int(pos[i]), branches, w.R, w.W, w.S)
        assert ac[i] == len(ref)
        assert a[i, :ac[i]].tolist() == ref
        assert np.all(a[i, ac[i]:] == -1)


def test_two_topics_one_branch_reads_one_topic():
    # Two far-apart latent directions, one per half of the context: the
    # buckets of each half form one super-bucket.  A query on topic A with one
    # branch reads only topic-A buckets; with two branches, once topic A is
    # exhausted the fill continues with topic B.
    T, p, G, k, R, W, S = 4096, 4, 64, 4, 2000, 16, 2
    e = np.zeros((2, 64), np.float32)
    e[0, 0] = 1.0
    e[1, 1] = 1.0
    rng = np.random.default_rng(7)
    lat = np.empty((T, 64), np.float32)
    lat[: T // 2] = e[0] + 0.05 * rng.standard_normal((T // 2, 64)).astype(np.float32)
    lat[T // 2:] = e[1] + 0.05 * rng.standard_normal((T // 2, 64)).astype(np.float32)
    orc = oracle.Index(T, p, G, k, 3, rt_bf16=False)
    orc.extend(lat, 0, T)
    tree = oracle.Tree(orc, 2, 3)
    nb = orc.n_buckets
    half = nb // 2
    groups = [set(tree.members[tree.offsets[h]:tree.offsets[h + 1]].tolist()) for h in range(2)]
    assert sorted(map(sorted, groups)) == [list(range(half)), list(range(half, nb))]
    q = (0.9 * e[0] + 0.1 * e[1])[None]
    pos = np.array([T - 1])
    sel1, c1 = oracle.tree_select(orc, tree, q, pos, 1, R, W, S)
    lr1 = [t for t in sel1[0, :c1[0]].tolist() if S <= t <= T - 1 - W]
    assert len(lr1) == R and max(lr1) < T // 2          # topic A only, and it fills R
    sel2, c2 = oracle.tree_select(orc, tree, q, pos, 2, 3000, W, S)
    lr2 = [t for t in sel2[0, :c2[0]].tolist() if S <= t <= T - 1 - W]
    a_keys = [t for t in lr2 if t < T // 2]
    assert len(a_keys) == T // 2 - S                    # all of topic A first ...
    assert len(lr2) == 3000
    assert all(t < T // 2 for t in lr2[: len(a_keys)])
    assert all(t >= T // 2 for t in lr2[len(a_keys):])  # ... then topic B


def test_level_two_is_a_clustering_of_the_buckets():
    w = synth.workload("tiny", T=8192, nq=8)
    _, orc = _index(w, 9, False)
    tree = oracle.Tree(orc, 7, 3)
    nb = orc.n_buckets
    assert tree.offsets[0] == 0 and tree.offsets[-1] == nb
    assert sorted(tree.members.tolist()) == list(range(nb))            # bijection
    for h in range(tree.n_super):
        m = tree.members[tree.offsets[h]:tree.offsets[h + 1]]
        assert np.all(np.diff(m) > 0)                                  # ascending
        assert np.all(tree.assign[m] == h)
        if len(m):
            v = np.zeros(64, np.float64)
            for g in m:                                                # ascending, binary64
                v += orc.cent[g].astype(np.float64)
            ss = 0.0
            for x in v.tolist():                                       # ascending, binary64
                ss = ss + x * x
            c = (v / math.sqrt(ss)).astype(np.float32)
            assert np.array_equal(c, tree.sup[h])


def test_one_branch_invariants():
    w = synth.workload("tiny", T=8192, nq=64)
    inp, orc = _index(w, 11, False)
    tree = oracle.Tree(orc, 6, 3)
    pos = np.linspace(0, w.T - 1, w.nq).astype(np.int64)
    q = inp["latent_Q"][0].float().numpy()
    sel, cnt = oracle.tree_select(orc, tree, q, pos, 1, w.R, w.W, w.S)
    for i in range(w.nq):
        row = sel[i, :cnt[i]]
        assert len(set(row.tolist())) == cnt[i]                        # no duplicates
        assert np.all(row <= pos[i]) and np.all(row >= 0)              # causal
        n_s = min(w.S, pos[i] + 1)
        n_w = pos[i] + 1 - max(pos[i] - w.W + 1, n_s)
        assert cnt[i] <= n_s + w.R + n_w
        assert row[:n_s].tolist() == list(range(n_s))
