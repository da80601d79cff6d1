"""Pins for the oracle's index half: pooling, unit vectors, spherical k-means, CSR.

Each check is tied to something other than the oracle's own code: hand-worked
golden cases, closed forms, library routines (numpy matmul/argmax, torch's
bf16 conversion) or invariants the method fixes."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- pooling --

def test_pool_golden_order():
    for case in _golden("pool_order.json")["cases"]:
        p = case["p"]
        rows = np.array(case["rows"], np.float32)
        lat = np.repeat(rows[:, None], 64, axis=1)
        x = oracle.pool(lat, p)
        assert x.shape == (1, 64)
        assert np.all(x == np.float32(case["mean"])), case["derivation"]


def test_pool_constant_rows_bitwise():
    rng = np.random.default_rng(1)
    row = rng.standard_normal(64).astype(np.float32)
    lat = np.tile(row, (4 * 5, 1))
    x = oracle.pool(lat, 4)
    # (r + r + r + r) / 4 is exact in binary32 for any finite r.
    assert np.array_equal(x, np.tile(row, (5, 1)))


def test_pool_groups_are_consecutive():
    # Group j must combine keys jp .. jp+p-1 (not a strided or shifted set).
    lat = np.arange(12, dtype=np.float32)[:, None] * np.ones((1, 64), np.float32)
    x = oracle.pool(lat, 4)
    assert np.array_equal(x[:, 0], np.array([1.5, 5.5, 9.5], np.float32))


# ------------------------------------------------------------ unit vectors --

def test_unit_closed_forms():
    x = np.zeros((3, 64), np.float32)
    x[0, 0], x[0, 1] = 3.0, 4.0          # norm 5
    x[1, 5] = -2.0                        # norm 2
    u = oracle.unit(x)
    assert u[0, 0] == np.float32(0.6) and u[0, 1] == np.float32(0.8)
    assert np.count_nonzero(u[0]) == 2
    assert u[1, 5] == np.float32(-1.0) and np.count_nonzero(u[1]) == 1
    assert np.all(u[2] == 0.0)            # zero vector stays zero


def test_unit_is_unit_and_parallel():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((100, 64)).astype(np.float32) * 3
    u = oracle.unit(x).astype(np.float64)
    assert np.allclose(np.linalg.norm(u, axis=1), 1.0, atol=1e-6)
    cos = np.sum(u * x, axis=1) / np.linalg.norm(x.astype(np.float64), axis=1)
    assert np.allclose(cos, 1.0, atol=1e-6)


# ---------------------------------------------------------------- k-means --

@pytest.mark.parametrize("case", _golden("kmeans_hand.json")["cases"], ids=lambda c: c["name"])
def test_kmeans_golden(case):
    u = np.array(case["u"], np.float32)
    cent, assign, _ = oracle.kmeans_block(u, case["k"], case["L"])
    assert assign.tolist() == case["assign"], case["derivation"]
    if "cent" in case:
        assert np.array_equal(cent, np.array(case["cent"], np.float32)), case["derivation"]
    if "cent_hex" in case:
        want = np.array([[int(h, 16) for h in row] for row in case["cent_hex"]], np.uint32)
        assert np.array_equal(cent.view(np.uint32), want), case["derivation"]


def test_kmeans_identical_points_keep_initial_rows():
    u = np.tile(np.array([[0.6, 0.8]], np.float32), (4, 1))
    cent, assign, margin = oracle.kmeans_block(u, 2, 3)
    assert np.all(assign == 0)
    assert np.array_equal(cent[1], u[2])          # empty bucket keeps its init u[2]
    assert np.all(margin == 0.0)                  # exact tie


def _clustered_units(rng, G, k, dl, spread):
    dirs = rng.standard_normal((k, dl))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    lab = rng.integers(0, k, G)
    x = dirs[lab] + spread * rng.standard_normal((G, dl))
    return oracle.unit(x.astype(np.float32))


def test_kmeans_L1_is_argmax_then_normalised_mean():
    # One Lloyd iteration from the evenly spaced init reduces to a matmul, an
    # argmax (first maximum = lowest id) and a normalised mean.
    rng = np.random.default_rng(3)
    G, k, dl = 256, 8, 64
    u = _clustered_units(rng, G, k, dl, 0.5)
    cent, assign, _ = oracle.kmeans_block(u, k, 1)
    init = u[(np.arange(k) * G) // k].astype(np.float64)
    s = u.astype(np.float64) @ init.T
    want = np.argmax(s, axis=1)
    assert np.array_equal(assign, want)
    for m in range(k):
        mem = u[want == m].astype(np.float64)
        if len(mem) == 0:
            assert np.array_equal(cent[m], init[m].astype(np.float32))
            continue
        v = mem.sum(axis=0)
        assert np.allclose(cent[m], v / np.linalg.norm(v), atol=2e-7)


def test_kmeans_converged_assignment_is_nearest_final_centroid():
    # On well-separated clusters Lloyd converges; then every point's bucket is
    # the argmax against the final centroids, and each centroid is the
    # normalised mean of its members.
    rng = np.random.default_rng(4)
    G, k, dl = 512, 8, 64
    u = _clustered_units(rng, G, k, dl, 0.05)
    cent, assign, margin = oracle.kmeans_block(u, k, 12)
    s = u.astype(np.float64) @ cent.astype(np.float64).T
    assert np.array_equal(assign, np.argmax(s, axis=1))
    top2 = np.sort(s, axis=1)[:, -2:]
    assert np.allclose(margin, (top2[:, 1] - top2[:, 0]) / np.abs(top2[:, 1]), rtol=1e-9)
    for m in np.unique(assign):
        v = u[assign == m].astype(np.float64).sum(axis=0)
        assert np.allclose(cent[m], v / np.linalg.norm(v), atol=2e-7)


def test_kmeans_assignment_depends_on_first_index_for_ties():
    # Permuting which duplicate comes first changes the init and hence the
    # bucket ids: a pin on the floor(m*G/k) init index.
    u = np.array([[1, 0], [1, 0], [0, 1], [0, 1]], np.float32)
    _, a1, _ = oracle.kmeans_block(u, 2, 1)
    assert a1.tolist() == [0, 0, 1, 1]
    u2 = u[[2, 3, 0, 1]]
    _, a2, _ = oracle.kmeans_block(u2, 2, 1)
    assert a2.tolist() == [0, 0, 1, 1]          # init = u2[0], u2[2] = e1, e0


# -------------------------------------------------------------- full index --

@pytest.fixture(scope="module")
def tiny_index():
    w = synth.workload("tiny")
    inp = synth.prefill_inputs(w, 0, "cpu")
    lat = inp["latent_K"][0].numpy()
    idx = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    idx.extend(lat, 0, w.T)
    return w, lat, idx


def test_index_pool_and_unit_rows(tiny_index):
    w, lat, idx = tiny_index
    assert np.array_equal(idx.pooled, oracle.pool(lat, w.p))
    assert np.array_equal(idx.unit, oracle.unit(idx.pooled))


def test_index_csr_invariants(tiny_index):
    w, _, idx = tiny_index
    nb = idx.n_buckets
    assert idx.n_blocks == w.T // (w.p * w.G) == 8
    off, mem = idx.csr()
    assert off[0] == 0 and off[-1] == idx.n_blocks * w.G
    assert np.all(np.diff(off) >= 0)
    for b in range(idx.n_blocks):
        assert off[b * w.k] == b * w.G                       # block starts
        blk = mem[b * w.G:(b + 1) * w.G]
        assert np.array_equal(np.sort(blk), np.arange(b * w.G, (b + 1) * w.G))  # bijection
    for g in range(nb):
        ms = mem[off[g]:off[g + 1]]
        assert np.all(np.diff(ms) > 0)                       # ascending
        assert np.all(idx.assign[ms] == g % w.k)             # members carry their bucket
        assert np.all(ms // w.G == g // w.k)                 # and stay in their block


def test_index_blocks_match_standalone_kmeans(tiny_index):
    w, _, idx = tiny_index
    for b in (0, 5, 7):
        cent, assign, _ = oracle.kmeans_block(idx.unit[b * w.G:(b + 1) * w.G], w.k, w.L)
        assert np.array_equal(cent, idx.cent[b * w.k:(b + 1) * w.k])
        assert np.array_equal(assign, idx.assign[b * w.G:(b + 1) * w.G])


def test_index_retrieval_copy_is_torch_bf16(tiny_index):
    _, _, idx = tiny_index
    want = torch.from_numpy(idx.cent).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(idx.cent_rt, want)
    assert np.array_equal(oracle.round_bf16(idx.cent), want)


def test_index_nonempty_centroids_are_normalised_member_means(tiny_index):
    w, _, idx = tiny_index
    off, mem = idx.csr()
    for g in range(idx.n_buckets):
        ms = mem[off[g]:off[g + 1]]
        if len(ms) == 0:
            continue
        v = idx.unit[ms].astype(np.float64).sum(axis=0)
        assert np.allclose(idx.cent[g], v / np.linalg.norm(v), atol=2e-7)


def test_index_extend_matches_full_build():
    w = synth.workload("tiny")
    inp = synth.prefill_inputs(w, 3, "cpu")
    lat = inp["latent_K"][0].numpy()
    full = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
    full.extend(lat, 0, w.T)
    inc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
    span = w.p * w.G
    inc.extend(lat, 0, 3 * span)
    inc.extend(lat, 3 * span, 5 * span + 100)   # trailing partial block -> open groups
    assert inc.n_blocks == 5
    assert np.all(inc.open_bucket[:100 // w.p] >= 0) and np.all(inc.open_bucket[100 // w.p:] == -1)
    inc.extend(lat, 5 * span, w.T)
    for name in ("pooled", "unit", "cent", "cent_rt", "offsets", "members", "assign"):
        assert np.array_equal(getattr(inc, name), getattr(full, name)), name
