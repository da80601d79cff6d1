"""Pins for the oracle's decode-time append (open block) and its effect on selection.

Decode-time index maintenance is a reading (the pages only say LSA also speeds
up decode): a completed pooled group after the last closed block is pooled,
normalised and appended to the bucket of its nearest closed centroid."""
import numpy as np

import oracle
import synth
from test_oracle_select import _brute_select


def _decode_state(seed=0):
    w = synth.workload("decode", T=4096, B=1, M=64, G=64, k=4, R=1024, W=8, S=4, steps=200,
                       Hq=4, Hkv=1, d=64, dtype="f32")
    inp = synth.decode_inputs(w, seed, "cpu")
    lat = inp["latent_K"][0].numpy()
    idx = oracle.Index(w.T + w.steps + w.p * w.G, w.p, w.G, w.k, w.L, rt_bf16=False)
    idx.extend(lat, 0, w.T)
    return w, inp, lat, idx


def test_open_assign_is_nearest_closed_centroid():
    w, inp, lat, idx = _decode_state()
    j0 = idx.n_blocks * w.G
    assert np.all(idx.open_bucket == -1)
    idx.append(lat, w.T + w.steps)
    n_new = w.steps // w.p
    assert np.all(idx.open_bucket[:n_new] >= 0) and np.all(idx.open_bucket[n_new:] == -1)
    u = oracle.unit(oracle.pool(lat[j0 * w.p:(j0 + n_new) * w.p], w.p))
    assert np.array_equal(idx.unit[j0:j0 + n_new], u)
    s = u.astype(np.float64) @ idx.cent[: idx.n_buckets].astype(np.float64).T
    assert np.array_equal(idx.open_bucket[:n_new], np.argmax(s, axis=1))


def test_append_is_incremental_and_idempotent():
    w, inp, lat, idx = _decode_state(1)
    ref = oracle.Index(w.T + w.steps + w.p * w.G, w.p, w.G, w.k, w.L, rt_bf16=False)
    ref.extend(lat, 0, w.T)
    ref.append(lat, w.T + w.steps)
    for t in range(w.T, w.T + w.steps + 1):
        idx.append(lat, t)                 # one token at a time, as in decode
    idx.append(lat, w.T + w.steps)
    assert np.array_equal(idx.open_bucket, ref.open_bucket)


def test_selection_reads_open_members_when_window_is_short():
    w, inp, lat, idx = _decode_state(2)
    idx.append(lat, w.T + w.steps)
    pos = np.arange(w.T, w.T + w.steps)
    # Queries aimed at a recently appended key, so its bucket ranks high.
    lq = lat[np.maximum(pos - w.W - 2, 0)].copy()
    out, cnt, _, nlr = oracle.select(idx, lq, pos, w.R, w.W, w.S)
    used_open = 0
    for i, p in enumerate(pos):
        # every completed group below pos - W is a candidate; rebuild with the
        # open lists as they stood at that step
        step = oracle.Index(w.T + w.steps + w.p * w.G, w.p, w.G, w.k, w.L, rt_bf16=False)
        step.__dict__.update({k: v.copy() if isinstance(v, np.ndarray) else v
                              for k, v in idx.__dict__.items()})
        n_done = (p + 1) // w.p - idx.n_blocks * w.G
        step.open_bucket[max(n_done, 0):] = -1
        o2, c2, _, _ = oracle.select(step, lq[i:i + 1], np.array([p]), w.R, w.W, w.S)
        s, lr, win = _brute_select(step, lq[i], int(p), w.R, w.W, w.S)
        assert o2[0, :c2[0]].tolist() == s + lr + win
        used_open += int(np.sum(np.array(lr, dtype=np.int64) >= w.T))
    assert used_open > 0


def test_open_assign_ties_go_to_lowest_bucket():
    # With every closed centroid equal, each appended group ties everywhere
    # and must land in bucket 0.
    w, inp, lat, idx = _decode_state(3)
    idx.cent[: idx.n_buckets] = idx.cent[5]
    idx.append(lat, w.T + w.steps)
    n_new = w.steps // w.p
    assert np.all(idx.open_bucket[:n_new] == 0)


def test_closing_a_filled_open_block_equals_building_the_longer_prefix():
    # The index past the open block: decode appends fill the open block, then
    # extend over that block closes it.  The result is the index built over
    # the longer prefix in one go (same pooled keys, centroids, CSR,
    # assignments), with an empty open block.
    w = synth.workload("decode", T=1024, B=1, M=16, G=16, k=4, R=200, W=8, S=4, steps=140,
                       Hq=4, Hkv=1, d=64, dtype="f32")
    inp = synth.decode_inputs(w, 5, "cpu")
    lat = inp["latent_K"][0].numpy()
    span = w.p * w.G
    t_cap = w.T + w.steps + span
    idx = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=False)
    idx.extend(lat, 0, w.T)
    t_end = w.T
    for pos in range(w.T, w.T + 2 * span):
        idx.append(lat, pos + 1)
        if (pos + 1) % span == 0:
            assert np.all(idx.open_bucket >= 0)            # the block's G groups are all assigned
            idx.extend(lat, pos + 1 - span, pos + 1)
            t_end = pos + 1
            assert np.all(idx.open_bucket == -1)
    assert t_end == w.T + 2 * span and idx.n_blocks == t_end // span
    ref = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=False)
    ref.extend(lat, 0, t_end)
    nb, npool = ref.n_buckets, t_end // w.p
    assert np.array_equal(idx.pooled[:npool], ref.pooled[:npool])
    assert np.array_equal(idx.unit[:npool], ref.unit[:npool])
    assert np.array_equal(idx.cent[:nb], ref.cent[:nb])
    assert np.array_equal(idx.offsets[:nb + 1], ref.offsets[:nb + 1])
    assert np.array_equal(idx.members[:npool], ref.members[:npool])
    assert np.array_equal(idx.assign[:npool], ref.assign[:npool])
    assert np.array_equal(idx.open_bucket, ref.open_bucket)
