"""The brute-force per-key indexer on the GPU against the oracle.

lsa_select_per_key must equal oracle.select_per_key row for row (integer
work with one correct answer: the R best long-range keys by exact binary64
score, ties to the lower position, emitted with the sinks and the window):
  * contexts where every key is its own strided group and where 4 to 32 keys
    share one; ragged query counts (and fewer than one 128-row tile),
    positions from 0 to the last key, keys past n_keys left unread, budgets
    0, 1 and 4096, window 0; positions outside the keys give empty rows and
    LSA_ERR_INVALID_ARG from the check;
  * tied scores (identical latent keys): rows with more than 8192 candidates
    take the exact fallback (counted), the others rank ties in the final
    kernel, both to the lowest positions;
  * scores beyond fp16's range (group maxima of +inf) and inside its
    subnormals;
  * the 1M workload's budget (2048) on a sample of its last chunk, with no
    fallback;
  * a wait limit of 0 makes the scoring passes give up (LSA_ERR_TIMEOUT from
    the check), and the next call on the same workspace is right.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


def _latents(T, B, M, seed, nq=8):
    w = synth.workload("tiny", T=T, nq=nq, B=B, M=M, Hq=1, Hkv=1, d=64, dtype="bf16")
    mix = synth.Mixture(w, seed, "cpu")
    lat = torch.empty(B, T, 64, dtype=torch.bfloat16)
    K = torch.empty(B, T, 1, 64, dtype=torch.bfloat16)
    V = torch.empty(B, T, 1, 64, dtype=torch.bfloat16)
    mix.keys(lat, K, V)
    return w, mix, lat


def _queries(mix, n, scale=1.0):
    lq, _ = mix.queries(n)
    return (lq * scale).to(torch.bfloat16).contiguous()


def _positions(rng, B, nq, lo, hi, edges=()):
    pos = rng.integers(lo, hi, size=(B, nq))
    for j, e in enumerate(edges):
        pos[:, j] = e
    return pos.astype(np.int32)


def _run(lat, lq, pos, R, W, S, n_keys=None, ws=None):
    idx, cnt, ws = lsa.lsa_select_per_key(lat.cuda(), lq.cuda(), torch.from_numpy(pos).cuda(), R,
                                          W, S, n_keys=n_keys, workspace=ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy(), ws


def _compare(lat, lq, pos, R, W, S, idx, cnt):
    for b in range(lat.shape[0]):
        o_idx, o_cnt = oracle.select_per_key(lat[b].float().numpy(), lq[b].float().numpy(), pos[b],
                                             R, W, S, s_max=idx.shape[-1])
        bad = np.nonzero((cnt[b] != o_cnt) | (idx[b] != o_idx).any(axis=1))[0]
        assert bad.size == 0, (b, bad[:8], cnt[b][bad[:4]], o_cnt[bad[:4]])


@pytest.mark.parametrize("T,B,nq,R,W,S,n_keys", [
    (8192, 2, 300, 512, 64, 4, None),        # one key per group
    (131072, 1, 256, 4096, 512, 4, None),    # four keys per group
    (50000, 1, 130, 2048, 512, 4, 40000),    # T_cap not a power of two, keys past n_keys
    (20000, 1, 129, 1, 0, 0, None),          # budget 1, no window, no sinks
    (20000, 1, 64, 0, 512, 4, None),         # no long-range budget
    (12000, 1, 20, 300, 64, 4, None),        # fewer query rows than one 128-row tile
])
def test_per_key_matches_oracle(T, B, nq, R, W, S, n_keys):
    w, mix, lat = _latents(T, B, 64 if T <= 8192 else 1024, T + R)
    lq = _queries(mix, nq)
    rng = np.random.default_rng(T + nq)
    top = n_keys or T
    edges = [0, 1, max(W - 1, 0), W, W + S, W + S + 1, W + S + R, top - 1]
    pos = _positions(rng, B, nq, 0, top, edges)
    idx, cnt, ws = _run(lat, lq, pos, R, W, S, n_keys=n_keys)
    assert lsa.lsa_select_per_key_check(ws) == 0
    _compare(lat, lq, pos, R, W, S, idx, cnt)


def test_per_key_positions_outside_the_keys():
    # a position at or past n_keys (or negative) reads nothing: its row is
    # empty and the check reports LSA_ERR_INVALID_ARG; every other row is right
    T, R, W, S, n_keys = 16384, 256, 64, 4, 12000
    _, mix, lat = _latents(T, 1, 64, 23)
    lq = _queries(mix, 140)
    rng = np.random.default_rng(29)
    pos = _positions(rng, 1, 140, 0, n_keys, [n_keys - 1, n_keys, T - 1, -5])
    idx, cnt, ws = _run(lat, lq, pos, R, W, S, n_keys=n_keys)
    with pytest.raises(lsa.LsaError, match="INVALID_ARG") as e:
        lsa.lsa_select_per_key_check(ws)
    assert e.value.code == 1
    bad = (pos[0] < 0) | (pos[0] >= n_keys)
    assert bad.sum() == 3 and (cnt[0][bad] == 0).all() and (idx[0][bad] == -1).all()
    ok = np.nonzero(~bad)[0]
    o_idx, o_cnt = oracle.select_per_key(lat[0].float().numpy(), lq[0].float().numpy()[ok],
                                         pos[0][ok], R, W, S, s_max=idx.shape[-1])
    assert np.array_equal(cnt[0][ok], o_cnt) and np.array_equal(idx[0][ok], o_idx)


def test_per_key_ties_take_the_lowest_positions():
    # identical latent keys: every score ties.  Rows with more than 8192
    # eligible keys overflow their candidate list and take the fallback.
    T, R, W, S = 24576, 700, 64, 4
    _, mix, lat = _latents(T, 1, 16, 3)
    lat[:] = lat[:, :1]
    lq = _queries(mix, 200)
    rng = np.random.default_rng(5)
    pos = _positions(rng, 1, 200, 0, T, [100, 8000, 8300, T - 1])
    idx, cnt, ws = _run(lat, lq, pos, R, W, S)
    fb = lsa.lsa_select_per_key_check(ws)
    over = int(((pos[0] - W - S + 1) > 8192).sum())
    assert fb == over and over > 0
    _compare(lat, lq, pos, R, W, S, idx, cnt)


@pytest.mark.parametrize("scale", [4.0e5, 1.0e-5])
def test_per_key_scores_outside_fp16(scale):
    # scores up to ~4e5 (group maxima round to +inf in fp16) and down to
    # ~1e-5 (fp16 subnormals): the threshold still holds the exact top set
    T, R, W, S = 32768, 1024, 128, 4
    _, mix, lat = _latents(T, 1, 256, 11)
    lq = _queries(mix, 160, scale)
    rng = np.random.default_rng(13)
    pos = _positions(rng, 1, 160, T // 2, T, [T - 1])
    idx, cnt, ws = _run(lat, lq, pos, R, W, S)
    lsa.lsa_select_per_key_check(ws)
    _compare(lat, lq, pos, R, W, S, idx, cnt)


def test_per_key_on_the_1m_workload():
    # the 1M workload's latents and budget (R = 2048), 1024 queries of the
    # last chunk; 48 rows spread over every 128-row tile checked
    w = synth.workload("1m")
    mix = synth.Mixture(w, 0, "cuda")
    lat = torch.empty(1, w.T, 64, dtype=torch.bfloat16, device="cuda")
    K = torch.empty(1, w.T, w.Hkv, w.d, dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    mix.keys(lat, K, V)
    del K, V
    nq = 1024
    lq, _ = mix.queries(nq)
    lq = lq.to(torch.bfloat16).contiguous()
    pos = torch.arange(w.T - nq, w.T, dtype=torch.int32, device="cuda")[None].contiguous()
    idx, cnt, ws = lsa.lsa_select_per_key(lat, lq, pos, w.R, w.W, w.S)
    torch.cuda.synchronize()
    assert lsa.lsa_select_per_key_check(ws) == 0
    rows = np.concatenate([np.arange(t * 128, t * 128 + 128, 23) for t in range(nq // 128)])
    lat_h = lat[0].float().cpu().numpy()
    lq_h = lq[0].float().cpu().numpy()
    pos_h = pos[0].cpu().numpy()
    o_idx, o_cnt = oracle.select_per_key(lat_h, lq_h[rows], pos_h[rows], w.R, w.W, w.S)
    assert np.array_equal(cnt[0].cpu().numpy()[rows], o_cnt)
    assert np.array_equal(idx[0].cpu().numpy()[rows], o_idx)


def test_per_key_wait_timeout_then_recovers():
    T, R, W, S = 16384, 512, 64, 4
    _, mix, lat = _latents(T, 1, 64, 17)
    lq = _queries(mix, 256)
    rng = np.random.default_rng(19)
    pos = _positions(rng, 1, 256, 0, T, [T - 1])
    try:
        lsa._check(lsa._lib.lsa_set_wait_limit(0))
        _, _, ws = _run(lat, lq, pos, R, W, S)
        with pytest.raises(lsa.LsaError, match="TIMEOUT") as e:
            lsa.lsa_select_per_key_check(ws)
        assert e.value.code == 5                          # LSA_ERR_TIMEOUT
    finally:
        lsa._check(lsa._lib.lsa_set_wait_limit(-1))
    idx, cnt, ws = _run(lat, lq, pos, R, W, S, ws=ws)
    assert lsa.lsa_select_per_key_check(ws) == 0
    _compare(lat, lq, pos, R, W, S, idx, cnt)
