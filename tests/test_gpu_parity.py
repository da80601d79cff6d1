"""GPU parity: liblsa's CUDA path against the CPU oracle on the same seeded inputs.

Bars (fixed semantics of the method):
  * index state (pooled, unit vectors, centroids, retrieval copy, CSR,
    assignments, open lists): identical bit for bit;
  * selections: identical index sets, except where the oracle's ranking margin
    is below 1e-4 relative, with such mismatches at most 1e-4 of the entries
    (the kernels rank with exact binary64 scores, so in practice every row is
    identical, order included);
  * attention: within 1e-4 max-abs (fp32) and within 2e-2 max-abs and 2e-3
    mean-abs (bf16) of the oracle evaluated on the same selections.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")

F32_TOL = 1e-4
BF16_MAX, BF16_MEAN = 2e-2, 2e-3


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def _dcode(w):
    return lsa.F32 if w.dtype == "f32" else lsa.BF16


def _compare_index(gpu, orc, b=0):
    ex = gpu.export()
    torch.cuda.synchronize()
    nb = orc.n_buckets
    NP = orc.n_blocks * orc.G
    assert np.array_equal(_np(ex["pooled"][b])[:NP], orc.pooled[:NP])
    assert np.array_equal(_np(ex["unit"][b])[:NP], orc.unit[:NP])
    assert np.array_equal(_np(ex["cent"][b])[:nb], orc.cent[:nb])
    assert np.array_equal(_np(ex["cent_rt"][b])[:nb], orc.cent_rt[:nb])
    assert np.array_equal(_np(ex["offsets"][b])[:nb + 1], orc.offsets[:nb + 1])
    assert np.array_equal(_np(ex["members"][b])[:NP], orc.members[:NP])
    assert np.array_equal(_np(ex["assign"][b])[:NP], orc.assign[:NP])
    assert np.array_equal(_np(ex["open_bucket"][b]), orc.open_bucket)
    return ex


def _compare_selection(g_idx, g_cnt, o_idx, o_cnt, o_margin):
    """Row-by-row set comparison with the margin exemption; returns #identical rows."""
    g_idx, g_cnt = _np(g_idx), _np(g_cnt)
    assert g_idx.shape == o_idx.shape
    bad = 0
    same = 0
    for r in range(o_idx.shape[0]):
        a = g_idx[r, :g_cnt[r]]
        b = o_idx[r, :o_cnt[r]]
        if g_cnt[r] == o_cnt[r] and np.array_equal(a, b):
            same += 1
            assert np.all(g_idx[r, g_cnt[r]:] == -1)
            continue
        if set(a.tolist()) == set(b.tolist()):
            same += 1
            continue
        assert o_margin[r] < 1e-4, "row %d differs with margin %g" % (r, o_margin[r])
        bad += len(set(a.tolist()) ^ set(b.tolist()))
    assert bad <= 1e-4 * o_idx.size
    return same


def _attn_check(O_gpu, O_ref, dtype):
    err = np.abs(_np(O_gpu).astype(np.float64) - O_ref.astype(np.float64))
    if dtype == "f32":
        assert err.max() <= F32_TOL, err.max()
    else:
        assert err.max() <= BF16_MAX, err.max()
        assert err.mean() <= BF16_MEAN, err.mean()
    return err.max(), err.mean()


def _setup(w, seed=0, t_build=None):
    inp = synth.prefill_inputs(w, seed, "cpu")
    lat = inp["latent_K"][0].float().numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=(w.dtype == "bf16"))
    orc.extend(lat, 0, t_build if t_build is not None else w.T)
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, _dcode(w))
    gpu.build(dev["latent_K"], t_build if t_build is not None else w.T)
    return inp, dev, orc, gpu


# --------------------------------------------------------------------------
# Full small workloads
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "128k"])
def test_workload_end_to_end(name):
    w = synth.workload(name)
    inp, dev, orc, gpu = _setup(w)
    _compare_index(gpu, orc)

    pos = inp["positions"][0].numpy()
    o_idx, o_cnt, o_mg, _ = oracle.select(orc, inp["latent_Q"][0].float().numpy(), pos, w.R, w.W,
                                          w.S)
    g_idx, g_cnt = lsa.lsa_select(gpu, dev["latent_Q"], dev["positions"].to(torch.int32), w.R,
                                  w.W, w.S)
    torch.cuda.synchronize()
    same = _compare_selection(g_idx[0], g_cnt[0], o_idx, o_cnt, o_mg)
    assert same == w.nq                       # exact ranking: every row identical
    fb = gpu.check()
    assert fb >= 0

    # attention on the oracle's selections (a sample of queries for 128k)
    rows = np.arange(w.nq) if w.nq <= 256 else np.arange(0, w.nq, 8)
    Qs = inp["Q"][0][rows].float().numpy()
    O_ref, lse_ref = oracle.attend(Qs, inp["K"][0].float().numpy(), inp["V"][0].float().numpy(),
                                   o_idx[rows], o_cnt[rows], oracle.default_scale(w.d))
    sel_i = torch.from_numpy(o_idx).cuda()[None]
    sel_c = torch.from_numpy(o_cnt).cuda()[None]
    O, lse = lsa.lsa_sparse_attn(dev["Q"], dev["K"], dev["V"], sel_i, sel_c, return_lse=True)
    torch.cuda.synchronize()
    _attn_check(O[0][torch.from_numpy(rows).cuda()], O_ref, w.dtype)
    assert np.abs(_np(lse[0])[rows] - lse_ref).max() < (1e-4 if w.dtype == "f32" else 2e-2)


@pytest.mark.parametrize("name", ["tiny", "128k"])
def test_prefill_chunk_matches_oracle(name):
    w = synth.workload(name)
    span = w.p * w.G
    T_old = w.T - w.nq
    inp, dev, orc, gpu = _setup(w, seed=1, t_build=(T_old // span) * span)
    # oracle: the chunk step extends the index over [T_old, T_new) first
    orc.extend(inp["latent_K"][0].float().numpy(), T_old, w.T)
    pos = inp["positions"][0].numpy()
    o_idx, o_cnt, o_mg, _ = oracle.select(orc, inp["latent_Q"][0].float().numpy(), pos, w.R, w.W,
                                          w.S)
    ws = torch.empty(lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    O = lsa.lsa_prefill_chunk(gpu, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"], dev["V"],
                              T_old, w.T, w.R, w.W, w.S, workspace=ws)
    torch.cuda.synchronize()
    _compare_index(gpu, orc)
    g_idx, g_cnt = lsa.prefill_selection_views(ws, 1, w.nq, w.s_max)
    assert _compare_selection(g_idx[0], g_cnt[0], o_idx, o_cnt, o_mg) == w.nq
    rows = np.arange(w.nq) if w.nq <= 256 else np.arange(3, w.nq, 16)
    O_ref, _ = oracle.attend(inp["Q"][0][rows].float().numpy(), inp["K"][0].float().numpy(),
                             inp["V"][0].float().numpy(), o_idx[rows], o_cnt[rows],
                             oracle.default_scale(w.d))
    _attn_check(O[0][torch.from_numpy(rows).cuda()], O_ref, w.dtype)
    # repeating the step reproduces it bit for bit (the timed loop relies on it)
    O2 = lsa.lsa_prefill_chunk(gpu, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"],
                               dev["V"], T_old, w.T, w.R, w.W, w.S, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(O, O2)


# --------------------------------------------------------------------------
# Selection edge cases
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("R", [0, 1, 7, 100, 5000])
def test_select_edges(dtype, R):
    w = synth.workload("tiny", T=4096, nq=64, G=32, k=4, W=16, S=3, M=16, dtype=dtype, R=R)
    inp, dev, orc, gpu = _setup(w, seed=2)
    _compare_index(gpu, orc)
    rng = np.random.default_rng(3)
    pos = np.concatenate([np.arange(0, 24), [w.W + w.S - 1, w.W + w.S, w.W + w.S + 1, 127, 128,
                                             129, w.T - 1], rng.integers(0, w.T, 40)])
    lq = inp["latent_Q"][0][rng.integers(0, w.nq, len(pos))]
    s_max = w.s_max + 5                                   # extra padding columns
    o_idx, o_cnt, o_mg, _ = oracle.select(orc, lq.float().numpy(), pos, w.R, w.W, w.S, s_max)
    g_idx, g_cnt = lsa.lsa_select(gpu, lq[None].cuda().contiguous(),
                                  torch.from_numpy(pos.astype(np.int32))[None].cuda(), w.R, w.W,
                                  w.S, s_max=s_max)
    torch.cuda.synchronize()
    assert _compare_selection(g_idx[0], g_cnt[0], o_idx, o_cnt, o_mg) == len(pos)


def test_select_exact_fallback_on_tied_scores():
    # Identical latent keys: every centroid is the same vector, so every
    # approximate score ties and no candidate set can prove the ranking; the
    # exact fallback must reproduce the oracle (ascending bucket ids).
    w = synth.workload("tiny", T=4096, nq=32, G=32, k=4, R=300, W=16, S=3, M=16)
    inp = synth.prefill_inputs(w, 4, "cpu")
    inp["latent_K"][:] = inp["latent_K"][0, 0]
    lat = inp["latent_K"][0].numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
    orc.extend(lat, 0, w.T)
    gpu = lsa.LsaIndex(1, w.T, w.p, w.G, w.k, w.L, lsa.F32)
    gpu.build(inp["latent_K"].cuda(), w.T)
    _compare_index(gpu, orc)
    pos = np.full(w.nq, w.T - 1) - np.arange(w.nq) * 7
    lq = inp["latent_Q"][0]
    o_idx, o_cnt, o_mg, _ = oracle.select(orc, lq.numpy(), pos, w.R, w.W, w.S)
    gpu.check()
    g_idx, g_cnt = lsa.lsa_select(gpu, lq[None].cuda(),
                                  torch.from_numpy(pos.astype(np.int32))[None].cuda(), w.R, w.W,
                                  w.S)
    torch.cuda.synchronize()
    assert gpu.check() > 0                                    # the fallback ran
    assert np.array_equal(_np(g_idx[0]), o_idx) and np.array_equal(_np(g_cnt[0]), o_cnt)


def test_open_block_appends_and_selection():
    # Extend to a position inside a block: the completed groups after the last
    # whole block join the open lists; with a short window they are selectable.
    w = synth.workload("tiny", T=4096, nq=64, G=32, k=4, R=400, W=8, S=4, M=16)
    inp = synth.prefill_inputs(w, 5, "cpu")
    lat = inp["latent_K"][0].numpy()
    t_now = 3 * w.p * w.G + 77
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
    orc.extend(lat, 0, t_now)
    gpu = lsa.LsaIndex(1, w.T, w.p, w.G, w.k, w.L, lsa.F32)
    gpu.build(inp["latent_K"].cuda(), t_now)
    _compare_index(gpu, orc)
    assert np.sum(orc.open_bucket >= 0) == (t_now // w.p) - 3 * w.G
    pos = np.arange(t_now - 40, t_now)
    lq = torch.from_numpy(lat[pos - w.W - 3]).contiguous()   # aim at recent keys
    o_idx, o_cnt, o_mg, _ = oracle.select(orc, lq.numpy(), pos, w.R, w.W, w.S)
    g_idx, g_cnt = lsa.lsa_select(gpu, lq[None].cuda(),
                                  torch.from_numpy(pos.astype(np.int32))[None].cuda(), w.R, w.W,
                                  w.S)
    torch.cuda.synchronize()
    assert _compare_selection(g_idx[0], g_cnt[0], o_idx, o_cnt, o_mg) == len(pos)
    assert np.any(o_idx[:, w.S:] >= 3 * w.p * w.G)            # open members were read


def test_multi_sequence_index_and_select():
    w = synth.workload("tiny", T=4096, nq=48, B=3, G=64, k=8, R=256, W=32, S=4, M=32)
    inp = synth.prefill_inputs(w, 6, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.F32)
    gpu.build(dev["latent_K"], w.T)
    g_idx, g_cnt = lsa.lsa_select(gpu, dev["latent_Q"], dev["positions"].to(torch.int32), w.R,
                                  w.W, w.S)
    torch.cuda.synchronize()
    for b in range(w.B):
        orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
        orc.extend(inp["latent_K"][b].numpy(), 0, w.T)
        _compare_index(gpu, orc, b)
        o_idx, o_cnt, o_mg, _ = oracle.select(orc, inp["latent_Q"][b].numpy(),
                                              inp["positions"][b].numpy(), w.R, w.W, w.S)
        assert _compare_selection(g_idx[b], g_cnt[b], o_idx, o_cnt, o_mg) == w.nq


# --------------------------------------------------------------------------
# Attention variants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("hpg,d", [(1, 64), (2, 128), (4, 64), (8, 128), (8, 64)])
def test_attention_shapes_and_ragged_counts(dtype, hpg, d):
    rng = np.random.default_rng(hpg * 1000 + d)
    Hkv = 2
    Hq = hpg * Hkv
    T, B, nq, s_max = 3000, 2, 9, 700
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator().manual_seed(hpg + d)
    K = torch.randn(B, T, Hkv, d, generator=g).to(tdt)
    V = torch.randn(B, T, Hkv, d, generator=g).to(tdt)
    Q = (torch.randn(B, nq, Hq, d, generator=g) * 2.0).to(tdt)
    counts = np.array([[1, 15, 16, 17, 63, 64, 65, 333, 700], [700, 2, 31, 32, 33, 128, 129, 5, 1]],
                      np.int32)
    idx = np.full((B, nq, s_max), -1, np.int32)
    for b in range(B):
        for i in range(nq):
            idx[b, i, :counts[b, i]] = rng.choice(T, counts[b, i], replace=False)
    O, lse = lsa.lsa_sparse_attn(Q.cuda(), K.cuda(), V.cuda(), torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(counts).cuda(), return_lse=True)
    torch.cuda.synchronize()
    for b in range(B):
        O_ref, lse_ref = oracle.attend(Q[b].float().numpy(), K[b].float().numpy(),
                                       V[b].float().numpy(), idx[b], counts[b],
                                       oracle.default_scale(d))
        _attn_check(O[b], O_ref, dtype)
        assert np.abs(_np(lse[b]) - lse_ref).max() < (1e-4 if dtype == "f32" else 2e-2)


def test_tensor_core_nomination_ragged_tiles_and_mixed_positions():
    # bf16 with Nq >= 128 takes the tcgen05 nominator: a ragged query count
    # (two full 128-row tiles + 44), two sequences, positions scattered from 0
    # to T-1 so rows of one tile see anywhere from 0 to 512 eligible buckets.
    w = synth.workload("tiny", T=16384, nq=300, B=2, G=32, k=4, R=700, W=64, S=4, M=64,
                       dtype="bf16", Hq=8, Hkv=1, d=64)
    inp = synth.prefill_inputs(w, 7, "cpu")
    rng = np.random.default_rng(7)
    pos = rng.integers(0, w.T, size=(w.B, w.nq))
    pos[:, :5] = [0, 1, w.W, w.W + 200, w.T - 1]
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(inp["latent_K"].cuda(), w.T)
    g_idx, g_cnt = lsa.lsa_select(gpu, inp["latent_Q"].cuda(),
                                  torch.from_numpy(pos.astype(np.int32)).cuda(), w.R, w.W, w.S)
    torch.cuda.synchronize()
    gpu.check()
    for b in range(w.B):
        orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
        orc.extend(inp["latent_K"][b].float().numpy(), 0, w.T)
        _compare_index(gpu, orc, b)
        o_idx, o_cnt, o_mg, _ = oracle.select(orc, inp["latent_Q"][b].float().numpy(), pos[b],
                                              w.R, w.W, w.S)
        assert _compare_selection(g_idx[b], g_cnt[b], o_idx, o_cnt, o_mg) == w.nq
