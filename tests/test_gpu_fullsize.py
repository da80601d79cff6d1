"""Parity at the full workload sizes, in the launch configuration bench.py times.

Prefill: the whole 1M and 10M chunks (32768 queries each) run through
lsa_prefill_chunk exactly as the benchmark calls it.  The oracle then checks
  * the whole exported index -- pooled and unit rows, fp32 and retrieval
    centroids, CSR offsets and members, assignments, open lists -- of every
    block, bit for bit;
  * every one of the chunk's 32768 selections, row for row (the margin rule
    of the parity bar applies to rows that differ; none is expected, because
    the kernels rank with exact binary64 scores);
  * the outputs of 1024 rows, four in every 128-query tile of the
    tensor-core scorer, against the bf16 bars.
Per-key indexer: the whole 10M chunk through lsa_select_per_key as
bench.py's per_key measurement calls it, no fallback, and six rows spread over
the chunk row for row against the oracle's per-key indexer.
Decode: the benchmark's 8 x 1M decode runs once eagerly and is then captured
in one CUDA graph and replayed twice, as bench.py does (it times the
replays); every step's selection and output is checked against the oracle on
every pass, and the final open lists bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

lsa = pytest.importorskip("long_context_indexing_b200")

BF16_MAX, BF16_MEAN = 2e-2, 2e-3
SELECT_SLICE = 4096        # oracle selections per call (OpenMP over the slice)
ATTEND_BATCH = 128         # rows per oracle attention call (bounds the host K/V gather)


def _gather_attend(Q_rows, K, V, sel, cnt, d):
    """Oracle attention for a few rows, with K/V rows gathered on the device
    (host copies of only the rows those queries read)."""
    uniq, inv = np.unique(np.where(sel >= 0, sel, 0), return_inverse=True)
    remap = np.where(sel >= 0, inv.reshape(sel.shape), -1).astype(np.int32)
    ui = torch.from_numpy(uniq).to(K.device)
    Kh = K.index_select(0, ui).float().cpu().numpy()
    Vh = V.index_select(0, ui).float().cpu().numpy()
    return oracle.attend(Q_rows, Kh, Vh, remap, cnt, oracle.default_scale(d))[0]


def _np(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _compare_whole_index(ex, orc, b=0):
    """Every array of the exported index against the oracle's, bit for bit."""
    NP = orc.n_blocks * orc.G
    nb = orc.n_buckets
    for key, ref, n in (("pooled", orc.pooled, NP), ("unit", orc.unit, NP),
                        ("cent", orc.cent, nb), ("cent_rt", orc.cent_rt, nb),
                        ("offsets", orc.offsets, nb + 1), ("members", orc.members, NP),
                        ("assign", orc.assign, NP)):
        got = _np(ex[key][b][:n])
        assert got.shape == ref[:n].shape, key
        eq = got == ref[:n]
        assert eq.all(), "%s differs at %d entries (first %s)" % (
            key, int((~eq).sum()), np.argwhere(~eq)[0])
    assert np.array_equal(_np(ex["open_bucket"][b]), orc.open_bucket)


def _compare_selection_slice(g_idx, g_cnt, o_idx, o_cnt, o_mg):
    """Rows identical, or (parity bar) a set difference only where the oracle's
    ranking margin is below 1e-4; returns (#rows identical, #entries differing)."""
    same = (g_cnt == o_cnt) & (g_idx == o_idx).all(axis=1)
    n_diff = 0
    for r in np.nonzero(~same)[0]:
        a = set(g_idx[r, :g_cnt[r]].tolist())
        b = set(o_idx[r, :o_cnt[r]].tolist())
        if a == b:
            continue
        assert o_mg[r] < 1e-4, "row %d differs with margin %g" % (r, o_mg[r])
        n_diff += len(a ^ b)
    return int(same.sum()), n_diff


@pytest.mark.parametrize("name", ["1m", "10m"])
def test_full_size_prefill_chunk(name):
    w = synth.workload(name)
    inp = synth.prefill_inputs(w, seed=0, device="cuda")
    span = w.p * w.G
    T_old = w.T - w.nq
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    idx.build(inp["latent_K"], (T_old // span) * span)
    ws = torch.empty(lsa.lsa_prefill_workspace_bytes(idx, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    O = lsa.lsa_prefill_chunk(idx, inp["latent_K"], inp["latent_Q"], inp["Q"], inp["K"],
                              inp["V"], T_old, w.T, w.R, w.W, w.S, workspace=ws)
    torch.cuda.synchronize()
    fallbacks = idx.check()
    g_idx_d, g_cnt_d = lsa.prefill_selection_views(ws, 1, w.nq, w.s_max)
    g_idx, g_cnt = g_idx_d[0].cpu().numpy(), g_cnt_d[0].cpu().numpy()

    # 1. the whole index, every block
    lat = inp["latent_K"][0].float().cpu().numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    orc.extend(lat, 0, T_old)
    orc.extend(lat, T_old, w.T)
    del lat
    assert orc.n_blocks == idx.num_blocks == w.T // span
    ex = idx.export()
    torch.cuda.synchronize()
    _compare_whole_index(ex, orc)
    del ex

    # 2. every selection of the chunk
    lq = inp["latent_Q"][0].float().cpu().numpy()
    n_same = n_diff = 0
    o_idx_all = np.empty_like(g_idx)
    o_cnt_all = np.empty_like(g_cnt)
    for r0 in range(0, w.nq, SELECT_SLICE):
        r1 = min(w.nq, r0 + SELECT_SLICE)
        o_idx, o_cnt, o_mg, _ = oracle.select(orc, lq[r0:r1], T_old + np.arange(r0, r1), w.R,
                                              w.W, w.S)
        s, dff = _compare_selection_slice(g_idx[r0:r1], g_cnt[r0:r1], o_idx, o_cnt, o_mg)
        n_same += s
        n_diff += dff
        o_idx_all[r0:r1] = o_idx
        o_cnt_all[r0:r1] = o_cnt
    assert n_diff <= 1e-4 * g_idx.size
    print("%s: %d of %d rows identical, %d entries differ, %d fallbacks"
          % (name, n_same, w.nq, n_diff, fallbacks))

    # 3. outputs of four rows in every 128-query scorer tile
    rows = (np.arange(w.nq // 128)[:, None] * 128 + np.array([0, 41, 86, 127])[None, :]).ravel()
    assert rows.size >= 1024
    errs = []
    for k0 in range(0, rows.size, ATTEND_BATCH):
        rb = rows[k0:k0 + ATTEND_BATCH]
        O_ref = _gather_attend(inp["Q"][0][torch.from_numpy(rb).cuda()].float().cpu().numpy(),
                               inp["K"][0], inp["V"][0], o_idx_all[rb], o_cnt_all[rb], w.d)
        got = O[0][torch.from_numpy(rb).cuda()].float().cpu().numpy()
        errs.append(np.abs(got.astype(np.float64) - O_ref))
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (err.max(), err.mean())


def test_full_size_per_key_indexer():
    w = synth.workload("10m")
    inp = synth.prefill_inputs(w, seed=0, device="cuda")
    pos = inp["positions"].to(torch.int32).contiguous()
    g_idx, g_cnt, ws = lsa.lsa_select_per_key(inp["latent_K"], inp["latent_Q"], pos, w.R, w.W,
                                              w.S)
    torch.cuda.synchronize()
    assert lsa.lsa_select_per_key_check(ws) == 0
    del ws
    rows = np.array([0, 4099, 12345, 20001, 27777, w.nq - 1])
    lat = inp["latent_K"][0].double().cpu().numpy()       # binary64 once, not per query
    lq = inp["latent_Q"][0].float().cpu().numpy()[rows]
    o_idx, o_cnt = oracle.select_per_key(lat, lq, pos[0].cpu().numpy()[rows], w.R, w.W, w.S)
    assert np.array_equal(g_cnt[0].cpu().numpy()[rows], o_cnt)
    assert np.array_equal(g_idx[0].cpu().numpy()[rows], o_idx)


def test_full_size_decode_eager_and_graph_replays():
    steps = 64                                  # 16 pooled groups complete on the way
    w = synth.workload("decode", steps=steps)
    span = w.p * w.G
    t_cap = w.T + span
    inp = synth.decode_inputs(w, seed=0, device="cuda", t_cap=t_cap)
    idx = lsa.LsaIndex(w.B, t_cap, w.p, w.G, w.k, w.L, lsa.BF16)
    idx.build(inp["latent_K"], w.T)
    ws = torch.empty(lsa.lsa_decode_workspace_bytes(idx, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    pos = (w.T + torch.arange(steps, device="cuda", dtype=torch.int32))[:, None]
    pos = pos.expand(steps, w.B).contiguous()
    O = torch.empty(steps, w.B, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    v_idx, v_cnt = lsa.decode_selection_views(ws, w.B, w.s_max)
    sel_i = torch.empty(steps, w.B, w.s_max, dtype=torch.int32, device="cuda")
    sel_c = torch.empty(steps, w.B, dtype=torch.int32, device="cuda")

    def step(s):
        lsa.lsa_decode_step(idx, inp["latent_K"], inp["K"], inp["V"], inp["new_latent_k"][s],
                            inp["new_k"][s], inp["new_v"][s], inp["latent_q"][s], inp["q"][s],
                            pos[s], w.R, w.W, w.S, workspace=ws, out=O[s])
        sel_i[s].copy_(v_idx)
        sel_c[s].copy_(v_cnt)

    # the oracle: each sequence's index, appended step by step, and every
    # step's selection and output
    o_sel = np.empty((steps, w.B, w.s_max), np.int32)
    o_cnt = np.empty((steps, w.B), np.int32)
    O_ref = np.empty((steps, w.B, w.Hq, w.d), np.float64)
    orcs = []
    for b in range(w.B):
        lat = inp["latent_K"][b, :w.T + steps].float().cpu().numpy()
        o = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=True)
        o.extend(lat, 0, w.T)
        for s in range(steps):
            o.append(lat, w.T + s + 1)
            si, sc, _, _ = oracle.select(o, inp["latent_q"][s][b:b + 1].float().cpu().numpy(),
                                         np.array([w.T + s]), w.R, w.W, w.S)
            o_sel[s, b], o_cnt[s, b] = si[0], sc[0]
        orcs.append(o)
        q_b = inp["q"][:, b].float().cpu().numpy()                 # [steps][Hq][d]
        O_ref[:, b] = _gather_attend(q_b, inp["K"][b], inp["V"][b], o_sel[:, b], o_cnt[:, b], w.d)

    def check_pass(what):
        torch.cuda.synchronize()
        assert idx.check() >= 0, what
        gi, gc = sel_i.cpu().numpy(), sel_c.cpu().numpy()
        assert np.array_equal(gc, o_cnt), what
        assert np.array_equal(gi, o_sel), what
        err = np.abs(O.float().cpu().numpy().astype(np.float64) - O_ref)
        assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (what, err.max(), err.mean())

    for s in range(steps):                      # eager pass (the bench's warm-up)
        step(s)
    check_pass("eager")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for s in range(steps):
            step(s)
    for rep in range(2):                        # the state the benchmark times: replays
        O.fill_(float("nan"))
        sel_i.fill_(-7)
        sel_c.fill_(-7)
        graph.replay()
        check_pass("replay %d" % rep)
    del graph
    ex = idx.export()
    torch.cuda.synchronize()
    for b in range(w.B):
        assert np.array_equal(ex["open_bucket"][b].cpu().numpy(), orcs[b].open_bucket)
