"""Parity at the full workload sizes, in the launch configuration bench.py times.

The whole 1M and 10M prefill chunks (32768 queries each) run through
lsa_prefill_chunk exactly as the benchmark calls it; the oracle then checks a
sample of the chunk's queries one by one: the index blocks the chunk rebuilt
(bit for bit), every sampled query's selection (row for row) and its outputs
(bf16 tolerance).  The decode test replays the benchmark's 8 x 1M decode for a
few steps and checks every sequence's selection and output each step.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

lsa = pytest.importorskip("long_context_indexing_b200")

BF16_MAX, BF16_MEAN = 2e-2, 2e-3


def _gather_attend(Q_rows, K, V, sel, cnt, d):
    """Oracle attention for sampled rows, with K/V rows gathered on the device
    (host copies of only the rows the sample reads)."""
    uniq, inv = np.unique(np.where(sel >= 0, sel, 0), return_inverse=True)
    remap = np.where(sel >= 0, inv.reshape(sel.shape), -1).astype(np.int32)
    ui = torch.from_numpy(uniq).to(K.device)
    Kh = K.index_select(0, ui).float().cpu().numpy()
    Vh = V.index_select(0, ui).float().cpu().numpy()
    return oracle.attend(Q_rows, Kh, Vh, remap, cnt, oracle.default_scale(d))[0]


@pytest.mark.parametrize("name", ["1m", "10m"])
def test_full_size_prefill_chunk_sampled(name):
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
    assert idx.check() >= 0
    g_idx, g_cnt = lsa.prefill_selection_views(ws, 1, w.nq, w.s_max)

    lat = inp["latent_K"][0].float().cpu().numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    orc.extend(lat, 0, w.T)
    # the chunk's blocks (and the first prefix block) bit for bit
    ex = idx.export()
    for b in (0, w.T // span - 8, w.T // span - 1):
        sl = slice(b * w.k, (b + 1) * w.k)
        assert np.array_equal(ex["cent"][0][sl].cpu().numpy(), orc.cent[sl])
        assert np.array_equal(ex["offsets"][0][sl].cpu().numpy(), orc.offsets[sl])
        ms = slice(b * w.G, (b + 1) * w.G)
        assert np.array_equal(ex["members"][0][ms].cpu().numpy(), orc.members[ms])
        assert np.array_equal(ex["assign"][0][ms].cpu().numpy(), orc.assign[ms])
    del ex

    rng = np.random.default_rng(0)
    rows = np.concatenate([[0, 1, 127, 128, w.nq - 1], rng.choice(w.nq, 59, replace=False)])
    o_idx, o_cnt, _, _ = oracle.select(orc, inp["latent_Q"][0][rows].float().cpu().numpy(),
                                       T_old + rows, w.R, w.W, w.S)
    gi = g_idx[0][torch.from_numpy(rows).cuda()].cpu().numpy()
    gc = g_cnt[0][torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.array_equal(gc, o_cnt)
    assert np.array_equal(gi, o_idx)
    O_ref = _gather_attend(inp["Q"][0][rows].float().cpu().numpy(), inp["K"][0], inp["V"][0],
                           o_idx, o_cnt, w.d)
    err = np.abs(O[0][torch.from_numpy(rows).cuda()].float().cpu().numpy() - O_ref)
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (err.max(), err.mean())


def test_full_size_decode_sampled():
    w = synth.workload("decode")
    span = w.p * w.G
    t_cap = w.T + span
    inp = synth.decode_inputs(w, seed=0, device="cuda", t_cap=t_cap)
    idx = lsa.LsaIndex(w.B, t_cap, w.p, w.G, w.k, w.L, lsa.BF16)
    idx.build(inp["latent_K"], w.T)
    ws = torch.empty(lsa.lsa_decode_workspace_bytes(idx, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    orcs = []
    for b in range(w.B):
        o = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=True)
        o.extend(inp["latent_K"][b].float().cpu().numpy(), 0, w.T)
        orcs.append(o)
    lat_host = [inp["latent_K"][b, :w.T + w.steps].float().cpu().numpy() for b in range(w.B)]
    for s in range(6):                                   # crosses a group completion
        pos = torch.full((w.B,), w.T + s, dtype=torch.int32, device="cuda")
        O = lsa.lsa_decode_step(idx, inp["latent_K"], inp["K"], inp["V"], inp["new_latent_k"][s],
                                inp["new_k"][s], inp["new_v"][s], inp["latent_q"][s],
                                inp["q"][s], pos, w.R, w.W, w.S, workspace=ws)
        g_idx, g_cnt = lsa.decode_selection_views(ws, w.B, w.s_max)
        torch.cuda.synchronize()
        for b in range(w.B):
            orcs[b].append(lat_host[b], w.T + s + 1)
            lq = inp["latent_q"][s][b:b + 1].float().cpu().numpy()
            o_idx, o_cnt, _, _ = oracle.select(orcs[b], lq, np.array([w.T + s]), w.R, w.W, w.S)
            assert int(g_cnt[b]) == o_cnt[0]
            assert np.array_equal(g_idx[b].cpu().numpy(), o_idx[0])
            O_ref = _gather_attend(inp["q"][s][b:b + 1].float().cpu().numpy(), inp["K"][b],
                                   inp["V"][b], o_idx, o_cnt, w.d)
            err = np.abs(O[b].float().cpu().numpy() - O_ref[0])
            assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN
    assert idx.check() >= 0
    ex = idx.export()
    for b in range(w.B):
        assert np.array_equal(ex["open_bucket"][b].cpu().numpy(), orcs[b].open_bucket)
