"""GPU parity of the fused decode step against the oracle, step by step.

Each step appends one token per sequence at its own position; a short window
(W = 8) makes the open-block members selectable, so the decode-time index
maintenance is exercised through the selections, not only through the
exported state."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


def _np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


@pytest.mark.parametrize("dtype,Hq,Hkv,d", [("bf16", 32, 4, 128), ("bf16", 8, 2, 64),
                                            ("f32", 4, 1, 64)])
def test_decode_steps_match_oracle(dtype, Hq, Hkv, d):
    w = synth.workload("decode", T=4096, B=3, M=64, G=64, k=4, L=3, R=600, W=8, S=4, steps=48,
                       Hq=Hq, Hkv=Hkv, d=d, dtype=dtype)
    inp = synth.decode_inputs(w, 11, "cpu")
    span = w.p * w.G
    t_cap = w.T + w.steps + 8 + span
    tdt = w.torch_dtype
    # caches hold the prefix only; the decode steps write the new rows
    lat = torch.zeros(w.B, t_cap, 64, dtype=tdt)
    Kc = torch.zeros(w.B, t_cap, w.Hkv, w.d, dtype=tdt)
    Vc = torch.zeros(w.B, t_cap, w.Hkv, w.d, dtype=tdt)
    for b in range(w.B):
        # sequence b starts decoding at T + (B-1-b): its rows before that exist
        t0 = w.T + (w.B - 1 - b)
        lat[b, :t0] = inp["latent_K"][b, :t0]
        Kc[b, :t0] = inp["K"][b, :t0]
        Vc[b, :t0] = inp["V"][b, :t0]
    full_lat = torch.zeros(w.B, t_cap, 64, dtype=tdt)
    full_lat[:, :w.T + w.steps] = inp["latent_K"]
    full_K = torch.zeros_like(Kc)
    full_V = torch.zeros_like(Vc)
    full_K[:, :w.T + w.steps] = inp["K"]
    full_V[:, :w.T + w.steps] = inp["V"]

    dev = dict(lat=lat.cuda(), K=Kc.cuda(), V=Vc.cuda())
    gidx = lsa.LsaIndex(w.B, t_cap, w.p, w.G, w.k, w.L, lsa.BF16 if dtype == "bf16" else lsa.F32)
    gidx.build(dev["lat"], w.T)
    orcs = []
    for b in range(w.B):
        o = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=(dtype == "bf16"))
        o.extend(full_lat[b].float().numpy(), 0, w.T)
        orcs.append(o)
    ws = torch.empty(lsa.lsa_decode_workspace_bytes(gidx, Hq, Hkv, d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    used_open = 0
    # sequence b runs `b` tokens behind sequence 0 (per-sequence positions)
    for s in range(w.steps - w.B):
        pos = np.array([w.T + s + (w.B - 1 - b) for b in range(w.B)], np.int64)
        src = pos - w.T
        new_lat = torch.stack([inp["new_latent_k"][src[b], b] for b in range(w.B)]).cuda()
        new_k = torch.stack([inp["new_k"][src[b], b] for b in range(w.B)]).cuda()
        new_v = torch.stack([inp["new_v"][src[b], b] for b in range(w.B)]).cuda()
        lq = torch.stack([inp["latent_q"][src[b], b] for b in range(w.B)])
        q = torch.stack([inp["q"][src[b], b] for b in range(w.B)])
        O = lsa.lsa_decode_step(gidx, dev["lat"], dev["K"], dev["V"], new_lat, new_k, new_v,
                                lq.cuda(), q.cuda(), torch.from_numpy(pos.astype(np.int32)).cuda(),
                                w.R, w.W, w.S, workspace=ws)
        g_idx, g_cnt = lsa.decode_selection_views(ws, w.B, w.s_max)
        torch.cuda.synchronize()
        for b in range(w.B):
            orcs[b].append(full_lat[b].float().numpy(), int(pos[b]) + 1)
            o_idx, o_cnt, _, _ = oracle.select(orcs[b], lq[b:b + 1].float().numpy(),
                                               pos[b:b + 1], w.R, w.W, w.S)
            assert int(g_cnt[b]) == o_cnt[0]
            assert np.array_equal(_np(g_idx[b]), o_idx[0]), (s, b)
            used_open += int(np.sum(o_idx[0, w.S:o_cnt[0] - w.W] >= w.T))
            O_ref, _ = oracle.attend(q[b:b + 1].float().numpy(), full_K[b].float().numpy(),
                                     full_V[b].float().numpy(), o_idx, o_cnt,
                                     oracle.default_scale(d))
            err = np.abs(_np(O[b]) - O_ref[0])
            if dtype == "f32":
                assert err.max() <= 1e-4
            else:
                assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert gidx.check() >= 0
    ex = gidx.export()
    for b in range(w.B):
        assert np.array_equal(_np(ex["open_bucket"][b]), orcs[b].open_bucket)
        # rows of every group pooled so far (later rows were never written)
        n_pooled = (w.T + w.steps - w.B + (w.B - 1 - b)) // w.p
        assert np.array_equal(_np(ex["unit"][b])[:n_pooled], orcs[b].unit[:n_pooled])
        assert np.array_equal(_np(ex["pooled"][b])[:n_pooled], orcs[b].pooled[:n_pooled])
    # the caches now hold the appended rows
    last = w.T + w.steps - w.B
    assert torch.equal(dev["K"][:, w.T:last].cpu(), full_K[:, w.T:last])
    assert used_open > 0


def test_decode_reports_full_open_block():
    w = synth.workload("decode", T=1024, B=1, M=16, G=16, k=4, R=64, W=8, S=4, steps=4, Hq=4,
                       Hkv=1, d=64, dtype="f32")
    span = w.p * w.G                       # 64 keys per block
    t_cap = 4 * span
    g = torch.Generator().manual_seed(0)
    lat = torch.randn(1, t_cap, 64, generator=g).cuda()
    Kc = torch.randn(1, t_cap, 1, 64, generator=g).cuda()
    Vc = torch.randn(1, t_cap, 1, 64, generator=g).cuda()
    idx = lsa.LsaIndex(1, t_cap, w.p, w.G, w.k, w.L, lsa.F32)
    idx.build(lat, 2 * span)
    args = (lat[:, 0].contiguous(), Kc[:, 0].contiguous(), Vc[:, 0].contiguous(),
            lat[:, 0].contiguous(), torch.randn(1, 4, 64, generator=g).cuda())
    # a position inside the open block is fine ...
    lsa.lsa_decode_step(idx, lat, Kc, Vc, *args, torch.tensor([2 * span + 3], dtype=torch.int32,
                                                              device="cuda"), w.R, w.W, w.S)
    assert idx.check() >= 0
    # ... a group beyond it is reported, not appended
    lsa.lsa_decode_step(idx, lat, Kc, Vc, *args, torch.tensor([3 * span + 3], dtype=torch.int32,
                                                              device="cuda"), w.R, w.W, w.S)
    with pytest.raises(lsa.LsaError) as e:
        idx.check()
    assert e.value.code == 6


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_past_block_ends_with_extend(dtype):
    # The index lifecycle beyond one open block: decode appends fill the open
    # block; when its last key is written the caller closes it with
    # lsa_index_extend over that block (k-means into buckets, open list
    # cleared), and decoding continues into the next block.  The oracle does
    # the same, and every step's selection, output and the final index agree.
    w = synth.workload("decode", T=1024, B=2, M=16, G=16, k=4, L=3, R=200, W=8, S=4, steps=150,
                       Hq=8, Hkv=2, d=64, dtype=dtype)
    inp = synth.decode_inputs(w, 12, "cpu")
    span = w.p * w.G                       # 64 keys per block
    t_cap = w.T + w.steps + 2 + span       # a whole number of groups, room for an open block
    tdt = w.torch_dtype
    lat = torch.zeros(w.B, t_cap, 64, dtype=tdt)
    Kc = torch.zeros(w.B, t_cap, w.Hkv, w.d, dtype=tdt)
    Vc = torch.zeros(w.B, t_cap, w.Hkv, w.d, dtype=tdt)
    lat[:, :w.T] = inp["latent_K"][:, :w.T]
    Kc[:, :w.T] = inp["K"][:, :w.T]
    Vc[:, :w.T] = inp["V"][:, :w.T]
    full_lat = torch.zeros(w.B, t_cap, 64, dtype=tdt)
    full_lat[:, :w.T + w.steps] = inp["latent_K"]
    full_K = torch.zeros_like(Kc)
    full_V = torch.zeros_like(Vc)
    full_K[:, :w.T + w.steps] = inp["K"]
    full_V[:, :w.T + w.steps] = inp["V"]
    dev = dict(lat=lat.cuda(), K=Kc.cuda(), V=Vc.cuda())
    gidx = lsa.LsaIndex(w.B, t_cap, w.p, w.G, w.k, w.L, lsa.BF16 if dtype == "bf16" else lsa.F32)
    gidx.build(dev["lat"], w.T)
    orcs = []
    for b in range(w.B):
        o = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=(dtype == "bf16"))
        o.extend(full_lat[b].float().numpy(), 0, w.T)
        orcs.append(o)
    ws = torch.empty(lsa.lsa_decode_workspace_bytes(gidx, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    closed = 0
    for s in range(w.steps):
        pos = w.T + s
        new_lat = inp["new_latent_k"][s].cuda()
        new_k = inp["new_k"][s].cuda()
        new_v = inp["new_v"][s].cuda()
        lq, q = inp["latent_q"][s], inp["q"][s]
        pos_t = torch.full((w.B,), pos, dtype=torch.int32, device="cuda")
        O = lsa.lsa_decode_step(gidx, dev["lat"], dev["K"], dev["V"], new_lat, new_k, new_v,
                                lq.cuda(), q.cuda(), pos_t, w.R, w.W, w.S, workspace=ws)
        g_idx, g_cnt = lsa.decode_selection_views(ws, w.B, w.s_max)
        torch.cuda.synchronize()
        for b in range(w.B):
            orcs[b].append(full_lat[b].float().numpy(), pos + 1)
            o_idx, o_cnt, _, _ = oracle.select(orcs[b], lq[b:b + 1].float().numpy(),
                                               np.array([pos]), w.R, w.W, w.S)
            assert int(g_cnt[b]) == o_cnt[0], (s, b)
            assert np.array_equal(_np(g_idx[b]), o_idx[0]), (s, b)
            O_ref, _ = oracle.attend(q[b:b + 1].float().numpy(), full_K[b].float().numpy(),
                                     full_V[b].float().numpy(), o_idx, o_cnt,
                                     oracle.default_scale(w.d))
            err = np.abs(_np(O[b]) - O_ref[0])
            if dtype == "f32":
                assert err.max() <= 1e-4
            else:
                assert err.max() <= 2e-2 and err.mean() <= 2e-3
        if (pos + 1) % span == 0:         # the open block is full: close it
            gidx.extend(dev["lat"], pos + 1 - span, pos + 1)
            for b in range(w.B):
                orcs[b].extend(full_lat[b].float().numpy(), pos + 1 - span, pos + 1)
            closed += 1
    assert closed == 2 and gidx.check() >= 0
    assert gidx.num_blocks == w.T // span + closed
    ex = gidx.export()
    nb = (w.T // span + closed) * w.k
    for b in range(w.B):
        assert np.array_equal(_np(ex["offsets"][b])[:nb + 1], orcs[b].offsets[:nb + 1])
        assert np.array_equal(_np(ex["members"][b])[:nb // w.k * w.G],
                              orcs[b].members[:nb // w.k * w.G])
        assert np.array_equal(_np(ex["cent"][b])[:nb], orcs[b].cent[:nb])
        assert np.array_equal(_np(ex["open_bucket"][b]), orcs[b].open_bucket)
