"""bf16 prefill chunks (bucket-major attention) against the oracle, whole chunk.

Each case runs lsa_prefill_chunk on a small bf16 workload and checks, for every
query of the chunk, the selection (row for row) and the output against
oracle.attend on the oracle's selection (bf16 bars: 2e-2 max-abs, 2e-3
mean-abs).  Cases: a chunk that ends inside a block (open-block members are
taken), a chunk that starts at position 0 (sinks and window overlap, block-0
buckets cut by the sinks bound), several sequences, every supported head
shape, pooling factors 2 and 8, workspaces with too few partial slots (some
or all rows then go through the per-query kernel), and exact-fallback rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")

BF16_MAX, BF16_MEAN = 2e-2, 2e-3


def _base(**kw):
    # 256-token blocks of 4 buckets (64 keys each); a budget of ~6 buckets
    args = dict(T=2760, nq=700, B=1, Hq=8, Hkv=2, d=64, M=48, p=4, G=64, k=4, L=3, R=384, W=48,
                S=4, dtype="bf16")
    args.update(kw)
    return synth.workload("tiny", **args)


def _run(w, seed=0, ws_bytes=None, same_latent=False, check_repeat=False):
    T_old = w.T - w.nq
    inp = synth.prefill_inputs(w, seed, "cpu")
    if same_latent:   # every approximate score ties: rows go to the exact fallback
        inp["latent_K"][:] = inp["latent_K"][:, :1]
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(dev["latent_K"], T_old)
    if ws_bytes is None:
        ws_bytes = lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    O = lsa.lsa_prefill_chunk(gpu, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"], dev["V"],
                              T_old, w.T, w.R, w.W, w.S, workspace=ws)
    torch.cuda.synchronize()
    fallbacks = gpu.check()
    g_idx, g_cnt = lsa.prefill_selection_views(ws, w.B, w.nq, w.s_max)
    g_idx, g_cnt = g_idx.cpu().numpy(), g_cnt.cpu().numpy()
    g_open = gpu.export()["open_bucket"].cpu().numpy()
    errs = []
    for b in range(w.B):
        lat = inp["latent_K"][b].float().numpy()
        orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
        orc.extend(lat, 0, T_old)
        orc.extend(lat, T_old, w.T)
        assert np.array_equal(g_open[b], orc.open_bucket)
        pos = inp["positions"][b].numpy()
        o_idx, o_cnt, _, _ = oracle.select(orc, inp["latent_Q"][b].float().numpy(), pos, w.R, w.W,
                                           w.S)
        assert np.array_equal(g_cnt[b], o_cnt)
        assert np.array_equal(g_idx[b], o_idx)
        O_ref, _ = oracle.attend(inp["Q"][b].float().numpy(), inp["K"][b].float().numpy(),
                                 inp["V"][b].float().numpy(), o_idx, o_cnt,
                                 oracle.default_scale(w.d))
        err = np.abs(O[b].float().cpu().numpy().astype(np.float64) - O_ref)
        assert err.max() <= BF16_MAX, (b, err.max())
        assert err.mean() <= BF16_MEAN, (b, err.mean())
        errs.append(err.max())
    if check_repeat:
        O2 = lsa.lsa_prefill_chunk(gpu, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"],
                                   dev["V"], T_old, w.T, w.R, w.W, w.S, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(O, O2)
    return fallbacks, max(errs)


def _ws_for_slots(w, want):
    """Smallest workspace giving at least `want` partial slots (binary search)."""
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    hi = lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    slots = lambda n: lsa.lsa_prefill_partial_slots(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S, n)
    assert slots(hi) >= want
    lo = 0
    while lo < hi:
        mid = (lo + hi) // 2
        if slots(mid) >= want:
            hi = mid
        else:
            lo = mid + 1
    return hi


def test_chunk_ending_inside_a_block():
    w = _base()
    span = w.p * w.G
    # the last queries' long-range keys reach into the open block
    assert w.T - 1 - w.W >= (w.T // span) * span + 64
    fb, _ = _run(w, seed=11, check_repeat=True)
    assert fb == 0


def test_chunk_from_position_zero():
    w = _base(T=2048, nq=2048, R=200, W=24, S=6)
    _run(w, seed=12)


def test_several_sequences():
    w = _base(T=4096, nq=512, B=3, R=512)
    _run(w, seed=13)


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 8, 64), (8, 4, 128), (16, 4, 64), (32, 4, 128),
                                      (8, 1, 128), (4, 2, 64)])
def test_head_shapes(Hq, Hkv, d):
    w = _base(T=3000, nq=400, Hq=Hq, Hkv=Hkv, d=d)
    _run(w, seed=14)


@pytest.mark.parametrize("p,G", [(2, 128), (8, 32)])
def test_pooling_factors(p, G):
    # other group sizes: p-row K/V boxes, and window groups that straddle the
    # sinks' end (S = 5 is no multiple of p)
    w = _base(T=3000, nq=500, p=p, G=G, S=5)
    _run(w, seed=20 + p)


def test_large_buckets_span_several_stages():
    # 2 buckets of 1024-token blocks: ~512 keys per bucket, 8 pipeline stages
    w = _base(T=6000, nq=600, G=256, k=2, R=1500, W=100)
    _run(w, seed=15)


def test_few_partial_slots():
    w = _base()
    ws = _ws_for_slots(w, w.nq * 2)     # room for a fraction of the rows
    _run(w, seed=16, ws_bytes=ws)


def test_no_partial_slots():
    w = _base()
    ws = _ws_for_slots(w, 0)            # minimum workspace: every row key by key
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    assert lsa.lsa_prefill_partial_slots(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S, ws) == 0
    assert lsa.lsa_prefill_partial_slots(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S, ws - 1) == -1
    _run(w, seed=17, ws_bytes=ws)


def test_workspace_below_minimum_is_refused():
    w = _base()
    ws = _ws_for_slots(w, 0) - 256
    with pytest.raises(lsa.LsaError):
        _run(w, seed=17, ws_bytes=ws)


def test_fallback_rows():
    w = _base(T=2048, nq=512, G=8, R=300)       # 256 buckets, all tied: more than the fill ranks
    fb, _ = _run(w, seed=18, same_latent=True)
    assert fb > 0


def test_blocks_too_large_for_the_tensor_core_tiles():
    # 2560 pooled groups per block: the member lists do not fit the
    # tensor-core kernel's shared memory, so the warp-MMA tile kernel runs
    w = _base(T=23000, nq=600, p=1, G=2560, k=8, R=1200, W=40)
    _run(w, seed=19)


def test_recommended_workspace_gives_the_recommended_slots():
    # 1.5 x (budget / mean bucket keys) + 2 slots per query row, capped at 65
    w = _base()
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    nbytes = lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    bk = w.p * w.G // w.k
    per_row = min(65, (3 * w.R + 2 * bk - 1) // (2 * bk) + 2)
    assert lsa.lsa_prefill_partial_slots(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S,
                                         nbytes) == w.B * w.nq * per_row


@pytest.mark.parametrize("dtype,B", [("bf16", 1), ("bf16", 2), ("f32", 2)])
def test_host_entry_matches_device_entry(dtype, B):
    # lsa_prefill_chunk_host copies the chunk's rows and queries in (K, V, Q on
    # a second stream, under the selection), runs the chunk and copies O out:
    # the same output as lsa_prefill_chunk on device inputs, bit for bit
    w = _base(B=B, dtype=dtype)
    T_old = w.T - w.nq
    inp = synth.prefill_inputs(w, 22, "cpu")
    lt = lsa.BF16 if dtype == "bf16" else lsa.F32

    def fresh_index(latent_K):
        idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lt)
        idx.build(latent_K, T_old)
        nb = lsa.lsa_prefill_workspace_bytes(idx, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
        return idx, torch.empty(nb, dtype=torch.uint8, device="cuda")

    dev = {k: v.cuda() for k, v in inp.items()}
    idx, ws = fresh_index(dev["latent_K"])
    O_dev = lsa.lsa_prefill_chunk(idx, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"],
                                  dev["V"], T_old, w.T, w.R, w.W, w.S, workspace=ws)
    torch.cuda.synchronize()

    # device caches hold only the prefix; the chunk's rows and queries come from host
    dev2 = {k: v.cuda() for k, v in inp.items()}
    for k in ("latent_K", "K", "V"):
        dev2[k][:, T_old:w.T] = 0
    dev2["latent_Q"].zero_()
    dev2["Q"].zero_()
    h = {k: inp[k][:, T_old:w.T].contiguous().pin_memory() for k in ("latent_K", "K", "V")}
    hq = {k: inp[k].contiguous().pin_memory() for k in ("latent_Q", "Q")}
    idx2, ws2 = fresh_index(dev2["latent_K"])
    O2 = torch.empty_like(dev2["Q"])
    hO = torch.empty(O2.shape, dtype=O2.dtype, pin_memory=True)
    lsa.lsa_prefill_chunk_host(idx2, h["latent_K"], h["K"], h["V"], hq["latent_Q"], hq["Q"],
                               dev2["latent_K"], dev2["K"], dev2["V"], dev2["latent_Q"], dev2["Q"],
                               T_old, w.T, w.R, w.W, w.S, ws2, O2, hO)
    torch.cuda.synchronize()
    assert idx2.check() == idx.check()
    assert torch.equal(hO, O_dev.cpu())
    assert torch.equal(dev2["K"], dev["K"]) and torch.equal(dev2["V"], dev["V"])
    assert torch.equal(dev2["latent_K"], dev["latent_K"])


def test_host_entry_rejects_one_stream():
    w = _base()
    T_old = w.T - w.nq
    inp = synth.prefill_inputs(w, 23, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    idx.build(dev["latent_K"], T_old)
    nb = lsa.lsa_prefill_workspace_bytes(idx, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    h = {k: inp[k][:, T_old:w.T].contiguous().pin_memory() for k in ("latent_K", "K", "V")}
    hq = {k: inp[k].contiguous().pin_memory() for k in ("latent_Q", "Q")}
    O = torch.empty_like(dev["Q"])
    hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    s = torch.cuda.current_stream()
    with pytest.raises(lsa.LsaError):
        lsa.lsa_prefill_chunk_host(idx, h["latent_K"], h["K"], h["V"], hq["latent_Q"], hq["Q"],
                                   dev["latent_K"], dev["K"], dev["V"], dev["latent_Q"], dev["Q"],
                                   T_old, w.T, w.R, w.W, w.S, ws, O, hO, stream=s, copy_stream=s)


def test_scorer_wait_that_runs_out_reports_a_timeout():
    # Failure detection without a fault: with the scorer's wait limit at 0
    # polls every one of its waits gives up at once; the kernel records
    # LSA_ERR_TIMEOUT, drains its copies and MMAs and leaves.  The context
    # stays usable: with the default limit back, a chunk matches the oracle.
    w = _base()
    T_old = w.T - w.nq
    inp = synth.prefill_inputs(w, 24, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(dev["latent_K"], T_old)
    nb = lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    lsa.set_wait_limit(0)
    try:
        lsa.lsa_prefill_select(gpu, dev["latent_K"], dev["latent_Q"], T_old, w.T, w.Hq, w.Hkv,
                               w.d, w.R, w.W, w.S, ws)
        torch.cuda.synchronize()
        with pytest.raises(lsa.LsaError, match="TIMEOUT"):
            gpu.check()
    finally:
        lsa.set_wait_limit(-1)
    gpu.check()                          # the status word was cleared by the report
    fb, _ = _run(w, seed=24)
    assert fb == 0


@pytest.mark.parametrize("cuts", [(0, 350, 700), (0, 128, 129, 700)])
def test_query_ranges_equal_the_whole_chunk(cuts):
    # A chunk that ends inside a block (open-block members are selectable),
    # split into query ranges with lsa_prefill_chunk_queries: every range
    # extends the index over the whole chunk; its rows' selections are the
    # whole chunk's bit for bit, and their outputs equal the whole chunk's up
    # to summation order (a sinks-and-window tile spans a run of consecutive
    # queries, so a cut through a run changes its stages): the bf16 bars.
    w = _base()
    T_old = w.T - w.nq
    inp = synth.prefill_inputs(w, 41, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(dev["latent_K"], T_old)
    ws = torch.empty(lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    O = lsa.lsa_prefill_chunk(gpu, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"], dev["V"],
                              T_old, w.T, w.R, w.W, w.S, workspace=ws)
    g_idx, g_cnt = lsa.prefill_selection_views(ws, w.B, w.nq, w.s_max)
    g_idx, g_cnt = g_idx.clone(), g_cnt.clone()
    parts_o, parts_i, parts_c = [], [], []
    for q0, q1 in zip(cuts[:-1], cuts[1:]):
        wsp = torch.empty(lsa.lsa_prefill_workspace_bytes(gpu, q1 - q0, w.Hq, w.Hkv, w.d, w.R,
                                                          w.W, w.S), dtype=torch.uint8,
                          device="cuda")
        Op = lsa.lsa_prefill_chunk_queries(gpu, dev["latent_K"],
                                           dev["latent_Q"][:, q0:q1].contiguous(),
                                           dev["Q"][:, q0:q1].contiguous(), dev["K"], dev["V"],
                                           T_old, w.T, q0, q1, w.R, w.W, w.S, workspace=wsp)
        pi, pc = lsa.prefill_selection_views(wsp, w.B, q1 - q0, w.s_max)
        parts_o.append(Op)
        parts_i.append(pi.clone())
        parts_c.append(pc.clone())
    torch.cuda.synchronize()
    assert gpu.check() >= 0
    assert torch.equal(torch.cat(parts_c, 1), g_cnt)
    assert torch.equal(torch.cat(parts_i, 1), g_idx)
    err = (torch.cat(parts_o, 1).float() - O.float()).abs()
    assert err.max().item() <= BF16_MAX and err.mean().item() <= BF16_MEAN
    with pytest.raises(lsa.LsaError):
        lsa.lsa_prefill_chunk_queries(gpu, dev["latent_K"], dev["latent_Q"][:, :10].contiguous(),
                                      dev["Q"][:, :10].contiguous(), dev["K"], dev["V"], T_old,
                                      w.T, w.nq - 5, w.nq + 5, w.R, w.W, w.S, workspace=ws)


def test_whole_context_chunk_by_chunk():
    # A whole context prefilled in chunks from position 0 (the index grows by
    # each chunk's blocks): every chunk's selections equal the oracle's, which
    # extends its index chunk by chunk in the same way, and the outputs are
    # within the bf16 bars.
    w = _base(T=4096, nq=4096, R=300, W=40, S=4)
    chunk = 512                                  # two blocks of 256 tokens
    inp = synth.prefill_inputs(w, 21, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(dev["latent_K"], 0)
    ws = torch.empty(lsa.lsa_prefill_workspace_bytes(gpu, chunk, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    lat = inp["latent_K"][0].float().numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    for t0 in range(0, w.T, chunk):
        t1 = t0 + chunk
        O = lsa.lsa_prefill_chunk(gpu, dev["latent_K"], dev["latent_Q"][:, t0:t1].contiguous(),
                                  dev["Q"][:, t0:t1].contiguous(), dev["K"], dev["V"], t0, t1,
                                  w.R, w.W, w.S, workspace=ws)
        torch.cuda.synchronize()
        assert gpu.check() == 0
        g_idx, g_cnt = lsa.prefill_selection_views(ws, 1, chunk, w.s_max)
        orc.extend(lat, t0, t1)
        pos = np.arange(t0, t1)
        o_idx, o_cnt, _, _ = oracle.select(orc, inp["latent_Q"][0, t0:t1].float().numpy(), pos,
                                           w.R, w.W, w.S)
        assert np.array_equal(g_cnt[0].cpu().numpy(), o_cnt), t0
        assert np.array_equal(g_idx[0].cpu().numpy(), o_idx), t0
        O_ref, _ = oracle.attend(inp["Q"][0, t0:t1].float().numpy(), inp["K"][0].float().numpy(),
                                 inp["V"][0].float().numpy(), o_idx, o_cnt,
                                 oracle.default_scale(w.d))
        err = np.abs(O[0].float().cpu().numpy().astype(np.float64) - O_ref)
        assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (t0, err.max(), err.mean())
