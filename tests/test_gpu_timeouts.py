"""Failure detection without a fault: every kernel that waits gives up cleanly.

With the wait limit at 0 polls (lsa_set_wait_limit, a test hook) every
bounded wait of the library's kernels gives up at once.  The kernel records
LSA_ERR_TIMEOUT in the index status word, waits for its own copies and MMAs
in flight with the default limit, frees its tensor memory and leaves; no
kernel traps, faults or spins.  The context stays usable: with the default
limit back, the same call on the same workspace matches the oracle.

Cases: the tensor-core attention tiles of a bf16 prefill chunk (and their
MMA issuer's no-progress counter), the per-query attention of prefill rows
that find no partial slot, and the split-KV attention of a decode step.
(The tensor-core scorer's case is in test_gpu_bucket_attn.py.)
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")

BF16_MAX, BF16_MEAN = 2e-2, 2e-3


def _chunk_setup(seed, **kw):
    args = dict(T=2760, nq=700, B=1, Hq=8, Hkv=2, d=64, M=48, p=4, G=64, k=4, L=3, R=384, W=48,
                S=4, dtype="bf16")
    args.update(kw)
    w = synth.workload("tiny", **args)
    inp = synth.prefill_inputs(w, seed, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(dev["latent_K"], w.T - w.nq)
    return w, inp, dev, gpu


def _oracle_chunk(w, inp):
    T_old = w.T - w.nq
    lat = inp["latent_K"][0].float().numpy()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    orc.extend(lat, 0, T_old)
    orc.extend(lat, T_old, w.T)
    o_idx, o_cnt, _, _ = oracle.select(orc, inp["latent_Q"][0].float().numpy(),
                                       inp["positions"][0].numpy(), w.R, w.W, w.S)
    O_ref, _ = oracle.attend(inp["Q"][0].float().numpy(), inp["K"][0].float().numpy(),
                             inp["V"][0].float().numpy(), o_idx, o_cnt,
                             oracle.default_scale(w.d))
    return o_idx, o_cnt, O_ref


def _bf16_close(O, O_ref):
    err = np.abs(O.float().cpu().numpy().astype(np.float64) - O_ref)
    assert err.max() <= BF16_MAX and err.mean() <= BF16_MEAN, (err.max(), err.mean())


def _attend_times_out_then_recovers(w, inp, dev, gpu, ws):
    T_old = w.T - w.nq
    lsa.lsa_prefill_select(gpu, dev["latent_K"], dev["latent_Q"], T_old, w.T, w.Hq, w.Hkv, w.d,
                           w.R, w.W, w.S, ws)
    torch.cuda.synchronize()
    assert gpu.check() == 0
    lsa.set_wait_limit(0)
    try:
        lsa.lsa_prefill_attend(gpu, dev["Q"], dev["K"], dev["V"], T_old, w.T, w.R, w.W, w.S, ws)
        torch.cuda.synchronize()
        with pytest.raises(lsa.LsaError, match="TIMEOUT"):
            gpu.check()
    finally:
        lsa.set_wait_limit(-1)
    gpu.check()                                  # the report cleared the status word
    # the same attention stage again, on the same workspace, with the default limit
    O = lsa.lsa_prefill_attend(gpu, dev["Q"], dev["K"], dev["V"], T_old, w.T, w.R, w.W, w.S, ws)
    torch.cuda.synchronize()
    assert gpu.check() == 0
    o_idx, o_cnt, O_ref = _oracle_chunk(w, inp)
    g_idx, g_cnt = lsa.prefill_selection_views(ws, 1, w.nq, w.s_max)
    assert np.array_equal(g_idx[0].cpu().numpy(), o_idx)
    assert np.array_equal(g_cnt[0].cpu().numpy(), o_cnt)
    _bf16_close(O[0], O_ref)


def test_attention_tiles_wait_that_runs_out_reports_a_timeout():
    w, inp, dev, gpu = _chunk_setup(31)
    nb = lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    assert lsa.lsa_prefill_partial_slots(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S, nb) > 0
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    _attend_times_out_then_recovers(w, inp, dev, gpu, ws)


def test_per_query_rows_wait_that_runs_out_reports_a_timeout():
    # The smallest workspace gives no partial slot: every row of the chunk is
    # attended key by key by the per-query kernel (row-list mode).
    w, inp, dev, gpu = _chunk_setup(32)
    full = lsa.lsa_prefill_workspace_bytes(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    slots = lambda n: lsa.lsa_prefill_partial_slots(gpu, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S, n)
    lo, hi = 0, full
    while lo < hi:                               # the minimum workspace
        mid = (lo + hi) // 2
        if slots(mid) >= 0:
            hi = mid
        else:
            lo = mid + 1
    assert slots(hi) == 0
    ws = torch.empty(hi, dtype=torch.uint8, device="cuda")
    _attend_times_out_then_recovers(w, inp, dev, gpu, ws)


def test_decode_split_attention_wait_that_runs_out_reports_a_timeout():
    w = synth.workload("decode", T=4096, B=3, M=64, G=64, k=4, L=3, R=600, W=64, S=4, steps=4,
                       Hq=32, Hkv=4, d=128)
    span = w.p * w.G
    t_cap = w.T + span
    inp = synth.decode_inputs(w, 17, "cuda", t_cap=t_cap)
    gpu = lsa.LsaIndex(w.B, t_cap, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(inp["latent_K"], w.T)
    ws = torch.empty(lsa.lsa_decode_workspace_bytes(gpu, w.Hq, w.Hkv, w.d, w.R, w.W, w.S),
                     dtype=torch.uint8, device="cuda")
    pos = torch.full((w.B,), w.T, dtype=torch.int32, device="cuda")

    def step():
        return lsa.lsa_decode_step(gpu, inp["latent_K"], inp["K"], inp["V"],
                                   inp["new_latent_k"][0], inp["new_k"][0], inp["new_v"][0],
                                   inp["latent_q"][0], inp["q"][0], pos, w.R, w.W, w.S,
                                   workspace=ws)

    lsa.set_wait_limit(0)
    try:
        step()
        torch.cuda.synchronize()
        with pytest.raises(lsa.LsaError, match="TIMEOUT"):
            gpu.check()
    finally:
        lsa.set_wait_limit(-1)
    gpu.check()
    O = step()                                   # the same step again: it rewrites the same rows
    torch.cuda.synchronize()
    assert gpu.check() == 0
    g_idx, g_cnt = lsa.decode_selection_views(ws, w.B, w.s_max)
    for b in range(w.B):
        orc = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=True)
        lat = inp["latent_K"][b].float().cpu().numpy()
        orc.extend(lat, 0, w.T)
        orc.append(lat, w.T + 1)
        o_idx, o_cnt, _, _ = oracle.select(orc, inp["latent_q"][0][b:b + 1].float().cpu().numpy(),
                                           np.array([w.T]), w.R, w.W, w.S)
        assert int(g_cnt[b]) == o_cnt[0]
        assert np.array_equal(g_idx[b].cpu().numpy(), o_idx[0])
        O_ref, _ = oracle.attend(inp["q"][0][b:b + 1].float().cpu().numpy(),
                                 inp["K"][b].float().cpu().numpy(),
                                 inp["V"][b].float().cpu().numpy(), o_idx, o_cnt,
                                 oracle.default_scale(w.d))
        _bf16_close(O[b], O_ref[0])
