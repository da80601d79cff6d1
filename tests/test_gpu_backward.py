"""Gradients of the sparse attention on the GPU against the oracle.

lsa_sparse_attn_backward (given the forward's O and lse from lsa_sparse_attn
and an upstream gradient) against oracle.attend_backward on the same inputs:
fp32 within 1e-4 of the gradients' scale, bf16 within the bf16 bars measured
against the gradients' scale (the forward's bf16 O enters D = <dO, O>, and dQ
is rounded to bf16).  Keys read by several queries accumulate their dK, dV
over every reader; a second call adds to the same accumulators.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


def _inputs(seed, nq, T, Hq, Hkv, d, s_max, dtype):
    rng = np.random.default_rng(seed)
    Q = (0.5 * rng.standard_normal((1, nq, Hq, d))).astype(np.float32)
    K = rng.standard_normal((1, T, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((1, T, Hkv, d)).astype(np.float32)
    dO = rng.standard_normal((1, nq, Hq, d)).astype(np.float32)
    idx = np.full((1, nq, s_max), -1, np.int32)
    cnt = rng.integers(1, s_max + 1, (1, nq)).astype(np.int32)
    hot = rng.choice(T, 16, replace=False)           # keys many queries read
    for i in range(nq):
        c = cnt[0, i]
        pick = np.unique(np.concatenate([hot[:min(c, 8)], rng.choice(T, c, replace=False)]))[:c]
        cnt[0, i] = len(pick)
        idx[0, i, :len(pick)] = rng.permutation(pick)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = {k: torch.from_numpy(v).to(tdt).cuda() for k, v in
           dict(Q=Q, K=K, V=V, dO=dO).items()}
    host = {k: dev[k].float().cpu().numpy() for k in dev}     # the values the GPU sees
    return dev, host, idx, cnt


def _rel(got, ref):
    err = np.abs(got.astype(np.float64) - ref)
    scale = np.abs(ref).max()
    return err.max() / scale, err.mean() / np.abs(ref).mean()


@pytest.mark.parametrize("dtype,Hq,Hkv,d", [("f32", 4, 1, 64), ("f32", 8, 2, 128),
                                            ("bf16", 8, 2, 128), ("bf16", 32, 4, 128),
                                            ("bf16", 4, 4, 64)])
def test_backward_matches_oracle(dtype, Hq, Hkv, d):
    nq, T, s_max = 48, 300, 80
    dev, host, idx, cnt = _inputs(Hq + d, nq, T, Hq, Hkv, d, s_max, dtype)
    i_d = torch.from_numpy(idx).cuda()
    c_d = torch.from_numpy(cnt).cuda()
    O, lse = lsa.lsa_sparse_attn(dev["Q"], dev["K"], dev["V"], i_d, c_d, return_lse=True)
    dQ, dK, dV = lsa.lsa_sparse_attn_backward(dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"],
                                              i_d, c_d)
    torch.cuda.synchronize()
    rQ, rK, rV = oracle.attend_backward(host["Q"][0], host["K"][0], host["V"][0], host["dO"][0],
                                        idx[0], cnt[0], oracle.default_scale(d))
    bars = (1e-4, 1e-4) if dtype == "f32" else (2e-2, 5e-3)
    for got, ref in ((dQ[0].float().cpu().numpy(), rQ), (dK[0].cpu().numpy(), rK),
                     (dV[0].cpu().numpy(), rV)):
        mx, mean = _rel(got, ref)
        assert mx <= bars[0] and mean <= bars[1], (mx, mean)
    # keys nobody reads keep zero gradients
    read = np.zeros(T, bool)
    for i in range(nq):
        read[idx[0, i, :cnt[0, i]]] = True
    assert not dK[0][torch.from_numpy(~read).cuda()].any()


def test_backward_accumulates_into_given_buffers():
    nq, T, Hq, Hkv, d, s_max = 20, 100, 8, 2, 64, 30
    dev, host, idx, cnt = _inputs(5, nq, T, Hq, Hkv, d, s_max, "f32")
    i_d = torch.from_numpy(idx).cuda()
    c_d = torch.from_numpy(cnt).cuda()
    O, lse = lsa.lsa_sparse_attn(dev["Q"], dev["K"], dev["V"], i_d, c_d, return_lse=True)
    _, dK1, dV1 = lsa.lsa_sparse_attn_backward(dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"],
                                               i_d, c_d)
    dK2, dV2 = dK1.clone(), dV1.clone()
    lsa.lsa_sparse_attn_backward(dev["Q"], dev["K"], dev["V"], O, lse, dev["dO"], i_d, c_d,
                                 dK=dK2, dV=dV2)
    torch.cuda.synchronize()
    assert torch.allclose(dK2, 2 * dK1, rtol=1e-5, atol=1e-6)
    assert torch.allclose(dV2, 2 * dV1, rtol=1e-5, atol=1e-6)
