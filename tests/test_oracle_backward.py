"""Pins of the oracle's attention backward (gradients over stored selections).

"Latent Sparse Attention: un indice gerarchico per contesti lunghi", paragraph
on N-LSA's memory: the selected indices are kept for the backward pass.  The
attention is ordinary softmax attention over the selected keys, so its
gradients have a plain definition; each pin would fail on a plausible mistake
in oracle.attend_backward:
  * torch autograd (binary64) through an independent dense formulation --
    every head scores every key, the unselected ones masked to -inf -- equals
    dQ, dK and dV (a dropped term of dS, a wrong sign, a transposed operand, a
    wrong GQA head or a key gradient not summed over queries shows);
  * a single selected key: dQ = 0 and dK = 0 for that head (a softmax over one
    key has no gradient), dV = dO summed over the heads that share the KV head;
  * keys selected by no query get zero gradients.
"""
import numpy as np
import pytest
import torch

import oracle


def _dense_grads(Q, K, V, dO, idx, cnt, scale):
    nq, Hq, d = Q.shape
    T, Hkv, _ = K.shape
    grp = Hq // Hkv
    q = torch.tensor(Q, dtype=torch.float64, requires_grad=True)
    k = torch.tensor(K, dtype=torch.float64, requires_grad=True)
    v = torch.tensor(V, dtype=torch.float64, requires_grad=True)
    mask = torch.zeros(nq, T, dtype=torch.bool)
    for i in range(nq):
        mask[i, torch.tensor(idx[i, :cnt[i]].astype(np.int64))] = True
    kh = k.repeat_interleave(grp, dim=1)              # [T][Hq][d]: head h reads KV head h // grp
    vh = v.repeat_interleave(grp, dim=1)
    s = torch.einsum("ihd,thd->iht", q, kh) * scale
    s = s.masked_fill(~mask[:, None, :], float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = torch.einsum("iht,thd->ihd", p, vh)
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (4, 2), (2, 2)])
def test_backward_equals_autograd_of_dense_attention(Hq, Hkv):
    rng = np.random.default_rng(Hq * 10 + Hkv)
    nq, T, d, s_max = 9, 40, 16, 12
    Q = rng.standard_normal((nq, Hq, d)).astype(np.float32)
    K = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    dO = rng.standard_normal((nq, Hq, d)).astype(np.float32)
    idx = np.full((nq, s_max), -1, np.int32)
    cnt = rng.integers(1, s_max + 1, nq).astype(np.int32)
    for i in range(nq):
        idx[i, :cnt[i]] = rng.choice(T - 5, cnt[i], replace=False)   # keys T-5.. never read
    scale = oracle.default_scale(d)
    dQ, dK, dV = oracle.attend_backward(Q, K, V, dO, idx, cnt, scale)
    rQ, rK, rV = _dense_grads(Q, K, V, dO, idx, cnt, scale)
    for got, ref in ((dQ, rQ), (dK, rK), (dV, rV)):
        assert np.allclose(got, ref, rtol=1e-5, atol=1e-5), np.abs(got - ref).max()
    assert not dK[T - 5:].any() and not dV[T - 5:].any()


def test_single_key_has_no_query_or_key_gradient():
    rng = np.random.default_rng(3)
    nq, T, Hq, Hkv, d = 3, 8, 4, 2, 8
    Q = rng.standard_normal((nq, Hq, d)).astype(np.float32)
    K = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    dO = rng.standard_normal((nq, Hq, d)).astype(np.float32)
    idx = np.array([[5], [2], [5]], np.int32)
    cnt = np.ones(nq, np.int32)
    dQ, dK, dV = oracle.attend_backward(Q, K, V, dO, idx, cnt)
    assert not dQ.any() and not dK.any()
    grp = Hq // Hkv
    ref = np.zeros_like(dV, dtype=np.float64)
    for i in range(nq):
        for h in range(Hq):
            ref[idx[i, 0], h // grp] += dO[i, h]
    assert np.allclose(dV, ref, rtol=0, atol=1e-6)
