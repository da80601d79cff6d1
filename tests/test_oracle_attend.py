"""Pins for the oracle's exact sparse attention.

When the budget covers every causal key, D-LSA Flat selects the whole causal
prefix and the attention must equal plain full causal attention, which is
checked against an explicit fp64 formula and torch's SDPA in fp64 on CPU."""
import json
import math
import os

import numpy as np
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_attend_golden():
    for c in json.load(open(os.path.join(GOLDEN, "attention_hand.json")))["cases"]:
        n = len(c["K"])
        Q = np.array(c["Q"], np.float32).reshape(1, 1, 1)
        K = np.array(c["K"], np.float32).reshape(n, 1, 1)
        V = np.array(c["V"], np.float32).reshape(n, 1, 1)
        idx = np.arange(n, dtype=np.int32)[None]
        O, lse = oracle.attend(Q, K, V, idx, np.array([n], np.int32), scale=c["scale"])
        assert abs(O[0, 0, 0] - c["O"]) < 1e-6, c["derivation"]
        assert abs(lse[0, 0] - c["lse"]) < 1e-6, c["derivation"]


def test_attend_single_key_returns_value_row():
    rng = np.random.default_rng(7)
    T, Hkv, Hq, d = 50, 2, 4, 64
    K = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    Q = rng.standard_normal((3, Hq, d)).astype(np.float32)
    idx = np.array([[17, -1], [0, -1], [49, -1]], np.int32)
    O, _ = oracle.attend(Q, K, V, idx, np.array([1, 1, 1], np.int32))
    for i, t in enumerate([17, 0, 49]):
        for h in range(Hq):
            assert np.array_equal(O[i, h], V[t, h // 2])     # heads 0,1 -> kv 0; 2,3 -> kv 1


def test_attend_is_permutation_invariant_and_ignores_padding():
    rng = np.random.default_rng(8)
    T, Hkv, Hq, d = 300, 1, 2, 64
    K = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    Q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    sel = rng.choice(T, 40, replace=False).astype(np.int32)
    a = np.full((1, 64), -1, np.int32)
    a[0, :40] = sel
    b = np.full((1, 64), -1, np.int32)
    b[0, :40] = sel[::-1]
    Oa, la = oracle.attend(Q, K, V, a, np.array([40], np.int32))
    Ob, lb = oracle.attend(Q, K, V, b, np.array([40], np.int32))
    assert np.allclose(Oa, Ob, atol=1e-6) and np.allclose(la, lb, atol=1e-6)


def _full_causal_fp64(Q, K, V, pos, scale):
    nq, Hq, d = Q.shape
    Hkv = K.shape[1]
    out = np.empty((nq, Hq, d))
    lse = np.empty((nq, Hq))
    for i, p in enumerate(pos):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            z = scale * (K[: p + 1, g].astype(np.float64) @ Q[i, h].astype(np.float64))
            w = np.exp(z - z.max())
            out[i, h] = w @ V[: p + 1, g].astype(np.float64) / w.sum()
            lse[i, h] = z.max() + math.log(w.sum())
    return out, lse


def test_budget_covering_everything_is_full_causal_attention():
    # Index + select + attend with R >= every key reduces to full causal attention.
    w = synth.workload("tiny", T=4096, nq=48)
    inp = synth.prefill_inputs(w, 9, "cpu")
    lat = inp["latent_K"][0].numpy()
    idx = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=False)
    idx.extend(lat, 0, w.T)
    rng = np.random.default_rng(9)
    pos = np.sort(rng.integers(0, w.T, w.nq))
    pos[:4] = [0, 1, 5, 70]
    R = w.T
    out, cnt, _, _ = oracle.select(idx, inp["latent_Q"][0].numpy(), pos, R, w.W, w.S,
                                   s_max=w.T + w.W + w.S)
    assert np.array_equal(cnt, pos + 1)
    Q, K, V = inp["Q"][0].numpy(), inp["K"][0].numpy(), inp["V"][0].numpy()
    scale = oracle.default_scale(w.d)
    O, lse = oracle.attend(Q, K, V, out, cnt, scale)
    ref, ref_lse = _full_causal_fp64(Q, K, V, pos, scale)
    assert np.max(np.abs(O - ref)) < 1e-6
    assert np.max(np.abs(lse - ref_lse)) < 1e-5

    # Library cross-check: torch SDPA in fp64 on CPU, one causal row per query.
    Qt = torch.from_numpy(Q).double()
    Kt = torch.from_numpy(K).double()
    Vt = torch.from_numpy(V).double()
    for i in (0, 3, 10, w.nq - 1):
        p = int(pos[i])
        q = Qt[i].unsqueeze(1)                               # [Hq][1][d]
        kk = Kt[: p + 1].permute(1, 0, 2).repeat_interleave(w.Hq // w.Hkv, 0)
        vv = Vt[: p + 1].permute(1, 0, 2).repeat_interleave(w.Hq // w.Hkv, 0)
        o = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, scale=scale)
        assert torch.max(torch.abs(o[:, 0] - torch.from_numpy(O[i]).double())) < 1e-6


def test_attend_uses_the_given_scale():
    rng = np.random.default_rng(10)
    K = rng.standard_normal((8, 1, 4)).astype(np.float32)
    V = rng.standard_normal((8, 1, 4)).astype(np.float32)
    Q = rng.standard_normal((1, 1, 4)).astype(np.float32)
    idx = np.arange(8, dtype=np.int32)[None]
    O1, _ = oracle.attend(Q, K, V, idx, np.array([8], np.int32), scale=0.5)
    O2, _ = oracle.attend(2 * Q, K, V, idx, np.array([8], np.int32), scale=0.25)
    assert np.allclose(O1, O2, atol=1e-7)
