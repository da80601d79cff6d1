"""D-LSA Tree on the GPU against the oracle.

The tree's level 2 (super-centroids, retrieval copy, CSR of bucket ids) must
equal the oracle's bit for bit; tree selections must equal the oracle's row
for row, for several branch counts (one branch: a narrow walk; every branch:
Flat's selection), for fp32 and bf16 indices, with an open block, on the path
of many rows (a warp per row) and of few rows (a CTA per row), and through the
exact fallback restricted to the chosen branches (tied scores).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


def _setup(w, seed, t_end=None, same_latent=False):
    inp = synth.prefill_inputs(w, seed, "cpu")
    if same_latent:
        inp["latent_K"][:] = inp["latent_K"][:, :1]
    end = t_end or w.T
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if w.dtype == "bf16" else lsa.F32)
    gpu.build(inp["latent_K"].cuda(), end)
    orcs = []
    for b in range(w.B):
        o = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=(w.dtype == "bf16"))
        o.extend(inp["latent_K"][b].float().numpy(), 0, end)
        orcs.append(o)
    return inp, gpu, orcs


def _np(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tree_build_matches_oracle(dtype):
    w = synth.workload("tiny", T=16384, nq=8, B=2, G=32, k=4, M=64, dtype=dtype)
    _, gpu, orcs = _setup(w, 3)
    tree = lsa.LsaTree(gpu, 13, 3)
    ex = tree.export()
    torch.cuda.synchronize()
    for b in range(w.B):
        ref = oracle.Tree(orcs[b], 13, 3)
        nb = orcs[b].n_buckets
        assert np.array_equal(_np(ex["sup"][b]), ref.sup)
        assert np.array_equal(_np(ex["sup_rt"][b]), ref.sup_rt)
        assert np.array_equal(_np(ex["offsets"][b]), ref.offsets)
        assert np.array_equal(_np(ex["members"][b])[:nb], ref.members)


@pytest.mark.parametrize("dtype,nq,branches,t_end", [
    ("bf16", 300, 1, None), ("bf16", 300, 3, None), ("f32", 97, 2, None),
    ("bf16", 20, 2, None), ("bf16", 300, 13, None), ("bf16", 200, 2, 16384 - 700)])
def test_tree_select_matches_oracle(dtype, nq, branches, t_end):
    w = synth.workload("tiny", T=16384, nq=nq, B=2, G=32, k=4, R=700, W=64, S=4, M=64,
                       dtype=dtype, Hq=8, Hkv=1, d=64)
    inp, gpu, orcs = _setup(w, 7, t_end)
    end = t_end or w.T
    tree = lsa.LsaTree(gpu, 13, 3)
    rng = np.random.default_rng(7)
    pos = rng.integers(0, end, size=(w.B, w.nq))
    pos[:, :4] = [0, w.W, w.W + 200, end - 1]
    g_idx, g_cnt = tree.select(inp["latent_Q"].cuda(), torch.from_numpy(pos.astype(np.int32)).cuda(),
                               branches, w.R, w.W, w.S)
    torch.cuda.synchronize()
    assert gpu.check() >= 0
    for b in range(w.B):
        ref = oracle.Tree(orcs[b], 13, 3)
        o_idx, o_cnt = oracle.tree_select(orcs[b], ref, inp["latent_Q"][b].float().numpy(),
                                          pos[b], branches, w.R, w.W, w.S)
        assert np.array_equal(_np(g_cnt[b]), o_cnt)
        assert np.array_equal(_np(g_idx[b]), o_idx)
    if branches == 13:                    # every branch: Flat's selection
        f_idx, f_cnt = lsa.lsa_select(gpu, inp["latent_Q"].cuda(),
                                      torch.from_numpy(pos.astype(np.int32)).cuda(), w.R, w.W,
                                      w.S)
        assert torch.equal(f_idx, g_idx) and torch.equal(f_cnt, g_cnt)


def test_tree_select_fallback_on_tied_scores():
    # identical latent keys: every approximate score ties, so no candidate
    # list proves the ranking; the fallback ranks the chosen branches exactly
    w = synth.workload("tiny", T=16384, nq=128, B=1, G=16, k=8, R=500, W=32, S=3, M=16,
                       dtype="bf16")
    inp, gpu, orcs = _setup(w, 9, same_latent=True)
    tree = lsa.LsaTree(gpu, 20, 2)
    pos = np.full((1, w.nq), w.T - 1) - np.arange(w.nq)[None] * 5
    gpu.check()
    g_idx, g_cnt = tree.select(inp["latent_Q"].cuda(), torch.from_numpy(pos.astype(np.int32)).cuda(),
                               4, w.R, w.W, w.S)
    torch.cuda.synchronize()
    assert gpu.check() > 0                          # the fallback ran
    ref = oracle.Tree(orcs[0], 20, 2)
    o_idx, o_cnt = oracle.tree_select(orcs[0], ref, inp["latent_Q"][0].float().numpy(), pos[0], 4,
                                      w.R, w.W, w.S)
    assert np.array_equal(_np(g_cnt[0]), o_cnt) and np.array_equal(_np(g_idx[0]), o_idx)


def test_tree_on_the_1m_index():
    # the 1M workload's index (4096 buckets), 64 super-buckets, 8 branches,
    # 1024 queries of the last chunk
    w = synth.workload("1m", nq=1024)
    inp = synth.prefill_inputs(w, 0, "cuda")
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(inp["latent_K"], w.T)
    tree = lsa.LsaTree(gpu, 64, 3)
    pos = torch.arange(w.T - w.nq, w.T, dtype=torch.int32, device="cuda")[None].contiguous()
    g_idx, g_cnt = tree.select(inp["latent_Q"], pos, 8, w.R, w.W, w.S)
    torch.cuda.synchronize()
    fb = gpu.check()
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    orc.extend(inp["latent_K"][0].float().cpu().numpy(), 0, w.T)
    ref = oracle.Tree(orc, 64, 3)
    ex = tree.export()
    assert np.array_equal(_np(ex["members"][0])[:orc.n_buckets], ref.members)
    o_idx, o_cnt = oracle.tree_select(orc, ref, inp["latent_Q"][0].float().cpu().numpy(),
                                      pos[0].cpu().numpy(), 8, w.R, w.W, w.S)
    assert np.array_equal(_np(g_cnt[0]), o_cnt)
    assert np.array_equal(_np(g_idx[0]), o_idx)
    assert fb == 0
