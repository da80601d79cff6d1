"""The tensor-core nomination with scores outside fp16's normal range.

The tensor-core scorer stores each (query, centroid) score as fp16 with one
fp16 maximum per 32 scores; the fill nominates candidates from them and proves
the exact ranking with binary64 rescoring, or sends the query to the exact
fallback.  Scaling the latent queries by a power of two scales every exact
score by the same factor (bf16 x bf16 products are exact in binary64), so the
exact ranking -- and the oracle's selection -- stays the same while the fp16
copies of the scores
  * overflow to infinity (2^17: scores up to ~1.3e5 > 65504),
  * fall among fp16 subnormals (2^-18: scores ~4e-6 < 6.1e-5),
  * round to zero altogether (2^-40),
or stay ordinary (2^0).  Selections must equal the oracle's row for row in
every case; where fp16 cannot rank at all (overflow, zero), queries must have
taken the fallback.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


@pytest.fixture(scope="module")
def setup():
    # 262144 keys in blocks of 64 pooled groups x 16 buckets: 16384 buckets,
    # 512 chunks of 32 scores per row (the chunk-maximum nomination path)
    w = synth.workload("tiny", T=262144, nq=384, B=1, Hq=1, Hkv=1, d=64, M=1024, p=4, G=64,
                       k=16, L=3, R=2048, W=512, S=4, dtype="bf16")
    inp = synth.prefill_inputs(w, 5, "cpu")
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    gpu.build(inp["latent_K"].cuda(), w.T)
    orc = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=True)
    orc.extend(inp["latent_K"][0].float().numpy(), 0, w.T)
    rng = np.random.default_rng(5)
    pos = rng.integers(w.T // 2, w.T, size=(w.B, w.nq))
    return w, inp, gpu, orc, pos


@pytest.mark.parametrize("exp2,must_fall_back", [(0, False), (17, True), (-18, False),
                                                 (-40, True)])
def test_selection_with_scaled_queries(setup, exp2, must_fall_back):
    w, inp, gpu, orc, pos = setup
    lq = (inp["latent_Q"].float() * (2.0 ** exp2)).to(torch.bfloat16)
    assert torch.equal(lq.float() / (2.0 ** exp2), inp["latent_Q"].float())   # exact scaling
    gpu.check()
    g_idx, g_cnt = lsa.lsa_select(gpu, lq.cuda(), torch.from_numpy(pos.astype(np.int32)).cuda(),
                                  w.R, w.W, w.S)
    torch.cuda.synchronize()
    fallbacks = gpu.check()
    o_idx, o_cnt, _, _ = oracle.select(orc, lq[0].float().numpy(), pos[0], w.R, w.W, w.S)
    assert np.array_equal(g_cnt[0].cpu().numpy(), o_cnt)
    assert np.array_equal(g_idx[0].cpu().numpy(), o_idx)
    if exp2 == 0:
        # the same selection as the unscaled query, by construction
        base_idx, _, _, _ = oracle.select(orc, inp["latent_Q"][0].float().numpy(), pos[0], w.R,
                                          w.W, w.S)
        assert np.array_equal(base_idx, o_idx)
    if must_fall_back:
        assert fallbacks > 0
