"""KV cache in shards (context parallel) against the oracle.

"Latent Sparse Attention: un indice gerarchico per contesti lunghi",
paragraph on memory: every rank keeps its share of the KV cache and a full
copy of the index, so every rank makes the same selection and reads the
selected keys it holds.  Here the shards are slices of one GPU's caches:
lsa_attend_key_range gives each slice's partial (output over its keys, and
their log-sum-exp), lsa_merge_partials weighs them together, and the result
equals the oracle's attention over the whole selection (bf16 bars, fp32
tolerance for fp32), and its lse the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


def _case(dtype, cuts, seed, **kw):
    args = dict(T=4096, nq=600, B=1, Hq=8, Hkv=2, d=64, M=48, p=4, G=64, k=4, L=3, R=384, W=48,
                S=4, dtype=dtype)
    args.update(kw)
    w = synth.workload("tiny", **args)
    inp = synth.prefill_inputs(w, seed, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    gpu = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if dtype == "bf16" else lsa.F32)
    gpu.build(dev["latent_K"], w.T)
    pos = dev["positions"].to(torch.int32).contiguous()
    idx, cnt = lsa.lsa_select(gpu, dev["latent_Q"], pos, w.R, w.W, w.S)
    edges = [0] + list(cuts) + [w.T]
    parts_o, parts_l = [], []
    for lo, hi in zip(edges[:-1], edges[1:]):
        Ks = dev["K"][:, lo:hi].contiguous()
        Vs = dev["V"][:, lo:hi].contiguous()
        o, l = lsa.lsa_attend_key_range(dev["Q"], Ks, Vs, idx, cnt, lo, hi)
        parts_o.append(o)
        parts_l.append(l)
    O_parts = torch.stack(parts_o).contiguous()
    L_parts = torch.stack(parts_l).contiguous()
    L = torch.empty_like(L_parts[0])
    O = lsa.lsa_merge_partials(O_parts, L_parts, lse=L)
    torch.cuda.synchronize()
    return w, inp, idx.cpu().numpy(), cnt.cpu().numpy(), O, L, L_parts


@pytest.mark.parametrize("cuts", [(1024, 2048, 3072), (256,), (3840,), (512, 700, 3000)])
def test_shards_merge_to_the_whole_attention_bf16(cuts):
    w, inp, idx, cnt, O, L, L_parts = _case("bf16", cuts, 3)
    O_ref, lse_ref = oracle.attend(inp["Q"][0].float().numpy(), inp["K"][0].float().numpy(),
                                   inp["V"][0].float().numpy(), idx[0], cnt[0],
                                   oracle.default_scale(w.d))
    err = np.abs(O[0].float().cpu().numpy().astype(np.float64) - O_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert np.allclose(L[0].cpu().numpy(), lse_ref, rtol=0, atol=2e-3)
    if len(cuts) >= 2:
        # a middle shard holds no key of some queries (every query's sinks
        # are in the first shard and its window in the last): lse -inf, weight 0
        assert bool(torch.isinf(L_parts).any())


def test_shards_merge_to_the_whole_attention_f32():
    w, inp, idx, cnt, O, L, _ = _case("f32", (1000, 2200), 5, Hq=4, Hkv=1, R=300)
    O_ref, lse_ref = oracle.attend(inp["Q"][0].numpy(), inp["K"][0].numpy(), inp["V"][0].numpy(),
                                   idx[0], cnt[0], oracle.default_scale(w.d))
    assert np.allclose(O[0].cpu().numpy(), O_ref, rtol=0, atol=1e-4)
    assert np.allclose(L[0].cpu().numpy(), lse_ref, rtol=0, atol=1e-4)


def test_one_shard_is_the_sparse_attention():
    # a single shard over the whole cache: the partial is lsa_sparse_attn's
    # result and the merge of one part returns it
    w, inp, idx, cnt, O, L, L_parts = _case("bf16", (), 7)
    dev_idx = torch.from_numpy(idx).cuda()
    dev_cnt = torch.from_numpy(cnt).cuda()
    Q, K, V = (inp[k].cuda() for k in ("Q", "K", "V"))
    O_full, lse_full = lsa.lsa_sparse_attn(Q, K, V, dev_idx, dev_cnt, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(O, O_full)
    assert torch.allclose(L, lse_full, rtol=0, atol=1e-6)
