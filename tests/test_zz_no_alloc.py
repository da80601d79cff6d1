"""lsa_select_noalloc: selection for callers that cannot allocate device memory.

Such a caller (a plug-in handed only input and output buffers, a serving loop
whose device memory was divided up at start-up) passes the same inputs and
outputs as to lsa_select but no workspace; the library's built-in device array
holds the scratch.  These checks call it through the C-ABI twice in a row and
require the same selections as lsa_select with a caller workspace (index work:
bit for bit), and that a request too large for the array is refused before any
launch.  The file sorts last so that a run stopping at its first failure has
already run every other test; it also passes on its own in a fresh process,
where its first call is the one that sets the array up.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

lsa = pytest.importorskip("long_context_indexing_b200")


def _case(dtype, nq, seed):
    w = synth.workload("tiny", T=16384, nq=nq, B=2, G=32, k=4, R=700, W=64, S=4, M=64,
                       dtype=dtype, Hq=8, Hkv=1, d=64)
    inp = synth.prefill_inputs(w, seed, "cpu")
    rng = np.random.default_rng(seed)
    pos = rng.integers(0, w.T, size=(w.B, w.nq)).astype(np.int32)
    pos[:, :3] = [0, w.W + 5, w.T - 1]
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if dtype == "bf16" else lsa.F32)
    idx.build(inp["latent_K"].cuda(), w.T)
    return w, idx, inp["latent_Q"].cuda(), torch.from_numpy(pos).cuda()


# bf16 with 300 queries takes the tensor-core nominator, f32 the SIMT one.
@pytest.mark.parametrize("dtype,nq", [("bf16", 300), ("f32", 97)])
def test_noalloc_select_matches_workspace_select_twice(dtype, nq):
    w, idx, lq, pos = _case(dtype, nq, seed=21)
    ref_i, ref_c = lsa.lsa_select(idx, lq, pos, w.R, w.W, w.S)
    torch.cuda.synchronize()
    for _ in range(2):                       # two calls in a row share the array
        out_i = torch.full_like(ref_i, 0x7f7f7f7f)
        out_c = torch.full_like(ref_c, -7)
        lsa.lsa_select_noalloc(idx, lq, pos, w.R, w.W, w.S, out_i, out_c)
        torch.cuda.synchronize()
        assert torch.equal(out_c, ref_c)
        assert torch.equal(out_i, ref_i)
    assert idx.check() >= 0


def test_noalloc_select_refuses_requests_beyond_its_array():
    w, idx, lq, pos = _case("f32", 40000, seed=22)   # about 40000 * 2 * 272 B of scratch
    out_i = torch.full((w.B, w.nq, w.s_max), 5, dtype=torch.int32, device="cuda")
    out_c = torch.full((w.B, w.nq), 5, dtype=torch.int32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_select_noalloc(idx, lq, pos, w.R, w.W, w.S, out_i, out_c)
    assert e.value.code == 3 and "built-in array" in str(e.value)
    torch.cuda.synchronize()
    assert int(out_c.min()) == 5 and int(out_c.max()) == 5   # nothing was launched


def test_noalloc_select_at_its_size_limit_with_two_sequences():
    # Two sequences on the tensor-core path (bf16, Nq >= 128): the largest
    # query count whose scratch fits the 8 MiB array gives lsa_select's
    # selections; one query more is refused before any launch.
    w, idx, lq, pos = _case("bf16", 12000, seed=23)
    limit = 8 << 20
    need = lambda n: int(lsa._lib.lsa_select_workspace_bytes(idx.handle, n))
    lo, hi = 128, w.nq
    assert need(lo) <= limit < need(hi)
    while hi - lo > 1:                       # need(lo) <= limit < need(hi)
        mid = (lo + hi) // 2
        if need(mid) <= limit:
            lo = mid
        else:
            hi = mid
    n_fit = lo
    lq_fit, pos_fit = lq[:, :n_fit].contiguous(), pos[:, :n_fit].contiguous()
    ref_i, ref_c = lsa.lsa_select(idx, lq_fit, pos_fit, w.R, w.W, w.S)
    out_i = torch.full_like(ref_i, 0x7f7f7f7f)
    out_c = torch.full_like(ref_c, -7)
    lsa.lsa_select_noalloc(idx, lq_fit, pos_fit, w.R, w.W, w.S, out_i, out_c)
    torch.cuda.synchronize()
    assert torch.equal(out_c, ref_c) and torch.equal(out_i, ref_i)
    n_over = n_fit + 1
    big_i = torch.full((w.B, n_over, w.s_max), 5, dtype=torch.int32, device="cuda")
    big_c = torch.full((w.B, n_over), 5, dtype=torch.int32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_select_noalloc(idx, lq[:, :n_over].contiguous(), pos[:, :n_over].contiguous(),
                               w.R, w.W, w.S, big_i, big_c)
    assert e.value.code == 3
    torch.cuda.synchronize()
    assert int(big_c.min()) == 5 and int(big_c.max()) == 5
    assert idx.check() >= 0
