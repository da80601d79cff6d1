"""The small pipeline that test_gpu_debug_checks.py runs with and without
LSA_DEBUG=1: a bf16 index over 8192 keys, one prefill chunk, a selection, a
per-key selection and a sparse attention of the chunk's queries."""
import synth


def case(lsa):
    import torch
    w = synth.workload("tiny", dtype="bf16", T=8192, nq=300, Hq=8, Hkv=2, d=64, M=64, p=4, G=256,
                       k=8, R=384, W=64, S=4)
    inp = synth.prefill_inputs(w, 21, "cpu")
    dev = {k: v.cuda() for k, v in inp.items()}
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16)
    T_old = w.T - w.nq
    idx.build(dev["latent_K"], T_old)
    O = lsa.lsa_prefill_chunk(idx, dev["latent_K"], dev["latent_Q"], dev["Q"], dev["K"], dev["V"],
                              T_old, w.T, w.R, w.W, w.S)
    pos = torch.arange(T_old, w.T, dtype=torch.int32, device="cuda")[None].contiguous()
    sel_idx, sel_cnt = lsa.lsa_select(idx, dev["latent_Q"], pos, w.R, w.W, w.S)
    pk_idx, pk_cnt, _ = lsa.lsa_select_per_key(dev["latent_K"], dev["latent_Q"], pos, w.R, w.W,
                                               w.S)
    O2 = lsa.lsa_sparse_attn(dev["Q"], dev["K"], dev["V"], sel_idx, sel_cnt)
    torch.cuda.synchronize()
    res = dict(O=O, sel_idx=sel_idx, sel_cnt=sel_cnt, pk_idx=pk_idx, pk_cnt=pk_cnt, O2=O2)
    return w, inp, dev, idx, res
