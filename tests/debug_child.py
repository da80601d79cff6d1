"""Child process of test_gpu_debug_checks.py: run with LSA_DEBUG=1 (read when
the library loads).  Runs a small pipeline through the checked entry points,
then plants three corruptions (on the host side, between calls) that the
checks must refuse before any kernel reads them.  Writes its findings as JSON
to argv[1] and the clean outputs to argv[2] (torch.save)."""
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import long_context_indexing_b200 as lsa  # noqa: E402
import synth  # noqa: E402

from debug_case import case  # noqa: E402


def refused(fn):
    try:
        fn()
        torch.cuda.synchronize()
    except lsa.LsaError as e:
        return {"code": e.code, "msg": str(e)}
    return None


def main(out_json, out_pt):
    w, inp, dev, idx, res = case(lsa)
    found = {"clean": True}
    torch.save({k: v.cpu() for k, v in res.items()}, out_pt)
    # 1. a gather index past T_cap handed to the sparse attention
    bad = res["sel_idx"].clone()
    bad[0, 3, 0] = w.T
    found["gather"] = refused(lambda: lsa.lsa_sparse_attn(dev["Q"], dev["K"], dev["V"], bad,
                                                          res["sel_cnt"]))
    # 2. a chunk selection whose long-range key lies after its query
    T_old = w.T - w.nq
    need = lsa.lsa_prefill_workspace_bytes(idx, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    work = torch.empty(need, dtype=torch.uint8, device="cuda")
    lsa.lsa_prefill_select(idx, dev["latent_K"], dev["latent_Q"], T_old, w.T, w.Hq, w.Hkv, w.d,
                           w.R, w.W, w.S, work)
    si, sc = lsa.prefill_selection_views(work, w.B, w.nq, w.s_max)
    row = 5                                          # position T_old + 5 < T - 1
    si[0, row, w.S] = T_old + row + 1
    found["selection"] = refused(lambda: lsa.lsa_prefill_attend(idx, dev["Q"], dev["K"], dev["V"],
                                                                T_old, w.T, w.R, w.W, w.S, work))
    # 3. the index's CSR: two members of a bucket swapped (no longer ascending)
    ex = idx.export()
    off, mem = ex["offsets"][0].cpu(), ex["members"][0].cpu()
    sizes = off[1: idx.k + 1] - off[: idx.k]           # buckets of block 0
    g = int(torch.nonzero(sizes >= 2)[0])
    o0 = int(off[g])
    raw = idx.buffer.cpu().numpy().tobytes()
    pat = mem[: idx.G].numpy().tobytes()                # block 0's members
    at = raw.find(pat)
    assert at >= 0 and at % 4 == 0 and raw.find(pat, at + 1) < 0, "members not found once"
    words = idx.buffer[at: at + idx.G * 4].view(torch.int32)
    a, b = int(words[o0]), int(words[o0 + 1])
    words[o0], words[o0 + 1] = b, a
    pos = torch.arange(T_old, w.T, dtype=torch.int32, device="cuda")[None].contiguous()
    found["index"] = refused(lambda: lsa.lsa_select(idx, dev["latent_Q"], pos, w.R, w.W, w.S))
    json.dump(found, open(out_json, "w"))


if __name__ == "__main__":
    main(sys.argv[1], sys.argv[2])
