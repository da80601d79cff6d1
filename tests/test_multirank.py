"""The N > 1 path of bench.py on CPU: world size 2 over gloo.

Under torchrun bench.py runs one process per GPU.  Every rank processes its
own chunk (the path shards by independent problems: no collective on the data
path), the step time is the max over ranks, the value is the units of all
ranks over that time, and rank 0 alone prints the JSON line.  Here the ranks
are CPU processes over gloo (bench picks gloo when no GPU is visible):
- the rank helpers agree on every rank (barrier, max over ranks, job rate);
- the reference arm under torchrun prints exactly one line, from rank 0,
  with n_gpus = 2, and every rank exits 0.
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import bench
    r, w = bench._dist(timeout_s=60)
    local_ms = 10.0 + 5.0 * r              # rank 1 is the slower one
    bench._barrier(w)
    mx = bench._max_over_ranks(local_ms, w)
    rate = bench._job_rate(32768, mx, w)
    backend = torch.distributed.get_backend()
    torch.distributed.destroy_process_group()
    q.put((r, w, mx, rate, backend))


def test_rank_helpers_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    for _, w, mx, rate, backend in res:
        assert w == 2 and backend == "gloo"
        assert mx == 15.0                                  # the slowest rank's time
        assert rate == 2 * 32768 / 0.015                   # both ranks' queries / that time


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "1", "--warmup", "3", "--ref-queries", "4", "--gpus", "2"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2 and j["scaling"] == "weak"
    assert j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"


def _split_worker(rank, ws, port, q):
    # One chunk's queries split over two ranks, the oracle standing in for the
    # GPU on each rank: the gathered rows equal the single-rank chunk.
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import oracle
    import synth
    r, w = bench._dist(timeout_s=60)
    wl = synth.workload("tiny", T=2048, nq=64, Hq=4, Hkv=1, d=64, M=16, G=64, k=4, R=200, W=32,
                        S=4)
    inp = synth.prefill_inputs(wl, 3, "cpu")                # every rank: the same chunk
    T_old = wl.T - wl.nq
    lat = inp["latent_K"][0].numpy()
    orc = oracle.Index(wl.T, wl.p, wl.G, wl.k, wl.L, rt_bf16=False)
    orc.extend(lat, 0, wl.T)
    q0, q1 = bench._query_slice(wl.nq, r, w)
    pos = T_old + np.arange(q0, q1)
    sel, cnt, _, _ = oracle.select(orc, inp["latent_Q"][0][q0:q1].numpy(), pos, wl.R, wl.W, wl.S)
    O, _ = oracle.attend(inp["Q"][0][q0:q1].numpy(), inp["K"][0].numpy(), inp["V"][0].numpy(),
                         sel, cnt)
    O_all = bench._gather_rows(torch.from_numpy(O), w)
    sel_all = bench._gather_rows(torch.from_numpy(sel), w)
    torch.distributed.destroy_process_group()
    if r == 0:
        pos_all = T_old + np.arange(wl.nq)
        ref_sel, ref_cnt, _, _ = oracle.select(orc, inp["latent_Q"][0].numpy(), pos_all, wl.R,
                                               wl.W, wl.S)
        ref_O, _ = oracle.attend(inp["Q"][0].numpy(), inp["K"][0].numpy(), inp["V"][0].numpy(),
                                 ref_sel, ref_cnt)
        q.put((bool(np.array_equal(sel_all.numpy(), ref_sel)),
               bool(np.array_equal(O_all.numpy(), ref_O)), (q0, q1)))
    else:
        q.put(None)


def test_query_split_over_gloo_matches_the_whole_chunk():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got = [x for x in res if x is not None]
    assert len(got) == 1
    same_sel, same_o, rng = got[0]
    assert same_sel and same_o
    assert rng == (0, 32)


def _context_worker(rank, ws, port, q):
    # The KV cache in two shards of whole blocks, the oracle standing in for
    # the GPU on each rank: every rank selects for the whole chunk, attends
    # over the selected keys of its shard (output and log-sum-exp), the
    # partials are exchanged by row blocks, and the LSE-weighted merge of a
    # rank's rows equals the single-rank attention of those rows.
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import oracle
    import synth
    r, w = bench._dist(timeout_s=60)
    wl = synth.workload("tiny", T=2048, nq=64, Hq=4, Hkv=1, d=64, M=16, G=64, k=4, R=200, W=32,
                        S=4)
    inp = synth.prefill_inputs(wl, 5, "cpu")
    T_old = wl.T - wl.nq
    orc = oracle.Index(wl.T, wl.p, wl.G, wl.k, wl.L, rt_bf16=False)
    orc.extend(inp["latent_K"][0].numpy(), 0, wl.T)
    pos = T_old + np.arange(wl.nq)
    sel, cnt, _, _ = oracle.select(orc, inp["latent_Q"][0].numpy(), pos, wl.R, wl.W, wl.S)
    lo, hi = bench._context_shard(wl.T, wl.p * wl.G, r, w)
    Q, K, V = (inp[k][0].numpy() for k in ("Q", "K", "V"))
    O_r = np.zeros(Q.shape, np.float32)
    L_r = np.full(Q.shape[:2], -np.inf, np.float32)
    loc = np.full(sel.shape, -1, np.int32)
    lc = np.zeros(cnt.shape, np.int32)
    for i in range(wl.nq):
        keep = [t for t in sel[i, :cnt[i]] if lo <= t < hi]
        loc[i, :len(keep)] = keep
        lc[i] = len(keep)
    has = lc > 0
    if has.any():
        o, l = oracle.attend(Q[has], K, V, loc[has], lc[has])
        O_r[has], L_r[has] = o, l
    O_parts = bench._exchange_rows(torch.from_numpy(O_r), r, w).double().numpy()
    L_parts = bench._exchange_rows(torch.from_numpy(L_r), r, w).double().numpy()
    torch.distributed.destroy_process_group()
    M = L_parts.max(0)
    wgt = np.exp(L_parts - M)                               # [parts][rows][heads]
    O_mine = (wgt[..., None] * O_parts).sum(0) / wgt.sum(0)[..., None]
    q0, q1 = bench._query_slice(wl.nq, r, w)
    ref_O, _ = oracle.attend(Q[q0:q1], K, V, sel[q0:q1], cnt[q0:q1])
    q.put((r, (lo, hi), float(np.abs(O_mine - ref_O).max()), bool(np.isinf(L_r).any())))


def test_context_split_over_gloo_matches_the_whole_chunk():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_context_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[1] for x in res] == [(0, 1024), (1024, 2048)]
    for _, _, err, _ in res:
        assert err < 1e-5


def test_context_shards_cover_the_cache():
    sys.path.insert(0, ROOT)
    import bench
    for T, span, ws in ((10485760, 4096, 8), (10485760, 4096, 3), (4096 * 5 + 100, 4096, 2)):
        got = [bench._context_shard(T, span, r, ws) for r in range(ws)]
        assert got[0][0] == 0 and got[-1][1] == T
        for (a, b), (c, _) in zip(got, got[1:]):
            assert b == c and a < b and b % span == 0


def test_query_slice_ranges():
    sys.path.insert(0, ROOT)
    import bench
    assert [bench._query_slice(32768, r, 4) for r in range(4)] == [
        (0, 8192), (8192, 16384), (16384, 24576), (24576, 32768)]
    import pytest
    with pytest.raises(ValueError):
        bench._query_slice(10, 0, 3)
