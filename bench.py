"""Benchmark of the D-LSA Flat hot path on B200.

Default workload: the last 32,768-query chunk of a 10,485,760-token context
(bf16, 32 query / 4 KV heads, d = 128, 64-d latent index with p = 4,
1024 pooled groups per block, 16 buckets per block, 3 Lloyd iterations,
4096 long-range + 512 recent + 4 sink keys per query).  One step is one call
of lsa_prefill_chunk: cluster the chunk's 8 blocks, select for every chunk
query, exact sparse attention.  Inputs are synthetic (the clustered mixture of
the `synth` module) and resident in HBM before the timed region; K and V
(21.5 GB) are far larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference]

Under torchrun every rank runs an independent chunk of its own sequence
(weak scaling, no collective on the data path); times are the max over
ranks.  `--impl reference` times the CPU oracle (the plain-C definition of
the method) on a bounded query sample of the same workload.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "prefill 32k-chunk queries/s and decode µs/step at 10M ctx; % of HBM/TC roofline"
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ------------------------------------------------------------------ helpers --

def _dist(timeout_s=300):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE / MASTER_*):
    NCCL on GPUs; gloo where no GPU is visible (the host-side logic, on CPU)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1 and not torch.distributed.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group(backend,
                                             timeout=datetime.timedelta(seconds=timeout_s))
    rank = torch.distributed.get_rank() if ws > 1 else 0
    return rank, ws


def _coll_device():
    return ("cuda" if torch.distributed.is_initialized()
            and torch.distributed.get_backend() == "nccl" else "cpu")


def _max_over_ranks(x, ws):
    """The largest of every rank's x (every rank gets it)."""
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_coll_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _sync():
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _barrier(ws):
    _sync()
    if ws > 1:
        torch.distributed.barrier()
        _sync()


def _job_rate(units_per_rank, ms_max, ws):
    """Whole-job throughput: the units all ranks processed / the slowest
    rank's time (weak scaling: every rank processes its own units)."""
    return ws * units_per_rank / (ms_max * 1e-3)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAK_FALLBACK), "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows, by_uuid = [], {}
        for ts, line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                row = (ts, float(parts[2]), float(parts[3]), parts[5:])
            except ValueError:
                continue
            by_uuid.setdefault(parts[1], []).append(row)
        if self.uuid in by_uuid:
            rows = by_uuid[self.uuid]
        elif len(by_uuid) == 1:
            rows = next(iter(by_uuid.values()))
        if not rows:
            return None
        inside = [r for r in rows if self.t0 - 0.05 <= r[0] <= self.t1 + 0.15] or rows
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in inside:
            for name, flag in zip(names, r[3][1:5]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": sorted(reasons),
                "samples": len(inside)}


def _gpu_uuid():
    try:
        u = torch.cuda.get_device_properties(torch.cuda.current_device()).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return None


def _events_time(fn, steps, stream):
    """Runs fn() `steps` times between two events on `stream`; returns ms per step."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / steps


# ---------------------------------------------------------------- workloads --

def _workload_desc(w):
    return ("D-LSA Flat prefill of the last %d-query chunk of a %d-token context "
            "(bf16, Hq=%d, Hkv=%d, d=%d; index p=%d, block=%d pooled, %d buckets/block, "
            "L=%d; reads %d long-range + %d recent + %d sinks)"
            % (w.nq, w.T, w.Hq, w.Hkv, w.d, w.p, w.G, w.k, w.L, w.R, w.W, w.S))


def _config(w, n_gpus):
    return {"workload": _workload_desc(w), "name": w.name, "T": w.T, "chunk_queries": w.nq,
            "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "p": w.p, "block": w.G, "buckets": w.k,
            "lloyd_iters": w.L, "budget": w.R, "window": w.W, "sinks": w.S,
            "l2": "no flush: K+V (%.1f GB) far exceed L2" % (2 * w.T * w.Hkv * w.d * 2 / 1e9),
            "parallelism": "dp%d (independent chunk per rank)" % n_gpus}


def _attn_floor_bytes(w, indices, counts, T_cap):
    """Compulsory bytes of one chunk's attention: every K and V row (all KV
    heads) that at least one query selected, read once, plus Q read and O
    written.  Counted from the chunk's selection."""
    elt = 2 if w.dtype == "bf16" else 4
    rows = 0
    for b in range(w.B):
        sel = indices[b]
        mask = torch.zeros(T_cap, dtype=torch.bool, device=sel.device)
        mask[sel[sel >= 0].long()] = True
        rows += int(mask.sum().item())
    kv = rows * w.Hkv * w.d * elt * 2
    qo = w.B * w.nq * w.Hq * w.d * elt * 2
    gather = int(counts.sum().item()) * w.Hkv * w.d * elt * 2 + qo
    return kv + qo, rows, gather


def _traffic_record(name):
    """DRAM bytes per call from a committed ncu summary, if none of the sources
    it was measured with has changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(name)
    if not rec:
        return None
    for src, want in rec["sources"].items():
        with open(os.path.join(ROOT, "long_context_indexing_b200", "csrc", src), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != want:
                return None
    return rec


# --------------------------------------------------------------- the oracle --

class OracleRun:
    """The CPU oracle on a bounded query sample of a prefill workload."""

    def __init__(self, w, inp, T_old):
        import oracle
        self.oracle = oracle
        self.w = w
        self.T_old = T_old
        lat = inp["latent_K"][0].float().cpu().numpy()
        self.lat = lat
        span = w.p * w.G
        self.idx = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=(w.dtype == "bf16"))
        t = time.time()
        self.idx.extend(lat, 0, (T_old // span) * span)
        self.setup_s = time.time() - t
        self.inp = inp

    def step(self, rows):
        """Chunk step on the sampled queries: extend the chunk's blocks, select,
        attend.  Host gathers of the selected K/V rows are outside the timing."""
        o, w, inp = self.oracle, self.w, self.inp
        t0 = time.time()
        self.idx.extend(self.lat, self.T_old, w.T)
        lq = inp["latent_Q"][0][rows].float().cpu().numpy()
        pos = (self.T_old + rows.cpu().numpy()).astype(np.int64)
        sel, cnt, _, _ = o.select(self.idx, lq, pos, w.R, w.W, w.S)
        t1 = time.time()
        uniq, inv = np.unique(np.where(sel >= 0, sel, 0), return_inverse=True)
        remap = np.where(sel >= 0, inv.reshape(sel.shape), -1).astype(np.int32)
        ui = torch.from_numpy(uniq).to(inp["K"].device)
        K = inp["K"][0].index_select(0, ui).float().cpu().numpy()
        V = inp["V"][0].index_select(0, ui).float().cpu().numpy()
        Q = inp["Q"][0][rows].float().cpu().numpy()
        t2 = time.time()
        O, _ = o.attend(Q, K, V, remap, cnt, o.default_scale(w.d))
        t3 = time.time()
        return (t1 - t0) + (t3 - t2), O


def _sample_rows(w, n, device):
    stride = max(1, w.nq // n)
    return torch.arange(0, n * stride, stride, device=device)[:n]


# -------------------------------------------------------- split of one chunk --

def _query_slice(nq, rank, ws):
    """Contiguous rows [q0, q1) of an nq-query chunk for `rank` of `ws` (equal
    shares; nq must be a multiple of ws)."""
    if nq % ws:
        raise ValueError("%d chunk queries do not split evenly over %d ranks" % (nq, ws))
    n = nq // ws
    return rank * n, (rank + 1) * n


def _gather_rows(part, ws):
    """All ranks' row blocks [n][...] concatenated in rank order ([ws * n][...]),
    on every rank."""
    if ws == 1:
        return part
    part = part.contiguous()
    if torch.distributed.get_backend() == "nccl":
        out = torch.empty((ws * part.shape[0],) + tuple(part.shape[1:]), dtype=part.dtype,
                          device=part.device)
        torch.distributed.all_gather_into_tensor(out, part)
        return out
    parts = [torch.empty_like(part) for _ in range(ws)]
    torch.distributed.all_gather(parts, part)
    return torch.cat(parts, 0)


def run_lsa_split(args, rank, ws):
    """One chunk's queries split over the ranks: every rank holds the same
    (replicated) caches and index, extends the index over the whole chunk,
    selects and attends its contiguous share of the queries, and the outputs
    are all-gathered (NCCL) inside the timed step.  Strong scaling: the job is
    one chunk whatever the rank count."""
    import long_context_indexing_b200 as lsa

    w = _bench_workload(args)
    dev = torch.device("cuda")
    inp = synth.prefill_inputs(w, seed=args.seed, device=dev)      # the same chunk on every rank
    span = w.p * w.G
    T_old = w.T - w.nq
    q0, q1 = _query_slice(w.nq, rank, ws)
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if w.dtype == "bf16" else lsa.F32)
    idx.build(inp["latent_K"], (T_old // span) * span)
    lq = inp["latent_Q"][:, q0:q1].contiguous()
    Qp = inp["Q"][:, q0:q1].contiguous()
    work = torch.empty(lsa.lsa_prefill_workspace_bytes(idx, q1 - q0, w.Hq, w.Hkv, w.d, w.R, w.W,
                                                       w.S), dtype=torch.uint8, device=dev)
    Op = torch.empty_like(Qp)
    stream = torch.cuda.current_stream()
    result = {}

    def step():
        lsa.lsa_prefill_chunk_queries(idx, inp["latent_K"], lq, Qp, inp["K"], inp["V"], T_old,
                                      w.T, q0, q1, w.R, w.W, w.S, workspace=work, out=Op)
        result["O"] = _gather_rows(Op[0], ws)

    for _ in range(args.warmup):
        step()
    _barrier(ws)
    launches0 = lsa.kernel_launches()
    ms = _max_over_ranks(_events_time(step, args.steps, stream), ws)
    launches = lsa.kernel_launches() - launches0
    _barrier(ws)
    fallbacks = idx.check()
    line = {"metric": METRIC, "value": round(w.nq / (ms * 1e-3), 2), "unit": "queries/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded clustered mixture; no model weights or datasets)",
            "config": dict(_config(w, ws), parallelism="query split of one chunk over %d ranks "
                           "(replicated caches and index, outputs all-gathered)" % ws),
            "e2e": None, "gpu_launches": launches, "selection_fallbacks": fallbacks}
    if rank == 0:
        print(json.dumps(line), flush=True)


def _context_shard(T, span, rank, ws):
    """Key rows [lo, hi) of `rank`'s shard of a T-token cache: whole blocks of
    `span` tokens, as even as they come; the last shard also takes a partial
    block at the end."""
    nb = T // span
    lo = (nb * rank // ws) * span
    hi = T if rank == ws - 1 else (nb * (rank + 1) // ws) * span
    return lo, hi


def _exchange_rows(part, rank, ws):
    """Every rank's [ws * n][...] tensor cut into ws row blocks; rank j gets
    block j of every rank, stacked by source rank ([ws][n][...])."""
    if ws == 1:
        return part[None]
    part = part.contiguous()
    n = part.shape[0] // ws
    if torch.distributed.get_backend() == "nccl":
        out = torch.empty_like(part)
        torch.distributed.all_to_all_single(out, part)
        return out.view((ws, n) + tuple(part.shape[1:]))
    parts = [torch.empty_like(part) for _ in range(ws)]
    torch.distributed.all_gather(parts, part)
    return torch.stack([p[rank * n:(rank + 1) * n] for p in parts])


def run_lsa_context(args, rank, ws):
    """One chunk with the KV cache in shards of whole blocks over the ranks
    (the pages' context-parallel layout): every rank holds its shard of K and
    V, the latent keys and the full index, extends the index and selects for
    every query of the chunk (the same selection on every rank), attends over
    the selected keys of its shard (lsa_attend_key_range: output and
    log-sum-exp per query head), and the partials are exchanged by row blocks
    (NCCL all-to-all) and merged by LSE weight (lsa_merge_partials) inside the
    timed step; each rank ends with its row block of the output.  Strong
    scaling: the job is one chunk whatever the rank count."""
    import long_context_indexing_b200 as lsa

    w = _bench_workload(args)
    dev = torch.device("cuda")
    inp = synth.prefill_inputs(w, seed=args.seed, device=dev)      # the same chunk on every rank
    span = w.p * w.G
    T_old = w.T - w.nq
    lo, hi = _context_shard(w.T, span, rank, ws)
    Ks = inp["K"][:, lo:hi].contiguous()
    Vs = inp["V"][:, lo:hi].contiguous()
    del inp["K"], inp["V"]                                          # a rank keeps its shard only
    torch.cuda.empty_cache()
    q0, q1 = _query_slice(w.nq, rank, ws)
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if w.dtype == "bf16" else lsa.F32)
    idx.build(inp["latent_K"], (T_old // span) * span)
    work = torch.empty(lsa.lsa_prefill_workspace_bytes(idx, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W,
                                                       w.S), dtype=torch.uint8, device=dev)
    sel_i, sel_c = lsa.prefill_selection_views(work, w.B, w.nq, w.s_max)
    Op = torch.empty_like(inp["Q"])
    Lp = torch.empty(w.B, w.nq, w.Hq, dtype=torch.float32, device=dev)
    Om = torch.empty((q1 - q0, w.Hq, w.d), dtype=inp["Q"].dtype, device=dev)
    kr_ws = torch.empty(lsa.lsa_attend_key_range_workspace_bytes(w.B, w.nq, w.s_max),
                        dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        lsa.lsa_prefill_select(idx, inp["latent_K"], inp["latent_Q"], T_old, w.T, w.Hq, w.Hkv,
                               w.d, w.R, w.W, w.S, work)
        lsa.lsa_attend_key_range(inp["Q"], Ks, Vs, sel_i, sel_c, lo, hi, workspace=kr_ws,
                                 out=Op, lse=Lp)
        O_parts = _exchange_rows(Op[0], rank, ws)
        L_parts = _exchange_rows(Lp[0], rank, ws)
        lsa.lsa_merge_partials(O_parts, L_parts, out=Om)

    for _ in range(args.warmup):
        step()
    _barrier(ws)
    launches0 = lsa.kernel_launches()
    ms = _max_over_ranks(_events_time(step, args.steps, stream), ws)
    launches = lsa.kernel_launches() - launches0
    _barrier(ws)
    fallbacks = idx.check()
    line = {"metric": METRIC, "value": round(w.nq / (ms * 1e-3), 2), "unit": "queries/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded clustered mixture; no model weights or datasets)",
            "config": dict(_config(w, ws), parallelism="KV cache in %d shards of whole blocks "
                           "(index replicated; per-shard partials merged by LSE weight after an "
                           "all-to-all of row blocks)" % ws),
            "e2e": None, "gpu_launches": launches, "selection_fallbacks": fallbacks}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- lsa --

def _bench_workload(args):
    over = {}
    if args.T:
        over["T"] = args.T
    if args.nq:
        over["nq"] = args.nq
    return synth.workload(args.workload, **over)


def run_lsa(args, rank, ws):
    import long_context_indexing_b200 as lsa

    w = _bench_workload(args)
    torch.manual_seed(rank)
    dev = torch.device("cuda")
    inp = synth.prefill_inputs(w, seed=args.seed + rank, device=dev)
    span = w.p * w.G
    T_old = w.T - w.nq
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if w.dtype == "bf16" else lsa.F32)
    t = time.time()
    idx.build(inp["latent_K"], (T_old // span) * span)
    torch.cuda.synchronize()
    build_s = time.time() - t
    ws_bytes = lsa.lsa_prefill_workspace_bytes(idx, w.nq, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    work = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    O = torch.empty_like(inp["Q"])
    stream = torch.cuda.current_stream()

    def step():
        lsa.lsa_prefill_chunk(idx, inp["latent_K"], inp["latent_Q"], inp["Q"], inp["K"],
                              inp["V"], T_old, w.T, w.R, w.W, w.S, workspace=work, out=O)

    for _ in range(args.warmup):
        step()
    _barrier(ws)
    sampler = ClockSampler(_gpu_uuid()) if rank == 0 else None
    if sampler:
        sampler.start()
    launches0 = lsa.kernel_launches()
    if sampler:
        sampler.mark("t0")
    ms = _events_time(step, args.steps, stream)
    if sampler:
        sampler.mark("t1")
    launches = lsa.kernel_launches() - launches0
    _barrier(ws)
    clocks = sampler.stop() if sampler else None
    ms = _max_over_ranks(ms, ws)
    fallbacks = idx.check()

    # Stage breakdown: the chunk's two halves through their own entry points
    # (same work, same stream, same workspace), and the index extension alone.
    sel_i, sel_c = lsa.prefill_selection_views(work, w.B, w.nq, w.s_max)
    stage_ms = {
        "index_extend": _events_time(lambda: idx.extend(inp["latent_K"], T_old, w.T),
                                     args.steps, stream),
        "extend_and_select": _events_time(
            lambda: lsa.lsa_prefill_select(idx, inp["latent_K"], inp["latent_Q"], T_old, w.T,
                                           w.Hq, w.Hkv, w.d, w.R, w.W, w.S, work),
            args.steps, stream),
        "attend": _events_time(
            lambda: lsa.lsa_prefill_attend(idx, inp["Q"], inp["K"], inp["V"], T_old, w.T, w.R,
                                           w.W, w.S, work, out=O),
            args.steps, stream),
    }
    attn_ms = _max_over_ranks(stage_ms["attend"], ws)
    peaks, peak_src = _peaks()
    floor, uniq_rows, gather = _attn_floor_bytes(w, sel_i, sel_c, w.T)
    achieved = floor / (attn_ms * 1e-3) / 1e9
    bucket = w.dtype == "bf16"
    traffic = _traffic_record("prefill_attend_" + args.workload)
    roofline = {"kernel": ("lsa_prefill_attend: bucket tiles (plan, scatter, tile records, "
                           "bucket_attn_tc_kernel, merge)" if bucket
                           else "lsa_prefill_attend: attn_f32_kernel"),
                "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": "%s (copy bandwidth)" % peak_src,
                "algorithmic_bytes_per_launch": floor,
                "algorithmic_bytes": "compulsory floor: %d distinct selected K/V rows x Hkv x d "
                                     "x 2 B x 2, plus Q and O" % uniq_rows,
                "per_query_gather_bytes": gather,
                "traffic": traffic["dram_bytes_per_call"] if traffic else None,
                "launch_ms": round(attn_ms, 4)}

    # End to end through the C-ABI with host buffers (lsa_prefill_chunk_host):
    # H2D of the step's inputs from page-locked memory (the chunk's new
    # latent/K/V rows, latent queries, queries), the chunk, D2H of the output.
    h = {k: inp[k][:, T_old:w.T].cpu().contiguous().pin_memory() for k in ("latent_K", "K", "V")}
    hq = {k: inp[k].cpu().pin_memory() for k in ("latent_Q", "Q")}
    hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in list(h.values()) + list(hq.values()))
    d2h = hO.numel() * hO.element_size()

    def e2e_step():
        lsa.lsa_prefill_chunk_host(idx, h["latent_K"], h["K"], h["V"], hq["latent_Q"], hq["Q"],
                                   inp["latent_K"], inp["K"], inp["V"], inp["latent_Q"], inp["Q"],
                                   T_old, w.T, w.R, w.W, w.S, work, O, hO)

    for _ in range(2):
        e2e_step()
    _barrier(ws)
    e2e_ms = _max_over_ranks(_events_time(e2e_step, args.steps, stream), ws)

    tree = None if args.tree_super <= 0 else _tree_measure(args, w, inp, idx, T_old, stream)
    full = None if args.no_full_prefill else _full_prefill(w, inp, work, O, stream)
    bwd = None if args.backward_queries <= 0 else _backward_measure(w, inp, idx, T_old, work,
                                                                     args.backward_queries, stream)
    per_key = None if args.no_per_key else _per_key_measure(w, inp, stage_ms, stream)

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        orc = OracleRun(w, inp, T_old)
        rows = _sample_rows(w, args.cpu_queries, dev)
        t_s, O_ref = orc.step(rows)
        err = float(np.abs(O[0][rows].float().cpu().numpy() - O_ref).max())
        cpu = {"value": round(len(rows) / t_s, 3), "unit": "queries/s",
               "cores": oracle.num_threads(), "kind": "oracle",
               "sample": "%d of the %d chunk queries (every %d-th); chunk index build + selection "
                         "+ attention; prefix index built untimed in %.1f s"
                         % (len(rows), w.nq, w.nq // len(rows), orc.setup_s),
               "max_abs_diff_vs_gpu": err}

    decode = None
    if not args.no_decode:
        del inp, idx, work, O, h, hq, hO, sel_i, sel_c
        torch.cuda.empty_cache()
        decode = run_decode(args, peaks, peak_src, ws)

    value = _job_rate(w.nq, ms, ws)
    line = {"metric": METRIC, "value": round(value, 2), "unit": "queries/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded clustered mixture; no model weights or datasets)",
            "config": _config(w, ws), "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": round(_job_rate(w.nq, e2e_ms, ws), 2), "unit": "queries/s",
                    "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches, "clocks": clocks,
            "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "index_build_prefix_s": round(build_s, 3), "selection_fallbacks": fallbacks,
            "tree": tree, "full_prefill": full, "backward": bwd, "per_key": per_key,
            "decode": decode}
    if rank == 0:
        print(json.dumps(line), flush=True)


def _tree_measure(args, w, inp, idx, T_old, stream):
    """D-LSA Tree beside Flat on the chunk's index (covering all T tokens):
    level-2 build time, tree selection of the chunk's queries against Flat
    selection (lsa_select) of the same queries, and on a row sample the share
    of Flat's long-range keys that the tree's walk also keeps."""
    import long_context_indexing_b200 as lsa

    pos = torch.arange(T_old, w.T, dtype=torch.int32, device="cuda")
    pos = pos[None].expand(w.B, -1).contiguous()
    s_max = w.R + w.W + w.S
    lq = inp["latent_Q"]
    t_ws = torch.empty(lsa.lsa_tree_select_workspace_bytes(idx, w.nq, args.tree_branches),
                       dtype=torch.uint8, device="cuda")
    f_ws = torch.empty(lsa.lsa_select_workspace_bytes(idx, w.nq), dtype=torch.uint8,
                       device="cuda")
    tr = lsa.LsaTree(idx, args.tree_super, w.L)
    build_ms = _events_time(lambda: tr.build(w.L), 3, stream)
    idx.check()
    tree_sel = lambda: tr.select(lq, pos, args.tree_branches, w.R, w.W, w.S, s_max, t_ws)
    flat_sel = lambda: lsa.lsa_select(idx, lq, pos, w.R, w.W, w.S, s_max, f_ws)
    for _ in range(3):
        tree_sel()
        flat_sel()
    idx.check()
    t_ms = _events_time(tree_sel, args.steps, stream)
    fb_tree = idx.check()
    f_ms = _events_time(flat_sel, args.steps, stream)
    t_idx, t_cnt = tree_sel()
    f_idx, f_cnt = flat_sel()
    rows = _sample_rows(w, 256, "cuda")
    kept = tot = 0
    for b in range(w.B):
        for r in rows.tolist():
            p = T_old + r
            lo, hi = w.S, p - w.W                     # long-range key positions
            fr = f_idx[b, r, :int(f_cnt[b, r])]
            tr_ = t_idx[b, r, :int(t_cnt[b, r])]
            fr = fr[(fr >= lo) & (fr <= hi)]
            tr_ = tr_[(tr_ >= lo) & (tr_ <= hi)]
            tot += fr.numel()
            kept += int(torch.isin(fr, tr_).sum())
    n_buckets = idx.n_buckets_max
    return {"n_super": args.tree_super, "branches": args.tree_branches, "lloyd_iters": w.L,
            "index_buckets": n_buckets, "level2_build_ms": round(build_ms, 4),
            "select_ms": round(t_ms, 4), "flat_select_ms": round(f_ms, 4),
            "select_fallbacks": fb_tree,
            "flat_long_range_keys_kept": round(kept / max(tot, 1), 4),
            "recall_sample": "%d rows (every %d-th) of the chunk" % (len(rows), w.nq // len(rows))}


def _full_prefill(w, inp, work, O, stream):
    """One layer's whole context prefilled chunk by chunk from position 0
    (lsa_prefill_chunk over [0, chunk), [chunk, 2 chunk), ...: the index
    grows by every chunk's blocks, every chunk's queries select and attend).
    The chunks reuse the bench chunk's latent queries and queries (their
    content does not change the work); one timed pass, CUDA events."""
    import long_context_indexing_b200 as lsa

    span = w.p * w.G
    chunk = w.nq
    if w.T % chunk or chunk % span:
        return None
    idx = lsa.LsaIndex(w.B, w.T, w.p, w.G, w.k, w.L, lsa.BF16 if w.dtype == "bf16" else lsa.F32)
    idx.build(inp["latent_K"], 0)
    n = w.T // chunk
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    ev[0].record(stream)
    for c in range(n):
        lsa.lsa_prefill_chunk(idx, inp["latent_K"], inp["latent_Q"], inp["Q"], inp["K"], inp["V"],
                              c * chunk, (c + 1) * chunk, w.R, w.W, w.S, workspace=work, out=O)
        ev[c + 1].record(stream)
    ev[n].synchronize()
    per = [ev[c].elapsed_time(ev[c + 1]) for c in range(n)]
    total = ev[0].elapsed_time(ev[n])
    fb = idx.check()
    del idx
    return {"what": "whole %d-token context of one layer prefilled in %d chunks of %d queries "
                    "(index built chunk by chunk from position 0)" % (w.T, n, chunk),
            "total_ms": round(total, 2), "queries_per_s": round(w.T * w.B / (total * 1e-3), 1),
            "first_chunk_ms": round(per[0], 4), "last_chunk_ms": round(per[-1], 4),
            "selection_fallbacks": fb}


def _backward_measure(w, inp, idx, T_old, work, n, stream):
    """Gradients of the attention over stored selections (lsa_sparse_attn_backward)
    for n of the chunk's queries (every (nq/n)-th): their selections from a
    fresh chunk call, the forward's O and lse from lsa_sparse_attn, a random
    upstream gradient, fp32 dK / dV accumulators over the whole cache.  One
    timed call after one untimed one, CUDA events."""
    import long_context_indexing_b200 as lsa

    lsa.lsa_prefill_chunk(idx, inp["latent_K"], inp["latent_Q"], inp["Q"], inp["K"], inp["V"],
                          T_old, w.T, w.R, w.W, w.S, workspace=work)
    sel_i, sel_c = lsa.prefill_selection_views(work, w.B, w.nq, w.s_max)
    rows = _sample_rows(w, n, "cuda")
    Qs = inp["Q"][:, rows].contiguous()
    ii = sel_i[:, rows].contiguous()
    cc = sel_c[:, rows].contiguous()
    O, lse = lsa.lsa_sparse_attn(Qs, inp["K"], inp["V"], ii, cc, return_lse=True)
    gen = torch.Generator(device="cuda").manual_seed(0)
    dO = torch.randn(Qs.shape, generator=gen, device="cuda").to(Qs.dtype)
    dK = torch.zeros(inp["K"].shape, dtype=torch.float32, device="cuda")
    dV = torch.zeros_like(dK)
    lsa.lsa_sparse_attn_backward(Qs, inp["K"], inp["V"], O, lse, dO, ii, cc, dK=dK, dV=dV)
    ms = _events_time(lambda: lsa.lsa_sparse_attn_backward(Qs, inp["K"], inp["V"], O, lse, dO,
                                                           ii, cc, dK=dK, dV=dV), 1, stream)
    keys = int(cc.sum().item())
    del dK, dV
    torch.cuda.empty_cache()
    return {"what": "gradients of the attention over stored selections for %d of the chunk's "
                    "queries (every %d-th), fp32 dK/dV accumulators" % (len(rows), w.nq // len(rows)),
            "ms": round(ms, 3), "queries_per_s": round(len(rows) / (ms * 1e-3), 1),
            "selected_keys": keys}


def _per_key_measure(w, inp, stage_ms, stream):
    """The brute-force latent per-key indexer (lsa_select_per_key) on the same
    chunk: every long-range key of each of the chunk's queries scored on the
    tensor cores (two passes), the exact top-R read, emitted like the bucket
    selection.  One timed call after one untimed one, CUDA events; compared
    with the bucket selection and attention stages of the chunk."""
    import long_context_indexing_b200 as lsa

    pos = inp["positions"].to(torch.int32).contiguous()
    sel = lsa.lsa_select_per_key(inp["latent_K"], inp["latent_Q"], pos, w.R, w.W, w.S)
    work = sel[2]
    fb = lsa.lsa_select_per_key_check(work)
    ms = _events_time(lambda: lsa.lsa_select_per_key(inp["latent_K"], inp["latent_Q"], pos, w.R,
                                                     w.W, w.S, workspace=work), 1, stream)
    fb = max(fb, lsa.lsa_select_per_key_check(work))
    # scores per pass: every query against its long-range keys [S, pos - W]
    scored = int((pos.to(torch.int64) - w.W - w.S + 1).clamp(min=0).sum().item())
    flops = 2 * 2.0 * scored * 64
    sel_ms, att_ms = stage_ms.get("extend_and_select"), stage_ms.get("attend")
    del sel, work
    torch.cuda.empty_cache()
    return {"what": "brute-force latent per-key indexer over the chunk's %d queries: every "
                    "long-range key scored on the tensor cores (two passes), exact top-%d by "
                    "binary64 rescoring, the baseline the bucket selection replaces" % (w.nq, w.R),
            "ms": round(ms, 3), "queries_per_s": round(w.B * w.nq / (ms * 1e-3), 1),
            "keys_scored_per_pass": scored, "tensor_tflops_effective": round(flops / ms * 1e-9, 1),
            "fallbacks": int(fb),
            "vs_bucket_selection": round(ms / sel_ms, 2) if sel_ms else None,
            "indexer_share_with_bucket_attention": round(ms / (ms + att_ms), 3) if att_ms else None}


# ------------------------------------------------------------------- decode --

def run_decode(args, peaks, peak_src, ws=1):
    """Decode workload: 8 sequences of 1,048,576-token context, one new token
    per sequence per step, 256 steps captured once in a CUDA graph and
    replayed.  Each step appends the token (and, every p-th token, the
    completed pooled group), selects 4096 + 512 + 4 keys and attends over them.
    Replays are idempotent: they rewrite the same rows and re-derive the same
    open-list entries."""
    import long_context_indexing_b200 as lsa

    w = synth.workload("decode", **({"T": args.decode_T} if args.decode_T else {}))
    dev = torch.device("cuda")
    span = w.p * w.G
    t_cap = w.T + span                      # room for the open block
    inp = synth.decode_inputs(w, seed=args.seed, device=dev, t_cap=t_cap)
    idx = lsa.LsaIndex(w.B, t_cap, w.p, w.G, w.k, w.L, lsa.BF16)
    idx.build(inp["latent_K"], w.T)
    pos = (w.T + torch.arange(w.steps, device=dev, dtype=torch.int32))[:, None]
    pos = pos.expand(w.steps, w.B).contiguous()
    O = torch.empty(w.steps, w.B, w.Hq, w.d, dtype=torch.bfloat16, device=dev)
    ws_bytes = lsa.lsa_decode_workspace_bytes(idx, w.Hq, w.Hkv, w.d, w.R, w.W, w.S)
    work = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step(s):
        lsa.lsa_decode_step(idx, inp["latent_K"], inp["K"], inp["V"], inp["new_latent_k"][s],
                            inp["new_k"][s], inp["new_v"][s], inp["latent_q"][s], inp["q"][s],
                            pos[s], w.R, w.W, w.S, workspace=work, out=O[s])

    for s in range(w.steps):                # eager warm-up pass
        step(s)
    torch.cuda.synchronize()
    idx.check()
    l0 = lsa.kernel_launches()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for s in range(w.steps):
            step(s)
    launches_per_step = (lsa.kernel_launches() - l0) / w.steps
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    reps = max(1, args.steps // 2)
    ms = _events_time(graph.replay, reps, stream)
    us = _max_over_ranks(1e3 * ms / w.steps, ws)
    fallbacks = idx.check()
    _, counts = lsa.decode_selection_views(work, w.B, w.s_max)
    n_sel = int(counts.sum().item())
    kv = n_sel * w.Hkv * w.d * 2 * 2
    qo = w.B * w.Hq * w.d * 2 * 2
    cent = w.B * (w.T // span) * w.k * 64 * 2
    alg = kv + qo + cent + n_sel * 4
    achieved = alg / (us * 1e-6) / 1e9
    del graph
    cpu = None
    if not args.no_cpu_baseline and (not torch.distributed.is_initialized()
                                     or torch.distributed.get_rank() == 0):
        cpu = _decode_cpu_baseline(w, inp, t_cap, args.cpu_decode_steps)
    return {"value": round(us, 3), "unit": "µs/step", "higher_is_better": False,
            "cpu_baseline": cpu,
            "workload": "D-LSA Flat decode: %d sequences x %d-token context, 1 query/sequence/step, "
                        "%d steps in one CUDA graph, replayed %d times" % (w.B, w.T, w.steps, reps),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "peak_source": "%s (copy bandwidth)" % peak_src,
                         "algorithmic_bytes_per_step": alg},
            "gpu_launches_per_step": launches_per_step,
            "selection_fallbacks": fallbacks}


def _decode_cpu_baseline(w, inp, t_cap, steps):
    """The oracle on the decode workload's first `steps` steps for all
    sequences: per step and sequence, the append of the new key, the selection
    and the attention (host gathers of the selected K/V rows untimed)."""
    import oracle
    orcs, lats = [], []
    t = time.time()
    for b in range(w.B):
        lat = inp["latent_K"][b, :w.T + steps].float().cpu().numpy()
        o = oracle.Index(t_cap, w.p, w.G, w.k, w.L, rt_bf16=True)
        o.extend(lat, 0, w.T)
        orcs.append(o)
        lats.append(lat)
    setup_s = time.time() - t
    timed = 0.0
    for s in range(steps):
        for b in range(w.B):
            t0 = time.time()
            orcs[b].append(lats[b], w.T + s + 1)
            sel, cnt, _, _ = oracle.select(orcs[b], inp["latent_q"][s][b:b + 1].float().cpu().numpy(),
                                           np.array([w.T + s]), w.R, w.W, w.S)
            t1 = time.time()
            uniq, inv = np.unique(np.where(sel >= 0, sel, 0), return_inverse=True)
            remap = np.where(sel >= 0, inv.reshape(sel.shape), -1).astype(np.int32)
            ui = torch.from_numpy(uniq).to(inp["K"].device)
            K = inp["K"][b].index_select(0, ui).float().cpu().numpy()
            V = inp["V"][b].index_select(0, ui).float().cpu().numpy()
            q = inp["q"][s][b:b + 1].float().cpu().numpy()
            t2 = time.time()
            oracle.attend(q, K, V, remap, cnt, oracle.default_scale(w.d))
            timed += (t1 - t0) + (time.time() - t2)
    return {"value": round(1e6 * timed / steps, 1), "unit": "µs/step",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "the first %d of the %d decode steps, all %d sequences (append, selection, "
                      "attention); per-sequence prefix indices built untimed in %.1f s"
                      % (steps, w.steps, w.B, setup_s)}


# ---------------------------------------------------------------- reference --

def run_reference(args, rank, ws):
    if rank != 0:
        return
    import oracle
    w = _bench_workload(args)
    dev = torch.device("cuda") if torch.cuda.is_available() else torch.device("cpu")
    inp = synth.prefill_inputs(w, seed=args.seed, device=dev)
    T_old = w.T - w.nq
    orc = OracleRun(w, inp, T_old)
    rows = _sample_rows(w, args.ref_queries, dev)
    for _ in range(args.warmup):
        orc.step(rows)
    times = [orc.step(rows)[0] for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = len(rows) / t
    sample = ("%d of the %d chunk queries per step (every %d-th): chunk index build + selection "
              "+ attention" % (len(rows), w.nq, w.nq // len(rows)))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "queries/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, ws),
            "cpu_baseline": {"value": round(value, 3), "unit": "queries/s",
                             "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["lsa", "reference"], default="lsa")
    ap.add_argument("--workload", default="10m", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--T", type=int, default=None, help="override the context length")
    ap.add_argument("--nq", type=int, default=None, help="override the chunk query count")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-queries", type=int, default=256)
    ap.add_argument("--cpu-decode-steps", type=int, default=4)
    ap.add_argument("--ref-queries", type=int, default=32)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--backward-queries", type=int, default=512,
                    help="queries of the chunk whose attention gradients are timed (0: skip)")
    ap.add_argument("--no-per-key", action="store_true",
                    help="skip the brute-force per-key indexer measurement")
    ap.add_argument("--no-full-prefill", action="store_true",
                    help="skip the whole-context chunk-by-chunk prefill measurement")
    ap.add_argument("--tree-super", type=int, default=256,
                    help="D-LSA Tree beside Flat: super-buckets of level 2 (0: skip)")
    ap.add_argument("--tree-branches", type=int, default=16,
                    help="D-LSA Tree beside Flat: super-buckets a query walks")
    ap.add_argument("--decode-T", type=int, default=None,
                    help="override the decode context length (a multiple of p * block)")
    ap.add_argument("--split", choices=["chunks", "queries", "context"], default="chunks",
                    help="several GPUs: every rank runs its own chunk (weak scaling), one "
                         "chunk's queries are split over the ranks, or the KV cache is held in "
                         "shards over the ranks (both strong scaling)")
    ap.add_argument("--per-key-only", action="store_true",
                    help="run only the per-key indexer measurement on the workload's chunk")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode measurement (prints its object)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, ws = _dist()
    try:
        if args.decode_only:
            peaks, src = _peaks()
            out = run_decode(args, peaks, src, ws)
            if rank == 0:
                print(json.dumps(out), flush=True)
        elif args.per_key_only:
            w = _bench_workload(args)
            inp = synth.prefill_inputs(w, args.seed, "cuda")
            out = _per_key_measure(w, inp, {}, torch.cuda.current_stream())
            if rank == 0:
                print(json.dumps(out), flush=True)
        elif args.impl == "reference":
            run_reference(args, rank, ws)
        elif args.split == "queries":
            run_lsa_split(args, rank, ws)
        elif args.split == "context":
            run_lsa_context(args, rank, ws)
        else:
            run_lsa(args, rank, ws)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
