"""Seeded synthetic workloads shaped like the pages' D-LSA Flat experiments.

This module is shared by the tests, the smoke check and the benchmark, and by
both sides of every parity check.  It holds none of the method's arithmetic:
it only draws inputs (a clustered latent/key mixture, values and queries) and
states each workload's sizes.

Workload shape, from "Latent Sparse Attention: un indice gerarchico per
contesti lunghi" (paragraph on the read budget: a 64-dimensional index,
4096 long-range keys, 512 recent keys, 4 sinks; 2048 long-range keys for the
GLM runs below 1M) and from "Prefrontal's Latent Sparse Attention speeds up
one attention layer 72x at 10M tokens ..." (section "The numbers, and which
ones to quote": the last 32k query chunk of a 10M-token context).  The pages
measure on real prompts that are not available here; this clustered mixture
stands in for them.

Recipe (identical on every device; the stream depends on the device):
  * M centres per space, rows of N(0, I) scaled to unit norm:
    C_lat [M][64] for the latent index space and C_k [Hkv][M][d] per KV head.
  * The context is cut into topic segments of SEG = 64 tokens; segment r of
    sequence b takes one uniform centre id m_r.  Token t of segment r:
      latent_k = C_lat[m_r] + (sigma / sqrt(64)) * eps
      K[t][g]  = C_k[g][m_r] + (sigma / sqrt(d)) * eps
      V[t][g]  ~ N(0, 1)
    sigma = 0.3 is the total noise norm.
  * Each query draws its own uniform centre m_q:
      latent_q = C_lat[m_q] + (sigma / sqrt(64)) * eps
      Q[h]     = beta * (C_k[h // (Hq / Hkv)][m_q] + (sigma / sqrt(d)) * eps),
    beta = 8 * sqrt(d), so that a matching key's scaled logit is about 8.
  * bf16 workloads round every array to bf16 (round to nearest even) after
    drawing it in fp32.
Tokens are drawn in slices of SLICE tokens, so large contexts never hold more
than one slice of fp32 temporaries.
"""
import math
from dataclasses import dataclass, replace

import torch

SEG = 64
SLICE = 1 << 19
SIGMA = 0.3
LATENT_DIM = 64


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # context length per sequence (keys 0 .. T-1 exist)
    nq: int           # queries per sequence: positions T-nq .. T-1
    B: int            # independent sequences
    Hq: int
    Hkv: int
    d: int
    M: int            # mixture centres
    p: int            # pool size
    G: int            # pooled groups per block
    k: int            # buckets per block
    L: int            # Lloyd iterations
    R: int            # long-range budget (keys)
    W: int            # recent window (keys)
    S: int            # sink keys
    dtype: str        # "f32" or "bf16"
    steps: int = 0    # decode steps (decode workload only)

    @property
    def s_max(self):
        return self.R + self.W + self.S

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    # Tiny fp32 prefill: whole index over 8 blocks, last 256 positions query.
    "tiny": Workload("tiny", T=8192, nq=256, B=1, Hq=4, Hkv=1, d=64, M=64, p=4, G=256,
                     k=8, L=3, R=512, W=64, S=4, dtype="f32"),
    # 128k bf16 prefill, last 4096 positions query.
    "128k": Workload("128k", T=131072, nq=4096, B=1, Hq=16, Hkv=2, d=128, M=4096, p=4,
                     G=1024, k=16, L=3, R=4096, W=512, S=4, dtype="bf16"),
    # 1M bf16 prefill with the GLM-style 2048-key long-range budget.
    "1m": Workload("1m", T=1048576, nq=32768, B=1, Hq=32, Hkv=4, d=128, M=16384, p=4,
                   G=1024, k=16, L=3, R=2048, W=512, S=4, dtype="bf16"),
    # 10M bf16 prefill: the last 32k chunk of a 10M-token context.
    "10m": Workload("10m", T=10485760, nq=32768, B=1, Hq=32, Hkv=4, d=128, M=65536, p=4,
                    G=1024, k=16, L=3, R=4096, W=512, S=4, dtype="bf16"),
    # Decode: 8 sequences of 1M context, one new token each per step, 256 steps.
    # T counts the prefix only; each sequence holds T + steps keys at the end.
    "decode": Workload("decode", T=1048576, nq=1, B=8, Hq=32, Hkv=4, d=128, M=16384, p=4,
                       G=1024, k=16, L=3, R=4096, W=512, S=4, dtype="bf16", steps=256),
}


def workload(name, **overrides):
    """A named workload, optionally with some fields replaced (smaller T for tests)."""
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _unit_rows(x):
    return x / x.norm(dim=-1, keepdim=True)


class Mixture:
    """Centres and segment labels of one workload (fp32, on `device`)."""

    def __init__(self, w: Workload, seed=0, device="cpu", t_total=None):
        self.w = w
        self.device = torch.device(device)
        self.gen = _gen(self.device, seed)
        g = self.gen
        self.t_total = t_total if t_total is not None else w.T
        self.C_lat = _unit_rows(torch.randn(w.M, LATENT_DIM, generator=g, device=self.device))
        self.C_k = _unit_rows(torch.randn(w.Hkv, w.M, w.d, generator=g, device=self.device))
        n_seg = (self.t_total + SEG - 1) // SEG
        self.seg_centre = torch.randint(0, w.M, (w.B, n_seg), generator=g, device=self.device)

    def keys(self, out_latent, out_k, out_v):
        """Fills latent_K [B][T][64], K and V [B][T][Hkv][d] (any float dtype,
        any device) for tokens 0 .. t_total-1, slice by slice."""
        w, g, dev = self.w, self.gen, self.device
        sl, sk = SIGMA / math.sqrt(LATENT_DIM), SIGMA / math.sqrt(w.d)
        for b in range(w.B):
            for t0 in range(0, self.t_total, SLICE):
                t1 = min(t0 + SLICE, self.t_total)
                n = t1 - t0
                ids = self.seg_centre[b, t0 // SEG: (t1 + SEG - 1) // SEG]
                ids = ids.repeat_interleave(SEG)[(t0 % SEG): (t0 % SEG) + n]
                lk = self.C_lat[ids] + sl * torch.randn(n, LATENT_DIM, generator=g, device=dev)
                kk = self.C_k[:, ids].transpose(0, 1) + sk * torch.randn(
                    n, w.Hkv, w.d, generator=g, device=dev)
                vv = torch.randn(n, w.Hkv, w.d, generator=g, device=dev)
                out_latent[b, t0:t1].copy_(lk.to(out_latent.dtype))
                out_k[b, t0:t1].copy_(kk.to(out_k.dtype))
                out_v[b, t0:t1].copy_(vv.to(out_v.dtype))

    def queries(self, n):
        """latent_Q [B][n][64] and Q [B][n][Hq][d] in fp32 (round to the
        workload dtype before use)."""
        w, g, dev = self.w, self.gen, self.device
        m_q = torch.randint(0, w.M, (w.B, n), generator=g, device=dev)
        sl, sk = SIGMA / math.sqrt(LATENT_DIM), SIGMA / math.sqrt(w.d)
        lq = self.C_lat[m_q] + sl * torch.randn(w.B, n, LATENT_DIM, generator=g, device=dev)
        kv_of_head = torch.arange(w.Hq, device=dev) // (w.Hq // w.Hkv)
        base = self.C_k[kv_of_head][:, m_q]            # [Hq][B][n][d]
        base = base.permute(1, 2, 0, 3)                # [B][n][Hq][d]
        beta = 8.0 * math.sqrt(w.d)
        q = beta * (base + sk * torch.randn(w.B, n, w.Hq, w.d, generator=g, device=dev))
        return lq, q


def prefill_inputs(w: Workload, seed=0, device="cpu"):
    """All inputs of a prefill workload, in the workload dtype, on `device`.

    Returns a dict with latent_K [B][T][64], K, V [B][T][Hkv][d],
    latent_Q [B][nq][64], Q [B][nq][Hq][d] and positions [B][nq] (int64,
    T-nq .. T-1)."""
    dt = w.torch_dtype
    mix = Mixture(w, seed, device)
    dev = mix.device
    latent_K = torch.empty(w.B, w.T, LATENT_DIM, dtype=dt, device=dev)
    K = torch.empty(w.B, w.T, w.Hkv, w.d, dtype=dt, device=dev)
    V = torch.empty(w.B, w.T, w.Hkv, w.d, dtype=dt, device=dev)
    mix.keys(latent_K, K, V)
    lq, q = mix.queries(w.nq)
    pos = torch.arange(w.T - w.nq, w.T, device=dev, dtype=torch.int64).expand(w.B, w.nq)
    return dict(latent_K=latent_K, K=K, V=V, latent_Q=lq.to(dt).contiguous(),
                Q=q.to(dt).contiguous(), positions=pos.contiguous())


def decode_inputs(w: Workload, seed=0, device="cpu", t_cap=None):
    """Inputs of a decode workload: caches sized T + steps per sequence, holding
    the prefix keys (0 .. T-1) AND the keys each step will append (T .. T+steps-1,
    also returned separately as the per-step new rows), plus one query per
    sequence per step.

    Returns a dict with latent_K [B][t_cap][64], K, V [B][t_cap][Hkv][d] (rows
    from T + steps on are zero; t_cap defaults to T + steps),
    new_latent_k [steps][B][64], new_k / new_v [steps][B][Hkv][d],
    latent_q [steps][B][64], q [steps][B][Hq][d]."""
    dt = w.torch_dtype
    t_all = w.T + w.steps
    t_cap = max(t_cap or t_all, t_all)
    mix = Mixture(w, seed, device, t_total=t_all)
    dev = mix.device
    latent_K = torch.zeros(w.B, t_cap, LATENT_DIM, dtype=dt, device=dev)
    K = torch.zeros(w.B, t_cap, w.Hkv, w.d, dtype=dt, device=dev)
    V = torch.zeros(w.B, t_cap, w.Hkv, w.d, dtype=dt, device=dev)
    mix.keys(latent_K, K, V)
    lq, q = mix.queries(w.steps)          # [B][steps][...]
    new_lat = latent_K[:, w.T:t_all].transpose(0, 1).contiguous()
    new_k = K[:, w.T:t_all].transpose(0, 1).contiguous()
    new_v = V[:, w.T:t_all].transpose(0, 1).contiguous()
    return dict(latent_K=latent_K, K=K, V=V, new_latent_k=new_lat, new_k=new_k, new_v=new_v,
                latent_q=lq.to(dt).transpose(0, 1).contiguous(),
                q=q.to(dt).transpose(0, 1).contiguous())
