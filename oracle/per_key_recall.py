"""Recall of the bucket selection against the brute-force per-key indexer.

TEST INFRASTRUCTURE / ANALYSIS ONLY (CPU, oracle functions only).  For a
sample of a workload's chunk queries, both indexers fill the same long-range
budget; the recall is the fraction of the per-key indexer's long-range keys
that the bucket selection also reads.

usage: python -m oracle.per_key_recall [workload] [T] [queries] [seed]
"""
import sys

import numpy as np

import oracle
import synth


def main(argv):
    name = argv[1] if len(argv) > 1 else "1m"
    T = int(argv[2]) if len(argv) > 2 else 131072
    nq_sample = int(argv[3]) if len(argv) > 3 else 32
    seed = int(argv[4]) if len(argv) > 4 else 0
    w = synth.workload(name, T=T, nq=4096, B=1)
    inp = synth.prefill_inputs(w, seed, "cpu")
    lat = inp["latent_K"][0].float().numpy()
    idx = oracle.Index(w.T, w.p, w.G, w.k, w.L, rt_bf16=(w.dtype == "bf16"))
    idx.extend(lat, 0, w.T)
    rows = np.linspace(0, w.nq - 1, nq_sample).astype(np.int64)
    q = inp["latent_Q"][0].float().numpy()[rows]
    if w.dtype == "bf16":
        q = oracle.round_bf16(q)
    pos = inp["positions"][0].numpy()[rows]
    bi, bc, _, _ = oracle.select(idx, q, pos, w.R, w.W, w.S)
    ki, kc = oracle.select_per_key(lat, q, pos, w.R, w.W, w.S)
    r = oracle.recall(bi, bc, ki, kc, pos, w.S, w.W)
    print("workload %s, T=%d, budget %d, window %d, sinks %d, p=%d, block %d, %d buckets/block: "
          "%d queries, recall of the per-key top-%d: mean %.4f, min %.4f, max %.4f"
          % (name, w.T, w.R, w.W, w.S, w.p, w.G, w.k, len(rows), w.R, r.mean(), r.min(), r.max()))


if __name__ == "__main__":
    main(sys.argv)
