"""The bucket selection's exactness check, restated on the CPU.

The tensor-core scorer only nominates (k_score_tc.cu, k_select.cu): with s~ an
approximation of every bucket's exact score s (binary64) and
|s~ - s| <= eps = 2^-12 ||q||_1 (centroid entries are at most 1), theta is
the m-th largest maximum of s~ over groups of gw consecutive buckets, each
maximum rounded down to fp16; the list holds every bucket with s~ >= theta up
to its capacity, and tau = max(theta, the largest s~ that found the list
full).  The fill ranks the listed buckets by exact score (desc, lower id on
ties), takes whole buckets while they fit the budget and the next one in part,
and accepts the result only when the last bucket it touched has an exact score
above tau + eps and the listed buckets did not run out while other buckets
still hold available keys; otherwise the row takes the exhaustive fallback.

This test checks, with numpy and independently of the kernels, that every
accepted result equals the exhaustive selection, on approximations pushed to
the worst case the bound allows, with empty buckets, tied scores and lists
that overflow; and that the check accepts the ordinary cases.
"""
import zlib

import numpy as np
import pytest

EPS_SHIFT = -12


def _fill(order, avail, R):
    """(bucket, keys taken) of a greedy fill over buckets in `order`."""
    out, rem = [], R
    for g in order:
        if rem <= 0:
            break
        a = int(avail[g])
        if a == 0:
            continue
        take = min(a, rem)
        out.append((int(g), take))
        rem -= take
    return out


def _rank(ids, exact):
    ids = np.asarray(ids)
    return ids[np.lexsort((ids, -exact[ids]))]


def _select(exact, approx, avail, R, gw, m, cap, eps):
    nb = exact.size
    ng = (nb + gw - 1) // gw
    gm = np.full(ng * gw, -np.inf)
    gm[:nb] = approx
    gmax = gm.reshape(ng, gw).max(axis=1).astype(np.float32)
    g16 = gmax.astype(np.float16)
    down = g16.astype(np.float32) > gmax                 # round down, as __float2half_rd
    g16[down] = np.nextafter(g16[down], np.float16(-np.inf))
    theta = float(np.sort(g16.astype(np.float64))[::-1][m - 1]) if ng > m else -np.inf
    hit = np.nonzero(approx >= theta)[0]
    listed, lost = hit[:cap], hit[cap:]
    tau = max(theta, float(approx[lost].max())) if lost.size else theta
    taken = _fill(_rank(listed, exact), avail, R)
    if not taken:
        return None
    if sum(n for _, n in taken) < min(R, int(avail.sum())):
        return None                                      # the list ran out: fallback
    cut = taken[-1][0]
    return taken if exact[cut] > tau + eps else None    # None: the exhaustive fallback


def _case(rng, case, nb):
    """exact scores, eps and the budget of one trial."""
    if case == "overflow":
        # 150 medium buckets at the lowest ids fill the list before the 200
        # best buckets, at high ids, are reached: the best ones are lost
        exact = rng.uniform(-1.0, 0.2, nb)
        exact[:150] = 0.5 + 0.01 * rng.random(150)
        exact[3000:3200] = 0.9 + 0.01 * rng.random(200)
        return exact, 1e-4, 1024
    C = rng.standard_normal((nb, 64))
    C /= np.linalg.norm(C, axis=1, keepdims=True)
    if case == "ties":
        C[:] = C[:1]
    q = rng.standard_normal(64)
    # a budget of about 48 buckets puts the cut next to theta (the 48th group maximum)
    R = 6144 if case == "push" else 1024
    return C @ q, np.ldexp(np.abs(q).sum(), EPS_SHIFT), R


@pytest.mark.parametrize("case", ["random", "push", "empty", "ties", "overflow"])
def test_accepted_selections_equal_the_exhaustive_one(case):
    rng = np.random.default_rng(zlib.crc32(case.encode()))
    nb, gw, m, cap = 4096, 16, 48, 128
    accepted = 0
    trials = 100
    for trial in range(trials):
        exact, eps, R = _case(rng, case, nb)
        avail = rng.integers(0, 257, nb)
        if case == "empty":
            avail[rng.random(nb) < 0.5] = 0
        ref = _fill(_rank(np.arange(nb), exact), avail, R)
        if case in ("push", "ties", "overflow"):
            # the worst the bound allows: the exhaustive choice scored eps low, the rest eps high
            chosen = np.zeros(nb, bool)
            chosen[[g for g, _ in ref]] = True
            approx = (exact + np.where(chosen, -eps, eps)).astype(np.float32)
        else:
            approx = (exact + rng.uniform(-eps, eps, nb)).astype(np.float32)
        got = _select(exact, approx, avail, R, gw, m, cap, eps)
        if got is not None:
            accepted += 1
            assert got == ref, (case, trial)
    if case in ("random", "empty"):
        assert accepted >= 0.9 * trials, accepted        # ordinary rows need no fallback
    if case == "push":
        assert accepted >= 0.5 * trials, accepted        # the check still accepts most rows
