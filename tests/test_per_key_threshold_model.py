"""The per-key indexer's candidate threshold, restated on the CPU.

lsa_select_per_key proves its exact top R through a threshold (k_perkey.cu):
with s~ any approximation of the exact score s (binary64) such that
|s~ - s| <= eps = 2^-12 sum_d |q_d| max_t |k_t,d| for every eligible key, take
h = the R-th largest maximum of s~ over the strided groups {t : t mod ng = c},
each maximum rounded to the nearest fp16, theta = h less half an fp16 ulp
(|h| 2^-10 + 2^-24; 65504 when h is +inf), and keep every key with
s~ >= theta - 2 eps (rounded down to binary32).  Claim: the kept keys always
hold the exact top R (score desc, lower position on ties).

This test checks the claim with numpy, independently of the kernels, on
approximations pushed to the worst case the bound allows (every top-R key
scored eps too low, every other key eps too high) and on clustered keys,
scores beyond fp16's range, scores in its subnormals and tied scores; and that
on the clustered mixture the kept set stays within the 8192-entry list.  In
the pushed cases one eligible key of large entries and a very low score makes
eps dominate fp16's rounding, so that both eps of the margin are needed.
"""
import zlib

import numpy as np
import pytest

import oracle

R, W, S = 256, 64, 4


def _mixture(rng, T, M=64, seg=64, sigma=0.3):
    C = rng.standard_normal((M, 64))
    C /= np.linalg.norm(C, axis=1, keepdims=True)
    ids = np.repeat(rng.integers(0, M, (T + seg - 1) // seg), seg)[:T]
    lat = C[ids] + sigma / 8 * rng.standard_normal((T, 64))
    q = C[rng.integers(0, M)] + sigma / 8 * rng.standard_normal(64)
    return lat.astype(np.float32), q.astype(np.float32)


def _kept(lat, q, pos, ng, push):
    lo, hi = S, pos - W
    t = np.arange(lo, hi + 1)
    exact = oracle.per_key_scores(lat[lo:hi + 1], q)              # binary64
    colmax = np.abs(lat[: pos + 1].astype(np.float64)).max(axis=0)
    eps = np.ldexp(np.sum(np.abs(q.astype(np.float64)) * colmax), -12)
    order = np.lexsort((t, -exact))
    top = np.zeros(t.size, bool)
    top[order[:R]] = True
    # the worst approximation the bound allows, rounded to binary32
    approx = exact + (np.where(top, -eps, eps) if push else 0.0)
    approx = approx.astype(np.float32)
    gmax = np.full(ng, -np.inf, np.float32)
    np.maximum.at(gmax, t % ng, approx)
    with np.errstate(over="ignore"):
        g16 = gmax.astype(np.float16)                              # nearest (inf past 65504)
    h = float(np.sort(g16.astype(np.float64))[::-1][R - 1])
    theta = 65504.0 if np.isinf(h) and h > 0 else h - (abs(h) * 2.0 ** -10 + 2.0 ** -24)
    th2 = np.float32(theta - 2 * eps)
    if th2 > theta - 2 * eps:                                      # round down
        th2 = np.nextafter(th2, np.float32(-np.inf))
    keep = approx >= th2
    return keep, top


@pytest.mark.parametrize("case", ["mixture", "mixture_push", "large", "tiny", "ties", "ties_push"])
def test_kept_keys_hold_the_exact_top_r(case):
    rng = np.random.default_rng(zlib.crc32(case.encode()))
    T, ng = 40000, 4096
    lat, q = _mixture(rng, T)
    if case == "large":
        q = (q * 4.0e5).astype(np.float32)          # group maxima beyond fp16's range
    elif case == "tiny":
        q = (q * 1.0e-5).astype(np.float32)         # group maxima among fp16 subnormals
    elif case in ("ties", "ties_push"):
        lat[:] = lat[:1]                            # every score equal
    push = case in ("mixture_push", "ties_push")
    if push:
        # a key of 50s, scoring far below every other: eps grows ~50x
        lat[S + 10] = (-50.0 * np.sign(q)).astype(np.float32)
    for pos in (T - 1, T // 2, W + S + R + 5):
        keep, top = _kept(lat, q, pos, ng, push)
        assert keep[top].all(), (case, pos)
        if case in ("mixture", "mixture_push"):
            assert keep.sum() <= 8192, (case, pos, int(keep.sum()))
