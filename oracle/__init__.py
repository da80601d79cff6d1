"""CPU oracle for D-LSA Flat: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (``long_context_indexing_b200``) never imports it and shares no code with
it; the two meet only through the seeded generators in ``synth``.

The arithmetic lives in ``lsa_oracle.c`` (plain C, binary64 reductions,
OpenMP over blocks and queries); this module marshals numpy arrays and
composes the C primitives into the per-sequence index, selection, attention
and decode-append steps.  Every function cites the passage it restates:

  [P4] "Prefrontal's Latent Sparse Attention speeds up one attention layer 72x
       at 10M tokens; end to end, the gain is 9x", section "What it changes"
       (attention is unchanged, the index only decides which keys are read).
  [P5] "Latent Sparse Attention: un indice gerarchico per contesti lunghi",
       paragraphs on index construction, on retrieval and on the read budget.

Parity is pinned for every function by ``tests/test_oracle_*.py`` (closed
forms, hand-built clusters, brute force on tiny inputs, full causal attention
when the budget covers every key).
"""
import ctypes
import math
import os

import numpy as np

from . import _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.orc_pool.argtypes = [P, I64, I, I, P]
        lib.orc_pool.restype = None
        lib.orc_unit.argtypes = [P, I64, I, P]
        lib.orc_unit.restype = None
        lib.orc_kmeans_block.argtypes = [P, I, I, I, I, P, P, P]
        lib.orc_kmeans_block.restype = I
        lib.orc_build_blocks.argtypes = [P, I, I, I, I, I, I, I64, I64,
                                         P, P, P, P, P, P, P, P]
        lib.orc_build_blocks.restype = I
        lib.orc_open_assign.argtypes = [P, I, I, I, I, I64, I64, P, P, P, P]
        lib.orc_open_assign.restype = I
        lib.orc_select.argtypes = [P, I, P, I64, I64, P, P, P, P, I64, I,
                                   I, I, I, I, I, P, P, P, P]
        lib.orc_select.restype = I
        lib.orc_tree_select.argtypes = [P, I, P, I64, I64, P, P, P, P, I64, I, I64, P, P, P,
                                        I, I, I, I, I, I, P, P]
        lib.orc_tree_select.restype = I
        lib.orc_attend.argtypes = [P, P, P, I64, I64, I, I, I, P, P, I,
                                   ctypes.c_double, P, P]
        lib.orc_attend.restype = I
        lib.orc_attend_backward.argtypes = [P, P, P, P, I64, I64, I, I, I, P, P, I,
                                            ctypes.c_double, P, P, P]
        lib.orc_attend_backward.restype = I
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = I
        lib.orc_set_num_threads.argtypes = [I]
        lib.orc_set_num_threads.restype = None
        _LIB = lib
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with code %d" % (what, rc))


def num_threads() -> int:
    return _lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    _lib().orc_set_num_threads(int(n))


# --------------------------------------------------------------------------
# Index [P5, index construction]
# --------------------------------------------------------------------------

def pool(lat, p):
    """Mean of p consecutive latent keys, summed left to right in binary32."""
    lat = _f32(lat)
    n, dl = lat.shape[0] // p, lat.shape[1]
    out = np.empty((n, dl), np.float32)
    _lib().orc_pool(_p(lat), n, dl, p, _p(out))
    return out


def unit(x):
    """x / ||x|| with the norm in binary64; the zero vector stays zero."""
    x = _f32(x)
    out = np.empty_like(x)
    _lib().orc_unit(_p(x), x.shape[0], x.shape[1], _p(out))
    return out


def kmeans_block(u, k, L):
    """Spherical k-means of one block: evenly spaced init, L Lloyd iterations.

    Returns (centroids [k][dl] fp32, assignment [G] int16, margin [G] fp64)."""
    u = _f32(u)
    G, dl = u.shape
    cent = np.empty((k, dl), np.float32)
    assign = np.empty(G, np.int16)
    margin = np.empty(G, np.float64)
    _check(_lib().orc_kmeans_block(_p(u), G, dl, k, L, _p(cent), _p(assign), _p(margin)),
           "kmeans_block")
    return cent, assign, margin


def round_bf16(x):
    """binary32 -> bf16 (round to nearest even) -> binary32, in numpy."""
    x = _f32(x)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(x.shape)


class Index:
    """One sequence's D-LSA Flat index, sized for t_max keys.

    Block b covers pooled ids [bG, (b+1)G), keys [bGp, (b+1)Gp).  Bucket ids
    are global: g = b*k + m.  The open block (decode-time appends) keeps a
    bucket id per completed pooled group, -1 when not yet assigned."""

    def __init__(self, t_max, p, G, k, L, rt_bf16, dl=64):
        self.p, self.G, self.k, self.L, self.dl = p, G, k, L, dl
        self.rt_bf16 = bool(rt_bf16)
        self.n_pooled_max = t_max // p
        self.n_blocks_max = self.n_pooled_max // G
        nb = self.n_blocks_max * k
        self.pooled = np.zeros((self.n_pooled_max, dl), np.float32)
        self.unit = np.zeros((self.n_pooled_max, dl), np.float32)
        self.cent = np.zeros((nb, dl), np.float32)
        self.cent_rt = np.zeros((nb, dl), np.float32)
        self.offsets = np.zeros(nb + 1, np.int32)
        self.members = np.zeros(self.n_pooled_max, np.int32)
        self.assign = np.zeros(self.n_pooled_max, np.int16)
        self.margin = np.full(self.n_pooled_max, np.inf, np.float64)
        self.n_blocks = 0
        self.open_bucket = np.full(G, -1, np.int32)

    @property
    def n_buckets(self):
        return self.n_blocks * self.k

    def extend(self, lat, t_old, t_new):
        """(Re)builds every whole block that overlaps [t_old, t_new), then
        assigns the completed pooled groups after the last whole block to the
        open lists (READING for keys after the last closed block).

        lat: [>= t_new][dl] fp32 latent keys of this sequence."""
        span = self.p * self.G
        b0, b1 = t_old // span, t_new // span
        if b0 > self.n_blocks or b1 > self.n_blocks_max:
            raise ValueError("extend would leave a gap or overflow the index")
        lat = _f32(lat)
        if b1 > b0:
            _check(_lib().orc_build_blocks(
                _p(lat), self.dl, self.p, self.G, self.k, self.L, int(self.rt_bf16), b0, b1,
                _p(self.pooled), _p(self.unit), _p(self.cent), _p(self.cent_rt),
                _p(self.offsets), _p(self.members), _p(self.assign), _p(self.margin)),
                "build_blocks")
        if b1 > self.n_blocks or b1 > b0:
            self.n_blocks = max(self.n_blocks, b1)
            self.open_bucket[:] = -1
        self.append(lat, t_new)

    def append(self, lat, t_end):
        """Assigns every completed pooled group in the open block whose keys
        are all below t_end to its nearest closed centroid (decode append)."""
        if self.n_blocks == 0:
            return
        j_end = min(t_end // self.p, (self.n_blocks + 1) * self.G)
        if j_end <= self.n_blocks * self.G:
            return
        lat = _f32(lat)
        _check(_lib().orc_open_assign(
            _p(lat), self.dl, self.p, self.G, self.k, self.n_blocks, j_end, _p(self.cent),
            _p(self.pooled), _p(self.unit), _p(self.open_bucket)), "open_assign")

    def csr(self):
        """(offsets, members) restricted to the closed blocks."""
        nb = self.n_buckets
        return self.offsets[: nb + 1].copy(), self.members[: self.n_blocks * self.G].copy()


# --------------------------------------------------------------------------
# Retrieval [P5, retrieval and read budget]
# --------------------------------------------------------------------------

def select(index, q, pos, R, W, S, s_max=None):
    """Per query: rank buckets by <q, c~_g> (desc; ties lowest g), fill R
    long-range keys greedily (whole buckets while they fit, the next one
    truncated in ascending position), add sinks and the recent window.

    Returns (indices [nq][s_max] int32, counts [nq], margin [nq], n_lr [nq])."""
    q = _f32(q)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    nq = q.shape[0]
    if s_max is None:
        s_max = R + W + S
    out = np.empty((nq, s_max), np.int32)
    cnt = np.empty(nq, np.int32)
    mg = np.empty(nq, np.float64)
    nlr = np.empty(nq, np.int32)
    ob = np.ascontiguousarray(index.open_bucket, dtype=np.int32)
    _check(_lib().orc_select(
        _p(q), index.dl, _p(pos), nq, index.n_buckets, _p(index.cent_rt), _p(index.offsets),
        _p(index.members), _p(ob), index.n_blocks * index.G, index.G, index.p, R, W, S, s_max,
        _p(out), _p(cnt), _p(mg), _p(nlr)), "select")
    return out, cnt, mg, nlr


# --------------------------------------------------------------------------
# D-LSA Tree [P4 "What it changes": clusters grouped into a hierarchy that a
# query walks down; P2 multi-level index; P5 Flat vs Tree]
# --------------------------------------------------------------------------

class Tree:
    """Level 2 of a two-level D-LSA Tree over one sequence's Flat index.

    READING (the pages give no construction): the closed buckets' fp32
    centroids are clustered like a block -- spherical k-means (kmeans_block:
    evenly spaced init, L Lloyd iterations, ties to the lowest id, an empty
    super-bucket keeps its centroid) -- into n_super super-buckets; each holds
    the ascending list of its bucket ids (CSR), and its retrieval copy is
    rounded to bf16 for bf16 indices, as the buckets' is."""

    def __init__(self, index, n_super, L):
        nb = index.n_buckets
        if not 1 <= n_super <= nb:
            raise ValueError("n_super must lie in [1, %d]" % nb)
        sup, assign, _ = kmeans_block(index.cent[:nb], n_super, L)
        self.n_super = n_super
        self.sup = sup
        self.sup_rt = round_bf16(sup) if index.rt_bf16 else sup.copy()
        self.assign = assign.astype(np.int32)
        counts = np.bincount(self.assign, minlength=n_super)
        self.offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        self.members = np.argsort(self.assign, kind="stable").astype(np.int32)


def tree_select(index, tree, q, pos, branches, R, W, S, s_max=None):
    """Per query: the `branches` best super-buckets (exact <q, c~2_h>, score
    desc, lowest id on ties), then the Flat ranking and greedy fill of their
    buckets only (see select); sinks and window as Flat.

    Returns (indices [nq][s_max] int32, counts [nq] int32)."""
    q = _f32(q)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    nq = q.shape[0]
    if s_max is None:
        s_max = R + W + S
    out = np.empty((nq, s_max), np.int32)
    cnt = np.empty(nq, np.int32)
    ob = np.ascontiguousarray(index.open_bucket, dtype=np.int32)
    _check(_lib().orc_tree_select(
        _p(q), index.dl, _p(pos), nq, index.n_buckets, _p(index.cent_rt), _p(index.offsets),
        _p(index.members), _p(ob), index.n_blocks * index.G, index.G, tree.n_super,
        _p(_f32(tree.sup_rt)), _p(tree.offsets), _p(tree.members), int(branches), index.p, R, W,
        S, s_max, _p(out), _p(cnt)), "tree_select")
    return out, cnt


# --------------------------------------------------------------------------
# Attention [P4 "What it changes"; P5 retrieval]
# --------------------------------------------------------------------------

def attend(Q, K, V, idx, cnt, scale=None):
    """Exact softmax attention of every head over its query's selected keys.

    Q [nq][Hq][d], K/V [T][Hkv][d], idx [nq][s_max], cnt [nq].
    KV head of query head h = h // (Hq // Hkv) (READING).
    Returns (O [nq][Hq][d] fp32, lse [nq][Hq] fp32)."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    nq, Hq, d = Q.shape
    T, Hkv, _ = K.shape
    if scale is None:
        scale = float(np.float32(1.0 / math.sqrt(d)))
    O = np.empty((nq, Hq, d), np.float32)
    lse = np.empty((nq, Hq), np.float32)
    _check(_lib().orc_attend(_p(Q), _p(K), _p(V), T, nq, Hq, Hkv, d, _p(idx), _p(cnt),
                             idx.shape[1], float(scale), _p(O), _p(lse)), "attend")
    return O, lse


def attend_backward(Q, K, V, dO, idx, cnt, scale=None):
    """Gradients of attend's output O for an upstream gradient dO [nq][Hq][d]
    (the selected indices kept from the forward pass): dQ [nq][Hq][d], dK and
    dV [T][Hkv][d], each summed over every query and head that read the key.
    p = softmax(scale <q, k_t>) over the query's keys; dV_t += p_t dO,
    dS_t = p_t (<dO, v_t> - sum_u p_u <dO, v_u>), dQ = scale sum_t dS_t k_t,
    dK_t += scale dS_t q; binary64 inside (lsa_oracle.c orc_attend_backward)."""
    Q, K, V, dO = _f32(Q), _f32(K), _f32(V), _f32(dO)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    nq, Hq, d = Q.shape
    T, Hkv, _ = K.shape
    if scale is None:
        scale = float(np.float32(1.0 / math.sqrt(d)))
    dQ = np.empty((nq, Hq, d), np.float32)
    dK = np.empty((T, Hkv, d), np.float32)
    dV = np.empty((T, Hkv, d), np.float32)
    _check(_lib().orc_attend_backward(_p(Q), _p(K), _p(V), _p(dO), T, nq, Hq, Hkv, d, _p(idx),
                                      _p(cnt), idx.shape[1], float(scale), _p(dQ), _p(dK),
                                      _p(dV)), "attend_backward")
    return dQ, dK, dV


def default_scale(d):
    """1/sqrt(d) rounded to binary32 (READING: the usual softmax scale)."""
    return float(np.float32(1.0 / math.sqrt(d)))


# --------------------------------------------------------------------------
# Per-key indexer: the comparison baseline LSA replaces [P4 "What it changes"]
# --------------------------------------------------------------------------

def per_key_scores(lat, q):
    """<q, latent_k[t]> for every key row of lat [n][dl]: the exact products
    summed in binary64 in ascending dimension (R10's rule, applied per key)."""
    lat = np.asarray(lat, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    s = np.zeros(lat.shape[0], np.float64)
    for d in range(lat.shape[1]):
        s += lat[:, d] * q[d]
    return s


def select_per_key(lat, q, pos, R, W, S, s_max=None):
    """Brute-force latent per-key indexer (READING of the indexer that LSA's
    bucket retrieval replaces: every earlier key scored against the query, the
    best ones read).  Per query at pos: every long-range-available key t
    (S <= t <= pos - W, R11) is scored by per_key_scores; the R best keys are
    taken (score descending, lowest position on ties).  Emitted: sinks, the
    taken keys in ascending position, the recent window ascending (R13); -1
    pads to s_max.

    lat [>= max(pos)+1][dl] latent keys of the sequence, q [nq][dl], pos [nq].
    Returns (indices [nq][s_max] int32, counts [nq] int32)."""
    q = np.asarray(q)
    pos = np.asarray(pos, dtype=np.int64)
    nq = q.shape[0]
    if s_max is None:
        s_max = R + W + S
    out = np.full((nq, s_max), -1, np.int32)
    cnt = np.zeros(nq, np.int32)
    for i in range(nq):
        p = int(pos[i])
        n_s = min(S, p + 1)
        w0 = max(p - W + 1, n_s)
        lo, hi = S, p - W                        # long-range keys [lo, hi]
        taken = np.zeros(0, np.int64)
        if hi >= lo and R > 0:
            t = np.arange(lo, hi + 1, dtype=np.int64)
            sc = per_key_scores(lat[lo:hi + 1], q[i])
            order = np.lexsort((t, -sc))         # score desc, then position asc
            taken = np.sort(t[order[:R]])
        row = np.concatenate([np.arange(n_s, dtype=np.int64), taken,
                              np.arange(w0, p + 1, dtype=np.int64)])
        out[i, :row.size] = row
        cnt[i] = row.size
    return out, cnt


def recall(sel_idx, sel_cnt, ref_idx, ref_cnt, pos, S, W):
    """Per query at pos, the fraction of the reference's long-range keys
    (S <= t <= pos - W) that the selection also reads; 1.0 where the reference
    takes none."""
    out = np.ones(len(sel_cnt), np.float64)
    for i in range(len(sel_cnt)):
        lo, hi = S, int(pos[i]) - W
        ref = {int(x) for x in ref_idx[i, :ref_cnt[i]] if lo <= x <= hi}
        if ref:
            sel = {int(x) for x in sel_idx[i, :sel_cnt[i]]}
            out[i] = len(ref & sel) / len(ref)
    return out
