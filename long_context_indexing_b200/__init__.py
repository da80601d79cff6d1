"""Python binding of liblsa, the D-LSA Flat hot path for B200 (sm_100a).

Argument marshalling only: every step of the path runs in liblsa's CUDA
kernels.  PyTorch provides device memory and streams.  The names mirror the
C-ABI in include/lsa.h; see that header for the semantics of every call.

Method: Latent Sparse Attention in its D-LSA Flat form ("Latent Sparse
Attention: un indice gerarchico per contesti lunghi", paragraphs on index
construction, retrieval and the read budget; "Prefrontal's Latent Sparse
Attention speeds up one attention layer 72x at 10M tokens ...", section
"What it changes").
"""
import ctypes
import math
import os

import torch

__all__ = [
    "LsaError", "LsaIndex", "lsa_index_bytes", "lsa_build_index", "lsa_select",
    "lsa_select_workspace_bytes", "lsa_tree_select_workspace_bytes",
    "lsa_sparse_attn", "lsa_prefill_chunk", "lsa_prefill_workspace_bytes",
    "lsa_attend_key_range", "lsa_attend_key_range_workspace_bytes", "lsa_merge_partials",
    "lsa_sparse_attn_backward",
    "lsa_prefill_partial_slots", "lsa_prefill_select", "lsa_prefill_attend",
    "lsa_prefill_chunk_host", "lsa_prefill_chunk_queries", "LsaTree", "set_wait_limit",
    "lsa_decode_workspace_bytes", "lsa_decode_step", "lsa_select_noalloc", "library_path", "kernel_launches", "F32",
    "BF16",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblsa.so")

F32, BF16 = 0, 1
_STATUS = {0: "LSA_OK", 1: "LSA_ERR_INVALID_ARG", 2: "LSA_ERR_ALIGNMENT", 3: "LSA_ERR_WORKSPACE",
           4: "LSA_ERR_CUDA", 5: "LSA_ERR_TIMEOUT", 6: "LSA_ERR_INTERNAL",
           7: "LSA_ERR_UNSUPPORTED"}


class LsaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("%s: %s" % (_STATUS.get(code, str(code)), msg))
        self.code = code


class IndexParams(ctypes.Structure):
    _fields_ = [("p", ctypes.c_int), ("block", ctypes.c_int), ("n_buckets", ctypes.c_int),
                ("lloyd_iters", ctypes.c_int)]


class SelectParams(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_int), ("window", ctypes.c_int), ("sinks", ctypes.c_int)]


def _declare(lib):
    P, I, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                        ctypes.c_float)
    sigs = {
        "lsa_last_error": ([], ctypes.c_char_p),
        "lsa_version": ([], ctypes.c_char_p),
        "lsa_kernel_launches": ([], ctypes.c_uint64),
        "lsa_index_bytes": ([I64, I64, IndexParams, I], SZ),
        "lsa_index_init": ([P, SZ, I64, I64, IndexParams, I, ctypes.POINTER(P)], I),
        "lsa_index_release": ([P], None),
        "lsa_build_index": ([P, P, I64, P], I),
        "lsa_index_extend": ([P, P, I64, I64, P], I),
        "lsa_index_num_blocks": ([P], I64),
        "lsa_index_export": ([P, P, P, P, P, P, P, P, P, P], I),
        "lsa_index_check": ([P, ctypes.POINTER(I64), P], I),
        "lsa_select_workspace_bytes": ([P, I64], SZ),
        "lsa_select": ([P, P, P, I64, SelectParams, P, P, I, P, SZ, P], I),
        "lsa_sparse_attn": ([P, P, P, I, I64, I64, I64, I, I, I, P, P, I, F, P, P, P], I),
        "lsa_sparse_attn_backward": ([P, P, P, P, P, P, I, I64, I64, I64, I, I, I, P, P, I, F,
                                      P, P, P, P], I),
        "lsa_attend_key_range_workspace_bytes": ([I64, I64, I], SZ),
        "lsa_attend_key_range": ([P, P, P, I, I64, I64, I, I, I, P, P, I, I64, I64, F, P, SZ, P,
                                  P, P], I),
        "lsa_merge_partials": ([P, P, I, I, I64, I, I, P, P, P], I),
        "lsa_prefill_workspace_bytes": ([P, I64, I, I, I, SelectParams], SZ),
        "lsa_prefill_partial_slots": ([P, I64, I, I, I, SelectParams, SZ], I64),
        "lsa_prefill_chunk": ([P, P, P, P, P, P, I64, I64, I, I, I, SelectParams, P, SZ, P, P],
                              I),
        "lsa_prefill_select": ([P, P, P, I64, I64, I, I, I, SelectParams, P, SZ, P], I),
        "lsa_prefill_attend": ([P, P, P, P, I64, I64, I, I, I, SelectParams, P, SZ, P, P], I),
        "lsa_prefill_chunk_host": ([P, P, P, P, P, P, P, P, P, P, P, I64, I64, I, I, I,
                                    SelectParams, P, SZ, P, P, P, P], I),
        "lsa_decode_workspace_bytes": ([P, I, I, I, SelectParams], SZ),
        "lsa_set_wait_limit": ([I64], I),
        "lsa_tree_bytes": ([P, I], SZ),
        "lsa_tree_build": ([P, P, SZ, I, I, P], I),
        "lsa_tree_select_workspace_bytes": ([P, I64, I], SZ),
        "lsa_tree_export": ([P, P, I, P, P, P, P, P], I),
        "lsa_tree_select": ([P, P, I, I, P, P, I64, SelectParams, P, P, I, P, SZ, P], I),
        "lsa_prefill_chunk_queries": ([P, P, P, P, P, P, I64, I64, I64, I64, I, I, I, SelectParams,
                                       P, SZ, P, P], I),
        "lsa_select_noalloc": ([P, P, P, I64, SelectParams, P, P, I, P], I),
        "lsa_select_per_key_workspace_bytes": ([I64, I64, I64], SZ),
        "lsa_select_per_key": ([P, I, I64, I64, I64, P, P, I64, SelectParams, P, P, I, P, SZ, P],
                               I),
        "lsa_select_per_key_check": ([P, ctypes.POINTER(I64), P], I),
        "lsa_decode_step": ([P, P, P, P, P, P, P, P, P, P, I, I, I, SelectParams, P, SZ, P, P], I),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError("liblsa.so is not built; run `python -m long_context_indexing_b200._build`"
                          " (or __graft_entry__.build())")
    return _declare(ctypes.CDLL(_LIB_PATH))


_lib = _load()


def library_path():
    return _LIB_PATH


def kernel_launches():
    """Kernel launches liblsa has enqueued in this process so far."""
    return int(_lib.lsa_kernel_launches())


def _check(rc):
    if rc != 0:
        raise LsaError(rc, _lib.lsa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _hptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("tensors must be float32 or bfloat16, got %s" % t.dtype)


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def lsa_index_bytes(B, T_cap, p, block, n_buckets, lloyd_iters, dtype=BF16):
    n = _lib.lsa_index_bytes(B, T_cap, IndexParams(p, block, n_buckets, lloyd_iters), dtype)
    if n == 0:
        raise LsaError(1, _lib.lsa_last_error().decode())
    return n


class LsaIndex:
    """A D-LSA Flat content index over B sequences of capacity T_cap keys.

    The device storage is one torch uint8 buffer owned by this object; the
    library only records pointers into it."""

    def __init__(self, B, T_cap, p, block, n_buckets, lloyd_iters, dtype=BF16, device="cuda"):
        self.B, self.T_cap = int(B), int(T_cap)
        self.p, self.G, self.k, self.L = int(p), int(block), int(n_buckets), int(lloyd_iters)
        self.dtype = dtype
        self.params = IndexParams(self.p, self.G, self.k, self.L)
        nbytes = lsa_index_bytes(self.B, self.T_cap, self.p, self.G, self.k, self.L, dtype)
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        h = ctypes.c_void_p()
        _check(_lib.lsa_index_init(_ptr(self.buffer), nbytes, self.B, self.T_cap, self.params,
                                   dtype, ctypes.byref(h)))
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            _lib.lsa_index_release(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    @property
    def num_blocks(self):
        return int(_lib.lsa_index_num_blocks(self._h))

    @property
    def n_pooled(self):
        return self.T_cap // self.p

    @property
    def n_buckets_max(self):
        return (self.n_pooled // self.G) * self.k

    def build(self, latent_K, T, stream=None):
        _cuda(latent_K)
        _check(_lib.lsa_build_index(self._h, _ptr(latent_K), int(T), _stream(stream)))
        return self

    def extend(self, latent_K, T_old, T_new, stream=None):
        _cuda(latent_K)
        _check(_lib.lsa_index_extend(self._h, _ptr(latent_K), int(T_old), int(T_new),
                                     _stream(stream)))
        return self

    def export(self, stream=None):
        """Copies of the index state as torch tensors on the index's device."""
        dev = self.buffer.device
        B, NP, NBK = self.B, self.n_pooled, self.n_buckets_max
        rt = torch.bfloat16 if self.dtype == BF16 else torch.float32
        out = dict(
            pooled=torch.empty(B, NP, 64, dtype=torch.float32, device=dev),
            unit=torch.empty(B, NP, 64, dtype=torch.float32, device=dev),
            cent=torch.empty(B, NBK, 64, dtype=torch.float32, device=dev),
            cent_rt=torch.empty(B, NBK, 64, dtype=rt, device=dev),
            offsets=torch.empty(B, NBK + 1, dtype=torch.int32, device=dev),
            members=torch.empty(B, NP, dtype=torch.int32, device=dev),
            assign=torch.empty(B, NP, dtype=torch.int16, device=dev),
            open_bucket=torch.empty(B, self.G, dtype=torch.int32, device=dev),
        )
        _check(_lib.lsa_index_export(self._h, *[_ptr(out[k]) for k in (
            "pooled", "unit", "cent", "cent_rt", "offsets", "members", "assign", "open_bucket")],
            _stream(stream)))
        return out

    def check(self, stream=None):
        """Raises LsaError if a kernel recorded an error; returns the number of
        queries that took the exact selection fallback since the last check."""
        fb = ctypes.c_int64(0)
        _check(_lib.lsa_index_check(self._h, ctypes.byref(fb), _stream(stream)))
        return int(fb.value)


def lsa_build_index(latent_K, T, p, block, n_buckets, lloyd_iters=3, T_cap=None, stream=None):
    """Builds an index over keys [0, T) of latent_K [B][T_cap][64]."""
    _cuda(latent_K)
    B, cap = latent_K.shape[0], latent_K.shape[1]
    idx = LsaIndex(B, T_cap or cap, p, block, n_buckets, lloyd_iters, _dtype_code(latent_K),
                   latent_K.device)
    return idx.build(latent_K, T, stream)


def lsa_select_workspace_bytes(index, Nq):
    """Workspace bytes lsa_select needs for Nq queries per sequence."""
    return int(_lib.lsa_select_workspace_bytes(index.handle, int(Nq)))


def lsa_tree_select_workspace_bytes(index, Nq, branches):
    """Workspace bytes lsa_tree_select needs for Nq queries and `branches`."""
    return int(_lib.lsa_tree_select_workspace_bytes(index.handle, int(Nq), int(branches)))


def lsa_select(index, latent_Q, positions, budget, window, sinks, s_max=None, workspace=None,
               stream=None):
    """Per-query selection: returns (indices [B][Nq][s_max] int32, counts [B][Nq] int32)."""
    _cuda(latent_Q, positions)
    if positions.dtype != torch.int32:
        raise TypeError("positions must be int32")
    B, Nq = latent_Q.shape[0], latent_Q.shape[1]
    s_max = s_max or (budget + window + sinks)
    dev = latent_Q.device
    indices = torch.empty(B, Nq, s_max, dtype=torch.int32, device=dev)
    counts = torch.empty(B, Nq, dtype=torch.int32, device=dev)
    need = _lib.lsa_select_workspace_bytes(index.handle, Nq)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(_lib.lsa_select(index.handle, _ptr(latent_Q), _ptr(positions), Nq,
                           SelectParams(budget, window, sinks), _ptr(indices), _ptr(counts),
                           s_max, _ptr(workspace), workspace.numel(), _stream(stream)))
    return indices, counts


def lsa_select_noalloc(index, latent_Q, positions, budget, window, sinks, indices, counts,
                       stream=None):
    """lsa_select without a workspace, for callers that cannot allocate device
    memory: the outputs `indices` [B][Nq][s_max] and `counts` [B][Nq] (int32)
    are caller buffers and the scratch is the library's built-in device array
    (see include/lsa.h for its limit and for the race between overlapping
    calls)."""
    _cuda(latent_Q, positions, indices, counts)
    Nq = latent_Q.shape[1]
    _check(_lib.lsa_select_noalloc(index.handle, _ptr(latent_Q), _ptr(positions), Nq,
                                   SelectParams(budget, window, sinks), _ptr(indices),
                                   _ptr(counts), indices.shape[-1], _stream(stream)))
    return indices, counts


def lsa_select_per_key_workspace_bytes(B, Nq, T_cap):
    return int(_lib.lsa_select_per_key_workspace_bytes(B, Nq, T_cap))


def lsa_select_per_key(latent_K, latent_Q, positions, budget, window, sinks, n_keys=None,
                       s_max=None, workspace=None, stream=None):
    """Brute-force per-key indexer over latent_K [B][T_cap][64] (keys
    0 .. n_keys-1, default T_cap) for latent_Q [B][Nq][64] at positions
    [B][Nq] (int32).  Returns (indices [B][Nq][s_max] int32, counts [B][Nq]
    int32, workspace); lsa_select_per_key_check(workspace) reads the call's
    status and fallback count."""
    _cuda(latent_K, latent_Q, positions)
    if positions.dtype != torch.int32:
        raise TypeError("positions must be int32")
    B, T_cap = latent_K.shape[0], latent_K.shape[1]
    Nq = latent_Q.shape[1]
    n_keys = T_cap if n_keys is None else int(n_keys)
    s_max = s_max or (budget + window + sinks)
    dev = latent_Q.device
    indices = torch.empty(B, Nq, s_max, dtype=torch.int32, device=dev)
    counts = torch.empty(B, Nq, dtype=torch.int32, device=dev)
    need = _lib.lsa_select_per_key_workspace_bytes(B, Nq, T_cap)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(_lib.lsa_select_per_key(_ptr(latent_K), _dtype_code(latent_K), B, T_cap, n_keys,
                                   _ptr(latent_Q), _ptr(positions), Nq,
                                   SelectParams(budget, window, sinks), _ptr(indices),
                                   _ptr(counts), s_max, _ptr(workspace), workspace.numel(),
                                   _stream(stream)))
    return indices, counts, workspace


def lsa_select_per_key_check(workspace, stream=None):
    """Status of the last lsa_select_per_key on `workspace` (raises LsaError
    on a device error); returns the number of queries that took the exact
    fallback."""
    fb = ctypes.c_int64(0)
    _check(_lib.lsa_select_per_key_check(_ptr(workspace), ctypes.byref(fb), _stream(stream)))
    return fb.value


def lsa_sparse_attn(Q, K, V, indices, counts, scale=None, return_lse=False, out=None,
                    stream=None):
    """Exact attention of Q [B][Nq][Hq][d] over the selected rows of K, V [B][T_cap][Hkv][d]."""
    _cuda(Q, K, V, indices, counts, out)
    B, Nq, Hq, d = Q.shape
    T_cap, Hkv = K.shape[1], K.shape[2]
    if scale is None:
        scale = float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
    O = out if out is not None else torch.empty_like(Q)
    lse = torch.empty(B, Nq, Hq, dtype=torch.float32, device=Q.device) if return_lse else None
    _check(_lib.lsa_sparse_attn(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(Q), B, Nq, T_cap, Hq, Hkv,
                                d, _ptr(indices), _ptr(counts), indices.shape[-1], scale, _ptr(O),
                                _ptr(lse), _stream(stream)))
    return (O, lse) if return_lse else O


def lsa_sparse_attn_backward(Q, K, V, O, lse, dO, indices, counts, scale=None, dK=None, dV=None,
                             stream=None):
    """Gradients of lsa_sparse_attn (C: lsa_sparse_attn_backward): returns (dQ, dK, dV); dK and
    dV (fp32 [B][T_cap][Hkv][d]) are added to when given, else start from zero."""
    _cuda(Q, K, V, O, lse, dO, indices, counts, dK, dV)
    B, Nq, Hq, d = Q.shape
    T_cap, Hkv = K.shape[1], K.shape[2]
    if scale is None:
        scale = float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
    dQ = torch.empty_like(Q)
    if dK is None:
        dK = torch.zeros(B, T_cap, Hkv, d, dtype=torch.float32, device=Q.device)
    if dV is None:
        dV = torch.zeros(B, T_cap, Hkv, d, dtype=torch.float32, device=Q.device)
    _check(_lib.lsa_sparse_attn_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _ptr(dO),
                                         _dtype_code(Q), B, Nq, T_cap, Hq, Hkv, d, _ptr(indices),
                                         _ptr(counts), indices.shape[-1], scale, _ptr(dQ),
                                         _ptr(dK), _ptr(dV), _stream(stream)))
    return dQ, dK, dV


def lsa_attend_key_range_workspace_bytes(B, Nq, s_max):
    """Workspace bytes lsa_attend_key_range needs."""
    return int(_lib.lsa_attend_key_range_workspace_bytes(int(B), int(Nq), int(s_max)))


def lsa_attend_key_range(Q, K_shard, V_shard, indices, counts, key_lo, key_hi, scale=None,
                         workspace=None, out=None, lse=None, stream=None):
    """Attention over the selected keys in [key_lo, key_hi) (C: lsa_attend_key_range), the
    caches' rows key_lo .. key_hi-1 in K_shard, V_shard [B][key_hi-key_lo][Hkv][d]: returns
    (O_part [B][Nq][Hq][d], lse_part [B][Nq][Hq] f32)."""
    _cuda(Q, K_shard, V_shard, indices, counts, out, lse)
    B, Nq, Hq, d = Q.shape
    Hkv = K_shard.shape[2]
    s_max = indices.shape[-1]
    if scale is None:
        scale = float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
    O = out if out is not None else torch.empty_like(Q)
    L = lse if lse is not None else torch.empty(B, Nq, Hq, dtype=torch.float32, device=Q.device)
    need = int(_lib.lsa_attend_key_range_workspace_bytes(B, Nq, s_max))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    _check(_lib.lsa_attend_key_range(_ptr(Q), _ptr(K_shard), _ptr(V_shard), _dtype_code(Q), B, Nq,
                                     Hq, Hkv, d, _ptr(indices), _ptr(counts), s_max, int(key_lo),
                                     int(key_hi), scale, _ptr(workspace), workspace.numel(),
                                     _ptr(O), _ptr(L), _stream(stream)))
    return O, L


def lsa_merge_partials(O_parts, lse_parts, out=None, lse=None, stream=None):
    """LSE-weighted merge (C: lsa_merge_partials) of O_parts [n][rows...][Hq][d] with
    lse_parts [n][rows...][Hq]; returns O [rows...][Hq][d] (and lse when given)."""
    _cuda(O_parts, lse_parts, out, lse)
    n = O_parts.shape[0]
    Hq, d = O_parts.shape[-2], O_parts.shape[-1]
    rows = O_parts[0].numel() // (Hq * d)
    O = out if out is not None else torch.empty(O_parts.shape[1:], dtype=O_parts.dtype,
                                                device=O_parts.device)
    _check(_lib.lsa_merge_partials(_ptr(O_parts), _ptr(lse_parts), _dtype_code(O_parts), n, rows,
                                   Hq, d, _ptr(O), _ptr(lse), _stream(stream)))
    return O


def lsa_prefill_workspace_bytes(index, Nq, Hq, Hkv, d, budget, window, sinks):
    """Recommended workspace bytes of lsa_prefill_chunk."""
    n = int(_lib.lsa_prefill_workspace_bytes(index.handle, Nq, Hq, Hkv, d,
                                             SelectParams(budget, window, sinks)))
    if n == 0:
        raise LsaError(1, "bad arguments")
    return n


def lsa_prefill_partial_slots(index, Nq, Hq, Hkv, d, budget, window, sinks, ws_bytes):
    """Softmax partial slots a workspace of ws_bytes gives (-1: below the minimum)."""
    return int(_lib.lsa_prefill_partial_slots(index.handle, Nq, Hq, Hkv, d,
                                              SelectParams(budget, window, sinks), ws_bytes))


def lsa_prefill_chunk(index, latent_K, latent_Q, Q, K, V, T_old, T_new, budget, window, sinks,
                      workspace=None, out=None, stream=None):
    """One fused prefill chunk (queries at positions [T_old, T_new)); returns O.

    The chunk's selection (indices [B][Nq][R+W+S] then counts [B][Nq]) is left
    at the start of `workspace`."""
    _cuda(latent_K, latent_Q, Q, K, V, out)
    B, Nq, Hq, d = Q.shape
    Hkv = K.shape[2]
    if workspace is None:
        need = lsa_prefill_workspace_bytes(index, Nq, Hq, Hkv, d, budget, window, sinks)
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    O = out if out is not None else torch.empty_like(Q)
    _check(_lib.lsa_prefill_chunk(index.handle, _ptr(latent_K), _ptr(latent_Q), _ptr(Q), _ptr(K),
                                  _ptr(V), int(T_old), int(T_new), Hq, Hkv, d,
                                  SelectParams(budget, window, sinks), _ptr(workspace),
                                  workspace.numel(), _ptr(O), _stream(stream)))
    return O


class LsaTree:
    """Level 2 of a D-LSA Tree over an LsaIndex (C: lsa_tree_build): n_super
    super-buckets of the index's closed buckets; rebuild after extending the
    index."""

    def __init__(self, index, n_super, lloyd_iters=3, stream=None):
        self.index = index
        self.n_super = int(n_super)
        n = int(_lib.lsa_tree_bytes(index.handle, self.n_super))
        if n == 0:
            raise LsaError(1, "bad tree arguments")
        self.buffer = torch.empty(n + 256, dtype=torch.uint8, device=index.buffer.device)
        off = (-self.buffer.data_ptr()) % 256
        self.view = self.buffer[off:off + n]
        self.build(lloyd_iters, stream)

    def build(self, lloyd_iters=3, stream=None):
        _check(_lib.lsa_tree_build(self.index.handle, _ptr(self.view), self.view.numel(),
                                   self.n_super, int(lloyd_iters), _stream(stream)))

    def export(self, stream=None):
        """Copies of the tree (C: lsa_tree_export) as torch tensors."""
        ix = self.index
        dev = ix.buffer.device
        rt = torch.bfloat16 if ix.dtype == BF16 else torch.float32
        out = dict(sup=torch.empty(ix.B, self.n_super, 64, dtype=torch.float32, device=dev),
                   sup_rt=torch.empty(ix.B, self.n_super, 64, dtype=rt, device=dev),
                   offsets=torch.empty(ix.B, self.n_super + 1, dtype=torch.int32, device=dev),
                   members=torch.empty(ix.B, ix.n_buckets_max, dtype=torch.int32, device=dev))
        _check(_lib.lsa_tree_export(ix.handle, _ptr(self.view), self.n_super, *[
            _ptr(out[k]) for k in ("sup", "sup_rt", "offsets", "members")], _stream(stream)))
        return out

    def select(self, latent_Q, positions, branches, budget, window, sinks, s_max=None,
               workspace=None, stream=None):
        """Tree selection (C: lsa_tree_select): (indices [B][Nq][s_max], counts [B][Nq])."""
        _cuda(latent_Q, positions)
        if positions.dtype != torch.int32:
            raise TypeError("positions must be int32")
        B, Nq = latent_Q.shape[0], latent_Q.shape[1]
        s_max = s_max or (budget + window + sinks)
        dev = latent_Q.device
        indices = torch.empty(B, Nq, s_max, dtype=torch.int32, device=dev)
        counts = torch.empty(B, Nq, dtype=torch.int32, device=dev)
        need = int(_lib.lsa_tree_select_workspace_bytes(self.index.handle, Nq, int(branches)))
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        _check(_lib.lsa_tree_select(self.index.handle, _ptr(self.view), self.n_super,
                                    int(branches), _ptr(latent_Q), _ptr(positions), Nq,
                                    SelectParams(budget, window, sinks), _ptr(indices),
                                    _ptr(counts), s_max, _ptr(workspace), workspace.numel(),
                                    _stream(stream)))
        return indices, counts


def lsa_prefill_chunk_queries(index, latent_K, latent_Q, Q, K, V, T_old, T_new, q_begin, q_end,
                              budget, window, sinks, workspace=None, out=None, stream=None):
    """lsa_prefill_chunk for the chunk's query rows [q_begin, q_end) (positions
    T_old + q_begin ..); latent_Q, Q and O hold those rows only."""
    _cuda(latent_K, latent_Q, Q, K, V, out)
    B, Nq, Hq, d = Q.shape
    Hkv = K.shape[2]
    if Nq != q_end - q_begin:
        raise ValueError("Q holds %d rows, the range %d" % (Nq, q_end - q_begin))
    if workspace is None:
        need = lsa_prefill_workspace_bytes(index, Nq, Hq, Hkv, d, budget, window, sinks)
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    O = out if out is not None else torch.empty_like(Q)
    _check(_lib.lsa_prefill_chunk_queries(index.handle, _ptr(latent_K), _ptr(latent_Q), _ptr(Q),
                                          _ptr(K), _ptr(V), int(T_old), int(T_new), int(q_begin),
                                          int(q_end), Hq, Hkv, d,
                                          SelectParams(budget, window, sinks), _ptr(workspace),
                                          workspace.numel(), _ptr(O), _stream(stream)))
    return O


def set_wait_limit(polls):
    """Test hook (C: lsa_set_wait_limit): polls each bounded wait of the
    library's kernels (tensor-core scorer, attention tiles, per-query
    attention) makes before it gives up; polls < 0 restores the defaults."""
    _check(_lib.lsa_set_wait_limit(int(polls)))


_copy_streams = {}


def lsa_prefill_chunk_host(index, h_latent_K, h_K, h_V, h_latent_Q, h_Q, latent_K, K, V,
                           latent_Q, Q, T_old, T_new, budget, window, sinks, workspace, out,
                           h_out, stream=None, copy_stream=None):
    """A prefill chunk from host inputs to a host output (C: lsa_prefill_chunk_host).

    h_latent_K [B][Nq][64], h_K and h_V [B][Nq][Hkv][d] are the chunk's new cache
    rows, h_latent_Q and h_Q its queries (page-locked CPU tensors); they are
    copied into the device tensors latent_K, K, V (at rows [T_old, T_new)),
    latent_Q and Q, and O (`out`) is copied back to `h_out`.  K, V and Q
    travel on `copy_stream` (one per device is kept when not given) under the
    selection.  Returns h_out, valid once `stream` has synchronised."""
    _cuda(latent_K, K, V, latent_Q, Q, workspace, out)
    for t in (h_latent_K, h_K, h_V, h_latent_Q, h_Q, h_out):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host tensors must be contiguous CPU tensors")
    B, Nq, Hq, d = Q.shape
    Hkv = K.shape[2]
    if copy_stream is None:
        dev = Q.device.index
        if dev not in _copy_streams:
            _copy_streams[dev] = torch.cuda.Stream(device=Q.device)
        copy_stream = _copy_streams[dev]
    _check(_lib.lsa_prefill_chunk_host(
        index.handle, _hptr(h_latent_K), _hptr(h_K), _hptr(h_V), _hptr(h_latent_Q), _hptr(h_Q),
        _ptr(latent_K), _ptr(K), _ptr(V), _ptr(latent_Q), _ptr(Q), int(T_old), int(T_new), Hq,
        Hkv, d, SelectParams(budget, window, sinks), _ptr(workspace), workspace.numel(),
        _ptr(out), _hptr(h_out), _stream(stream), _stream(copy_stream)))
    return h_out


def lsa_prefill_select(index, latent_K, latent_Q, T_old, T_new, Hq, Hkv, d, budget, window,
                       sinks, workspace, stream=None):
    """First half of a prefill chunk: index extension and selection into `workspace`."""
    _cuda(latent_K, latent_Q, workspace)
    _check(_lib.lsa_prefill_select(index.handle, _ptr(latent_K), _ptr(latent_Q), int(T_old),
                                   int(T_new), Hq, Hkv, d, SelectParams(budget, window, sinks),
                                   _ptr(workspace), workspace.numel(), _stream(stream)))


def lsa_prefill_attend(index, Q, K, V, T_old, T_new, budget, window, sinks, workspace, out=None,
                       stream=None):
    """Second half of a prefill chunk: attention from the selection in `workspace`."""
    _cuda(Q, K, V, workspace, out)
    B, Nq, Hq, d = Q.shape
    Hkv = K.shape[2]
    O = out if out is not None else torch.empty_like(Q)
    _check(_lib.lsa_prefill_attend(index.handle, _ptr(Q), _ptr(K), _ptr(V), int(T_old),
                                   int(T_new), Hq, Hkv, d, SelectParams(budget, window, sinks),
                                   _ptr(workspace), workspace.numel(), _ptr(O), _stream(stream)))
    return O


def prefill_selection_views(workspace, B, Nq, s_max):
    """(indices, counts) views of the selection a prefill chunk left in `workspace`."""
    n_idx = B * Nq * s_max
    al = (n_idx * 4 + 255) // 256 * 256
    indices = workspace[: n_idx * 4].view(torch.int32).view(B, Nq, s_max)
    counts = workspace[al: al + B * Nq * 4].view(torch.int32).view(B, Nq)
    return indices, counts


def lsa_decode_workspace_bytes(index, Hq, Hkv, d, budget, window, sinks):
    n = int(_lib.lsa_decode_workspace_bytes(index.handle, Hq, Hkv, d,
                                            SelectParams(budget, window, sinks)))
    if n == 0:
        raise LsaError(1, _lib.lsa_last_error().decode())
    return n


def lsa_decode_step(index, latent_K, K, V, new_latent_k, new_k, new_v, latent_q, q, pos, budget,
                    window, sinks, workspace=None, out=None, stream=None):
    """One decode step for every sequence (new token at pos[b]); returns O [B][Hq][d].

    The caches latent_K, K, V [B][T_cap][...] are updated in place at pos."""
    _cuda(latent_K, K, V, new_latent_k, new_k, new_v, latent_q, q, pos, out)
    if pos.dtype != torch.int32:
        raise TypeError("pos must be int32")
    B, Hq, d = q.shape
    Hkv = K.shape[2]
    need = lsa_decode_workspace_bytes(index, Hq, Hkv, d, budget, window, sinks)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    O = out if out is not None else torch.empty_like(q)
    _check(_lib.lsa_decode_step(index.handle, _ptr(latent_K), _ptr(K), _ptr(V), _ptr(new_latent_k),
                                _ptr(new_k), _ptr(new_v), _ptr(latent_q), _ptr(q), _ptr(pos), Hq,
                                Hkv, d, SelectParams(budget, window, sinks), _ptr(workspace),
                                workspace.numel(), _ptr(O), _stream(stream)))
    return O


def decode_selection_views(workspace, B, s_max):
    """(indices [B][s_max], counts [B]) views of the selection a decode step left in
    `workspace`."""
    n_idx = B * s_max
    al = (n_idx * 4 + 255) // 256 * 256
    indices = workspace[: n_idx * 4].view(torch.int32).view(B, s_max)
    counts = workspace[al: al + B * 4].view(torch.int32).view(B)
    return indices, counts
