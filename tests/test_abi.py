"""The C-ABI library loads on a host without a GPU, exports every entry point
that include/lsa.h declares, and rejects bad arguments on the host before any
launch.  No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

import long_context_indexing_b200 as lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(lsa.library_path())
    names = _declared()
    assert len(names) >= 15
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_version_and_empty_error():
    assert b"D-LSA" in lsa._lib.lsa_version()


def test_index_bytes_validation():
    P = lsa.IndexParams
    good = P(4, 1024, 16, 3)
    n = lsa._lib.lsa_index_bytes(1, 1 << 20, good, lsa.BF16)
    # pooled + unit (2 * NP * 64 * 4) dominate; everything 256-byte aligned
    NP = (1 << 20) // 4
    assert n >= 2 * NP * 64 * 4 and n % 256 == 0
    for bad in [P(0, 1024, 16, 3), P(4, 1024, 0, 3), P(4, 16, 32, 3), P(4, 1024, 16, 0),
                P(4, 1024, 64, 3)]:
        assert lsa._lib.lsa_index_bytes(1, 1 << 20, bad, lsa.BF16) == 0
        assert lsa._lib.lsa_last_error() != b""
    assert lsa._lib.lsa_index_bytes(0, 1 << 20, good, lsa.BF16) == 0
    assert lsa._lib.lsa_index_bytes(1, 100, good, lsa.BF16) == 0        # no whole block
    assert lsa._lib.lsa_index_bytes(1, 1 << 20, good, 7) == 0           # bad dtype


def test_index_init_checks_buffer():
    P = lsa.IndexParams(4, 256, 8, 3)
    need = lsa._lib.lsa_index_bytes(1, 8192, P, lsa.F32)
    h = ctypes.c_void_p()
    # NULL buffer, misaligned buffer, short buffer: all rejected on the host
    assert lsa._lib.lsa_index_init(None, need, 1, 8192, P, lsa.F32, ctypes.byref(h)) == 1
    assert lsa._lib.lsa_index_init(ctypes.c_void_p(4096 + 16), need, 1, 8192, P, lsa.F32,
                                   ctypes.byref(h)) == 2
    assert lsa._lib.lsa_index_init(ctypes.c_void_p(4096), need - 1, 1, 8192, P, lsa.F32,
                                   ctypes.byref(h)) == 3
    # a fake (never dereferenced on the host) aligned address is accepted
    assert lsa._lib.lsa_index_init(ctypes.c_void_p(1 << 20), need, 1, 8192, P, lsa.F32,
                                   ctypes.byref(h)) == 0
    assert lsa._lib.lsa_index_num_blocks(h) == 0
    # select / prefill argument checks fire before any launch
    fake = ctypes.c_void_p(1 << 21)
    S = lsa.SelectParams
    ws = lsa._lib.lsa_select_workspace_bytes(h, 16)
    assert ws > 0
    rc = lsa._lib.lsa_select(h, fake, fake, 16, S(512, 64, 4), fake, fake, 100, fake, ws, None)
    assert rc == 1 and b"s_max" in lsa._lib.lsa_last_error()
    rc = lsa._lib.lsa_select(h, fake, fake, 16, S(512, 2, 4), fake, fake, 600, fake, ws, None)
    assert rc == 7                                                      # window < p - 1
    rc = lsa._lib.lsa_select(h, fake, fake, 16, S(-1, 64, 4), fake, fake, 600, fake, ws, None)
    assert rc == 1
    rc = lsa._lib.lsa_select(h, fake, fake, 16, S(512, 64, 4), fake, fake, 580, fake, ws - 1, None)
    assert rc == 3
    rc = lsa._lib.lsa_select(h, ctypes.c_void_p((1 << 21) + 4), fake, 16, S(512, 64, 4), fake, fake,
                             580, fake, ws, None)
    assert rc == 2
    # extend: gap and range checks
    assert lsa._lib.lsa_index_extend(h, fake, 2048, 4096, None) == 1      # block 2 > 0 blocks
    assert lsa._lib.lsa_index_extend(h, fake, 0, 9000, None) == 1         # beyond T_cap
    lsa._lib.lsa_index_release(h)


def test_sparse_attn_argument_checks():
    fake = ctypes.c_void_p(1 << 22)
    f = lsa._lib.lsa_sparse_attn
    assert f(fake, fake, fake, lsa.BF16, 1, 4, 100, 12, 4, 128, fake, fake, 8, 0.1, fake, None,
             None) == 7                                                 # Hq/Hkv = 3
    assert f(fake, fake, fake, lsa.BF16, 1, 4, 100, 8, 3, 128, fake, fake, 8, 0.1, fake, None,
             None) == 1                                                 # Hq % Hkv
    assert f(fake, fake, fake, lsa.BF16, 1, 4, 100, 8, 1, 96, fake, fake, 8, 0.1, fake, None,
             None) == 7                                                 # d = 96
    assert f(fake, fake, fake, lsa.BF16, 1, 4, 100, 8, 1, 64, fake, fake, 8, 0.0, fake, None,
             None) == 1                                                 # scale
    assert f(None, fake, fake, lsa.BF16, 1, 4, 100, 8, 1, 64, fake, fake, 8, 0.1, fake, None,
             None) == 1
    assert f(ctypes.c_void_p((1 << 22) + 8), fake, fake, lsa.BF16, 1, 4, 100, 8, 1, 64, fake, fake,
             8, 0.1, fake, None, None) == 2


def test_calls_without_gpu_fail_cleanly():
    # With no device, a well-formed call reaches the CUDA runtime and must come
    # back with LSA_ERR_CUDA rather than crash.  (Skipped where a GPU exists.)
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    fake = ctypes.c_void_p(1 << 22)
    rc = lsa._lib.lsa_sparse_attn(fake, fake, fake, lsa.BF16, 1, 4, 100, 8, 1, 64, fake, fake, 8,
                                  0.125, fake, None, None)
    assert rc == 4


def test_host_entry_and_wait_hook_argument_checks():
    P = lsa.IndexParams(4, 256, 8, 3)
    need = lsa._lib.lsa_index_bytes(1, 8192, P, lsa.BF16)
    h = ctypes.c_void_p()
    assert lsa._lib.lsa_index_init(ctypes.c_void_p(1 << 20), need, 1, 8192, P, lsa.BF16,
                                   ctypes.byref(h)) == 0
    fake = ctypes.c_void_p(1 << 22)
    S = lsa.SelectParams(512, 64, 4)
    f = lsa._lib.lsa_prefill_chunk_host
    s1, s2 = ctypes.c_void_p(1 << 10), ctypes.c_void_p(1 << 11)
    args = [fake] * 10                     # 5 host inputs, 5 device tensors
    # NULL host input; one stream for both roles; the prefill checks (block-aligned T_old)
    assert f(h, None, *args[1:], 4096, 4160, 8, 2, 64, S, fake, 1 << 30, fake, fake, s1, s2) == 1
    assert f(h, *args, 4096, 4160, 8, 2, 64, S, fake, 1 << 30, fake, fake, s1, s1) == 1
    assert b"copy_stream" in lsa._lib.lsa_last_error()
    assert f(h, *args, 4000, 4160, 8, 2, 64, S, fake, 1 << 30, fake, fake, s1, s2) != 0
    # a misaligned device buffer is refused before any copy
    mis = ctypes.c_void_p((1 << 22) + 8)
    bad = [fake] * 5 + [mis] + [fake] * 4
    ws = lsa._lib.lsa_prefill_workspace_bytes(h, 64, 8, 2, 64, S)
    rc = f(h, *bad, 4096, 4160, 8, 2, 64, S, fake, ws, fake, fake, s1, s2)
    assert rc != 0
    lsa._lib.lsa_index_release(h)


def test_wait_hook_without_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lsa._lib.lsa_set_wait_limit(0) == 4                           # LSA_ERR_CUDA


def test_query_range_entry_argument_checks():
    # lsa_prefill_chunk_queries refuses an empty or out-of-chunk query range,
    # a NULL argument and a short workspace before any launch.
    P = lsa.IndexParams(4, 256, 8, 3)
    need = lsa._lib.lsa_index_bytes(1, 8192, P, lsa.BF16)
    h = ctypes.c_void_p()
    assert lsa._lib.lsa_index_init(ctypes.c_void_p(1 << 20), need, 1, 8192, P, lsa.BF16,
                                   ctypes.byref(h)) == 0
    fake = ctypes.c_void_p(1 << 22)
    S = lsa.SelectParams(512, 64, 4)
    f = lsa._lib.lsa_prefill_chunk_queries
    ws = lsa._lib.lsa_prefill_workspace_bytes(h, 32, 8, 2, 64, S)
    args = [fake] * 6                       # latent_K, latent_Q, Q, K, V (and O below)
    for q0, q1 in ((10, 10), (-1, 5), (0, 65), (70, 80)):
        assert f(h, *args[:5], 4096, 4160, q0, q1, 8, 2, 64, S, fake, ws, fake, None) == 1
        assert b"query range" in lsa._lib.lsa_last_error()
    assert f(h, None, *args[1:5], 4096, 4160, 0, 32, 8, 2, 64, S, fake, ws, fake, None) == 1
    assert f(h, *args[:5], 4096, 4160, 0, 32, 8, 2, 64, S, fake, 16, fake, None) == 3
    lsa._lib.lsa_index_release(h)


def test_context_parallel_entry_argument_checks():
    # lsa_attend_key_range refuses an empty or negative key range, NULL
    # arguments, a short workspace and misaligned pointers, and
    # lsa_merge_partials a part count outside 1 .. 32, before any launch.
    fake = ctypes.c_void_p(1 << 22)
    f = lsa._lib.lsa_attend_key_range
    ws = lsa._lib.lsa_attend_key_range_workspace_bytes(1, 16, 64)
    assert ws >= 16 * 64 * 4 + 16 * 4
    assert lsa._lib.lsa_attend_key_range_workspace_bytes(0, 16, 64) == 0
    base = [fake, fake, fake, lsa.BF16, 1, 16, 8, 2, 64, fake, fake, 64]
    for lo, hi in ((100, 100), (-1, 50), (50, 10)):
        assert f(*base, lo, hi, 0.125, fake, ws, fake, fake, None) == 1
    assert f(None, *base[1:], 0, 256, 0.125, fake, ws, fake, fake, None) == 1
    assert f(*base, 0, 256, 0.125, fake, ws, fake, None, None) == 1          # lse required
    assert f(*base, 0, 256, 0.125, fake, 16, fake, fake, None) == 3          # workspace
    odd = ctypes.c_void_p((1 << 22) + 4)
    assert f(odd, *base[1:], 0, 256, 0.125, fake, ws, fake, fake, None) == 2  # alignment
    m = lsa._lib.lsa_merge_partials
    for n in (0, 33):
        assert m(fake, fake, lsa.BF16, n, 16, 8, 64, fake, None, None) == 1
    assert m(None, fake, lsa.BF16, 2, 16, 8, 64, fake, None, None) == 1


def test_backward_entry_argument_checks():
    # lsa_sparse_attn_backward refuses NULL arguments, unsupported head
    # shapes and misaligned pointers before any launch.
    fake = ctypes.c_void_p(1 << 22)
    f = lsa._lib.lsa_sparse_attn_backward
    ok = [fake] * 6 + [lsa.BF16, 1, 16, 256, 8, 2, 64, fake, fake, 32, 0.125, fake, fake, fake, None]
    bad = list(ok)
    bad[0] = None
    assert f(*bad) == 1
    shape = list(ok)
    shape[10], shape[11] = 16, 1          # 16 query heads per KV head
    assert f(*shape) == 7                 # LSA_ERR_UNSUPPORTED
    odd = list(ok)
    odd[5] = ctypes.c_void_p((1 << 22) + 8)
    assert f(*odd) == 2


def test_per_key_entry_argument_checks():
    # lsa_select_per_key refuses bad arguments before any launch: NULL
    # pointers, fp32 latents, budgets above 4096, a short s_max or workspace,
    # misaligned pointers.
    need = lsa._lib.lsa_select_per_key_workspace_bytes(1, 32768, 10485760)
    # [rows][32768] fp16 group maxima + [rows][8192] candidates + per-row words
    assert 32768 * (2 * 32768 + 4 * 8192) < need < 32768 * (2 * 32768 + 4 * 8192 + 64) + (1 << 20)
    assert lsa._lib.lsa_select_per_key_workspace_bytes(0, 16, 1024) == 0
    assert lsa._lib.lsa_select_per_key_workspace_bytes(4, 16, 1 << 30) == 0   # B*T_cap >= 2^31
    fake = ctypes.c_void_p(1 << 22)
    f = lsa._lib.lsa_select_per_key
    sp = lsa.SelectParams(256, 64, 4)
    small = lsa._lib.lsa_select_per_key_workspace_bytes(1, 16, 8192)
    ok = [fake, lsa.BF16, 1, 8192, 8192, fake, fake, 16, sp, fake, fake, 324, fake, small, None]
    bad = list(ok)
    bad[0] = None
    assert f(*bad) == 1
    f32 = list(ok)
    f32[1] = lsa.F32
    assert f(*f32) == 7                                 # LSA_ERR_UNSUPPORTED
    big = list(ok)
    big[8] = lsa.SelectParams(5000, 64, 4)
    big[11] = 5068
    assert f(*big) == 7
    short = list(ok)
    short[11] = 323                                      # s_max < budget + window + sinks
    assert f(*short) == 1
    keys = list(ok)
    keys[4] = 8193                                       # n_keys > T_cap
    assert f(*keys) == 1
    ws = list(ok)
    ws[13] = small - 1
    assert f(*ws) == 3                                   # LSA_ERR_WORKSPACE
    odd = list(ok)
    odd[6] = ctypes.c_void_p((1 << 22) + 4)
    assert f(*odd) == 2                                  # LSA_ERR_ALIGNMENT


def test_per_key_workspace_layout():
    # rows x (2 B per strided group + 4 B per candidate slot of 8192 + three
    # 4-byte words), the groups a power of two between 256 (one block of
    # 256-key columns) and 32768 that covers T_cap, every array 256-byte
    # aligned, plus the status and per-dimension maxima
    def groups(T_cap):
        ng = 256
        while ng < T_cap and ng < 32768:
            ng *= 2
        return ng

    def al(x):
        return (x + 255) // 256 * 256

    for B, Nq, T_cap in [(1, 1, 100), (1, 300, 5000), (2, 129, 8192), (1, 32768, 10485760),
                         (3, 7, 40000)]:
        rows = B * Nq
        want = (256 + al(B * 64 * 4) + 3 * al(rows * 4) + al(rows * groups(T_cap) * 2)
                + al(rows * 8192 * 4))
        assert lsa._lib.lsa_select_per_key_workspace_bytes(B, Nq, T_cap) == want, (B, Nq, T_cap)
