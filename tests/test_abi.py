"""The C-ABI library builds, loads and exports every entry point declared in include/lsa.h,
and its host-side argument checks reject bad calls before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

from learned_sparse_kv_b200 import build as lbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(lbuild.build())


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("lsa_nmi_select", "lsa_topk", "lsa_topk_from_scores", "lsa_sparse_decode",
                     "lsa_append_token", "lsa_gather_chunks", "lsa_label_vote", "lsa_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"


def test_build_targets_sm100a_only():
    assert lbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def _err(lib):
    lib.lsa_last_error.restype = ctypes.c_char_p
    return lib.lsa_last_error().decode()


def test_gather_rejects_unsorted_kept_list(lib):
    kept = (ctypes.c_int32 * 3)(5, 2, 9)
    table = (ctypes.c_int32 * 20)()
    hp = (ctypes.c_void_p * 1)(ctypes.addressof(table))
    dp = (ctypes.c_void_p * 1)(ctypes.addressof(table))
    cb = (ctypes.c_size_t * 1)(64)
    rc = lib.lsa_gather_chunks(1, hp, cb, dp, ctypes.c_int64(20), ctypes.c_int64(20), kept, 3, 15, 0,
                               table, table, 20, None, None, None)
    assert rc == 1 and "ascending" in _err(lib)


def test_gather_reports_slot_capacity(lib):
    kept = (ctypes.c_int32 * 4)(1, 2, 3, 4)
    table = (ctypes.c_int32 * 20)()
    hp = (ctypes.c_void_p * 1)(ctypes.addressof(table))
    cb = (ctypes.c_size_t * 1)(64)
    rc = lib.lsa_gather_chunks(1, hp, cb, hp, ctypes.c_int64(20), ctypes.c_int64(5), kept, 4, 15, 2,
                               table, table, 20, None, None, None)
    assert rc == 4 and "fit" in _err(lib)


def test_gather_rejects_chunk_outside_host_pool(lib):
    kept = (ctypes.c_int32 * 2)(1, 30)
    table = (ctypes.c_int32 * 40)()
    hp = (ctypes.c_void_p * 1)(ctypes.addressof(table))
    cb = (ctypes.c_size_t * 1)(64)
    rc = lib.lsa_gather_chunks(1, hp, cb, hp, ctypes.c_int64(20), ctypes.c_int64(100), kept, 2, 35, 0,
                               table, table, 40, None, None, None)
    assert rc == 6


def test_entry_points_reject_bad_shapes_before_launch(lib):
    P = ctypes.c_void_p(16)  # never dereferenced: the calls fail validation first
    f = lib.lsa_sparse_decode
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    rc = f(P, P, 576, None, 0, 10, P, 4, P, P, 16, P, P, 100, 1, 96, 576, 512, 0.04, P, None, None, P, 1 << 20, None)
    assert rc == 2 and "unsupported" in _err(lib)
    rc = lib.lsa_label_vote(P, 65, 4, 128, ctypes.c_float(0.6), 3, 0, P, None, P, ctypes.c_size_t(1 << 20), None)
    assert rc == 2
    rc = lib.lsa_label_vote(P, 4, 4, 128, ctypes.c_float(0.6), 3, 2, P, None, P, ctypes.c_size_t(1 << 20), None)
    assert rc == 1


def test_workspace_queries_are_host_only(lib):
    lib.lsa_label_vote_workspace_size.restype = ctypes.c_size_t
    lib.lsa_topk_workspace_size.restype = ctypes.c_size_t
    lib.lsa_nmi_select_workspace_size.restype = ctypes.c_size_t
    assert lib.lsa_label_vote_workspace_size(32, 64, 2048) == 64 * 2048 * 4
    assert lib.lsa_topk_workspace_size(8, 2048) >= 8 * 2048 * 64 * 4 + 8 * 4
    assert lib.lsa_nmi_select_workspace_size(8, 2048) >= 8 * 32 * 8


def test_topk_kernel_count_follows_the_indexer_shape(lib):
    # The tcgen05 indexer (Hl in {32, 64, 128}, dl in {64, 128}, B <= 64) counts the kept cold
    # chunks itself: 2 kernels per lsa_topk call; other accepted shapes add a counting kernel.
    assert lib.lsa_topk_kernel_count(8, 64, 128) == 2
    assert lib.lsa_topk_kernel_count(1, 32, 64) == 2
    assert lib.lsa_topk_kernel_count(64, 128, 128) == 2
    assert lib.lsa_topk_kernel_count(65, 64, 128) == 3
    assert lib.lsa_topk_kernel_count(1, 8, 64) == 3
    assert lib.lsa_topk_kernel_count(8, 48, 128) == 3
    # shapes lsa_topk rejects
    assert lib.lsa_topk_kernel_count(8, 7, 128) == 0
    assert lib.lsa_topk_kernel_count(8, 64, 96) == 0
    assert lib.lsa_topk_kernel_count(0, 64, 128) == 0


def test_append_entry_points_reject_unaligned_rows_before_launch(lib):
    # Rows move as 16-byte vectors: a base that is not 16-byte aligned is an argument error,
    # reported before anything is enqueued (the pointers are never dereferenced).
    P, U = ctypes.c_void_p(4096), ctypes.c_void_p(4096 + 2)
    f = lib.lsa_append_token
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_void_p]
    rc = f(U, None, P, P, 576, 576, None, 0, 0, P, 128, 16, P, 4, P, P, 1, None, None)
    assert rc == 1 and "16-byte" in _err(lib)
    g = lib.lsa_append_topk
    g.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_int] + [ctypes.c_void_p] * 4 + \
        [ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
         ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 5 + \
        [ctypes.c_size_t, ctypes.c_void_p]
    rc = g(P, U, P, 576, 576, P, P, P, P, 16, P, 4, P, P, 4, P, 1, 64, 128, 64, P, P, P, None, P, 1 << 20, None)
    assert rc == 1 and "16-byte" in _err(lib)
    rc = g(P, P, None, 576, 576, P, P, P, P, 16, P, 4, P, P, 4, P, 1, 64, 128, 64, P, P, P, None, P, 1 << 20, None)
    assert rc == 1 and "null" in _err(lib)


def test_append_topk_launch_count_follows_the_indexer_shape():
    # The tcgen05 indexer shapes append inside the indexer launch (2 kernels per call);
    # other shapes launch the append, the counting kernel, the indexer and the top-k.
    from learned_sparse_kv_b200 import lsa
    assert lsa.append_topk_kernel_count(8, 64, 128) == 2
    assert lsa.append_topk_kernel_count(1, 32, 64) == 2
    assert lsa.append_topk_kernel_count(65, 64, 128) == 4
    assert lsa.append_topk_kernel_count(8, 48, 128) == 4


def _gather_args(lib, np, kept, first_window_chunk, table):
    f = lib.lsa_gather_chunks
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    host = np.zeros((16, 64), np.uint8)
    HP = (ctypes.c_void_p * 1)(host.ctypes.data)
    DP = (ctypes.c_void_p * 1)(4096)            # never written: the first copy fails before enqueueing
    CB = (ctypes.c_size_t * 1)(64)
    return f, (1, HP, CB, DP, 16, 32, kept.ctypes.data, kept.size, first_window_chunk, 8,
               table.ctypes.data, ctypes.c_void_p(8192), table.size, None, None, None), host


@pytest.mark.parametrize("cold", [True, False])
def test_gather_copy_failure_leaves_the_host_table_unchanged(lib, cold):
    """Host-side fault injection: the first copy of lsa_gather_chunks (a chunk run, or the table
    itself when no kept chunk is cold) reports failure; the call returns LSA_ERR_CUDA before
    enqueueing anything and the caller's host table is as it was."""
    import numpy as np
    kept = np.array([1, 2, 5, 12], np.int32) if cold else np.array([12, 13], np.int32)
    table = np.arange(100, 116, dtype=np.int32)
    f, args, _ = _gather_args(lib, np, kept, 10, table)
    assert lib.lsa_test_fail_copy(0) == 0
    try:
        rc = f(*args)
    finally:
        lib.lsa_test_fail_copy(-1)
    assert rc == 3 and "failed" in _err(lib)
    np.testing.assert_array_equal(table, np.arange(100, 116, dtype=np.int32))


def test_fail_copy_switch_rejects_bad_counts(lib):
    assert lib.lsa_test_fail_copy(-2) == 1
    assert lib.lsa_test_fail_copy(-1) == 0


@pytest.mark.parametrize("k, shape, code, words", [(0, (64, 128), 1, "outside"), (65537, (64, 128), 1, "outside"),
                                                  (64, (64, 96), 2, "unsupported"), (64, (7, 128), 2, "unsupported")])
def test_topk_rejects_bad_k_and_indexer_shapes_before_launch(lib, k, shape, code, words):
    P = ctypes.c_void_p(4096)   # never dereferenced: the call fails validation first
    f = lib.lsa_topk
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 2 + \
        [ctypes.c_int, ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 5 + [ctypes.c_size_t, ctypes.c_void_p]
    Hl, dl = shape
    rc = f(P, P, P, 16, P, 4, P, P, 4, P, 2, Hl, dl, k, P, P, None, None, P, 1 << 30, None)
    assert rc == code and words in _err(lib)
