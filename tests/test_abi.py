"""The C ABI library loads, exports every symbol include/kvq.h declares, and
rejects bad arguments on the host before touching the GPU (runs without one)."""
import ctypes
import os
import re
import subprocess

import pytest

import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kvq.lib()


def declared_functions():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            text = open(os.path.join(ROOT, "include", hdr)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"kvq_quantize", "kvq_dequantize", "kvq_append", "kvq_decode_attn",
            "kvq_decode_attn_workspace_size", "kvq_status_string"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", kvq._LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (kvq_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)
    # nothing but the C ABI is exported
    assert all(e.startswith("kvq_") for e in exported)


def test_status_strings_and_version(L):
    assert L.kvq_status_string(0) == b"KVQ_OK"
    assert L.kvq_status_string(3) == b"KVQ_ERR_CAPACITY"
    assert L.kvq_status_string(99) == b"unknown status"
    assert L.kvq_abi_version() == 1


def test_view_struct_layout_matches_header():
    assert ctypes.sizeof(kvq.CView) == 80
    assert kvq.CView.n_packed.offset == 16
    assert kvq.CView.k_codes.offset == 32


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(0x10000)   # aligned, never dereferenced: validation fails first


def test_quantize_rejects_bad_arguments(L):
    ok_args = dict(x=FAKE, hs=8 * 128, ts=128, nh=2, nt=8, d=128, bits=4, codes=FAKE, sm=FAKE, cap=8)

    def call(**kw):
        a = dict(ok_args, **kw)
        return L.kvq_quantize(a["x"], a["hs"], a["ts"], a["nh"], a["nt"], a["d"], a["bits"], a["codes"], a["sm"],
                              a["cap"], NULL)

    assert call(bits=5) == kvq.KVQ_ERR_UNSUPPORTED
    assert call(bits=1) == kvq.KVQ_ERR_UNSUPPORTED
    assert call(d=96) == kvq.KVQ_ERR_UNSUPPORTED
    assert call(d=320) == kvq.KVQ_ERR_UNSUPPORTED
    assert call(x=NULL) == kvq.KVQ_ERR_INVALID_ARG
    assert call(codes=NULL) == kvq.KVQ_ERR_INVALID_ARG
    assert call(x=ctypes.c_void_p(0x10008)) == kvq.KVQ_ERR_INVALID_ARG   # not 16-B aligned
    assert call(ts=129) == kvq.KVQ_ERR_INVALID_ARG                       # stride not multiple of 8
    assert call(cap=7) == kvq.KVQ_ERR_INVALID_ARG                        # cap < n_tokens
    assert call(nt=0) == kvq.KVQ_OK                                      # empty: nothing enqueued
    assert call(nh=0, x=NULL) == kvq.KVQ_OK


def test_dequantize_rejects_overlapping_rows(L):
    r = L.kvq_dequantize(FAKE, FAKE, 8, 2, 8, 128, 4, FAKE, 8 * 128, 64, NULL)
    assert r == kvq.KVQ_ERR_INVALID_ARG


def cview(**kw):
    base = dict(bits=4, n_window=0, cap_window=0, window_head=0, n_packed=16, cap_packed=16,
                k_codes=0x10000, v_codes=0x20000, k_scalemin=0x30000, v_scalemin=0x40000,
                k_window=None, v_window=None)
    base.update(kw)
    return kvq.CView(**base)


def test_decode_attn_validation(L):
    arr = (kvq.CView * 1)(cview())
    ws = L.kvq_decode_attn_workspace_size(arr, 1, 8, 2, 128)
    assert ws > 0
    assert L.kvq_decode_attn_workspace_size(arr, 1, 7, 2, 128) == 0       # Hq % Hkv
    assert L.kvq_decode_attn_workspace_size(arr, 1, 8, 2, 96) == 0        # head_dim
    bad = (kvq.CView * 1)(cview(bits=5))
    assert L.kvq_decode_attn(bad, 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == kvq.KVQ_ERR_UNSUPPORTED
    empty = (kvq.CView * 1)(cview(n_packed=0))
    assert L.kvq_decode_attn(empty, 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == kvq.KVQ_ERR_INVALID_ARG
    odd = (kvq.CView * 1)(cview(cap_packed=17))
    assert L.kvq_decode_attn(odd, 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn(arr, 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws - 1, NULL) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn(arr, 1, 8, 2, 128, NULL, 0.1, FAKE, FAKE, ws, NULL) == kvq.KVQ_ERR_INVALID_ARG
    mis = (kvq.CView * 1)(cview(k_codes=0x10004))
    assert L.kvq_decode_attn(mis, 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == kvq.KVQ_ERR_INVALID_ARG
    win = (kvq.CView * 1)(cview(n_window=3, cap_window=2, k_window=0x50000, v_window=0x60000))
    assert L.kvq_decode_attn(win, 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == kvq.KVQ_ERR_INVALID_ARG


def test_decode_attn_seq_validation(L):
    def sb(*xs):
        return (ctypes.c_int32 * len(xs))(*xs)

    views = (kvq.CView * 4)(cview(), cview(bits=2, n_packed=0), cview(bits=8), cview(bits=3))
    ws = L.kvq_decode_attn_seq_workspace_size(views, 4, sb(0, 3, 4), 2, 8, 2, 128)
    assert ws > 0
    # one view per sequence needs the same scratch as kvq_decode_attn
    one = (kvq.CView * 2)(cview(), cview(bits=8))
    assert L.kvq_decode_attn_seq_workspace_size(one, 2, sb(0, 1, 2), 2, 8, 2, 128) == \
        L.kvq_decode_attn_workspace_size(one, 2, 8, 2, 128)
    for bad in [sb(1, 3, 4), sb(0, 3, 3), sb(0, 4, 4), sb(0, 0, 4), sb(0, 3, 5)]:
        assert L.kvq_decode_attn_seq_workspace_size(views, 4, bad, 2, 8, 2, 128) == 0
        assert L.kvq_decode_attn_seq(views, 4, bad, 2, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == \
            kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn_seq(views, 4, NULL, 2, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG
    # a sequence whose views hold no token
    empty = (kvq.CView * 2)(cview(), cview(n_packed=0))
    assert L.kvq_decode_attn_seq(empty, 2, sb(0, 1, 2), 2, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG
    # too many non-empty segments in one sequence
    n = kvq.MAX_SEGMENTS + 1
    many = (kvq.CView * n)(*[cview() for _ in range(n)])
    assert L.kvq_decode_attn_seq(many, n, sb(0, n), 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, 1 << 30, NULL) == \
        kvq.KVQ_ERR_UNSUPPORTED
    ok = (kvq.CView * (n - 1))(*[cview() for _ in range(n - 1)])
    assert L.kvq_decode_attn_seq_workspace_size(ok, n - 1, sb(0, n - 1), 1, 8, 2, 128) > 0
    # workspace too small, unaligned q
    assert L.kvq_decode_attn_seq(views, 4, sb(0, 3, 4), 2, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, ws - 1, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn_seq(views, 4, sb(0, 3, 4), 2, 8, 2, 128, ctypes.c_void_p(0x10008), 0.1, FAKE, FAKE,
                                 ws, NULL) == kvq.KVQ_ERR_INVALID_ARG


def test_sparse_decode_attn_validation(L):
    views = (kvq.CView * 2)(cview(n_packed=4096, cap_packed=4096), cview(bits=2, n_packed=16))
    ws = L.kvq_sparse_decode_attn_workspace_size(views, 2, 8, 2, 128, 64)
    assert ws >= 2 * 4096 * 4 + 2 * 2 * 64 * 4  # at least the scores and the selections
    assert L.kvq_sparse_decode_attn_workspace_size(views, 2, 8, 2, 128, 0) == 0
    assert L.kvq_sparse_decode_attn_workspace_size(views, 2, 7, 2, 128, 64) == 0
    # top_k above every view's packed count: no scores and no gathered rows
    big = L.kvq_sparse_decode_attn_workspace_size(views, 2, 8, 2, 128, 5000)
    assert 0 < big
    call = lambda **kw: L.kvq_sparse_decode_attn(
        kw.get("views", views), 2, 8, 2, 128, kw.get("q", FAKE), 0.1, kw.get("k", 64), FAKE, kw.get("sel", NULL),
        FAKE, kw.get("ws", ws), NULL)
    assert call(k=0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(ws=ws - 1) == kvq.KVQ_ERR_INVALID_ARG
    assert call(q=NULL) == kvq.KVQ_ERR_INVALID_ARG
    assert call(sel=ctypes.c_void_p(0x10002)) == kvq.KVQ_ERR_INVALID_ARG
    bad = (kvq.CView * 2)(cview(bits=5), cview())
    assert call(views=bad) == kvq.KVQ_ERR_UNSUPPORTED
    empty = (kvq.CView * 2)(cview(), cview(n_packed=0))
    assert call(views=empty) == kvq.KVQ_ERR_INVALID_ARG


def test_workspace_grows_with_views(L):
    one = (kvq.CView * 1)(cview(n_packed=4096, cap_packed=4096))
    many = (kvq.CView * 200)(*[cview(n_packed=4096, cap_packed=4096) for _ in range(200)])
    assert L.kvq_decode_attn_workspace_size(many, 200, 8, 2, 128) > L.kvq_decode_attn_workspace_size(one, 1, 8, 2, 128)


def test_append_capacity_checked_before_launch(L):
    full = (kvq.CView * 2)(cview(n_packed=4, cap_packed=8), cview(n_packed=8, cap_packed=8))
    r = L.kvq_append(full, 2, 2, 128, FAKE, FAKE, NULL)
    assert r == kvq.KVQ_ERR_CAPACITY
    # no view was advanced
    assert full[0].n_packed == 4 and full[1].n_packed == 8
    # a view with room in its window never flushes, so it needs no packed room
    ok_win = (kvq.CView * 1)(cview(n_packed=8, cap_packed=8, n_window=1, cap_window=4,
                                   k_window=0x50000, v_window=0x60000))
    assert L.kvq_append(ok_win, 1, 2, 128, NULL, FAKE, NULL) == kvq.KVQ_ERR_INVALID_ARG  # null k_new


def test_fused_step_checks_before_launch(L):
    # capacity: nothing enqueued, no counter changed
    full = (kvq.CView * 2)(cview(n_packed=4, cap_packed=8), cview(n_packed=8, cap_packed=8))
    ws = 1 << 20
    r = L.kvq_append_decode_attn(full, 2, 8, 2, 128, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, ws, NULL)
    assert r == kvq.KVQ_ERR_CAPACITY
    assert full[0].n_packed == 4 and full[1].n_packed == 8
    # attention arguments are checked before the append is enqueued
    ok = (kvq.CView * 1)(cview(n_packed=4, cap_packed=8))
    assert L.kvq_append_decode_attn(ok, 1, 7, 2, 128, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, ws, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG                                                    # Hq % Hkv
    assert L.kvq_append_decode_attn(ok, 1, 8, 2, 128, FAKE, FAKE, NULL, 0.1, FAKE, FAKE, ws, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG                                                    # null q
    assert L.kvq_append_decode_attn(ok, 1, 8, 2, 128, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, 16, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG                                                    # workspace too small
    assert ok[0].n_packed == 4


def test_view_count_is_bounded(L):
    # the bound is checked before the views are read
    one = (kvq.CView * 1)(cview())
    assert L.kvq_decode_attn(one, (1 << 22) + 1, 8, 2, 128, FAKE, 0.1, FAKE, FAKE, 1 << 30, NULL) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attn_workspace_size(one, (1 << 22) + 1, 8, 2, 128) == 0
