"""CacheCard host logic without a GPU: the card size follows the documented
layout (recomputed here from the header's description), and a card is
validated before anything is enqueued (magic, version, sizes, offsets,
counts, widths, capacities)."""
import ctypes
import struct

import numpy as np
import pytest

import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import build as kbuild

FAKE = 0x100000  # aligned, never dereferenced


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kvq.lib()


def up(x, a):
    return (x + a - 1) // a * a


def layout(H, D, recs):
    """recs: (bits, n_packed, n_window) per view -> (total, [data_offset], [data_bytes])."""
    off = up(64 + 64 * len(recs), 256)
    offs, sizes = [], []
    for b, n_p, n_w in recs:
        codes = H * n_p * D * b // 8
        sm = H * n_p * (D // 64) * 8
        win = H * n_w * D * 2
        start = off
        for size in (codes, codes, sm, sm, win, win):
            off = up(off + size, 16)
        offs.append(start)
        sizes.append(off - start)
        off = up(off, 256)
    return off, offs, sizes


def cview(bits, n_p, cap_p, n_w, cap_w, head=0):
    return kvq.CView(bits=bits, n_window=n_w, cap_window=cap_w, window_head=head, n_packed=n_p, cap_packed=cap_p,
                     k_codes=FAKE, v_codes=FAKE, k_scalemin=FAKE, v_scalemin=FAKE,
                     k_window=FAKE if cap_w else None, v_window=FAKE if cap_w else None)


def make_card(H, D, recs, model_id=7, positions=None):
    total, offs, sizes = layout(H, D, recs)
    buf = bytearray(total)
    struct.pack_into("<8sIIIIQQ24x", buf, 0, b"KVQCARD1", 1, len(recs), H, D, model_id, total)
    for i, (b, n_p, n_w) in enumerate(recs):
        pos = positions[i] if positions else 0
        struct.pack_into("<IIQqQQQ16x", buf, 64 + 64 * i, b, n_w, n_p, pos, offs[i], sizes[i], n_p + n_w)
    return np.frombuffer(bytes(buf), dtype=np.uint8).copy()


def test_card_bytes_follow_the_layout(L):
    recs = [(4, 4096, 128), (2, 1000, 0), (3, 333, 17), (8, 0, 5)]
    arr = (kvq.CView * 4)(*[cview(b, n_p, n_p + (n_p & 1) + 2, n_w, max(n_w, 1) if n_w else 0)
                            for b, n_p, n_w in recs])
    for H, D in ((8, 128), (2, 64), (4, 256)):
        assert L.kvq_card_bytes(arr, 4, H, D) == layout(H, D, recs)[0]


def test_header_round_trip_and_records(L):
    card = make_card(8, 128, [(4, 4096, 128), (3, 77, 0)], model_id=0xABCDEF, positions=[5, -3])
    n, hk, d, mid = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_uint64()
    p = card.ctypes.data_as(ctypes.c_void_p)
    assert L.kvq_card_read_header(p, card.size, ctypes.byref(n), ctypes.byref(hk), ctypes.byref(d),
                                  ctypes.byref(mid)) == kvq.KVQ_OK
    assert (n.value, hk.value, d.value, mid.value) == (2, 8, 128, 0xABCDEF)
    b, w, np_, pos = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int64(), ctypes.c_int64()
    assert L.kvq_card_view_info(p, card.size, 1, ctypes.byref(b), ctypes.byref(np_), ctypes.byref(w),
                                ctypes.byref(pos)) == kvq.KVQ_OK
    assert (b.value, np_.value, w.value, pos.value) == (3, 77, 0, -3)
    assert L.kvq_card_view_info(p, card.size, 2, None, None, None, None) == kvq.KVQ_ERR_INVALID_ARG


def test_malformed_cards_are_rejected(L):
    good = make_card(2, 64, [(4, 64, 8)])

    def status(card, size=None):
        return L.kvq_card_read_header(card.ctypes.data_as(ctypes.c_void_p), card.size if size is None else size,
                                      None, None, None, None)

    assert status(good) == kvq.KVQ_OK
    bad = good.copy(); bad[0] = ord("X")
    assert status(bad) == kvq.KVQ_ERR_INVALID_ARG                       # magic
    bad = good.copy(); struct.pack_into("<I", bad, 8, 2)
    assert status(bad) == kvq.KVQ_ERR_INVALID_ARG                       # version
    assert status(good, good.size - 1) == kvq.KVQ_ERR_INVALID_ARG       # truncated
    bad = good.copy(); struct.pack_into("<Q", bad, 64 + 24, 0)
    assert status(bad) == kvq.KVQ_ERR_INVALID_ARG                       # data not where the layout puts it
    bad = good.copy(); struct.pack_into("<Q", bad, 64 + 40, 99)
    assert status(bad) == kvq.KVQ_ERR_INVALID_ARG                       # seq_len != n_packed + n_window
    bad = good.copy(); struct.pack_into("<I", bad, 64, 5)
    assert status(bad) == kvq.KVQ_ERR_UNSUPPORTED                       # width 5


def test_unpack_checks_views_before_launch(L):
    card = make_card(2, 64, [(4, 64, 8), (2, 10, 0)])
    p = card.ctypes.data_as(ctypes.c_void_p)
    dev = ctypes.c_void_p(FAKE)

    def unpack(views, n=2, H=2, D=64):
        arr = (kvq.CView * len(views))(*views)
        return L.kvq_card_unpack(p, dev, card.size, arr, n, H, D, None), arr

    ok = [cview(4, 0, 64, 0, 8), cview(2, 0, 10, 0, 0)]
    assert unpack(ok, n=1)[0] == kvq.KVQ_ERR_INVALID_ARG                # view count differs
    assert unpack(ok, H=4)[0] == kvq.KVQ_ERR_INVALID_ARG                # heads differ
    r, arr = unpack([cview(3, 0, 64, 0, 8), cview(2, 0, 10, 0, 0)])
    assert r == kvq.KVQ_ERR_INVALID_ARG                                 # width differs
    r, arr = unpack([cview(4, 0, 62, 0, 8), cview(2, 0, 10, 0, 0)])
    assert r == kvq.KVQ_ERR_CAPACITY and arr[0].n_packed == 0          # packed capacity; view untouched
    r, arr = unpack([cview(4, 0, 64, 0, 4), cview(2, 0, 10, 0, 0)])
    assert r == kvq.KVQ_ERR_CAPACITY                                    # window capacity


def test_random_corruption_never_crashes_the_parser(L):
    # a card read from a file is untrusted input: random bytes in the header
    # and records, and random truncations, give a status (or a valid reading),
    # never a read outside the buffer
    rng = np.random.default_rng(7)
    good = make_card(4, 128, [(4, 300, 16), (2, 0, 7), (8, 33, 0)], model_id=3, positions=[1, 2, 3])
    meta = 64 + 64 * 3
    outcomes = set()
    for trial in range(3000):
        card = good.copy()
        if trial % 3 == 0:
            card = card[:int(rng.integers(0, len(card)))].copy()
        for _ in range(int(rng.integers(1, 4))):
            if len(card) == 0:
                break
            i = int(rng.integers(0, min(meta, len(card))))
            card[i] = rng.integers(0, 256)
        p = card.ctypes.data_as(ctypes.c_void_p) if len(card) else ctypes.c_void_p(0)
        n, hk, d, mid = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32(), ctypes.c_uint64()
        st = L.kvq_card_read_header(p, len(card), ctypes.byref(n), ctypes.byref(hk), ctypes.byref(d),
                                    ctypes.byref(mid))
        outcomes.add(st)
        if st == kvq.KVQ_OK:
            for i in range(n.value):
                b, w = ctypes.c_int32(), ctypes.c_int32()
                np_, off = ctypes.c_int64(), ctypes.c_int64()
                assert L.kvq_card_view_info(p, len(card), i, ctypes.byref(b), ctypes.byref(np_), ctypes.byref(w),
                                            ctypes.byref(off)) == kvq.KVQ_OK
    assert kvq.KVQ_ERR_INVALID_ARG in outcomes and kvq.KVQ_OK in outcomes
