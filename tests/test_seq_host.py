"""Host logic of sequences of several views, without a GPU: View.new_segment
hands the window ring over (same memory, same tokens) and freezes the old
view's packed rows; the sequence planner accepts the pair and rejects
malformed sequences."""
import ctypes

import pytest

import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import build as kbuild


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()


def test_new_segment_takes_over_the_window():
    old = kvq.View(2, 128, 4, 64, 8, device="cpu")
    old.set_state(n_packed=40, n_window=8, window_head=3)
    kw, vw = old.k_window.data_ptr(), old.v_window.data_ptr()
    seg = old.new_segment(2, 100)
    assert (seg.bits, seg.n_packed, seg.n_window, seg.window_head, seg.cap_window) == (2, 0, 8, 3, 8)
    assert seg.c.k_window == kw and seg.c.v_window == vw and seg.c.cap_packed == 100
    assert (old.bits, old.n_packed, old.n_window, old.cap_window) == (4, 40, 0, 0)
    assert old.c.k_window is None and old.c.v_window is None
    # the pair is one sequence for the planner; either alone is one too
    n = kvq.seq_workspace_size([old, seg], [0, 2], 8)
    assert n > 0
    assert kvq.seq_workspace_size([old, seg], [0, 1, 2], 8) > 0
    # an empty sequence, a sequence past the views, a decreasing boundary
    empty = kvq.View(2, 128, 2, 16, 0, device="cpu")
    assert kvq.seq_workspace_size([old, empty], [0, 1, 2], 8) == 0
    assert kvq.seq_workspace_size([old, seg], [0, 3], 8) == 0
    assert kvq.seq_workspace_size([old, seg, empty], [0, 2, 1, 3], 8) == 0
    # an empty view inside a sequence with tokens is fine
    assert kvq.seq_workspace_size([old, empty, seg], [0, 3], 8) > 0


def test_segments_of_a_sequence_may_differ_in_width_only():
    views = [kvq.View(2, 64, b, 32, 0, device="cpu") for b in (2, 3, 4, 8)]
    for v in views:
        v.set_state(n_packed=32, n_window=0)
    assert kvq.seq_workspace_size(views, [0, 4], 4) > 0
    # every view needs the same heads and head_dim: the call takes them once
    arr = (kvq.CView * 4)(*[v.c for v in views])
    sb = (ctypes.c_int32 * 2)(0, 4)
    assert kvq.lib().kvq_decode_attn_seq_workspace_size(arr, 4, sb, 1, 4, 2, 96) == 0
