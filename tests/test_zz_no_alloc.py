"""kvq_decode_attn_noalloc against kvq_decode_attn, through the C ABI.

The no-allocation variant takes its scratch from a fixed per-device array in
the library instead of a caller workspace.  It runs the same plan on the same
kernels as kvq_decode_attn, so two calls in a row (different view sets, so the
second reuses scratch the first one wrote) must each give bitwise the outputs
of kvq_decode_attn on the same inputs (and therefore lie within the attention
tolerance of it); the scratch's status word reads 0 after each call.  A call
whose plan needs more than the array holds is refused with KVQ_ERR_CAPACITY
before anything is enqueued.  This file sorts last so that it also runs after
every other GPU test in the same process.
"""
import math

import numpy as np
import pytest
import torch

import quantized_kv_cache_dequantize_b200 as kvq
from helpers import ViewSpec, assert_close, build_case

pytestmark = pytest.mark.gpu


def _noalloc(case, scale):
    out = torch.empty((len(case.views), case.n_q_heads, case.head_dim), dtype=torch.float32,
                      device=case.q.device)
    kvq.decode_attn_noalloc(case.views, case.q, scale, out)
    status = kvq.decode_attn_noalloc_status()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "a bounded copy wait gave up"
    return out.cpu().numpy().astype(np.float64)


def _with_workspace(case, scale):
    out = kvq.decode_attn(case.views, case.q, scale)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def test_two_calls_in_a_row_match_workspace_path(cuda_device):
    # call 1: Llama-3.1-8B decode shape, 3 views, wrapped 128-token rings
    a = build_case(32, 8, 128, [ViewSpec(4096, 128, 128, 4, head=37 * i % 128, seed=700 + i)
                                for i in range(3)], q_seed=71)
    # call 2: mixed widths, ragged lengths, D 256, one view without a window
    b = build_case(16, 4, 256, [ViewSpec(1500, 40, 64, 2, head=9, seed=710),
                                ViewSpec(333, 0, 0, 8, seed=711),
                                ViewSpec(2048, 64, 64, 3, head=63, seed=712)], q_seed=72)
    sa, sb = 1 / math.sqrt(128), 1 / 16
    assert kvq.workspace_size(a.views, 32) <= kvq.NOALLOC_SCRATCH_BYTES
    assert kvq.workspace_size(b.views, 16) <= kvq.NOALLOC_SCRATCH_BYTES
    got_a = _noalloc(a, sa)
    got_b = _noalloc(b, sb)
    ref_a = _with_workspace(a, sa)
    ref_b = _with_workspace(b, sb)
    for i in range(len(a.views)):
        assert_close(got_a[i], ref_a[i], f"noalloc call 1, view {i}")
    for i in range(len(b.views)):
        assert_close(got_b[i], ref_b[i], f"noalloc call 2, view {i}")
    # the same plan on the same kernels: bitwise the workspace path's outputs
    assert np.array_equal(got_a, ref_a) and np.array_equal(got_b, ref_b)
    # and once more on the first set, after the second call overwrote the scratch
    again = _noalloc(a, sa)
    for i in range(len(a.views)):
        assert_close(again[i], ref_a[i], f"noalloc call 3, view {i}")
    assert np.array_equal(again, ref_a)


def test_rejects_plans_beyond_the_scratch_array(cuda_device, monkeypatch):
    # 16 views x 32768 packed tokens (8 kv heads, D 128) cut into 128-token
    # chunks merged through the workspace: about 69 MiB of partials, more than
    # the array holds
    monkeypatch.setenv("KVQ_CHUNK_TOKENS", "128")
    views = []
    for i in range(16):
        v = kvq.View(8, 128, 4, 32768, 128, device=cuda_device)
        v.set_state(32768, 128)
        views.append(v)
    need = kvq.workspace_size(views, 32)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((16, 32, 128), dtype=torch.bfloat16, device=cuda_device)
    out = torch.full((16, 32, 128), 7.0, dtype=torch.float32, device=cuda_device)
    with pytest.raises(kvq.KvqError) as e:
        kvq.decode_attn_noalloc(views, q, 1 / math.sqrt(128), out)
    assert e.value.status == kvq.KVQ_ERR_CAPACITY
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was enqueued
