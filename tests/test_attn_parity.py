"""kvq_decode_attn on the GPU against the fp64 oracle (tolerance: 2e-3
max-abs and 1e-3 relative L2 per (view, head)), over the five workload shapes
at sizes the oracle finishes quickly, plus the edge cases: empty packed part,
no window, ragged tiles, ring wrap, every width, GQA 1..16, head_dim 64..256."""
import math

import numpy as np
import pytest
import torch

from helpers import ViewSpec, assert_close, build_case, oracle_view, run_gpu

pytestmark = pytest.mark.gpu


def check_case(case, scale, what):
    out = run_gpu(case, scale)
    for i in range(len(case.specs)):
        ref = oracle_view(case, i, scale)
        assert_close(out[i], ref, f"{what} view {i} {case.specs[i]}")
    return out


def test_tiny_single_agent(cuda_device):
    """1 view, 4 q / 2 kv heads, D 64, 256 packed tokens @4b, no window, K
    channels 0-3 x10, scale 1/8."""
    case = build_case(4, 2, 64, [ViewSpec(256, 0, 0, 4, seed=1, first4=True)], q_seed=1)
    check_case(case, 1 / 8, "tiny")


def test_llama8b_shape_small(cuda_device):
    """32 q / 8 kv heads, D 128, 4096 packed @4b + full 128-token window (ring wrapped)."""
    specs = [ViewSpec(4096, 128, 128, 4, head=37 * i % 128, seed=30 + i) for i in range(3)]
    check_case(build_case(32, 8, 128, specs, q_seed=3), 1 / math.sqrt(128), "llama8b")


def test_gemma12b_shape_small(cuda_device):
    """16 q / 8 kv heads, D 256, varied lengths, 256-token window, K outliers."""
    specs = [ViewSpec(n, 256, 256, 4, head=11 * i, seed=40 + i, outlier_frac=0.01)
             for i, n in enumerate((4096, 1000, 8192))]
    check_case(build_case(16, 8, 256, specs, q_seed=4), 1 / 16, "gemma12b")


def test_qwen32b_shape_mixed_bits_small(cuda_device):
    """64 q / 8 kv heads, D 128, widths {2,3,4,8} per view, ragged lengths."""
    rng = np.random.default_rng(5)
    specs = []
    for i, b in enumerate((2, 3, 4, 8, 2, 3, 2, 8)):
        n = int(rng.integers(500, 3000))
        specs.append(ViewSpec(n, 128, 128, b, head=int(rng.integers(0, 128)), seed=50 + i, outlier_frac=0.01))
    check_case(build_case(64, 8, 128, specs, q_seed=5), 1 / math.sqrt(128), "qwen32b")


@pytest.mark.parametrize("bits", (2, 3, 4, 8))
@pytest.mark.parametrize("D", (64, 128, 192, 256))
def test_every_width_and_head_dim(cuda_device, bits, D):
    specs = [ViewSpec(333, 20, 32, bits, head=25, seed=bits * 100 + D, first4=True),
             ViewSpec(16, 0, 0, bits, seed=bits * 100 + D + 1)]
    check_case(build_case(8, 2, D, specs, q_seed=D + bits), 1 / math.sqrt(D), f"b{bits} D{D}")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (6, 2), (16, 1), (24, 2), (12, 4)])
def test_gqa_group_sizes(cuda_device, hq, hkv):
    specs = [ViewSpec(700, 9, 16, 4, head=12, seed=hq * 10 + hkv)]
    check_case(build_case(hq, hkv, 128, specs, q_seed=hq), 0.1, f"GQA {hq}/{hkv}")


def test_edge_lengths_and_ring_states(cuda_device):
    specs = [
        ViewSpec(0, 5, 8, 4, head=0, seed=1),        # window only
        ViewSpec(0, 8, 8, 4, head=6, seed=2),        # window only, wrapped
        ViewSpec(1, 0, 0, 4, seed=3),                # one packed token
        ViewSpec(17, 0, 0, 3, seed=4),               # one full tile + 1
        ViewSpec(15, 1, 4, 2, head=3, seed=5),       # partial tile + one window token
        ViewSpec(16, 4, 8, 8, head=6, seed=6),       # window wraps around slot 0
        ViewSpec(4097, 3, 1024, 4, head=1023, seed=7),  # wrap at the last slot
        ViewSpec(2, 0, 0, 3, seed=8),
    ]
    check_case(build_case(8, 2, 64, specs, q_seed=7), 0.125, "edges")


def test_single_call_over_many_views_spanning_launches(cuda_device):
    """More views than one launch holds (parameter-space batching)."""
    specs = [ViewSpec(64 + 7 * i, 8, 8, (2, 3, 4, 8)[i % 4], head=i % 8, seed=900 + i) for i in range(200)]
    case = build_case(4, 2, 64, specs, q_seed=9)
    out = run_gpu(case, 0.125)
    for i in (0, 1, 95, 96, 97, 150, 199):
        assert_close(out[i], oracle_view(case, i, 0.125), f"many view {i}")


def test_chunking_changes_only_rounding(cuda_device, monkeypatch):
    specs = [ViewSpec(3000, 64, 64, 4, head=9, seed=77), ViewSpec(1200, 64, 64, 2, head=0, seed=78)]
    case = build_case(16, 4, 128, specs, q_seed=11)
    ref = [oracle_view(case, i, 0.09) for i in range(2)]
    outs = []
    for chunk in ("16", "64", "256", "1024", "8192"):
        monkeypatch.setenv("KVQ_CHUNK_TOKENS", chunk)
        out = run_gpu(case, 0.09)
        for i in range(2):
            assert_close(out[i], ref[i], f"chunk {chunk}")
        outs.append(out)


@pytest.mark.parametrize("D,bits", [(256, 4), (128, 8), (128, 2), (64, 3)])
def test_long_single_chunk(cuda_device, monkeypatch, D, bits):
    """32768 packed tokens forced into ONE chunk, so one warp (or team) sweeps
    the whole view: the error must not grow with the tokens a warp
    accumulates.  A PV accumulator chained through every tile's MMA drops low
    bits at each tile, always downward, and fails here (about 4e-2 relative L2
    at head_dim 256)."""
    hq, hkv = (16, 8) if D == 256 else (8, 2)
    specs = [ViewSpec(32768, 64, 64, bits, head=5, seed=90 + bits, outlier_frac=0.01)]
    case = build_case(hq, hkv, D, specs, q_seed=14)
    monkeypatch.setenv("KVQ_CHUNK_TOKENS", "32768")
    scale = 1 / math.sqrt(D)
    out = run_gpu(case, scale)
    assert_close(out[0], oracle_view(case, 0, scale), f"one chunk, D {D}, {bits} bits")


def test_bitwise_deterministic(cuda_device):
    specs = [ViewSpec(5000, 128, 128, 4, head=3, seed=60), ViewSpec(777, 100, 128, 3, head=120, seed=61)]
    case = build_case(32, 8, 128, specs, q_seed=12)
    a = run_gpu(case, 0.088)
    b = run_gpu(case, 0.088)
    assert np.array_equal(a, b)


def test_workspace_status_word_stays_clear(cuda_device):
    import quantized_kv_cache_dequantize_b200 as kvq
    specs = [ViewSpec(2048, 16, 16, 4, seed=70)]
    case = build_case(8, 2, 128, specs, q_seed=13)
    ws = kvq.new_workspace(case.views, 8)
    run_gpu(case, 0.1, workspace=ws)
    run_gpu(case, 0.1, workspace=ws)
    torch.cuda.synchronize()
    status = int(ws[:4].view(torch.int32).item())
    assert status == 0
