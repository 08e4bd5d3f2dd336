"""kvq_width_sensitivity on the GPU against the oracle's fp64 bound
coefficient (fp32 on the GPU: 1e-5 relative), over widths, head_dims, GQA
groups, ring states and empty windows; then a whole allocation step: the
sensitivities of a mixed workload feed kvq_allocate_widths."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from helpers import ViewSpec, build_case

pytestmark = pytest.mark.gpu


def window_bits(case, i):
    s, h = case.specs[i], case.host[i]
    return h["k"][:, s.n_packed:], h["v"][:, s.n_packed:]


@pytest.mark.parametrize("D,hq,hkv", [(64, 4, 2), (128, 32, 8), (256, 16, 8), (128, 64, 8)])
def test_sensitivity_matches_oracle(cuda_device, D, hq, hkv):
    specs = [ViewSpec(64, 16, 16, 4, head=5, seed=800, outlier_frac=0.02),
             ViewSpec(0, 7, 8, 2, head=3, seed=801),
             ViewSpec(32, 0, 0, 8, seed=802),                       # no window: 0
             ViewSpec(10, 128, 128, 3, head=127, seed=803, first4=True)]
    case = build_case(hq, hkv, D, specs)
    scale = 1 / np.sqrt(D)
    got = kvq.width_sensitivity(case.views, case.q, scale).cpu().numpy().astype(np.float64)
    for i in range(len(specs)):
        kw, vw = window_bits(case, i)
        want = oracle.width_sensitivity(case.q_bits[i], kw, vw, scale)[0]
        assert got[i] == pytest.approx(want, rel=1e-5, abs=1e-30), (i, got[i], want)
    assert got[2] == 0.0


def test_allocation_from_measured_sensitivities(cuda_device):
    # the mixed-precision workload's shape, small: 8 agents x 4 layers
    specs = [ViewSpec(256, 32, 32, 4, head=i % 32, seed=900 + i, outlier_frac=0.01 * (i % 3)) for i in range(32)]
    case = build_case(16, 2, 128, specs)
    sens = kvq.width_sensitivity(case.views, case.q, 1 / np.sqrt(128)).cpu().numpy()
    cap = np.full(32, 4096)
    per = lambda b: 2 * 2 * (128 * b // 8 + 16)
    budget = int(cap.sum() * per(3))  # an average of 3 bits' storage
    bits, total = kvq.allocate_widths(sens, cap, 2, 128, budget)
    want = oracle.allocate_widths(sens, cap, 2, 128, budget)
    assert bits == want[0] and total == want[1]
    assert sum(c * per(b) for c, b in zip(cap, bits)) <= budget
    assert len(set(bits)) > 1  # the sensitivities differ enough to mix widths
