"""kvq_allocate_widths (host code in the C library) against the oracle's
allocation: the same widths and the same total on random instances, the
budget extremes, and argument checks.  Runs without a GPU."""
import numpy as np
import pytest

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import build as kbuild


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()


@pytest.mark.parametrize("seed", range(8))
def test_allocation_matches_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 40))
    sens = rng.exponential(1.0, n).astype(np.float32)
    cap = rng.integers(0, 20000, n)
    H, D = int(rng.choice([1, 2, 8])), int(rng.choice([64, 128, 256]))
    per = lambda b: 2 * H * (D * b // 8 + D // 64 * 8)
    lo, hi = int((cap * per(2)).sum()), int((cap * per(8)).sum())
    for f in (1.0, 0.3, 0.7, 1.2):
        budget = int(lo + f * (hi - lo))
        want = oracle.allocate_widths(sens, cap, H, D, budget, units=512)
        got = kvq.allocate_widths(sens, cap, H, D, budget, units=512)
        assert want is not None
        assert got[0] == want[0] and got[1] == want[1], (seed, f)
        used = sum(c * per(b) for c, b in zip(cap, got[0]))
        assert used <= budget


def test_allocation_budget_extremes_and_errors():
    sens, cap, H, D = [2.0, 0.5], [1000, 3000], 8, 128
    per = lambda b: 2 * H * (D * b // 8 + D // 64 * 8)
    bits, total = kvq.allocate_widths(sens, cap, H, D, 10 ** 12)
    assert bits == [8, 8] and total == pytest.approx(2.0 / 255 + 0.5 / 255)
    floor = sum(c * per(2) for c in cap)
    with pytest.raises(kvq.KvqError) as e:
        kvq.allocate_widths(sens, cap, H, D, floor - 1)
    assert e.value.status == kvq.KVQ_ERR_CAPACITY
    with pytest.raises(kvq.KvqError) as e:
        kvq.allocate_widths(sens, cap, H, D, floor, units=0)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    with pytest.raises(kvq.KvqError) as e:
        kvq.allocate_widths([-1.0, 0.5], cap, H, D, floor * 4)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    with pytest.raises(kvq.KvqError) as e:
        kvq.allocate_widths(sens, cap, H, 96, floor * 4)
    assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED
    # views with nothing left to quantize cost nothing and take 8 bits (costs
    # are rounded up to whole units, so an exact fit needs a little slack)
    bits, _ = kvq.allocate_widths([1.0, 1.0], [0, 1000], H, D, int(1000 * per(2) * 1.01))
    assert bits == [8, 2]


def test_allocation_refuses_oversized_tables():
    n = 2048
    with pytest.raises(kvq.KvqError) as e:
        kvq.allocate_widths(np.ones(n, np.float32), np.full(n, 1000), 8, 128, 10 ** 12, units=1 << 20)
    assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED


def test_allocation_costs_wider_than_64_bits():
    # at the argument limits a width's byte cost, 2^40 tokens x 2 x 65535 heads
    # x 288 bytes at 8 bits and head_dim 256, needs more than 64 bits: it must
    # come out unaffordable, not wrap around to a small cost that fits the
    # budget (wrapped, 8 bits would cost about 934 of 4096 units here)
    H, D = 65535, 256
    per = lambda b: 2 * H * (D * b // 8 + D // 64 * 8)
    cap = [1 << 40]
    assert cap[0] * per(8) >= 1 << 64 > cap[0] * per(2)
    budget = (1 << 64) - 1
    want = oracle.allocate_widths([1.0], cap, H, D, budget, units=4096)
    got = kvq.allocate_widths([1.0], cap, H, D, budget, units=4096)
    assert got[0] == want[0] and got[1] == want[1]
    assert got[0] == [2]
    # below the 2-bit cost nothing fits
    with pytest.raises(kvq.KvqError) as e:
        kvq.allocate_widths([1.0], cap, H, D, cap[0] * per(2) - 1, units=4096)
    assert e.value.status == kvq.KVQ_ERR_CAPACITY
