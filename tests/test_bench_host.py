"""bench.py's host-side oracle timing runs on the CPU: the single-thread
sample and its split over (view, KV head) on host threads count the same
bytes and compute the same outputs (checked on the tiny workload)."""
import numpy as np

import bench
import oracle
from quantized_kv_cache_dequantize_b200 import workloads as wl


def test_threaded_oracle_timing_counts_the_same_bytes():
    w = wl.tiny()
    secs1, nb1 = bench.oracle_sample(w, [(0, 0)], device="cpu")
    secs2, nb2, threads = bench.oracle_threaded(w, [(0, 0)], device="cpu")
    assert nb1 == nb2 > 0 and secs1 > 0 and secs2 > 0 and threads >= 1


def test_one_call_per_kv_head_gives_the_whole_view():
    # the split the threaded timing uses computes exactly what one call does
    g = wl.generator(3)
    Hq, Hkv, D, n = 8, 2, 64, 40
    k, v = wl.kv_pair(g, Hkv, n, D, None)
    q = wl.bf16_bits(wl.normal_bf16(g, (Hq, D)))
    kb, vb = wl.bf16_bits(k), wl.bf16_bits(v)
    kc, ks = oracle.quantize(kb[:, :32], 4)
    vc, vs = oracle.quantize(vb[:, :32], 4)
    whole = oracle.decode_attn(q, 4, kc, ks, vc, vs, kb[:, 32:], vb[:, 32:], 0.125)
    G = Hq // Hkv
    for hk in range(Hkv):
        h = slice(hk, hk + 1)
        part = oracle.decode_attn(q[hk * G:(hk + 1) * G], 4, kc[h], ks[h], vc[h], vs[h], kb[h, 32:], vb[h, 32:], 0.125)
        assert np.array_equal(part, whole[hk * G:(hk + 1) * G])
