"""kvq_quantize / kvq_dequantize on the GPU against the oracle: bit-exact codes,
packed bytes, scales, mins and bf16 outputs, on ragged sizes, strided inputs,
special values, and sampled rows of the full bulk-handoff workload."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu
BITS = (2, 3, 4, 8)
DIMS = (64, 128, 192, 256)


def special_rows(D, bits, rng):
    """bf16 bit patterns of rows that stress the format's corner cases."""
    qmax = (1 << bits) - 1
    rows = []
    z = np.zeros(D, np.float32)
    rows.append(z.copy())                                          # all +0
    r = z.copy(); r[::2] = -0.0; rows.append(r)                    # +0 / -0 mix
    rows.append(np.full(D, 1.5, np.float32))                       # constant
    r = np.zeros(D, np.float32)                                    # exact ties
    for g in range(D // 64):
        r[64 * g] = 0.0
        r[64 * g + 1] = float(qmax)
        k = np.arange(62) % min(qmax, 127)
        r[64 * g + 2: 64 * g + 64] = k + 0.5
    rows.append(r)
    r = rng.integers(0, qmax + 1, D).astype(np.float32) * 0.25 - 3.0   # on grid, s = 1/4
    for g in range(D // 64):
        r[64 * g] = -3.0
        r[64 * g + 1] = -3.0 + 0.25 * qmax
    rows.append(r)
    rows.append((rng.standard_normal(D) * 1e30).astype(np.float32))    # huge range
    rows.append((rng.standard_normal(D) * 1e-3).astype(np.float32))
    out = torch.tensor(np.stack(rows)).to(torch.bfloat16)
    bits_u16 = out.view(torch.int16).numpy().view(np.uint16).copy()
    # subnormal bf16 values and zeros
    sub = rng.integers(0, 0x80, D).astype(np.uint16)
    sub[::3] |= 0x8000
    bits_u16 = np.concatenate([bits_u16, sub[None]], axis=0)
    return bits_u16


def to_bf16_tensor(bits_u16):
    return torch.from_numpy(bits_u16.view(np.int16).copy()).view(torch.bfloat16)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("D", DIMS)
def test_quantize_dequantize_bit_exact(cuda_device, bits, D):
    rng = np.random.default_rng(bits * 1000 + D)
    g = wl.generator(bits * 31 + D)
    H, T, cap, T0 = 3, 37, 45, 5
    mask = wl.outlier_mask(g, H, D, 0.0, first4=True)
    big = wl.normal_bf16(g, (H, T0 + T + 3, D), scale_mask=mask)
    sp = to_bf16_tensor(special_rows(D, bits, rng))
    big[1, T0 + 3:T0 + 3 + sp.shape[0]] = sp
    x = big[:, T0:T0 + T, :]                         # strided view: token offset, head stride of `big`
    xg = big.to(cuda_device)[:, T0:T0 + T, :]
    rb = kvq.row_bytes(D, bits)
    codes = torch.full((H, cap, rb), 0xAB, dtype=torch.uint8, device=cuda_device)
    sm = torch.full((H, cap, D // 64, 2), -7.0, dtype=torch.float32, device=cuda_device)
    kvq.quantize(xg, bits, codes, sm)
    torch.cuda.synchronize()
    want_c, want_s = oracle.quantize(wl.bf16_bits(x), bits)
    got_c = codes.cpu().numpy()
    got_s = sm.cpu().numpy()
    assert np.array_equal(got_c[:, :T], want_c)
    assert np.array_equal(got_s[:, :T].view(np.uint32), want_s.view(np.uint32))   # bit patterns (+0 vs -0)
    assert np.all(got_c[:, T:] == 0xAB) and np.all(got_s[:, T:] == -7.0)       # rows past n_tokens untouched

    y = kvq.dequantize(codes, sm, T, D, bits)
    torch.cuda.synchronize()
    want_y = oracle.dequantize(want_c, want_s, D, bits)
    assert np.array_equal(wl.bf16_bits(y), want_y)


@pytest.mark.parametrize("bits", BITS)
def test_dequantize_into_strided_output(cuda_device, bits):
    g = wl.generator(500 + bits)
    H, T, D = 2, 20, 128
    x = wl.normal_bf16(g, (H, T, D))
    codes, sm = kvq.quantize(x.to(cuda_device), bits)
    out_big = torch.full((H, T + 4, D + 64), 3.0, dtype=torch.bfloat16, device=cuda_device)
    out = out_big[:, 2:T + 2, 32:32 + D]
    kvq.dequantize(codes, sm, T, D, bits, out=out)
    torch.cuda.synchronize()
    want = oracle.dequantize(*oracle.quantize(wl.bf16_bits(x), bits), D, bits)
    assert np.array_equal(wl.bf16_bits(out), want)
    ob = out_big.cpu()
    assert torch.all(ob[:, :2] == 3.0) and torch.all(ob[:, T + 2:] == 3.0)
    assert torch.all(ob[:, :, :32] == 3.0) and torch.all(ob[:, :, 32 + D:] == 3.0)


def test_empty_inputs_enqueue_nothing(cuda_device):
    x = torch.empty((4, 0, 128), dtype=torch.bfloat16, device=cuda_device)
    codes, sm = kvq.quantize(x, 4)
    assert codes.shape == (4, 0, 64)


def test_bulk_handoff_full_size_sampled(cuda_device):
    """Bulk cache handoff, Llama-3.1-8B shape (32 layers x 8 KV heads x 32768
    tokens x 128, K and V, 4-bit, 1% K outlier channels): full-size quantize and
    dequantize on the GPU, sampled rows checked bit-exactly against the oracle,
    and the round-trip error bound checked on every element."""
    w = wl.handoff_llama8b()
    H = w.n_layers * w.n_kv_heads
    gm = wl.generator(w.seed)
    mask = torch.stack([wl.outlier_mask(gm, w.n_kv_heads, w.head_dim, w.outlier_frac)
                        for _ in range(w.n_layers)]).view(H, w.head_dim)
    g = wl.generator(w.seed, device=cuda_device)
    k, v = wl.kv_pair(g, H, w.n_tokens, w.head_dim, mask, cuda_device)
    rng = np.random.default_rng(0)
    rows_h = rng.integers(0, H, 1024)
    rows_t = rng.integers(0, w.n_tokens, 1024)
    rows_t[:8] = [0, 1, w.n_tokens - 1, w.n_tokens - 2, 15, 16, 17, 12345]
    for name, x in (("K", k), ("V", v)):
        codes, sm = kvq.quantize(x, w.bits)
        y = kvq.dequantize(codes, sm, w.n_tokens, w.head_dim, w.bits)
        torch.cuda.synchronize()
        # every element: |y - x| <= s/2 (+ fp32 slack) + half a bf16 ulp of y
        s = sm[..., 0].repeat_interleave(64, dim=-1)
        err = (y.float() - x.float()).abs()
        bound = s * (0.5 + 2.0 ** (w.bits - 23)) + y.float().abs() * 2.0 ** -8 + 1e-30
        assert bool((err <= bound).all()), name
        del err, bound, s
        xs = wl.bf16_bits(x[rows_h, rows_t])
        want_c, want_s = oracle.quantize(xs, w.bits)
        assert np.array_equal(codes[rows_h, rows_t].cpu().numpy(), want_c), name
        assert np.array_equal(sm[rows_h, rows_t].cpu().numpy().view(np.uint32), want_s.view(np.uint32)), name
        assert np.array_equal(wl.bf16_bits(y[rows_h, rows_t]), oracle.dequantize(want_c, want_s, w.head_dim, w.bits))
        del codes, sm, y
    torch.cuda.empty_cache()
