"""kvq_quantize / kvq_dequantize on the GPU against the oracle: bit-exact codes,
packed bytes, scales, mins and bf16 outputs, on ragged sizes, strided inputs,
special values, and every row of the full bulk-handoff workload."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from helpers import OracleRunner

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


def offset_rows(D, bits, rng):
    """bf16 rows whose groups sit far from zero against their range: each
    group is min = +-2^e plus 0..J bf16 ulps of 2^e (exact in bf16, both ends
    present, ties among them), so |min| / scale = 128 * (2^bits - 1) / J runs
    from about 2^bits to 2^(bits+7), across the point 2^(bits+2) where the
    quantizer's fast path changes its arithmetic."""
    rows = []
    for J in (1, 3, 8, 20, 32, 48, 100, 127):
        for sign in (1.0, -1.0):
            r = np.zeros(D, np.float32)
            for g in range(D // 64):
                e = int(rng.integers(-8, 9))
                ulp = 2.0 ** (e - 7)
                j = rng.integers(0, J + 1, 64).astype(np.float32)
                j[0], j[1] = 0, J
                r[64 * g:64 * g + 64] = sign * 2.0 ** e + j * ulp
            rows.append(r)
    out = torch.tensor(np.stack(rows)).to(torch.bfloat16)
    assert np.array_equal(out.float().numpy(), np.stack(rows))   # exact in bf16
    return out.view(torch.int16).numpy().view(np.uint16).copy()


@pytest.mark.parametrize("bits", BITS)
def test_quantize_groups_far_from_zero(cuda_device, bits):
    rng = np.random.default_rng(77 + bits)
    for D in (64, 192):
        xb = offset_rows(D, bits, rng)
        x = to_bf16_tensor(xb)[None]                 # [1, rows, D]
        codes, sm = kvq.quantize(x.to(cuda_device), bits)
        torch.cuda.synchronize()
        want_c, want_s = oracle.quantize(xb[None], bits)
        assert np.array_equal(codes.cpu().numpy(), want_c), (bits, D)
        assert np.array_equal(sm.cpu().numpy().view(np.uint32), want_s.view(np.uint32)), (bits, D)
        y = kvq.dequantize(codes, sm, xb.shape[0], D, bits)
        torch.cuda.synchronize()
        assert np.array_equal(wl.bf16_bits(y), oracle.dequantize(want_c, want_s, D, bits)), (bits, D)


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


def test_bulk_handoff_full_size(cuda_device):
    """Bulk cache handoff, Llama-3.1-8B shape (32 layers x 8 KV heads x 32768
    tokens x 128, K and V, 4-bit, 1% K outlier channels): full-size quantize and
    dequantize on the GPU, one launch each as the bench runs them, and every
    row of both checked bit for bit against the oracle (codes, scale/min bit
    patterns and dequantized bf16), one KV head per oracle call on host
    threads."""
    w = wl.handoff_llama8b()
    H = w.n_layers * w.n_kv_heads
    gm = wl.generator(w.seed)
    mask = torch.stack([wl.outlier_mask(gm, w.n_kv_heads, w.head_dim, w.outlier_frac)
                        for _ in range(w.n_layers)]).view(H, w.head_dim)
    g = wl.generator(w.seed, device=cuda_device)
    k, v = wl.kv_pair(g, H, w.n_tokens, w.head_dim, mask, cuda_device)

    def check_head(name, h, xs, gc, gs, gy):
        want_c, want_s = oracle.quantize(xs, w.bits)
        if not np.array_equal(gc, want_c):
            return f"{name} head {h}: codes differ in {int((gc != want_c).any(-1).sum())} rows"
        if not np.array_equal(gs.view(np.uint32), want_s.view(np.uint32)):
            return f"{name} head {h}: scale/min differ"
        if not np.array_equal(gy, oracle.dequantize(want_c, want_s, w.head_dim, w.bits)):
            return f"{name} head {h}: dequantized values differ"
        return None

    run = OracleRunner()
    for name, x in (("K", k), ("V", v)):
        codes, sm = kvq.quantize(x, w.bits)
        y = kvq.dequantize(codes, sm, w.n_tokens, w.head_dim, w.bits)
        torch.cuda.synchronize()
        for h0 in range(0, H, 8):  # one layer's heads per host copy
            xs = wl.bf16_bits(x[h0:h0 + 8])
            gc = codes[h0:h0 + 8].cpu().numpy()
            gs = sm[h0:h0 + 8].cpu().numpy()
            gy = wl.bf16_bits(y[h0:h0 + 8])
            for j in range(8):
                run.submit(check_head, name, h0 + j, xs[j], gc[j], gs[j], gy[j])
        del codes, sm, y
    assert run.finish() == 2 * H
    torch.cuda.empty_cache()
