"""Small cases of every kernel family, run through the library the
environment selects (KVQ_DEBUG=1: the debug build with device bounds checks).
Prints one line "flags=<word> checked=<n>" after checking the outputs against
the oracle; exits non-zero on a mismatch.  Run by tests/test_debug_build.py in
a child process, so that the debug library is the one loaded."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import quantized_kv_cache_dequantize_b200 as kvq  # noqa: E402
from quantized_kv_cache_dequantize_b200 import workloads as wl  # noqa: E402
from helpers import ViewSpec, assert_close, build_case, oracle_view  # noqa: E402


def main():
    dev = torch.device("cuda:0")
    checked = 0
    assert kvq.lib().kvq_debug_build() == (1 if os.environ.get("KVQ_DEBUG") == "1" else 0)
    kvq.debug_flags(clear=True)
    # codec: every width, a ragged length, strided input, bit-exact
    g = wl.generator(11)
    for bits in (2, 3, 4, 8):
        for D in (64, 256):
            x = wl.normal_bf16(g, (3, 37, D)).to(dev)
            codes, sm = kvq.quantize(x, bits)
            y = kvq.dequantize(codes, sm, 37, D, bits)
            torch.cuda.synchronize()
            want_c, want_s = oracle.quantize(wl.bf16_bits(x), bits)
            assert np.array_equal(codes.cpu().numpy(), want_c)
            assert np.array_equal(sm.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
            assert np.array_equal(wl.bf16_bits(y), oracle.dequantize(want_c, want_s, D, bits))
            checked += 1
    # attention: mixed widths, windows, GQA 4, a window-only view, forced chunks
    scale = 1 / np.sqrt(128)
    case = build_case(8, 2, 128, [ViewSpec(300, 16, 16, 4, head=3, seed=1), ViewSpec(97, 0, 0, 2, seed=2),
                                  ViewSpec(0, 5, 8, 3, head=6, seed=3), ViewSpec(513, 8, 8, 8, head=1, seed=4)],
                      extra_packed=8)  # room for the decode steps below
    out = kvq.decode_attn(case.views, case.q, scale)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for i in range(4):
        assert_close(got[i], oracle_view(case, i, scale), f"debug decode view {i}")
        checked += 1
    os.environ["KVQ_CHUNK_TOKENS"] = "48"
    out2 = kvq.decode_attn(case.views, case.q, scale)
    os.environ.pop("KVQ_CHUNK_TOKENS")
    torch.cuda.synchronize()
    for i in range(4):
        assert_close(out2[i].cpu().numpy().astype(np.float64), oracle_view(case, i, scale), f"chunked view {i}")
        checked += 1
    # decode steps (append + attention), then appends alone, on the same views
    kn = wl.normal_bf16(g, (4, 2, 128)).to(dev)
    for _ in range(3):
        kvq.append_decode_attn(case.views, kn, kn, case.q, scale)
    kvq.append(case.views, kn, kn)
    # sequences of several views, top-K sparse decode, sensitivity, cards
    kvq.decode_attn_seq(case.views, [0, 2, 4], case.q[:2].contiguous(), scale)
    kvq.sparse_decode_attn(case.views, case.q, scale, 40)
    kvq.width_sensitivity(case.views, case.q, scale)
    card = kvq.card_pack(case.views)
    fresh = kvq.views_for_card(card.cpu(), device=dev)
    kvq.card_unpack(card.cpu(), fresh)
    assert torch.equal(kvq.decode_attn(fresh, case.q, scale), kvq.decode_attn(case.views, case.q, scale))
    checked += 1
    torch.cuda.synchronize()
    flags = kvq.debug_flags(clear=True)
    print(f"flags={flags} checked={checked}", flush=True)


if __name__ == "__main__":
    main()
