"""The Python binding refuses tensors the C calls would misread, before it
calls into the library: the C ABI sees only pointers, so a q or out with the
wrong dtype, shape, layout or device would become an out-of-bounds device
access.  Runs without a GPU: every case is refused on the host."""
import pytest
import torch

import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import build as kbuild


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()


H, D, HQ = 2, 64, 4


def _views(n=2, head_dim=D):
    vs = []
    for _ in range(n):
        v = kvq.View(H, head_dim, 4, 64, 16, device="cpu")
        v.set_state(32, 8)
        vs.append(v)
    return vs


def _q(n, hq=HQ, d=D, dtype=torch.bfloat16):
    return torch.zeros((n, hq, d), dtype=dtype)


def _out(n, hq=HQ, d=D, dtype=torch.float32):
    return torch.zeros((n, hq, d), dtype=dtype)


@pytest.mark.parametrize("q, why", [
    (_q(1), "shape"),                                    # fewer rows than views
    (_q(3), "shape"),                                    # more rows than views
    (_q(2, d=128), "shape"),                             # another head_dim
    (_q(2, hq=3), "multiple"),                           # H_q not a multiple of H_kv
    (_q(2, dtype=torch.float32), "bfloat16"),            # fp32 q
    (torch.zeros((HQ, 2, D), dtype=torch.bfloat16).transpose(0, 1), "contiguous"),
    (torch.zeros((2, HQ * D), dtype=torch.bfloat16), "3-d"),
    (_q(2), "CUDA"),                                     # right shape, but host memory
])
def test_decode_attn_rejects_bad_q(q, why):
    with pytest.raises(ValueError, match=why):
        kvq.decode_attn(_views(), q, 0.125, out=_out(2), workspace=torch.zeros(1 << 16, dtype=torch.uint8))


@pytest.mark.parametrize("out, why", [
    (_out(1), "shape"),
    (_out(2, d=128), "shape"),
    (_out(2, dtype=torch.bfloat16), "float32"),
    (torch.zeros((2, D, HQ), dtype=torch.float32).transpose(1, 2), "contiguous"),
])
def test_attention_entry_points_reject_bad_out(out, why):
    views = _views()
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match=why):
        kvq.decode_attn(views, _q(2), 0.125, out=out, workspace=ws)
    with pytest.raises(ValueError, match=why):
        kvq.decode_attn_noalloc(views, _q(2), 0.125, out)
    kn = torch.zeros((2, H, D), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match=why):
        kvq.append_decode_attn(views, kn, kn, _q(2), 0.125, out=out, workspace=ws)
    with pytest.raises(ValueError, match=why):
        kvq.decode_attn_seq(views, [0, 1, 2], _q(2), 0.125, out=out, workspace=ws)


@pytest.mark.parametrize("kn, why", [
    (torch.zeros((1, H, D), dtype=torch.bfloat16), "shape"),
    (torch.zeros((2, H + 1, D), dtype=torch.bfloat16), "shape"),
    (torch.zeros((2, H, D), dtype=torch.float16), "bfloat16"),
    (torch.zeros((2, D, H), dtype=torch.bfloat16).transpose(1, 2), "contiguous"),
])
def test_append_entry_points_reject_bad_new_tokens(kn, why):
    views = _views()
    good = torch.zeros((2, H, D), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match=why):
        kvq.append(views, kn, good)
    with pytest.raises(ValueError, match=why):
        kvq.append(views, good, kn)
    with pytest.raises(ValueError, match=why):
        kvq.append_decode_attn(views, kn, good, _q(2), 0.125, out=_out(2))
    # nothing was appended
    assert all(v.n_packed == 32 and v.n_window == 8 for v in views)


def test_views_of_one_call_must_agree():
    views = _views(1) + _views(1, head_dim=128)
    with pytest.raises(ValueError, match="same n_kv_heads and head_dim"):
        kvq.decode_attn(views, _q(2), 0.125, out=_out(2), workspace=torch.zeros(16, dtype=torch.uint8))


def test_sparse_and_sensitivity_check_their_outputs():
    views = _views()
    with pytest.raises(ValueError, match="shape"):
        kvq.sparse_decode_attn(views, _q(2), 0.125, 8, out=_out(2), workspace=torch.zeros(16, dtype=torch.uint8),
                               selected=torch.zeros((2, H, 7), dtype=torch.int32))
    with pytest.raises(ValueError, match="shape"):
        kvq.width_sensitivity(views, _q(2), 0.125, out=torch.zeros(3, dtype=torch.float32))
    with pytest.raises(ValueError, match="uint8"):
        kvq.decode_attn(views, _q(2), 0.125, out=_out(2), workspace=torch.zeros(16, dtype=torch.int32))
