"""Quantized KV-cache handoff and decode attention for NVIDIA B200 (sm_100a).

A thin binding over the C ABI of ``libkvq.so`` (declared in ``include/kvq.h``).
Every computation of the method runs in the library's CUDA kernels; this module
only marshals torch tensors (device memory and the current stream) into the C
calls.  There is no CPU fallback: if the library is missing, every entry point
raises.

Entry points (same names as the C ABI, without the ``kvq_`` prefix):
  quantize, dequantize          -- bf16 rows <-> packed b-bit codes + {s, mn}
  View, append                  -- one (agent, layer) cache; add a decode token
  decode_attn, workspace_size   -- batched split-K attention over many views
  sparse_decode_attn            -- top-K sparse decode: the K best packed tokens
                                   per (view, KV head) by query score, plus the
                                   bf16 window
  decode_attn_seq               -- the same over sequences held by several views
                                   (segments) of any widths; View.new_segment
                                   starts a segment at a new width
  append_decode_attn            -- one decode step: append, then attend, in one call
  width_sensitivity, allocate_widths
                                -- per-view sensitivity to the width from the
                                   recent window and query; exact width choice
                                   under a shared byte budget
  card_pack, card_unpack, ...   -- CacheCard: several views' caches as one
                                   artifact (transfer, save_card / load_card)
  decode_attn_noalloc           -- the same without a workspace: scratch is a
                                   fixed per-device array inside the library
                                   (NOALLOC_SCRATCH_BYTES), for callers that
                                   cannot allocate device memory when they attend
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import workloads  # noqa: F401  (seeded input generators)

__all__ = ["quantize", "dequantize", "View", "append", "decode_attn", "workspace_size", "append_decode_attn",
           "step_workspace_size", "decode_attn_noalloc", "decode_attn_noalloc_status", "decode_attn_seq", "seq_workspace_size",
           "new_seq_workspace", "MAX_SEGMENTS", "sparse_decode_attn", "sparse_workspace_size",
           "width_sensitivity", "allocate_widths", "card_bytes", "card_pack", "card_info", "card_unpack",
           "views_for_card", "save_card", "load_card", "NOALLOC_SCRATCH_BYTES", "KvqError", "lib", "debug_flags",
           "row_bytes", "GROUP"]

GROUP = 64
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024   # KVQ_NOALLOC_SCRATCH_BYTES in kvq.h
MAX_SEGMENTS = 64                          # KVQ_MAX_SEGMENTS in kvq.h
_HERE = os.path.dirname(os.path.abspath(__file__))
# KVQ_DEBUG=1 in the environment selects the debug build (device bounds
# checks recorded in a flags word, see debug_flags); read once, at first use
_LIB_PATH = os.path.join(_HERE, "libkvq_debug.so" if os.environ.get("KVQ_DEBUG") == "1" else "libkvq.so")
_lib = None

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_CUDA = range(5)


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        name = lib().kvq_status_string(status).decode()
        super().__init__(f"{where}: {name}")
        self.status = status


class CView(ctypes.Structure):
    """ctypes mirror of ``kvq_view``."""
    _fields_ = [("bits", ctypes.c_int32), ("n_window", ctypes.c_int32),
                ("cap_window", ctypes.c_int32), ("window_head", ctypes.c_int32),
                ("n_packed", ctypes.c_int64), ("cap_packed", ctypes.c_int64),
                ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_scalemin", ctypes.c_void_p), ("v_scalemin", ctypes.c_void_p),
                ("k_window", ctypes.c_void_p), ("v_window", ctypes.c_void_p)]


def lib():
    """The loaded ``libkvq.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libkvq.so not found at {_LIB_PATH}; build it with "
                               "`python -m quantized_kv_cache_dequantize_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.kvq_status_string.argtypes = [i32]
        L.kvq_status_string.restype = ctypes.c_char_p
        L.kvq_abi_version.argtypes = []
        L.kvq_abi_version.restype = i32
        L.kvq_quantize.argtypes = [P, i64, i64, i32, i64, i32, i32, P, P, i64, P]
        L.kvq_quantize.restype = i32
        L.kvq_dequantize.argtypes = [P, P, i64, i32, i64, i32, i32, P, i64, i64, P]
        L.kvq_dequantize.restype = i32
        L.kvq_append.argtypes = [ctypes.POINTER(CView), i32, i32, i32, P, P, P]
        L.kvq_append.restype = i32
        L.kvq_decode_attn_workspace_size.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32]
        L.kvq_decode_attn_workspace_size.restype = sz
        L.kvq_decode_attn.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32, P, f32, P, P, sz, P]
        L.kvq_decode_attn.restype = i32
        L.kvq_decode_attn_seq_workspace_size.argtypes = [ctypes.POINTER(CView), i32, P, i32, i32, i32, i32]
        L.kvq_decode_attn_seq_workspace_size.restype = sz
        L.kvq_decode_attn_seq.argtypes = [ctypes.POINTER(CView), i32, P, i32, i32, i32, i32, P, f32, P, P, sz, P]
        L.kvq_decode_attn_seq.restype = i32
        L.kvq_sparse_decode_attn_workspace_size.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32, i32]
        L.kvq_sparse_decode_attn_workspace_size.restype = sz
        L.kvq_sparse_decode_attn.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32, P, f32, i32, P, P, P, sz,
                                             P]
        L.kvq_sparse_decode_attn.restype = i32
        L.kvq_width_sensitivity.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32, P, f32, P, P]
        L.kvq_width_sensitivity.restype = i32
        L.kvq_allocate_widths.argtypes = [P, P, i32, i32, i32, ctypes.c_uint64, i32, P, P]
        L.kvq_allocate_widths.restype = i32
        L.kvq_append_decode_attn.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32, P, P, P, f32, P, P, sz, P]
        L.kvq_append_decode_attn.restype = i32
        u64 = ctypes.c_uint64
        L.kvq_card_bytes.argtypes = [ctypes.POINTER(CView), i32, i32, i32]
        L.kvq_card_bytes.restype = sz
        L.kvq_card_pack.argtypes = [ctypes.POINTER(CView), i32, i32, i32, u64, P, P, sz, P]
        L.kvq_card_pack.restype = i32
        L.kvq_card_read_header.argtypes = [P, sz, P, P, P, P]
        L.kvq_card_read_header.restype = i32
        L.kvq_card_view_info.argtypes = [P, sz, i32, P, P, P, P]
        L.kvq_card_view_info.restype = i32
        L.kvq_card_unpack.argtypes = [P, P, sz, ctypes.POINTER(CView), i32, i32, i32, P]
        L.kvq_card_unpack.restype = i32
        L.kvq_decode_attn_noalloc.argtypes = [ctypes.POINTER(CView), i32, i32, i32, i32, P, f32, P, P]
        L.kvq_decode_attn_noalloc.restype = i32
        L.kvq_decode_attn_noalloc_status.argtypes = [P, P]
        L.kvq_decode_attn_noalloc_status.restype = i32
        L.kvq_debug_build.argtypes = []
        L.kvq_debug_build.restype = i32
        L.kvq_debug_flags.argtypes = [P, i32, P]
        L.kvq_debug_flags.restype = i32
        _lib = L
    return _lib


def row_bytes(head_dim: int, bits: int) -> int:
    return head_dim // 8 * bits


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != KVQ_OK:
        raise KvqError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _views_device(views):
    return views[0].k_codes.device


def _check_tensor(name, t, dtype, shape, device):
    """A tensor the C call reads or writes as a dense array: dtype, shape,
    contiguity and device must match, since the library sees only a pointer."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the views are on {device}")


def _require_cuda(dev):
    """Last of the checks: the views (and so every tensor checked against
    them) must be in device memory."""
    if dev.type != "cuda":
        raise ValueError(f"the views and tensors must be CUDA tensors, not {dev}")


def _check_views(views):
    """The views of one call share n_kv_heads and head_dim (the C ABI takes them once)."""
    if not views:
        raise ValueError("at least one view is needed")
    H, D = views[0].n_kv_heads, views[0].head_dim
    dev = _views_device(views)
    for v in views:
        if v.n_kv_heads != H or v.head_dim != D:
            raise ValueError("all views of a call must have the same n_kv_heads and head_dim")
        if v.k_codes.device != dev:
            raise ValueError("all views of a call must be on one device")
    return H, D, dev


def _check_q(views, q, n_rows):
    """q: bf16 [n_rows, H_q, D] with H_q a multiple of the views' n_kv_heads."""
    H, D, dev = _check_views(views)
    if not isinstance(q, torch.Tensor) or q.dim() != 3:
        raise ValueError("q must be a 3-d tensor [rows, H_q, D]")
    Hq = q.shape[1]
    if Hq <= 0 or Hq % H:
        raise ValueError(f"q has {Hq} query heads, not a multiple of n_kv_heads {H}")
    _check_tensor("q", q, torch.bfloat16, (n_rows, Hq, D), dev)
    return Hq, D, dev


def _check_out(out, n_rows, Hq, D, dev):
    _check_tensor("out", out, torch.float32, (n_rows, Hq, D), dev)


def _check_new_tokens(views, k_new, v_new):
    H, D, dev = _check_views(views)
    _check_tensor("k_new", k_new, torch.bfloat16, (len(views), H, D), dev)
    _check_tensor("v_new", v_new, torch.bfloat16, (len(views), H, D), dev)


def _check_workspace(ws, dev):
    if ws is None:
        return
    if not isinstance(ws, torch.Tensor) or ws.dtype != torch.uint8 or ws.dim() != 1 or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous 1-d uint8 tensor")
    if ws.device != dev:
        raise ValueError(f"workspace is on {ws.device}, the views are on {dev}")


# -------------------------------------------------------------- codec -----

def quantize(x: torch.Tensor, bits: int, codes: torch.Tensor | None = None,
             scalemin: torch.Tensor | None = None, head_cap: int | None = None, stream=None):
    """x: bf16 CUDA tensor [H, T, D] (d contiguous; head/token strides free).

    Returns (codes u8 [H, cap, D*bits/8], scalemin f32 [H, cap, D/64, 2]);
    pass preallocated outputs to write in place."""
    if x.dtype != torch.bfloat16 or x.dim() != 3 or x.stride(2) != 1:
        raise ValueError("x must be a bf16 [H, T, D] tensor with contiguous last dim")
    H, T, D = x.shape
    cap = head_cap if head_cap is not None else (codes.shape[1] if codes is not None else T)
    if codes is None:
        codes = torch.empty((H, cap, row_bytes(D, bits)), dtype=torch.uint8, device=x.device)
    if scalemin is None:
        scalemin = torch.empty((H, cap, D // GROUP, 2), dtype=torch.float32, device=x.device)
    _check(lib().kvq_quantize(_ptr(x), x.stride(0), x.stride(1), H, T, D, bits,
                              _ptr(codes), _ptr(scalemin), cap, _stream(stream)), "kvq_quantize")
    return codes, scalemin


def dequantize(codes: torch.Tensor, scalemin: torch.Tensor, n_tokens: int, head_dim: int, bits: int,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Inverse of quantize: bf16 [H, n_tokens, D] (or into ``out``)."""
    H, cap = codes.shape[0], codes.shape[1]
    if out is None:
        out = torch.empty((H, n_tokens, head_dim), dtype=torch.bfloat16, device=codes.device)
    _check(lib().kvq_dequantize(_ptr(codes), _ptr(scalemin), cap, H, n_tokens, head_dim, bits,
                                _ptr(out), out.stride(0), out.stride(1), _stream(stream)),
           "kvq_dequantize")
    return out


# -------------------------------------------------------------- views -----

class View:
    """One (agent, layer) cache: packed tokens + bf16 recent-window ring.

    Owns (or borrows) the torch tensors behind a ``kvq_view``:
      k_codes, v_codes          u8  [H_kv, cap_packed, D*bits/8]
      k_scalemin, v_scalemin    f32 [H_kv, cap_packed, D/64, 2]
      k_window, v_window        bf16 [H_kv, cap_window, D]
    """

    def __init__(self, n_kv_heads: int, head_dim: int, bits: int, cap_packed: int, cap_window: int,
                 device="cuda", tensors: dict | None = None):
        if cap_packed % 2:
            cap_packed += 1
        self.n_kv_heads, self.head_dim, self.bits = n_kv_heads, head_dim, bits
        t = tensors or {}
        rb = row_bytes(head_dim, bits)
        ng = head_dim // GROUP
        self.k_codes = t.get("k_codes", torch.zeros((n_kv_heads, cap_packed, rb), dtype=torch.uint8, device=device))
        self.v_codes = t.get("v_codes", torch.zeros((n_kv_heads, cap_packed, rb), dtype=torch.uint8, device=device))
        self.k_scalemin = t.get("k_scalemin", torch.zeros((n_kv_heads, cap_packed, ng, 2), dtype=torch.float32,
                                                          device=device))
        self.v_scalemin = t.get("v_scalemin", torch.zeros((n_kv_heads, cap_packed, ng, 2), dtype=torch.float32,
                                                          device=device))
        self.k_window = t.get("k_window", torch.zeros((n_kv_heads, cap_window, head_dim), dtype=torch.bfloat16,
                                                      device=device))
        self.v_window = t.get("v_window", torch.zeros((n_kv_heads, cap_window, head_dim), dtype=torch.bfloat16,
                                                      device=device))
        self.c = CView(bits=bits, n_window=0, cap_window=cap_window, window_head=0, n_packed=0,
                       cap_packed=cap_packed)
        self._sync_ptrs()

    def _sync_ptrs(self):
        c = self.c
        c.k_codes, c.v_codes = self.k_codes.data_ptr(), self.v_codes.data_ptr()
        c.k_scalemin, c.v_scalemin = self.k_scalemin.data_ptr(), self.v_scalemin.data_ptr()
        c.k_window = self.k_window.data_ptr() if self.c.cap_window else None
        c.v_window = self.v_window.data_ptr() if self.c.cap_window else None

    # state accessors
    @property
    def n_packed(self) -> int:
        return self.c.n_packed

    @property
    def n_window(self) -> int:
        return self.c.n_window

    @property
    def cap_window(self) -> int:
        return self.c.cap_window

    @property
    def window_head(self) -> int:
        return self.c.window_head

    def set_state(self, n_packed: int, n_window: int, window_head: int = 0, bits: int | None = None):
        self.c.n_packed, self.c.n_window, self.c.window_head = n_packed, n_window, window_head
        if bits is not None:
            self.c.bits = self.bits = bits

    def new_segment(self, bits: int, cap_packed: int, device=None) -> "View":
        """Continue this cache at another width without requantizing it: a new
        view of width ``bits`` with room for ``cap_packed`` packed rows takes
        over this view's window ring (the same memory, the same tokens), so
        later flushes are quantized at the new width.  This view keeps its
        packed rows and gives up its window (cap_window 0).  Attend to both
        with decode_attn_seq; append to the new one."""
        dev = self.k_codes.device if device is None else device
        t = dict(k_window=self.k_window, v_window=self.v_window)
        seg = View(self.n_kv_heads, self.head_dim, bits, cap_packed, self.c.cap_window, device=dev, tensors=t)
        seg.c.n_window, seg.c.window_head = self.c.n_window, self.c.window_head
        self.c.n_window = self.c.window_head = self.c.cap_window = 0
        self.k_window = self.k_window[:, :0]
        self.v_window = self.v_window[:, :0]
        self._sync_ptrs()
        return seg

    def fill_packed(self, k: torch.Tensor, v: torch.Tensor, stream=None):
        """Quantize bf16 K/V [H, T, D] into packed rows [0, T) (prefill handoff)."""
        T = k.shape[1]
        quantize(k, self.bits, self.k_codes, self.k_scalemin, stream=stream)
        quantize(v, self.bits, self.v_codes, self.v_scalemin, stream=stream)
        self.c.n_packed = T

    def fill_window(self, k: torch.Tensor, v: torch.Tensor, head: int = 0):
        """Place bf16 K/V [H, n, D] as the window, oldest first, starting at ring slot ``head``."""
        n = k.shape[1]
        W = self.c.cap_window
        if n > W:
            raise ValueError("more window tokens than ring slots")
        idx = (torch.arange(n, device=k.device) + head) % W
        self.k_window[:, idx] = k
        self.v_window[:, idx] = v
        self.c.n_window, self.c.window_head = n, head


def _view_array(views):
    arr = (CView * len(views))()
    for i, v in enumerate(views):
        arr[i] = v.c
    return arr


def append(views, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
    """Append one token per view: k_new, v_new bf16 [n_views, H_kv, D]."""
    views = list(views)
    _check_new_tokens(views, k_new, v_new)
    arr = _view_array(views)
    H, D = views[0].n_kv_heads, views[0].head_dim
    _require_cuda(views[0].k_codes.device)
    _check(lib().kvq_append(arr, len(views), H, D, _ptr(k_new), _ptr(v_new), _stream(stream)),
           "kvq_append")
    for i, v in enumerate(views):
        v.c.n_packed, v.c.n_window, v.c.window_head = arr[i].n_packed, arr[i].n_window, arr[i].window_head


def workspace_size(views, n_q_heads: int) -> int:
    views = list(views)
    arr = _view_array(views)
    return int(lib().kvq_decode_attn_workspace_size(arr, len(views), n_q_heads, views[0].n_kv_heads,
                                                    views[0].head_dim))


def new_workspace(views, n_q_heads: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace of the size kvq_decode_attn needs for these views."""
    n = workspace_size(views, n_q_heads)
    if n == 0:
        raise KvqError(KVQ_ERR_INVALID_ARG, "kvq_decode_attn_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_attn(views, q: torch.Tensor, softmax_scale: float, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None, _arr=None) -> torch.Tensor:
    """q: bf16 [n_views, H_q, D] -> fp32 [n_views, H_q, D]."""
    views = list(views)
    Hq, D, dev = _check_q(views, q, len(views))
    n = len(views)
    arr = _arr if _arr is not None else _view_array(views)
    if workspace is None:
        workspace = new_workspace(views, Hq, device=q.device)
    _check_workspace(workspace, dev)
    if out is None:
        out = torch.empty((n, Hq, D), dtype=torch.float32, device=q.device)
    _check_out(out, n, Hq, D, dev)
    _require_cuda(dev)
    _check(lib().kvq_decode_attn(arr, len(views), Hq, views[0].n_kv_heads, D, _ptr(q), float(softmax_scale),
                                 _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "kvq_decode_attn")
    return out


def _seq_array(seq_begin):
    sb = [int(x) for x in seq_begin]
    return (ctypes.c_int32 * len(sb))(*sb), len(sb) - 1


def seq_workspace_size(views, seq_begin, n_q_heads: int) -> int:
    """kvq_decode_attn_seq_workspace_size (0 if the arguments are invalid)."""
    views = list(views)
    sb, n_seqs = _seq_array(seq_begin)
    return int(lib().kvq_decode_attn_seq_workspace_size(_view_array(views), len(views), sb, n_seqs, n_q_heads,
                                                        views[0].n_kv_heads, views[0].head_dim))


def new_seq_workspace(views, seq_begin, n_q_heads: int, device="cuda") -> torch.Tensor:
    n = seq_workspace_size(views, seq_begin, n_q_heads)
    if n == 0:
        raise KvqError(KVQ_ERR_INVALID_ARG, "kvq_decode_attn_seq_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode_attn_seq(views, seq_begin, q: torch.Tensor, softmax_scale: float, out: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """kvq_decode_attn_seq: sequence s is views seq_begin[s] .. seq_begin[s+1]-1.
    q: bf16 [n_seqs, H_q, D] -> fp32 [n_seqs, H_q, D]."""
    views = list(views)
    sb, n_seqs = _seq_array(seq_begin)
    Hq, D, dev = _check_q(views, q, n_seqs)
    n = n_seqs
    if workspace is None:
        workspace = new_seq_workspace(views, seq_begin, Hq, device=q.device)
    _check_workspace(workspace, dev)
    if out is None:
        out = torch.empty((n, Hq, D), dtype=torch.float32, device=q.device)
    _check_out(out, n, Hq, D, dev)
    _require_cuda(dev)
    _check(lib().kvq_decode_attn_seq(_view_array(views), len(views), sb, n_seqs, Hq, views[0].n_kv_heads, D,
                                     _ptr(q), float(softmax_scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "kvq_decode_attn_seq")
    return out


def sparse_workspace_size(views, n_q_heads: int, top_k: int) -> int:
    """kvq_sparse_decode_attn_workspace_size (0 if the arguments are invalid)."""
    views = list(views)
    return int(lib().kvq_sparse_decode_attn_workspace_size(_view_array(views), len(views), n_q_heads,
                                                           views[0].n_kv_heads, views[0].head_dim, int(top_k)))


def sparse_decode_attn(views, q: torch.Tensor, softmax_scale: float, top_k: int, out: torch.Tensor | None = None,
                       selected: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """kvq_sparse_decode_attn.  q: bf16 [n_views, H_q, D]; returns (out fp32
    [n_views, H_q, D], selected int32 [n_views, H_kv, top_k] or None)."""
    views = list(views)
    Hq, D, dev = _check_q(views, q, len(views))
    n = len(views)
    if workspace is None:
        nb = sparse_workspace_size(views, Hq, top_k)
        if nb == 0:
            raise KvqError(KVQ_ERR_INVALID_ARG, "kvq_sparse_decode_attn_workspace_size")
        workspace = torch.zeros(nb, dtype=torch.uint8, device=q.device)
    _check_workspace(workspace, dev)
    if out is None:
        out = torch.empty((n, Hq, D), dtype=torch.float32, device=q.device)
    _check_out(out, n, Hq, D, dev)
    if selected is not None:
        _check_tensor("selected", selected, torch.int32, (n, views[0].n_kv_heads, int(top_k)), dev)
    _require_cuda(dev)
    _check(lib().kvq_sparse_decode_attn(_view_array(views), len(views), Hq, views[0].n_kv_heads, D, _ptr(q),
                                        float(softmax_scale), int(top_k), _ptr(out),
                                        _ptr(selected) if selected is not None else None, _ptr(workspace),
                                        workspace.numel(), _stream(stream)), "kvq_sparse_decode_attn")
    return out, selected


def width_sensitivity(views, q: torch.Tensor, softmax_scale: float, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """kvq_width_sensitivity: q bf16 [n_views, H_q, D] -> fp32 [n_views] (device)."""
    views = list(views)
    Hq, D, dev = _check_q(views, q, len(views))
    n = len(views)
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=q.device)
    _check_tensor("out", out, torch.float32, (n,), dev)
    _require_cuda(dev)
    _check(lib().kvq_width_sensitivity(_view_array(views), len(views), Hq, views[0].n_kv_heads, D, _ptr(q),
                                       float(softmax_scale), _ptr(out), _stream(stream)), "kvq_width_sensitivity")
    return out


def allocate_widths(sens, capacity, n_kv_heads: int, head_dim: int, budget_bytes: int, units: int = 4096):
    """kvq_allocate_widths (host): returns (bits list, total estimated error)."""
    import numpy as np
    s = np.ascontiguousarray(np.asarray(sens, dtype=np.float32))
    c = np.ascontiguousarray(np.asarray(capacity, dtype=np.int64))
    bits = np.zeros(len(s), dtype=np.int32)
    total = ctypes.c_double()
    _check(lib().kvq_allocate_widths(s.ctypes.data, c.ctypes.data, len(s), n_kv_heads, head_dim, int(budget_bytes),
                                     int(units), bits.ctypes.data, ctypes.byref(total)), "kvq_allocate_widths")
    return [int(b) for b in bits], total.value


def _advanced(c: CView) -> CView:
    """A copy of a view's C struct with the counters one append later."""
    n = CView()
    ctypes.pointer(n)[0] = c
    if n.cap_window == 0:
        n.n_packed += 1
    elif n.n_window == n.cap_window:
        n.n_packed += 1
        n.window_head = (n.window_head + 1) % n.cap_window
    else:
        n.n_window += 1
    return n


def step_workspace_size(views, n_q_heads: int) -> int:
    """Workspace bytes append_decode_attn needs: kvq_decode_attn_workspace_size
    on the views as they will be after the append."""
    views = list(views)
    arr = (CView * len(views))()
    for i, v in enumerate(views):
        arr[i] = _advanced(v.c)
    return int(lib().kvq_decode_attn_workspace_size(arr, len(views), n_q_heads, views[0].n_kv_heads,
                                                    views[0].head_dim))


def append_decode_attn(views, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor, softmax_scale: float,
                       out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """One decode step (kvq_append_decode_attn): append k_new, v_new (bf16
    [n_views, H_kv, D]) to the views, then attend with q (bf16 [n_views, H_q,
    D]) over the appended views; returns fp32 [n_views, H_q, D]."""
    views = list(views)
    Hq, D, dev = _check_q(views, q, len(views))
    _check_new_tokens(views, k_new, v_new)
    n = len(views)
    if workspace is None:
        # 0 when the step is invalid: the call below then reports why
        nb = step_workspace_size(views, Hq)
        workspace = torch.zeros(nb, dtype=torch.uint8, device=q.device) if nb else None
    _check_workspace(workspace, dev)
    if out is None:
        out = torch.empty((n, Hq, D), dtype=torch.float32, device=q.device)
    _check_out(out, n, Hq, D, dev)
    arr = _view_array(views)
    _require_cuda(dev)
    _check(lib().kvq_append_decode_attn(arr, len(views), Hq, views[0].n_kv_heads, D, _ptr(k_new), _ptr(v_new),
                                        _ptr(q), float(softmax_scale), _ptr(out), _ptr(workspace),
                                        workspace.numel() if workspace is not None else 0, _stream(stream)),
           "kvq_append_decode_attn")
    for i, v in enumerate(views):
        v.c.n_packed, v.c.n_window, v.c.window_head = arr[i].n_packed, arr[i].n_window, arr[i].window_head
    return out


def decode_attn_noalloc(views, q: torch.Tensor, softmax_scale: float, out: torch.Tensor, stream=None,
                        _arr=None) -> torch.Tensor:
    """kvq_decode_attn_noalloc: like decode_attn, but the library allocates
    nothing: its scratch is a fixed per-device array of NOALLOC_SCRATCH_BYTES.
    ``out`` (fp32 [n_views, H_q, D]) must be given, so this call allocates no
    device memory either.  Calls that may overlap on the GPU race on the one
    array; the first call on a device should come before any stream capture."""
    views = list(views)
    Hq, D, dev = _check_q(views, q, len(views))
    _check_out(out, len(views), Hq, D, dev)
    arr = _arr if _arr is not None else _view_array(views)
    _require_cuda(dev)
    _check(lib().kvq_decode_attn_noalloc(arr, len(views), Hq, views[0].n_kv_heads, D, _ptr(q),
                                         float(softmax_scale), _ptr(out), _stream(stream)),
           "kvq_decode_attn_noalloc")
    return out


def debug_flags(clear: bool = True, stream=None) -> int:
    """The debug build's flags word (0: every device bounds check passed;
    one bit per kernel family otherwise), read after the work enqueued on
    ``stream`` so far, and cleared when ``clear``.  Synchronizes the stream.
    Raises KvqError (KVQ_ERR_UNSUPPORTED) in the normal build."""
    out = torch.zeros(1, dtype=torch.int32).pin_memory()
    _check(lib().kvq_debug_flags(_ptr(out), 1 if clear else 0, _stream(stream)), "kvq_debug_flags")
    (stream if stream is not None else torch.cuda.current_stream()).synchronize()
    return int(out.item()) & 0xFFFFFFFF


def decode_attn_noalloc_status(out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """kvq_decode_attn_noalloc_status: the status word the last
    decode_attn_noalloc call enqueued on ``stream`` left in the scratch array
    (0: outputs valid; 1: a bounded copy wait gave up), copied into ``out``
    (an int32 tensor of one element: device, or pinned host memory; a new
    pinned host tensor when None).  Stream-ordered: synchronize the stream
    before reading a host tensor."""
    if out is None:
        out = torch.zeros(1, dtype=torch.int32).pin_memory()
    if out.dtype != torch.int32 or out.numel() != 1 or not out.is_contiguous():
        raise ValueError("out must be a contiguous int32 tensor of one element")
    _check(lib().kvq_decode_attn_noalloc_status(_ptr(out), _stream(stream)), "kvq_decode_attn_noalloc_status")
    return out


# ---------------------------------------------------------- CacheCard -----

def card_bytes(views) -> int:
    views = list(views)
    return int(lib().kvq_card_bytes(_view_array(views), len(views), views[0].n_kv_heads, views[0].head_dim))


def card_pack(views, model_id: int = 0, position_offsets=None, out: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """kvq_card_pack: the card of these views as a DEVICE uint8 tensor."""
    views = list(views)
    n = card_bytes(views)
    if n == 0:
        raise KvqError(KVQ_ERR_INVALID_ARG, "kvq_card_bytes")
    dev = views[0].k_codes.device
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=dev)
    pos = None
    if position_offsets is not None:
        pos = (ctypes.c_int64 * len(views))(*[int(x) for x in position_offsets])
    _check(lib().kvq_card_pack(_view_array(views), len(views), views[0].n_kv_heads, views[0].head_dim,
                               int(model_id), ctypes.cast(pos, ctypes.c_void_p) if pos is not None else None,
                               _ptr(out), out.numel(), _stream(stream)), "kvq_card_pack")
    return out


def card_info(card_host: torch.Tensor) -> dict:
    """Header and per-view records of a card held in host memory."""
    if card_host.is_cuda:
        raise ValueError("card_info reads a host copy of the card")
    card_host = card_host.contiguous()
    nv, hk, d = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    mid = ctypes.c_uint64()
    _check(lib().kvq_card_read_header(_ptr(card_host), card_host.numel(), ctypes.byref(nv), ctypes.byref(hk),
                                      ctypes.byref(d), ctypes.byref(mid)), "kvq_card_read_header")
    recs = []
    for i in range(nv.value):
        b, w = ctypes.c_int32(), ctypes.c_int32()
        p, off = ctypes.c_int64(), ctypes.c_int64()
        _check(lib().kvq_card_view_info(_ptr(card_host), card_host.numel(), i, ctypes.byref(b), ctypes.byref(p),
                                        ctypes.byref(w), ctypes.byref(off)), "kvq_card_view_info")
        recs.append(dict(bits=b.value, n_packed=p.value, n_window=w.value, position_offset=off.value))
    return dict(n_views=nv.value, n_kv_heads=hk.value, head_dim=d.value, model_id=mid.value, views=recs)


def views_for_card(card_host: torch.Tensor, cap_window: int | None = None, extra_packed: int = 0,
                   device="cuda") -> list:
    """Fresh views that can take the card: each view's width from its record,
    capacity for its tokens (plus extra_packed rows; window capacity
    cap_window, default the record's n_window)."""
    info = card_info(card_host)
    out = []
    for r in info["views"]:
        W = r["n_window"] if cap_window is None else cap_window
        out.append(View(info["n_kv_heads"], info["head_dim"], r["bits"], max(2, r["n_packed"] + extra_packed), W,
                        device=device))
    return out


def card_unpack(card_host: torch.Tensor, views, card: torch.Tensor | None = None, stream=None):
    """kvq_card_unpack: restore the card into views (uploads the host copy
    when no device copy is given)."""
    views = list(views)
    card_host = card_host.contiguous()
    if card is None:
        # upload on the stream the kernel runs on
        s = stream if stream is not None else torch.cuda.current_stream(views[0].k_codes.device)
        with torch.cuda.stream(s):
            card = card_host.to(views[0].k_codes.device, non_blocking=True)
    arr = _view_array(views)
    _check(lib().kvq_card_unpack(_ptr(card_host), _ptr(card), card_host.numel(), arr, len(views),
                                 views[0].n_kv_heads, views[0].head_dim, _stream(stream)), "kvq_card_unpack")
    for i, v in enumerate(views):
        v.c.n_packed, v.c.n_window, v.c.window_head = arr[i].n_packed, arr[i].n_window, arr[i].window_head
    return views


def save_card(path: str, card: torch.Tensor):
    """Write a card (device or host tensor) to a file, byte for byte."""
    card.detach().cpu().numpy().tofile(path)


def load_card(path: str, pin: bool = True) -> torch.Tensor:
    """Read a card file into a host uint8 tensor (pinned for fast upload)."""
    import numpy as np
    t = torch.from_numpy(np.fromfile(path, dtype=np.uint8))
    return t.pin_memory() if pin and torch.cuda.is_available() else t
