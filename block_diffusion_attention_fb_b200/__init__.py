"""Per-denoise-step block-diffusion attention on B200 (FlashBlock, LoSA).

Thin Python binding of the C ABI declared in include/fb.h: every function here
has the C entry point's name and only marshals arguments (torch tensors ->
device pointers, the current CUDA stream) before calling into libfb_b200.so.
All computation happens in the library's CUDA kernels; there is no fallback.
Build the library with ``python -m block_diffusion_attention_fb_b200.build``.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfb_b200.so")

FB_OK = 0
FB_ERR_ARG = -1
FB_ERR_SHAPE = -2
FB_ERR_ALIGN = -3
FB_ERR_WORKSPACE = -4
FB_ERR_CUDA = -5
FB_ERR_TIMEOUT = -6
FB_F32 = 0
FB_BF16 = 1
FB_THRESHOLD = 0
FB_PER_HEAD = 1
FB_LOSA = 2
FB_SPARSE_RESIDUAL = 3

# Every entry point include/fb.h declares.
EXPORTS = ("fb_workspace_size", "fb_prefix_attn", "fb_block_attn", "fb_merge", "fb_page_summary",
           "losa_select", "losa_gather", "fb_step", "fb_device_status", "fb_last_error",
           "fb_kernel_launches", "fb_prefix_attn_noalloc", "fb_block_commit",
           "fb_selftest_timeout", "fb_prefix_attn_varlen", "fb_block_attn_varlen",
           "fb_step_varlen", "fb_workspace_page_scores")


class FbError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class fb_kv(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("seq_len", ctypes.c_void_p), ("n_slots", ctypes.c_int64),
                ("batch", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class fb_policy(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("tau", ctypes.c_int32), ("gamma", ctypes.c_double),
                ("n_active", ctypes.c_int32), ("topk_pages", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class fb_cache(ctypes.Structure):
    _fields_ = [("a_out", ctypes.c_void_p), ("l_out", ctypes.c_void_p),
                ("a_out_prev", ctypes.c_void_p), ("head_mask", ctypes.c_void_p),
                ("head_cos", ctypes.c_void_p), ("q_prev", ctypes.c_void_p),
                ("active_rows", ctypes.c_void_p), ("row_scores", ctypes.c_void_p),
                ("union_bitmap", ctypes.c_void_p), ("union_list", ctypes.c_void_p),
                ("union_count", ctypes.c_void_p), ("step", ctypes.c_int32),
                ("recomputed", ctypes.c_int32), ("a_res", ctypes.c_void_p),
                ("l_res", ctypes.c_void_p), ("comp_list", ctypes.c_void_p),
                ("comp_count", ctypes.c_void_p)]


_lib = None


def load_library() -> ctypes.CDLL:
    """Loads libfb_b200.so; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_diffusion_attention_fb_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    KV = ctypes.POINTER(fb_kv)
    sig = {
        "fb_workspace_size": (SZ, [KV, I32, I32, I32, I32, I32]),
        "fb_workspace_page_scores": (SZ, [KV, I32, I32, I32, I32, I32]),
        "fb_prefix_attn": (ctypes.c_int, [P, I32, I32, F32, KV, P, P, P, P, SZ, P]),
        "fb_block_attn": (ctypes.c_int, [P, P, P, I32, I32, I32, I32, I32, F32, ctypes.c_int, P, P, P]),
        "fb_merge": (ctypes.c_int, [P, P, P, P, I64, I32, P, P, P]),
        "fb_page_summary": (ctypes.c_int, [KV, P, P, P]),
        "losa_select": (ctypes.c_int, [P, P, I32, I32, P, P, KV, I32, I32, P, P, P, P, P, P, SZ, P]),
        "losa_gather": (ctypes.c_int, [P, I32, I32, P, I32, P, P, I32, KV, F32, P, P, P, SZ, P]),
        "fb_step": (ctypes.c_int, [ctypes.POINTER(fb_policy), ctypes.POINTER(fb_cache), P, P, P, I32,
                                   I32, KV, P, P, P, P, P, P, SZ, P]),
        "fb_device_status": (ctypes.c_int, []),
        "fb_last_error": (ctypes.c_char_p, []),
        "fb_kernel_launches": (ctypes.c_uint64, []),
        "fb_prefix_attn_noalloc": (ctypes.c_int, [P, I32, I32, F32, KV, P, P, P, P]),
        "fb_block_commit": (ctypes.c_int, [KV, P, P, P, I32, P, P, P]),
        "fb_selftest_timeout": (ctypes.c_int, [P, P]),
        "fb_prefix_attn_varlen": (ctypes.c_int, [P, P, I32, I32, I32, F32, KV, P, P, P, SZ, P]),
        "fb_block_attn_varlen": (ctypes.c_int, [P, P, P, P, I32, I32, I32, I32, I32, I32, F32,
                                                ctypes.c_int, P, P, P]),
        "fb_step_varlen": (ctypes.c_int, [ctypes.POINTER(fb_policy), ctypes.POINTER(fb_cache), P, P,
                                          P, P, I32, I32, I32, KV, P, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int) -> None:
    if rc != FB_OK:
        raise FbError(rc, load_library().fb_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FB_BF16
    if t.dtype == torch.float32:
        return FB_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


@dataclass
class KV:
    """A block-external KV cache on the device and its fb_kv descriptor."""

    k: object
    v: object
    seq_len: object = None
    page_table: object = None
    page_size: int = 16
    max_seq_len: int = 0
    c: fb_kv = None

    def __post_init__(self):
        n_slots, hkv, d = self.k.shape
        batch = int(self.seq_len.shape[0]) if self.seq_len is not None else (
            int(self.page_table.shape[0]) if self.page_table is not None else n_slots // self.max_seq_len)
        max_pages = int(self.page_table.shape[1]) if self.page_table is not None else 0
        self.c = fb_kv(_ptr(self.k), _ptr(self.v), _ptr(self.page_table), _ptr(self.seq_len),
                       n_slots, batch, hkv, d, self.page_size, max_pages, self.max_seq_len,
                       _dtype_code(self.k))

    @property
    def batch(self) -> int:
        return self.c.batch

    @property
    def n_pages(self) -> int:
        """Logical pages per sequence (the LoSA summary / union extent)."""
        if self.page_table is not None:
            return int(self.page_table.shape[1])
        return -(-self.max_seq_len // self.page_size)


def fb_workspace_size(kv: KV, block: int, n_heads_q: int, n_active: int = 0, topk_pages: int = 0,
                      num_sms: int = 0) -> int:
    n = load_library().fb_workspace_size(ctypes.byref(kv.c), block, n_heads_q, n_active, topk_pages,
                                         num_sms)
    if n == 0:
        raise FbError(FB_ERR_ARG, "fb_workspace_size: invalid arguments")
    return int(n)


def fb_workspace_page_scores(kv: KV, block: int, n_heads_q: int, n_active: int, topk_pages: int,
                             num_sms: int = 0) -> int:
    """Byte offset of the LoSA page scores inside the workspace."""
    n = load_library().fb_workspace_page_scores(ctypes.byref(kv.c), block, n_heads_q, n_active,
                                                topk_pages, num_sms)
    if n == 0:
        raise FbError(FB_ERR_ARG, "fb_workspace_page_scores: invalid arguments")
    return int(n)


def fb_prefix_attn(q, kv: KV, a_out, l_out, workspace, scale: float = 1.0, head_mask=None,
                   stream=None) -> None:
    batch, B, Hq, d = q.shape
    _check(load_library().fb_prefix_attn(_ptr(q), B, Hq, scale, ctypes.byref(kv.c), _ptr(head_mask),
                                         _ptr(a_out), _ptr(l_out), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def fb_block_attn(q, k_in, v_in, a_in, l_in, scale: float = 1.0, stream=None) -> None:
    batch, B, Hq, d = q.shape
    Hkv = k_in.shape[2]
    _check(load_library().fb_block_attn(_ptr(q), _ptr(k_in), _ptr(v_in), batch, B, Hq, Hkv, d,
                                        scale, _dtype_code(q), _ptr(a_in), _ptr(l_in),
                                        _stream(stream)))


def fb_merge(a_out, l_out, a_in, l_in, a_full, l_full=None, stream=None) -> None:
    d = a_out.shape[-1]
    rows = a_out.numel() // d
    _check(load_library().fb_merge(_ptr(a_out), _ptr(l_out), _ptr(a_in), _ptr(l_in), rows, d,
                                   _ptr(a_full), _ptr(l_full), _stream(stream)))


def fb_page_summary(kv: KV, page_min, page_max, stream=None) -> None:
    _check(load_library().fb_page_summary(ctypes.byref(kv.c), _ptr(page_min), _ptr(page_max),
                                          _stream(stream)))


def losa_select(q_cur, q_prev, page_min, page_max, kv: KV, n_active: int, topk_pages: int,
                active_rows, union_bitmap, union_list, union_count, workspace, row_scores=None,
                stream=None) -> None:
    batch, B, Hq, d = q_cur.shape
    _check(load_library().losa_select(_ptr(q_cur), _ptr(q_prev), B, Hq, _ptr(page_min),
                                      _ptr(page_max), ctypes.byref(kv.c), n_active, topk_pages,
                                      _ptr(active_rows), _ptr(row_scores), _ptr(union_bitmap),
                                      _ptr(union_list), _ptr(union_count), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)))


def losa_gather(q, active_rows, n_active: int, union_list, union_count, kv: KV, a_out, l_out,
                workspace, scale: float = 1.0, max_union: int = 0, stream=None) -> None:
    batch, B, Hq, d = q.shape
    _check(load_library().losa_gather(_ptr(q), B, Hq, _ptr(active_rows), n_active,
                                      _ptr(union_list), _ptr(union_count), max_union,
                                      ctypes.byref(kv.c), scale, _ptr(a_out), _ptr(l_out),
                                      _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)))


def fb_step(policy: fb_policy, cache: fb_cache, q, k_in, v_in, kv: KV, a_full, l_full=None,
            m_updated: Optional[Sequence[int]] = None, page_min=None, page_max=None,
            workspace=None, stream=None) -> None:
    batch, B, Hq, d = q.shape
    m_arr = _m_array(m_updated, kv.batch)
    _check(load_library().fb_step(ctypes.byref(policy), ctypes.byref(cache), _ptr(q), _ptr(k_in),
                                  _ptr(v_in), B, Hq, ctypes.byref(kv.c), _ptr(page_min),
                                  _ptr(page_max),
                                  ctypes.cast(m_arr, ctypes.c_void_p) if m_arr is not None else None,
                                  _ptr(a_full), _ptr(l_full), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def _m_array(m_updated, batch):
    if m_updated is None:
        return None
    if len(m_updated) < batch:  # the library reads one count per sequence
        raise ValueError(f"m_updated holds {len(m_updated)} counts for {batch} sequences")
    return (ctypes.c_int32 * len(m_updated))(*[int(x) for x in m_updated])


def fb_prefix_attn_varlen(q, cu_rows, max_rows: int, kv: KV, a_out, l_out, workspace,
                          scale: float = 1.0, stream=None) -> None:
    """Packed rows q [total, Hq, d]; cu_rows: device int32 [batch + 1] offsets;
    max_rows: the most rows any sequence has (host)."""
    total, Hq, d = q.shape
    _check(load_library().fb_prefix_attn_varlen(_ptr(q), _ptr(cu_rows), max_rows, total, Hq, scale,
                                                ctypes.byref(kv.c), _ptr(a_out), _ptr(l_out),
                                                _ptr(workspace),
                                                workspace.numel() * workspace.element_size(),
                                                _stream(stream)))


def fb_block_attn_varlen(q, k_in, v_in, cu_rows, max_rows: int, a_in, l_in, scale: float = 1.0,
                         stream=None) -> None:
    total, Hq, d = q.shape
    batch = int(cu_rows.shape[0]) - 1
    _check(load_library().fb_block_attn_varlen(_ptr(q), _ptr(k_in), _ptr(v_in), _ptr(cu_rows),
                                               batch, max_rows, total, Hq, int(k_in.shape[1]), d,
                                               scale, _dtype_code(q), _ptr(a_in), _ptr(l_in),
                                               _stream(stream)))


def fb_step_varlen(policy: fb_policy, cache: fb_cache, q, k_in, v_in, cu_rows, max_rows: int,
                   kv: KV, a_full, l_full=None, m_updated: Optional[Sequence[int]] = None,
                   workspace=None, stream=None) -> None:
    total, Hq, d = q.shape
    m_arr = _m_array(m_updated, kv.batch)
    _check(load_library().fb_step_varlen(ctypes.byref(policy), ctypes.byref(cache), _ptr(q),
                                         _ptr(k_in), _ptr(v_in), _ptr(cu_rows), max_rows, total,
                                         Hq, ctypes.byref(kv.c),
                                         ctypes.cast(m_arr, ctypes.c_void_p) if m_arr is not None
                                         else None, _ptr(a_full), _ptr(l_full), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def fb_device_status() -> None:
    _check(load_library().fb_device_status())


def fb_last_error() -> str:
    return load_library().fb_last_error().decode()


def fb_prefix_attn_noalloc(q, kv: KV, a_out, l_out, scale: float = 1.0, head_mask=None,
                           stream=None) -> None:
    """fb_prefix_attn with the library's static scratch instead of a workspace
    (for callers that cannot allocate device memory; see include/fb.h)."""
    batch, B, Hq, d = q.shape
    _check(load_library().fb_prefix_attn_noalloc(_ptr(q), B, Hq, scale, ctypes.byref(kv.c),
                                                 _ptr(head_mask), _ptr(a_out), _ptr(l_out),
                                                 _stream(stream)))


def fb_block_commit(kv: KV, seq_len_host, k_in, v_in, page_min=None, page_max=None,
                    stream=None) -> None:
    """Appends the block k_in / v_in [batch, B, Hkv, d] to the cache at the
    positions given by seq_len_host (host int32 lengths before the call) and
    updates the device lengths and, if given, the page summaries in place."""
    import numpy as _np
    lens = _np.ascontiguousarray(_np.asarray(seq_len_host, dtype=_np.int32))
    if lens.shape != (kv.batch,):
        raise ValueError("seq_len_host must hold one length per sequence")
    _check(load_library().fb_block_commit(
        ctypes.byref(kv.c), lens.ctypes.data_as(ctypes.c_void_p), _ptr(k_in), _ptr(v_in),
        int(k_in.shape[1]), _ptr(page_min), _ptr(page_max), _stream(stream)))


def fb_selftest_timeout(gave_up=None, stream=None) -> None:
    """Launches the failure-path self-test kernel (a wait that must give up)."""
    _check(load_library().fb_selftest_timeout(_ptr(gave_up), _stream(stream)))


def fb_kernel_launches() -> int:
    return int(load_library().fb_kernel_launches())
