"""The C-ABI library loads without a GPU and exports every entry point that
include/fb.h declares; the Python binding mirrors the same names."""

import ctypes
import os
import re

import block_diffusion_attention_fb_b200 as fb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fb.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_the_expected_entry_points():
    assert set(declared_functions()) == set(fb.EXPORTS)


def test_library_exports_every_declared_symbol():
    from block_diffusion_attention_fb_b200 import build as _build
    _build.build()
    lib = ctypes.CDLL(fb.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    for name in declared_functions():
        assert callable(getattr(fb, name)), name


def test_last_error_is_empty_string_initially():
    assert fb.load_library().fb_last_error() == b""


def test_host_validation_without_a_gpu():
    # argument checks run on the host before any CUDA call
    lib = fb.load_library()
    kv = fb.fb_kv()
    rc = lib.fb_prefix_attn(None, 4, 4, 1.0, ctypes.byref(kv), None, None, None, None, 0, None)
    assert rc == fb.FB_ERR_ARG
    assert b"NULL" in lib.fb_last_error()
    kv.k = kv.v = 16
    kv.batch, kv.n_heads_kv, kv.head_dim, kv.page_size = 1, 2, 96, 16
    kv.max_seq_len, kv.n_slots = 64, 64
    rc = lib.fb_prefix_attn(16, 4, 4, 1.0, ctypes.byref(kv), None, 16, 16, None, 0, None)
    assert rc == fb.FB_ERR_SHAPE
    assert lib.fb_workspace_size(None, 4, 4, 0, 0, 148) == 0
