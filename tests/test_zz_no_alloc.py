"""fb_prefix_attn_noalloc: the prefix partial for callers that cannot allocate
device memory on the call path (plugin hosts that pass no scratch pointer,
engines that pre-reserve all device memory in their own pool, latency-bound
loops where cudaMalloc may synchronise). Its split-KV scratch is a static
device array inside the library instead of a caller workspace.

The test calls the entry point through the C ABI and compares it with
fb_prefix_attn (the workspace entry point) on the same inputs, within the
bf16 tolerances of the other parity tests, on two calls in a row: the second
call uses different shapes and inputs, so results left in the shared array by
the first call must not leak into it. It lives in its own file, named to be
collected last, and passes alone or after the other tests.
"""

import ctypes

import pytest
import torch

import block_diffusion_attention_fb_b200 as fb
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _both(wl):
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    q = dev(next(wl.steps(1)).q, sp.dtype)
    shape = (sp.batch, sp.block, sp.n_heads_q, sp.head_dim)
    ws_bytes = fb.fb_workspace_size(kv, sp.block, sp.n_heads_q)
    assert ws_bytes > (1 << 20), "the case must use split-KV scratch"
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    A1 = torch.full(shape, 3.0, device="cuda")
    L1 = torch.full(shape[:3], 3.0, device="cuda")
    fb.fb_prefix_attn(q, kv, A1, L1, ws)
    A2 = torch.full(shape, -3.0, device="cuda")
    L2 = torch.full(shape[:3], -3.0, device="cuda")
    lib = fb.load_library()
    rc = lib.fb_prefix_attn_noalloc(q.data_ptr(), sp.block, sp.n_heads_q, ctypes.c_float(1.0),
                                    ctypes.byref(kv.c), None, A2.data_ptr(), L2.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == fb.FB_OK, lib.fb_last_error()
    sync()
    return cpu(A1), cpu(L1), cpu(A2), cpu(L2)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    calls = [
        make_workload("dllm", prefix_min=5000, prefix_max=5000, n_heads_q=4, n_heads_kv=4),
        make_workload("gqa", prefix_min=300, prefix_max=2000, batch=3, block=24, n_heads_q=8,
                      n_heads_kv=2),
    ]
    for wl in calls:
        A1, L1, A2, L2 = _both(wl)
        assert_close_A(A2, A1, "bf16", wl.spec.name)
        assert_close_L(L2, L1, wl.spec.name)
    fb.fb_device_status()


def test_noalloc_rejects_shapes_beyond_its_static_scratch():
    # A video-shaped request (24 heads, 1664 block rows, 4096-token prefix) is
    # split twice per 128-row tile on 140-148 SMs: its partials (41 MB) exceed
    # the 32 MiB static array, so the call is refused on the host. The buffers
    # are real and sized for the shapes, so even a launch would only read memory
    # it owns.
    assert 140 <= torch.cuda.get_device_properties(0).multi_processor_count <= 148
    L, B, H = 4096, 1664, 24
    k = torch.zeros(L, H, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    q = torch.zeros(1, B, H, 128, dtype=torch.bfloat16, device="cuda")
    A = torch.full((1, B, H, 128), 5.0, device="cuda")
    Lo = torch.full((1, B, H), 5.0, device="cuda")
    kv = fb.KV(k, v, seq_len=None, page_table=None, page_size=16, max_seq_len=L)
    lib = fb.load_library()
    rc = lib.fb_prefix_attn_noalloc(q.data_ptr(), B, H, ctypes.c_float(1.0), ctypes.byref(kv.c),
                                    None, A.data_ptr(), Lo.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == fb.FB_ERR_WORKSPACE, rc
    assert b"static" in lib.fb_last_error()
    sync()
    assert float(A.min()) == 5.0 and float(A.max()) == 5.0  # nothing was launched
