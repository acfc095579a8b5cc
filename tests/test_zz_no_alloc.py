"""fb_prefix_attn_noalloc: the prefix partial for callers that cannot allocate
device memory on the call path (plugin hosts that pass no scratch pointer,
engines that pre-reserve all device memory in their own pool, latency-bound
loops where cudaMalloc may synchronise). Its split-KV scratch is a static
device array inside the library instead of a caller workspace.

The tests call the entry point through the C ABI and compare it with
fb_prefix_attn (the workspace entry point) and with the oracle, within the
bf16 tolerances of the other parity tests, on calls in a row: each call uses
other shapes and inputs, so results left in the shared array by an earlier
call must not leak into a later one (one earlier call leaves NaN there). The
file is named to be collected last, and passes alone or after the other tests.
"""

import ctypes
import os

import numpy as np
import pytest
import torch

import block_diffusion_attention_fb_b200 as fb
import oracle
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _noalloc(q, kv, B, Hq, A, L, head_mask=None):
    lib = fb.load_library()
    rc = lib.fb_prefix_attn_noalloc(q.data_ptr(), B, Hq, ctypes.c_float(1.0), ctypes.byref(kv.c),
                                    None if head_mask is None else head_mask.data_ptr(),
                                    A.data_ptr(), L.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    return rc, lib


def _both(wl, q_np=None, head_mask=None):
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    q = dev(next(wl.steps(1)).q if q_np is None else q_np, sp.dtype)
    shape = (sp.batch, sp.block, sp.n_heads_q, sp.head_dim)
    ws_bytes = fb.fb_workspace_size(kv, sp.block, sp.n_heads_q)
    assert ws_bytes > (1 << 20), "the case must use split-KV scratch"
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    hm = None if head_mask is None else torch.from_numpy(head_mask.astype(np.uint8)).cuda()
    A1 = torch.full(shape, 3.0, device="cuda")
    L1 = torch.full(shape[:3], 3.0, device="cuda")
    fb.fb_prefix_attn(q, kv, A1, L1, ws, head_mask=hm)
    A2 = torch.full(shape, 3.0, device="cuda")
    L2 = torch.full(shape[:3], 3.0, device="cuda")
    rc, lib = _noalloc(q, kv, sp.block, sp.n_heads_q, A2, L2, hm)
    assert rc == fb.FB_OK, lib.fb_last_error()
    sync()
    return cpu(A1), cpu(L1), cpu(A2), cpu(L2)


def test_noalloc_matches_workspace_entry_point_and_oracle_on_calls_in_a_row():
    # 1: long prefix, all heads; 2: paged GQA with ragged lengths and a head mask;
    # 3: NaN queries fill the shared scratch with NaN partials; 4: a short prefix
    #    planned for a long one, so most splits are empty and their (stale, NaN)
    #    scratch must carry no weight
    wl1 = make_workload("dllm", prefix_min=5000, prefix_max=5000, n_heads_q=4, n_heads_kv=4)
    wl2 = make_workload("gqa", prefix_min=300, prefix_max=2000, batch=3, block=24, n_heads_q=8,
                        n_heads_kv=2)
    wl3 = make_workload("dllm", prefix_min=9000, prefix_max=9000, n_heads_q=4, n_heads_kv=4)
    mask2 = np.zeros((3, 8), dtype=np.uint8)
    mask2[0, [0, 5]] = 1
    mask2[1, :] = 1
    mask2[2, 7] = 1
    for wl, q_np, mask in ((wl1, None, None), (wl2, None, mask2)):
        sp = wl.spec
        st = next(wl.steps(1))
        A1, L1, A2, L2 = _both(wl, q_np, mask)
        A_ref, L_ref = oracle.prefix_partial(wl.prefix, st.q, sp.dtype, head_mask=mask)
        on = np.ones((sp.batch, sp.n_heads_q), bool) if mask is None else mask.astype(bool)
        for b in range(sp.batch):
            for h in range(sp.n_heads_q):
                if on[b, h]:
                    assert_close_A(A2[b, :, h], A1[b, :, h], "bf16", f"{sp.name} b{b} h{h}")
                    assert_close_L(L2[b, :, h], L1[b, :, h], f"{sp.name} b{b} h{h}")
                    assert_close_A(A2[b, :, h], A_ref[b, :, h], "bf16", f"oracle b{b} h{h}")
                    assert_close_L(L2[b, :, h], L_ref[b, :, h], f"oracle b{b} h{h}")
                else:  # masked heads are left untouched
                    assert np.all(A2[b, :, h] == 3.0) and np.all(L2[b, :, h] == 3.0)
    # NaN partials left in the shared array by one call ...
    sp = wl3.spec
    kv3 = make_kv(wl3.prefix, sp.dtype)
    qn = torch.full((1, sp.block, sp.n_heads_q, sp.head_dim), float("nan"), dtype=torch.bfloat16,
                    device="cuda")
    A = torch.zeros(1, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(1, sp.block, sp.n_heads_q, device="cuda")
    rc, lib = _noalloc(qn, kv3, sp.block, sp.n_heads_q, A, L)
    assert rc == fb.FB_OK, lib.fb_last_error()
    sync()
    # ... carry no weight in the next call, whose short sequence leaves most of
    # the splits of the same plan empty
    kv3.seq_len.fill_(700)
    st = next(wl3.steps(1))
    q = dev(st.q, sp.dtype)
    rc, lib = _noalloc(q, kv3, sp.block, sp.n_heads_q, A, L)
    assert rc == fb.FB_OK, lib.fb_last_error()
    sync()
    tokens = list(range(700))
    for h in range(sp.n_heads_q):
        K, V = oracle.attention.prefix_keys(wl3.prefix, 0, h, sp.dtype, tokens=tokens)
        a, l = oracle.partial(oracle.to_f64(st.q[0, :, h], sp.dtype), K, V)
        assert_close_A(cpu(A)[0, :, h], a, "bf16", f"short prefix h{h}")
        assert_close_L(cpu(L)[0, :, h], l, f"short prefix h{h}")
    fb.fb_device_status()


def test_noalloc_rejects_shapes_beyond_its_static_scratch():
    # A video-shaped request (24 heads, 1664 block rows, 4096-token prefix) with
    # the tcgen05 plan forced to 32 splits per row tile needs about 650 MB of
    # split partials on any SM count, far above the 32 MiB static array, so the
    # call is refused on the host. The buffers are real and sized for the shapes,
    # so even a launch would only read memory it owns.
    L, B, H = 4096, 1664, 24
    k = torch.zeros(L, H, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    q = torch.zeros(1, B, H, 128, dtype=torch.bfloat16, device="cuda")
    A = torch.full((1, B, H, 128), 5.0, device="cuda")
    Lo = torch.full((1, B, H), 5.0, device="cuda")
    kv = fb.KV(k, v, seq_len=None, page_table=None, page_size=16, max_seq_len=L)
    old = os.environ.get("FB_TC_SPLITS")
    os.environ["FB_TC_SPLITS"] = "32"
    try:
        rc, lib = _noalloc(q, kv, B, H, A, Lo)
    finally:
        if old is None:
            del os.environ["FB_TC_SPLITS"]
        else:
            os.environ["FB_TC_SPLITS"] = old
    assert rc == fb.FB_ERR_WORKSPACE, rc
    assert b"static" in lib.fb_last_error()
    sync()
    assert float(A.min()) == 5.0 and float(A.max()) == 5.0  # nothing was launched
