"""GPU parity of the packed-row (variable-length) entry points against the
oracle: several blocks of different sizes, each with its own prefix (or one
prefix shared through the page table), in one launch.

BlockBatch page, "Optimización del Sistema" (all active branches' query
positions in one variable-length buffer); FlashBlock technical summary §2 for
what each segment computes.
"""

import numpy as np
import pytest
import torch

import block_diffusion_attention_fb_b200 as fb
from block_diffusion_attention_fb_b200.runtime import VarlenBlockAttention
from oracle import varlen as ov
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads.varlen import BLOCKBATCH_ROWS, make_varlen_workload

pytestmark = pytest.mark.gpu

CASES = {
    # BlockBatch branch sizes 4..128 over one shared paged prefix, GQA G = 4: up to
    # 512 stacked rows per kv head (tcgen05 kernel for the prefix and the block)
    "blockbatch_shared_gqa": ("gqa", BLOCKBATCH_ROWS, True,
                              dict(prefix_min=700, prefix_max=1500, n_heads_q=8, n_heads_kv=2)),
    # distinct paged prefixes, an empty branch, at most 60 stacked rows (mma.sync kernel)
    "paged_gqa_short": ("gqa", (3, 0, 15, 9), False,
                        dict(prefix_min=200, prefix_max=2100, n_heads_q=8, n_heads_kv=2)),
    # contiguous MHA prefixes, single-row and full blocks
    "dllm_contig": ("dllm", (1, 32, 7), False,
                    dict(prefix_min=1500, prefix_max=1500, n_heads_q=4, n_heads_kv=4)),
    # rows of 70..200 in one launch: video-sized blocks on the tcgen05 kernel
    "video_long_blocks": ("video", (200, 70, 129), False,
                          dict(prefix_min=600, prefix_max=600, n_heads_q=2, n_heads_kv=2)),
    # fp32 (CUDA-core kernels), head_dim 64
    "tiny_f32": ("tiny", (5, 16, 2), False, dict(prefix_min=1000, prefix_max=1000)),
}


def _setup(case, steps=1):
    base, rows, shared, ovr = CASES[case]
    wl = make_varlen_workload(base, rows, shared_prefix=shared, steps=steps, **ovr)
    kv = make_kv(wl.prefix, wl.spec.dtype)
    cu = torch.from_numpy(wl.cu).cuda()
    return wl, kv, cu


@pytest.mark.parametrize("case", sorted(CASES))
def test_prefix_and_block_varlen_match_oracle(case):
    wl, kv, cu = _setup(case)
    sp = wl.spec
    st = next(wl.steps(1))
    H, d, T = sp.n_heads_q, sp.head_dim, wl.total
    max_rows = max(wl.rows)
    q = dev(st.q, sp.dtype)
    A = torch.full((T, H, d), 7.0, device="cuda")
    L = torch.full((T, H), 7.0, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, max_rows, H), dtype=torch.uint8, device="cuda")
    fb.fb_prefix_attn_varlen(q, cu, max_rows, kv, A, L, ws)
    Ai = torch.full((T, H, d), 7.0, device="cuda")
    Li = torch.full((T, H), 7.0, device="cuda")
    fb.fb_block_attn_varlen(q, dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), cu, max_rows, Ai,
                            Li)
    sync()
    fb.fb_device_status()
    A_ref, L_ref = ov.prefix_partial_varlen(wl.prefix, st.q, wl.cu, sp.dtype)
    assert_close_A(cpu(A), A_ref, sp.dtype, "prefix")
    assert_close_L(cpu(L), L_ref, "prefix")
    A_ref, L_ref = ov.block_partial_varlen(st.q, st.k_in, st.v_in, wl.cu, sp.dtype)
    assert_close_A(cpu(Ai), A_ref, sp.dtype, "block")
    assert_close_L(cpu(Li), L_ref, "block")


@pytest.mark.parametrize("case,tau", [("blockbatch_shared_gqa", 3), ("paged_gqa_short", 3),
                                      ("dllm_contig", 2), ("tiny_f32", 2),
                                      ("video_long_blocks", 0)])
def test_step_varlen_matches_oracle(case, tau):
    """Threshold reuse over packed rows, step by step: per-sequence decisions
    from each branch's update count, A_full of every packed row."""
    wl, kv, cu = _setup(case, steps=6)
    sp = wl.spec
    H, d, T = sp.n_heads_q, sp.head_dim, wl.total
    blk = VarlenBlockAttention(kv, wl.cu, H, tau=tau)
    ctl = ov.ThresholdVarlenController(wl.prefix, sp.dtype, tau)
    A = torch.zeros(T, H, d, device="cuda")
    L = torch.zeros(T, H, device="cuda")
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, wl.cu, st.m_updated)
        sync()
        assert blk.recomputed == int(ref["recompute"].sum()), st.step
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")
    fb.fb_device_status()


@pytest.mark.parametrize("bad_cu", [[0, 5, 9, 7], [0, 4, 12, 9]])
def test_bad_row_offsets_read_as_empty_and_are_reported(bad_cu):
    """Offsets that decrease or leave the packed buffer are checked on the
    device before use: that sequence is treated as empty (its rows keep their
    old contents), the others are computed, and fb_device_status reports
    FB_ERR_ARG."""
    wl = make_varlen_workload("dllm", (5, 4, 0), prefix_min=300, prefix_max=300, n_heads_q=2,
                              n_heads_kv=2)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    st = next(wl.steps(1))
    T, H, d = 9, sp.n_heads_q, sp.head_dim
    q = dev(st.q, sp.dtype)
    cu = torch.tensor(bad_cu, dtype=torch.int32, device="cuda")
    A = torch.full((T, H, d), 7.0, device="cuda")
    L = torch.full((T, H), 7.0, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, 8, H), dtype=torch.uint8, device="cuda")
    fb.fb_prefix_attn_varlen(q, cu, 8, kv, A, L, ws)
    sync()
    with pytest.raises(fb.FbError) as e:
        fb.fb_device_status()
    assert e.value.code == fb.FB_ERR_ARG
    good = [(b, lo, hi) for b, (lo, hi) in enumerate(zip(bad_cu[:-1], bad_cu[1:]))
            if 0 <= lo <= hi <= T]
    ref_cu = np.array([0, 5, 9, 9], dtype=np.int32)  # the rows as drawn
    A_ref, L_ref = ov.prefix_partial_varlen(wl.prefix, st.q, ref_cu, sp.dtype)
    A, L = cpu(A), cpu(L)
    written = np.zeros(T, bool)
    for b, lo, hi in good:
        if hi == lo:
            continue
        assert_close_A(A[lo:hi], A_ref[lo:hi], sp.dtype, f"seq {b}")
        assert_close_L(L[lo:hi], L_ref[lo:hi], f"seq {b}")
        written[lo:hi] = True
    assert np.all(A[~written] == 7.0) and np.all(L[~written] == 7.0)
