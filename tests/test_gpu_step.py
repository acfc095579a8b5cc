"""GPU parity of fb_step (the reuse controllers) against the oracle's step
procedures, step by step over whole blocks at reduced sizes.

FlashBlock technical summary §2 "Adaptive reuse strategies" (threshold tau,
per-head gamma); LoSA §2 steps 1-4.
"""

import numpy as np
import pytest
import torch

from block_diffusion_attention_fb_b200.runtime import BlockAttention
from oracle.controllers import (LosaController, PerHeadController, ThresholdController,
                                head_cosine)
from oracle.residual import SparseResidualController
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _out(sp):
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    return A, L


@pytest.mark.parametrize("name,ov,tau", [
    ("tiny", {}, 3),
    ("tiny", {}, 0),
    ("dllm", dict(prefix_min=900, prefix_max=900, n_heads_q=4, n_heads_kv=4, steps=12), 2),
    ("gqa", dict(prefix_min=100, prefix_max=500, batch=3, block=16, n_heads_q=8, n_heads_kv=2,
                 steps=10), 3),
])
def test_threshold_steps_match_oracle(name, ov, tau):
    wl = make_workload(name, **ov)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "threshold", tau=tau)
    ctl = ThresholdController(wl.prefix, sp.dtype, tau)
    A, L = _out(sp)
    n_rec = 0
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        sync()
        assert blk.recomputed == int(ref["recompute"].sum()), f"step {st.step}"
        n_rec += blk.recomputed
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")
    assert blk.step_index == sp.steps
    if tau == 0:
        assert n_rec == sp.steps * sp.batch


@pytest.mark.parametrize("name", ["gqa", "tiny"])
def test_threshold_steps_with_an_empty_prefix_side(name):
    """A sequence with no prefix tokens has L_out = -inf: the fused merge must
    return its in-block partial alone (FlashBlock merge with one empty side)."""
    wl = make_workload(name, prefix_min=20, prefix_max=300, batch=3, block=24, n_heads_q=8,
                       n_heads_kv=2, steps=4)
    wl.prefix.seq_len[1] = 0
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "threshold", tau=2)
    ctl = ThresholdController(wl.prefix, sp.dtype, 2)
    A, L = _out(sp)
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        sync()
        assert np.isfinite(cpu(L)[1]).all()
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")


@pytest.mark.parametrize("block,tau", [(300, 0), (300, 3), (520, 0)])
def test_long_single_sequence_block_with_a_short_last_row_tile(block, tau):
    """One sequence, one q head per kv head, more than 256 block rows with at
    most 64 in the last 256-row tile: fb_step runs the full tiles on the
    tcgen05 kernel and the last rows on the streaming kernel (split over the
    block's keys); every row must match the oracle, merge included."""
    wl = make_workload("video", prefix_min=1200, prefix_max=1200, block=block, n_heads_q=3,
                       n_heads_kv=3, steps=3)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "threshold", tau=tau)
    ctl = ThresholdController(wl.prefix, sp.dtype, tau)
    A, L = _out(sp)
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        sync()
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")


def test_per_head_steps_match_oracle_with_bit_exact_cosine_replay():
    wl = make_workload("video", prefix_min=700, prefix_max=700, block=90, n_heads_q=6,
                       n_heads_kv=6, steps=8)
    sp = wl.spec
    # cosines of this case lie in [0.959, 0.9994]: 0.997 stops two heads at
    # step 1 and keeps the others computing, each with a margin above 1e-3
    gamma = 0.997
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "per_head", gamma=gamma)
    ctl = PerHeadController(wl.prefix, sp.dtype, gamma)
    A, L = _out(sp)
    prev_gpu_aout = None
    stopped_any = False
    for st in wl.steps():
        mask_before = cpu(blk.t["head_mask"]).astype(bool)
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L)
        sync()
        gpu_aout = cpu(blk.a_out).copy()
        # teacher forcing: the oracle computes exactly the heads the GPU computed
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, force_mask=mask_before,
                       a_out_for_decision=(gpu_aout, prev_gpu_aout))
        if st.step >= 1:
            cos_gpu = cpu(blk.t["head_cos"])
            for h in range(sp.n_heads_q):
                if mask_before[0, h]:
                    # replay: the oracle's cosine on the GPU's own float32 tiles
                    want = head_cosine(gpu_aout[0, :, h], cpu(blk.t["a_out_prev"])[0, :, h])
                    assert cos_gpu[0, h] == want, (st.step, h, cos_gpu[0, h], want)
                    assert ref["cos"][0, h] == want
            np.testing.assert_array_equal(cpu(blk.t["head_mask"]).astype(bool), ref["next_mask"])
            stopped_any |= bool((~ref["next_mask"]).any())
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")
        prev_gpu_aout = gpu_aout
    assert stopped_any, "gamma chosen so that some heads start reusing"


def test_per_head_oracle_mask_agrees_away_from_the_threshold():
    """End to end: the oracle's own float64 A_out gives the same decisions as
    the GPU wherever |c - gamma| > 1e-4."""
    wl = make_workload("video", prefix_min=400, prefix_max=400, block=60, n_heads_q=4,
                       n_heads_kv=4, steps=6)
    sp = wl.spec
    gamma = 0.999
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "per_head", gamma=gamma)
    ctl = PerHeadController(wl.prefix, sp.dtype, gamma)
    A, L = _out(sp)
    for st in wl.steps():
        mask_before = cpu(blk.t["head_mask"]).astype(bool)
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L)
        sync()
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, force_mask=mask_before)
        if st.step >= 1:
            cos_gpu = cpu(blk.t["head_cos"])
            for h in range(sp.n_heads_q):
                if mask_before[0, h] and abs(ref["cos"][0, h] - gamma) > 1e-4:
                    assert (cos_gpu[0, h] >= gamma) == (ref["cos"][0, h] >= gamma)


@pytest.mark.parametrize("name,ov,n_active,topk", [
    ("losa", dict(prefix_min=3000, prefix_max=3000, n_heads_q=4, n_heads_kv=4, steps=6), 4, 16),
    ("losa", dict(prefix_min=2500, prefix_max=2500, n_heads_q=4, n_heads_kv=2, steps=5,
                  block=20), 3, 9),
    # paged pool, pages permuted, ragged lengths, batch 3, GQA (G = 4): per-sequence
    # active sets and per-(sequence, kv head) unions in one launch
    ("gqa", dict(prefix_min=700, prefix_max=3100, batch=3, block=16, n_heads_q=8, n_heads_kv=2,
                 steps=5), 4, 12),
    # 20 active rows x 4 q heads = 80 stacked rows per kv head: the tcgen05
    # kernel over page lists
    ("gqa", dict(prefix_min=1500, prefix_max=4000, batch=2, block=32, n_heads_q=8, n_heads_kv=2,
                 steps=4), 20, 8),
    # video block (200 of its 1560 rows, reduced prefix): per-head drift, long block
    # (in-block partial on the tcgen05 kernel), 8 active rows on the mma.sync kernel
    ("video", dict(prefix_min=2000, prefix_max=2000, block=200, n_heads_q=4, n_heads_kv=4,
                   steps=4), 8, 10),
    # 70 active rows of the video block: the tcgen05 kernel over page lists
    ("video", dict(prefix_min=1800, prefix_max=1800, block=200, n_heads_q=2, n_heads_kv=2,
                   steps=3), 70, 6),
])
def test_losa_steps_match_oracle(name, ov, n_active, topk):
    wl = make_workload(name, **ov)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "losa", n_active=n_active, topk_pages=topk)
    ctl = LosaController(wl.prefix, sp.dtype, n_active, topk)
    A, L = _out(sp)
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L)
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in)
        sync()
        if st.step >= 1:
            np.testing.assert_array_equal(cpu(blk.t["active_rows"]), ref["active"])
            for (b, hk), pages in ref["union"].items():
                cnt = int(cpu(blk.t["union_count"])[b, hk])
                assert cnt == len(pages)
                np.testing.assert_array_equal(cpu(blk.t["union_list"])[b, hk, :cnt], pages)
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")


@pytest.mark.parametrize("name,ov,tau,topk", [
    ("dllm", dict(prefix_min=1500, prefix_max=1500, n_heads_q=4, n_heads_kv=4, block=32,
                  steps=8), 2, 12),
    # paged, ragged lengths, GQA (16 rows x 4 q heads = 64 stacked rows per kv head)
    ("gqa", dict(prefix_min=100, prefix_max=900, batch=3, block=16, n_heads_q=8, n_heads_kv=2,
                 steps=6), 3, 5),
    ("tiny", dict(steps=6), 2, 9),  # float32, head_dim 64
    # every page selected: the complement is empty and every step is dense
    ("dllm", dict(prefix_min=700, prefix_max=700, n_heads_q=2, n_heads_kv=2, block=8, steps=4),
     2, 1000),
    # no page selected: plain threshold reuse of the cached residual
    ("dllm", dict(prefix_min=700, prefix_max=700, n_heads_q=2, n_heads_kv=2, block=8, steps=5),
     2, 0),
])
def test_sparse_residual_steps_match_oracle(name, ov, tau, topk):
    """FlashBlock with sparse attention (technical summary §2): fresh partial over
    the selected pages merged with the cached residual of the unselected ones."""
    wl = make_workload(name, **ov)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "sparse_residual", tau=tau, topk_pages=topk)
    ctl = SparseResidualController(wl.prefix, sp.dtype, tau, topk)
    A, L = _out(sp)
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        sync()
        assert blk.recomputed == (sp.batch if ref["refresh"] else 0), f"step {st.step}"
        if ref["refresh"]:  # the selection is bit-exact
            ul, uc = cpu(blk.t["union_list"]), cpu(blk.t["union_count"])
            cl, cc = cpu(blk.t["comp_list"]), cpu(blk.t["comp_count"])
            for (b, hk), (S, C) in ref["selection"].items():
                assert uc[b, hk] == len(S) and np.array_equal(ul[b, hk, :len(S)], S), (b, hk)
                assert cc[b, hk] == len(C) and np.array_equal(cl[b, hk, :len(C)], C), (b, hk)
        assert_close_A(cpu(A), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(cpu(L), ref["L_full"], f"step {st.step}")


@pytest.mark.parametrize("name,ov,tau,topk", [
    # 32 rows x 4 q heads = 128 stacked rows per kv head: two row groups of the
    # head scorer, tcgen05 page-list partials; paged ragged cache of two sequences
    ("gqa", dict(prefix_min=400, prefix_max=1500, batch=2, block=32, n_heads_q=8, n_heads_kv=2,
                 steps=4), 2, 9),
    # a 150-row video block: three row groups, tcgen05 in-block and page-list partials
    ("video", dict(prefix_min=900, prefix_max=900, block=150, n_heads_q=2, n_heads_kv=2,
                   steps=3), 0, 14),
])
def test_sparse_residual_beyond_64_rows_per_kv_head(name, ov, tau, topk):
    """The sparse-residual selection over more than 64 stacked rows per kv head
    (rows scored 64 at a time): selection bit-exact, outputs within tolerance."""
    test_sparse_residual_steps_match_oracle(name, ov, tau, topk)


@pytest.mark.parametrize("captured", [False, True])
def test_host_block_pipeline_matches_oracle(captured):
    """Steps fed from pinned host buffers with overlapped copies (eager, and
    captured as one CUDA graph per block) return the oracle's A_full / L_full."""
    from block_diffusion_attention_fb_b200.runtime import HostBlockPipeline
    from workloads.torch_io import to_torch
    wl = make_workload("dllm", prefix_min=1200, prefix_max=1200, n_heads_q=4, n_heads_kv=4,
                       steps=9)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "threshold", tau=2)
    pipe = HostBlockPipeline(blk, torch.bfloat16, depth=3)
    steps = list(wl.steps())
    host_in = [pipe.pack_inputs(to_torch(st.q, sp.dtype, "cpu"), to_torch(st.k_in, sp.dtype, "cpu"),
                                to_torch(st.v_in, sp.dtype, "cpu")) for st in steps]
    host_out = [pipe.new_output() for _ in steps]
    ms = [st.m_updated.tolist() for st in steps]
    if captured:
        pipe.enqueue_block(host_in, host_out, ms)  # eager warm-up
        sync()
        for o in host_out:
            o.fill_(7.0)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            pipe.enqueue_block(host_in, host_out, ms)
        g.replay()
    else:
        pipe.enqueue_block(host_in, host_out, ms)
    sync()
    ctl = ThresholdController(wl.prefix, sp.dtype, 2)
    for st, out in zip(steps, host_out):
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        A, L = pipe.unpack_output(out)
        assert_close_A(A.numpy(), ref["A_full"], sp.dtype, f"step {st.step}")
        assert_close_L(L.numpy(), ref["L_full"], f"step {st.step}")
