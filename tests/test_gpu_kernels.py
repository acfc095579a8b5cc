"""GPU parity of each C-ABI call against the oracle at sizes that span several
key tiles, several row tiles and ragged tails (seconds of oracle time).

Sources: FlashBlock technical summary §2 (partials, merge, reuse rules); LoSA
§2 steps 1-4 (locality score, active set, sparse selection, union).
"""

import numpy as np
import pytest
import torch

import block_diffusion_attention_fb_b200 as fb
import oracle
from oracle import losa as olosa
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads import make_workload

pytestmark = pytest.mark.gpu


def run_prefix(wl, q_np, head_mask=None):
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    q = dev(q_np, sp.dtype)
    A = torch.full((sp.batch, sp.block, sp.n_heads_q, sp.head_dim), 7.0, device="cuda")
    L = torch.full((sp.batch, sp.block, sp.n_heads_q), 7.0, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, sp.block, sp.n_heads_q), dtype=torch.uint8,
                     device="cuda")
    hm = None if head_mask is None else torch.from_numpy(head_mask.astype(np.uint8)).cuda()
    fb.fb_prefix_attn(q, kv, A, L, ws, head_mask=hm)
    sync()
    return cpu(A), cpu(L)


PREFIX_CASES = {
    # name: (workload, overrides)
    "tiny_full_f32": ("tiny", {}),
    "tiny_ragged_f32": ("tiny", dict(prefix_min=1001, prefix_max=1001, block=13)),
    # fp32, several tiles per split through the two-stage cp.async ring, ragged tail
    "tiny_long_f32": ("tiny", dict(prefix_min=20011, prefix_max=20011)),
    # fp32 paged pool, head_dim 128, GQA stacking over 5 row tiles, varied lengths
    "tiny_paged_gqa_d128_f32": ("tiny", dict(prefix_min=17, prefix_max=900, batch=3, block=20,
                                             head_dim=128, n_heads_q=8, n_heads_kv=2,
                                             paged=True)),
    "dllm_small_ragged": ("dllm", dict(prefix_min=1000, prefix_max=1000, n_heads_q=4,
                                       n_heads_kv=4)),
    "dllm_block16": ("dllm", dict(prefix_min=777, prefix_max=777, block=16, n_heads_q=2,
                                  n_heads_kv=2)),
    "dllm_block1": ("dllm", dict(prefix_min=300, prefix_max=300, block=1, n_heads_q=2,
                                 n_heads_kv=2)),
    "gqa_paged_small": ("gqa", dict(prefix_min=100, prefix_max=700, batch=3, block=20,
                                    n_heads_q=8, n_heads_kv=2)),
    "gqa_paged_rows_gt_64": ("gqa", dict(prefix_min=50, prefix_max=400, batch=2, block=40,
                                         n_heads_q=8, n_heads_kv=2)),
    "video_rows_many_tiles": ("video", dict(prefix_min=500, prefix_max=500, block=150,
                                            n_heads_q=2, n_heads_kv=2)),
    "losa_contig_d128": ("losa", dict(prefix_min=2000, prefix_max=2000, n_heads_q=3,
                                      n_heads_kv=3)),
    "d64_bf16": ("dllm", dict(prefix_min=600, prefix_max=600, head_dim=64, n_heads_q=2,
                              n_heads_kv=2)),
    # two long groups over many CTAs: partial segments at both ends of CTAs
    "dllm_two_heads_long": ("dllm", dict(prefix_min=20011, prefix_max=20011, n_heads_q=2,
                                         n_heads_kv=2)),
    # paged, varied lengths, 64 stacked rows per kv head (16 rows x 4 q heads)
    "gqa_paged_64_rows": ("gqa", dict(prefix_min=17, prefix_max=3000, batch=5, block=16,
                                      n_heads_q=8, n_heads_kv=2)),
    # more groups than CTAs, each a few tiles
    "many_groups": ("gqa", dict(prefix_min=64, prefix_max=500, batch=40, block=8,
                                n_heads_q=16, n_heads_kv=8)),
    # one sequence with a short last 256-row tile: full tiles on the tcgen05
    # kernel, the last rows (44; 24 stacked = 6 block rows x G 4) on the
    # streaming kernel
    "video_short_last_tile": ("video", dict(prefix_min=1300, prefix_max=1300, block=300,
                                            n_heads_q=2, n_heads_kv=2)),
    "gqa_one_seq_short_last_tile": ("gqa", dict(prefix_min=900, prefix_max=900, batch=1,
                                                block=70, n_heads_q=8, n_heads_kv=2)),
}


@pytest.mark.parametrize("case", sorted(PREFIX_CASES))
def test_prefix_attn_matches_oracle(case):
    name, ov = PREFIX_CASES[case]
    wl = make_workload(name, **ov)
    st = next(wl.steps(1))
    A, L = run_prefix(wl, st.q)
    A_ref, L_ref = oracle.prefix_partial(wl.prefix, st.q, wl.spec.dtype)
    assert_close_A(A, A_ref, wl.spec.dtype, case)
    assert_close_L(L, L_ref, case)


def test_prefix_attn_head_mask_leaves_other_rows():
    wl = make_workload("gqa", prefix_min=200, prefix_max=300, batch=2, block=8, n_heads_q=8,
                       n_heads_kv=2)
    st = next(wl.steps(1))
    mask = np.zeros((2, 8), dtype=bool)
    mask[0, 1] = mask[1, 4] = mask[1, 5] = True
    A, L = run_prefix(wl, st.q, head_mask=mask)
    A_ref, L_ref = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    sel = np.broadcast_to(mask[:, None, :], L.shape)
    assert_close_A(A[sel], A_ref[sel], "bf16")
    assert_close_L(L[sel], L_ref[sel])
    assert np.all(A[~sel] == 7.0) and np.all(L[~sel] == 7.0)


def test_prefix_attn_empty_and_short_sequences():
    wl = make_workload("gqa", prefix_min=1, prefix_max=40, batch=4, block=6, n_heads_q=4,
                       n_heads_kv=2)
    wl.prefix.seq_len[2] = 0  # an empty prefix: A = 0, L = -inf
    st = next(wl.steps(1))
    A, L = run_prefix(wl, st.q)
    A_ref, L_ref = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    assert np.all(A[2] == 0) and np.all(np.isneginf(L[2]))
    assert_close_A(A, A_ref, "bf16")
    assert_close_L(L, L_ref)


@pytest.mark.parametrize("name,ov", [
    ("tiny", {}),
    ("dllm", dict(block=32, n_heads_q=4, n_heads_kv=4, prefix_min=64, prefix_max=64)),
    ("gqa", dict(block=64, batch=2, n_heads_q=8, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    ("video", dict(block=130, n_heads_q=2, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    ("dllm", dict(block=5, n_heads_q=2, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    # short-block kernel: every key-tile count (B padded to 16, 32, 48, 64), GQA row
    # stacking with a ragged last row tile, head_dim 64, a single-token block
    ("dllm", dict(block=1, n_heads_q=3, n_heads_kv=3, prefix_min=64, prefix_max=64)),
    ("dllm", dict(block=17, n_heads_q=2, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    ("gqa", dict(block=45, batch=3, n_heads_q=12, n_heads_kv=3, prefix_min=64, prefix_max=64)),
    ("gqa", dict(block=64, batch=2, n_heads_q=32, n_heads_kv=8, prefix_min=64, prefix_max=64)),
    ("dllm", dict(block=33, head_dim=64, n_heads_q=4, n_heads_kv=2, prefix_min=64,
                  prefix_max=64)),
    ("video", dict(block=65, n_heads_q=2, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    # one sequence, 290 rows (a full 256-row tile and 34 rows) on the tcgen05 kernel
    ("video", dict(block=290, n_heads_q=2, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    # fp32 short-block kernel: one token, head_dim 128 with GQA stacking and keys past
    # 32, a full 64-token block with 256 stacked rows over 3 sequences; the last case
    # stacks too many rows for its shared memory and takes the general kernel
    ("tiny", dict(block=1, prefix_min=64, prefix_max=64)),
    ("tiny", dict(block=37, head_dim=128, n_heads_q=8, n_heads_kv=2, prefix_min=64,
                  prefix_max=64)),
    ("tiny", dict(block=64, batch=3, n_heads_q=8, n_heads_kv=2, prefix_min=64, prefix_max=64)),
    ("tiny", dict(block=64, head_dim=128, n_heads_q=16, n_heads_kv=2, prefix_min=64,
                  prefix_max=64)),
])
def test_block_attn_matches_oracle(name, ov):
    wl = make_workload(name, **ov)
    sp = wl.spec
    st = next(wl.steps(1))
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    fb.fb_block_attn(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L)
    sync()
    A_ref, L_ref = oracle.block_partial(st.q, st.k_in, st.v_in, sp.dtype)
    assert_close_A(cpu(A), A_ref, sp.dtype)
    assert_close_L(cpu(L), L_ref)


def test_merge_matches_oracle_including_empty_sides():
    rng = np.random.default_rng(0)
    rows, d = 1000, 128
    Ao = rng.normal(size=(rows, d)).astype(np.float32)
    Ai = rng.normal(size=(rows, d)).astype(np.float32)
    Lo = rng.normal(size=rows).astype(np.float32) * 5
    Li = rng.normal(size=rows).astype(np.float32) * 5
    Lo[:10] = -np.inf
    Li[5:15] = -np.inf
    Ao[:10] = np.nan  # a side with L = -inf is never read
    t = lambda x: torch.from_numpy(x).cuda()  # noqa: E731
    Af = torch.zeros(rows, d, device="cuda")
    Lf = torch.zeros(rows, device="cuda")
    fb.fb_merge(t(Ao), t(Lo), t(Ai), t(Li), Af, Lf)
    sync()
    Ao64 = np.where(np.isnan(Ao), 0.0, Ao)
    A_ref, L_ref = oracle.merge(Ao64, Lo, Ai, Li)
    np.testing.assert_allclose(cpu(Af), A_ref, rtol=0, atol=2e-6)
    assert_close_L(cpu(Lf), L_ref)
    assert np.all(cpu(Af)[5:10] == 0)


def _losa_small(**kw):
    args = dict(prefix_min=3001, prefix_max=3001, block=16, n_heads_q=4, n_heads_kv=4)
    args.update(kw)
    return make_workload("losa", **args)


def _bf16_bits(t):
    return cpu(t.view(torch.int16)).view(np.uint16)


@pytest.mark.parametrize("paged", [False, True])
def test_page_summary_is_exact(paged):
    if paged:
        wl = make_workload("gqa", prefix_min=100, prefix_max=600, batch=3, block=4, n_heads_q=4,
                           n_heads_kv=2)
    else:
        wl = _losa_small()
    kv = make_kv(wl.prefix, "bf16")
    npg = kv.n_pages
    pmin = torch.empty(kv.batch, npg, kv.c.n_heads_kv, 128, dtype=torch.bfloat16, device="cuda")
    pmax = torch.empty_like(pmin)
    fb.fb_page_summary(kv, pmin, pmax)
    sync()
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    gmin = cpu(pmin.float())
    gmax = cpu(pmax.float())
    for b in range(kv.batch):
        n = -(-int(wl.prefix.seq_len[b]) // 16)
        np.testing.assert_array_equal(gmin[b, :n], smin[b, :n])
        np.testing.assert_array_equal(gmax[b, :n], smax[b, :n])


def run_select(wl, q_cur, q_prev, n_active, topk):
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    npg, hkv = kv.n_pages, sp.n_heads_kv
    pmin = torch.empty(kv.batch, npg, hkv, sp.head_dim, dtype=torch.bfloat16, device="cuda")
    pmax = torch.empty_like(pmin)
    fb.fb_page_summary(kv, pmin, pmax)
    na = min(n_active, sp.block)
    act = torch.full((sp.batch, max(na, 1)), -1, dtype=torch.int32, device="cuda")
    rs = torch.zeros(sp.batch, sp.block, device="cuda")
    bm = torch.zeros(sp.batch, hkv, -(-npg // 32), dtype=torch.int32, device="cuda")
    ul = torch.full((sp.batch, hkv, npg), -1, dtype=torch.int32, device="cuda")
    uc = torch.zeros(sp.batch, hkv, dtype=torch.int32, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, sp.block, sp.n_heads_q, n_active, topk),
                     dtype=torch.uint8, device="cuda")
    fb.losa_select(dev(q_cur, "bf16"), dev(q_prev, "bf16"), pmin, pmax, kv, n_active, topk, act,
                   bm, ul, uc, ws, row_scores=rs)
    sync()
    return kv, act, rs, bm, ul, uc, ws


@pytest.mark.parametrize("ov,n_active,topk", [
    ({}, 4, 20),
    (dict(prefix_min=999, prefix_max=999), 3, 7),
    (dict(n_heads_q=4, n_heads_kv=2), 2, 9),
    ({}, 4, 1000),       # top-k larger than the page count: every page
    ({}, 40, 5),         # more active rows than block rows: all rows
    (dict(block=300), 4, 9),    # more rows than the selection block's threads
    (dict(block=70), 40, 5),    # more than 32 active rows: the rank path
])
def test_losa_select_is_bit_exact(ov, n_active, topk):
    wl = _losa_small(**ov)
    steps = list(wl.steps(2))
    q_prev, q_cur = steps[0].q, steps[1].q
    kv, act, rs, bm, ul, uc, ws = run_select(wl, q_cur, q_prev, n_active, topk)
    score = olosa.locality_score(q_cur, q_prev, "bf16")
    np.testing.assert_array_equal(cpu(rs), score)  # bit-exact float32 tree
    act_ref = olosa.active_rows(score, n_active)
    np.testing.assert_array_equal(cpu(act)[:, :act_ref.shape[1]], act_ref)
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    _, union = olosa.select_pages(wl.prefix, q_cur, "bf16", act_ref, topk, smin, smax)
    npg = kv.n_pages
    # every page bound, bit-exact (not only the ones near each top-k boundary)
    sp = wl.spec
    na, Hq, G = act_ref.shape[1], sp.n_heads_q, sp.n_heads_q // sp.n_heads_kv
    off = fb.fb_workspace_page_scores(kv, sp.block, Hq, n_active, topk)
    sc = cpu(ws[off:off + kv.batch * na * Hq * npg * 4].view(torch.float32)).reshape(
        kv.batch, na, Hq, npg)
    qf = olosa.to_f32(q_cur, "bf16")
    for b in range(kv.batch):
        n = -(-int(wl.prefix.seq_len[b]) // 16)
        for h in range(Hq):
            ref = olosa.page_scores(qf[b, act_ref[b], h], smin[b, :n, h // G], smax[b, :n, h // G])
            np.testing.assert_array_equal(sc[b, :, h, :n], ref, err_msg=f"b={b} h={h}")
    bm_ref = olosa.union_bitmap(union, kv.batch, kv.c.n_heads_kv, npg)
    np.testing.assert_array_equal(cpu(bm).view(np.uint32), bm_ref)
    for (b, hk), pages in union.items():
        assert int(cpu(uc)[b, hk]) == len(pages)
        np.testing.assert_array_equal(cpu(ul)[b, hk, :len(pages)], pages)


@pytest.mark.parametrize("period,topk", [(1, 20), (3, 7), (3, 100)])
def test_losa_select_breaks_page_ties_by_lower_page(period, topk):
    """Pages repeat with the given period (every page a copy of one of `period`
    distinct pages), so many page bounds are equal and the k-th largest is
    shared by more pages than are taken: the union must hold the lowest such
    pages, as the oracle's selection does."""
    wl = _losa_small()
    pre = wl.prefix
    n = int(pre.seq_len[0])
    t = np.arange(pre.k.shape[0]) % n  # position within its sequence
    src = (t // 16 % period) * 16 + t % 16 + (np.arange(pre.k.shape[0]) // n) * n
    pre.k[:] = pre.k[src]
    steps = list(wl.steps(2))
    q_prev, q_cur = steps[0].q, steps[1].q
    kv, act, rs, bm, ul, uc, ws = run_select(wl, q_cur, q_prev, 4, topk)
    act_ref = olosa.active_rows(olosa.locality_score(q_cur, q_prev, "bf16"), 4)
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    _, union = olosa.select_pages(wl.prefix, q_cur, "bf16", act_ref, topk, smin, smax)
    bm_ref = olosa.union_bitmap(union, kv.batch, kv.c.n_heads_kv, kv.n_pages)
    np.testing.assert_array_equal(cpu(bm).view(np.uint32), bm_ref)
    for (b, hk), pages in union.items():
        assert int(cpu(uc)[b, hk]) == len(pages)
        np.testing.assert_array_equal(cpu(ul)[b, hk, :len(pages)], pages)


def test_losa_gather_matches_oracle():
    wl = _losa_small(n_heads_q=4, n_heads_kv=2)
    steps = list(wl.steps(2))
    q_prev, q_cur = steps[0].q, steps[1].q
    n_active, topk = 3, 11
    kv, act, rs, bm, ul, uc, ws = run_select(wl, q_cur, q_prev, n_active, topk)
    A = torch.full((1, 16, 4, 128), 5.0, device="cuda")
    L = torch.full((1, 16, 4), 5.0, device="cuda")
    fb.losa_gather(dev(q_cur, "bf16"), act, n_active, ul, uc, kv, A, L, ws,
                   max_union=n_active * 2 * topk)
    sync()
    act_ref = olosa.active_rows(olosa.locality_score(q_cur, q_prev, "bf16"), n_active)
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    _, union = olosa.select_pages(wl.prefix, q_cur, "bf16", act_ref, topk, smin, smax)
    ref = olosa.sparse_partial(wl.prefix, q_cur, "bf16", act_ref, union)
    A, L = cpu(A), cpu(L)
    got_A = np.stack([A[b, i, h] for (b, i, h) in ref])
    want_A = np.stack([v[0] for v in ref.values()])
    assert_close_A(got_A, want_A, "bf16")
    assert_close_L(np.array([L[k] for k in ref]), np.array([v[1] for v in ref.values()]))
    stable = np.ones(16, dtype=bool)
    stable[act_ref[0]] = False
    assert np.all(A[0, stable] == 5.0) and np.all(L[0, stable] == 5.0)


def test_invalid_arguments_are_rejected_on_the_host():
    wl = make_workload("dllm", prefix_min=128, prefix_max=128, n_heads_q=2, n_heads_kv=2)
    kv = make_kv(wl.prefix, "bf16")
    q = dev(next(wl.steps(1)).q, "bf16")
    A = torch.zeros(1, 32, 2, 128, device="cuda")
    L = torch.zeros(1, 32, 2, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fb.FbError) as e:
        fb.fb_prefix_attn(q, kv, A, L, ws)  # workspace far too small
    assert e.value.code == fb.FB_ERR_WORKSPACE
    bad = make_kv(wl.prefix, "bf16")
    bad.c.head_dim = 96
    with pytest.raises(fb.FbError) as e:
        fb.fb_prefix_attn(q, bad, A, L, ws)
    assert e.value.code == fb.FB_ERR_SHAPE
    q3 = torch.zeros(1, 32, 3, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fb.FbError) as e:
        fb.fb_prefix_attn(q3, kv, A, L, ws)  # 3 q heads cannot share 2 kv heads
    assert e.value.code == fb.FB_ERR_SHAPE
    big = torch.empty(fb.fb_workspace_size(kv, 32, 2), dtype=torch.uint8, device="cuda")
    for bad_scale in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(fb.FbError) as e:
            fb.fb_prefix_attn(q, kv, A, L, big, scale=bad_scale)
        assert e.value.code == fb.FB_ERR_ARG
        with pytest.raises(fb.FbError) as e:
            fb.fb_block_attn(q, q, q, A, L, scale=bad_scale)
        assert e.value.code == fb.FB_ERR_ARG
    fb.fb_device_status()


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    """A wait that nothing satisfies (an mbarrier nobody arrives at) gives up
    after its cycle budget, flags FB_ERR_TIMEOUT to the host, and the next
    attention call on the same context is correct."""
    fb.fb_device_status()  # start clean
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    fb.fb_selftest_timeout(flag)
    sync()
    assert int(flag.item()) == 1
    with pytest.raises(fb.FbError) as e:
        fb.fb_device_status()
    assert e.value.code == fb.FB_ERR_TIMEOUT
    fb.fb_device_status()  # the word was cleared by the read
    name, ov = PREFIX_CASES["dllm_small_ragged"]
    wl = make_workload(name, **ov)
    st = next(wl.steps(1))
    A, L = run_prefix(wl, st.q)
    A_ref, L_ref = oracle.prefix_partial(wl.prefix, st.q, wl.spec.dtype)
    assert_close_A(A, A_ref, wl.spec.dtype)
    assert_close_L(L, L_ref)
    fb.fb_device_status()


def test_losa_active_rows_break_ties_by_lower_row():
    """Rows whose q did not move score exactly 0; the active set takes the moved
    rows by score, then the lowest-index unmoved rows (LoSA step 1, ties)."""
    wl = _losa_small(block=40)
    steps = list(wl.steps(2))
    q_prev = steps[0].q
    q_cur = q_prev.copy()
    q_cur[0, [7, 21, 33]] = steps[1].q[0, [7, 21, 33]]
    kv, act, rs, *_ = run_select(wl, q_cur, q_prev, 6, 4)
    score = olosa.locality_score(q_cur, q_prev, "bf16")
    act_ref = olosa.active_rows(score, 6)
    np.testing.assert_array_equal(cpu(act)[:, :6], act_ref)
    assert sorted(act_ref[0, :3].tolist()) == [7, 21, 33]
    assert act_ref[0, 3:].tolist() == [0, 1, 2]


@pytest.mark.parametrize("name,ov", [
    # bf16 (TMA producer) and fp32 (cp.async) read paths; GQA rows over 64 take the
    # tcgen05 kernel
    ("gqa", dict(prefix_min=300, prefix_max=700, batch=2, block=12, n_heads_q=8, n_heads_kv=2)),
    ("gqa", dict(prefix_min=300, prefix_max=700, batch=2, block=24, n_heads_q=8, n_heads_kv=2)),
    ("tiny", dict(prefix_min=300, prefix_max=700, batch=2, block=12, head_dim=128,
                  n_heads_q=8, n_heads_kv=2, paged=True)),
])
def test_page_table_entries_outside_the_pool_read_as_absent(name, ov):
    """A page-table entry outside the pool (past its end, or negative) is
    checked before any access: its tokens count as absent, the result equals
    the partial over the remaining tokens, and fb_device_status reports
    FB_ERR_ARG. The page summary skips the same pages."""
    wl = make_workload(name, steps=1, **ov)
    sp = wl.spec
    pre = wl.prefix
    n_pool_pages = pre.k.shape[0] // pre.page_size
    kv = make_kv(pre, sp.dtype)
    bad = {(0, 1): n_pool_pages + 3, (1, 0): -2}  # (sequence, logical page) -> bad entry
    for (b, p), e in bad.items():
        kv.page_table[b, p] = e
    st = next(wl.steps(1))
    A = torch.full((sp.batch, sp.block, sp.n_heads_q, sp.head_dim), 7.0, device="cuda")
    L = torch.full((sp.batch, sp.block, sp.n_heads_q), 7.0, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, sp.block, sp.n_heads_q), dtype=torch.uint8,
                     device="cuda")
    fb.fb_prefix_attn(dev(st.q, sp.dtype), kv, A, L, ws)
    sync()
    with pytest.raises(fb.FbError) as e:
        fb.fb_device_status()
    assert e.value.code == fb.FB_ERR_ARG
    fb.fb_device_status()  # the word was cleared
    A, L = cpu(A), cpu(L)
    G = sp.n_heads_q // sp.n_heads_kv
    P = pre.page_size
    for b in range(sp.batch):
        keep = [t for t in range(int(pre.seq_len[b])) if (b, t // P) not in bad]
        for hk in range(sp.n_heads_kv):
            K, V = oracle.attention.prefix_keys(pre, b, hk, sp.dtype, tokens=keep)
            for g in range(G):
                h = hk * G + g
                a, l = oracle.partial(oracle.to_f64(st.q[b, :, h], sp.dtype), K, V)
                assert_close_A(A[b, :, h], a, sp.dtype, f"b{b} h{h}")
                assert_close_L(L[b, :, h], l, f"b{b} h{h}")
    if sp.dtype == "bf16":
        pmin = torch.empty(sp.batch, kv.n_pages, sp.n_heads_kv, sp.head_dim, dtype=torch.bfloat16,
                           device="cuda")
        pmax = torch.empty_like(pmin)
        fb.fb_page_summary(kv, pmin, pmax)
        sync()
        with pytest.raises(fb.FbError):
            fb.fb_device_status()
        smin, smax = olosa.page_summary(pre, sp.dtype)
        gmin, gmax = cpu(pmin.float()), cpu(pmax.float())
        for b in range(sp.batch):
            for p in range(-(-int(pre.seq_len[b]) // P)):
                if (b, p) not in bad:
                    np.testing.assert_array_equal(gmin[b, p], smin[b, p])
                    np.testing.assert_array_equal(gmax[b, p], smax[b, p])
