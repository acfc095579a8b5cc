"""Pins of the oracle's FlashBlock + sparse-attention residual (oracle/residual.py).

FlashBlock technical summary §2: the keys a sparse method leaves out are
treated as the block-external set and their contribution is cached. Pins: at a
refresh the selected and complementary pages split J_out exactly, so the
prefix partial equals the dense one (merge identity); selecting every page is
dense attention at every step; selecting none is plain threshold reuse; the
head score is an upper bound of every q.k in its page, and the selection is a
top-k of it.
"""

import numpy as np
import pytest

import oracle
from oracle import losa as olosa
from oracle import residual as ores
from oracle.controllers import ThresholdController, dense_step
from workloads import make_workload


def _wl(**ov):
    base = dict(prefix_min=300, prefix_max=300, block=8, n_heads_q=2, n_heads_kv=2, head_dim=64,
                steps=5)
    base.update(ov)
    return make_workload("dllm", **base)


def test_refresh_step_equals_dense_prefix_partial():
    wl = _wl()
    ctl = ores.SparseResidualController(wl.prefix, "bf16", tau=3, topk=5)
    st = next(wl.steps(1))
    out = ctl.step(0, st.q, st.k_in, st.v_in, st.m_updated)
    A, L = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    assert out["refresh"]
    assert np.max(np.abs(out["A_out"] - A)) < 1e-12
    assert np.max(np.abs(out["L_out"] - L)) < 1e-12


def test_all_pages_selected_is_dense_every_step():
    wl = _wl()
    ctl = ores.SparseResidualController(wl.prefix, "bf16", tau=100, topk=10 ** 6)
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        A, L = dense_step(wl.prefix, "bf16", st.q, st.k_in, st.v_in)
        assert np.max(np.abs(out["A_full"] - A)) < 1e-12
        assert np.max(np.abs(out["L_full"] - L)) < 1e-12


def test_no_page_selected_is_threshold_reuse():
    wl = _wl(steps=8)
    ctl = ores.SparseResidualController(wl.prefix, "bf16", tau=2, topk=0)
    ref = ThresholdController(wl.prefix, "bf16", 2)
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        r = ref.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        assert bool(out["refresh"]) == bool(r["recompute"][0])
        assert np.max(np.abs(out["A_full"] - r["A_full"])) < 1e-12
        assert np.max(np.abs(out["L_full"] - r["L_full"])) < 1e-12


def test_selection_is_a_top_k_split_of_the_pages():
    wl = make_workload("gqa", prefix_min=50, prefix_max=400, batch=3, block=6, n_heads_q=4,
                       n_heads_kv=2, head_dim=64)
    st = next(wl.steps(1))
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    sel = ores.head_selection(wl.prefix, st.q, "bf16", 7, smin, smax)
    for (b, hk), (S, C) in sel.items():
        npg = olosa.n_pages(wl.prefix, b)
        assert len(S) == min(7, npg)
        assert np.array_equal(np.union1d(S, C), np.arange(npg))
        assert len(np.intersect1d(S, C)) == 0
        sc = ores.head_page_scores(wl.prefix, st.q, "bf16", b, hk, smin, smax)
        if len(C) and len(S):
            assert sc[S].min() >= sc[C].max()
            # equal scores straddling the cut: the lower page is the selected one
            tie = sc[S].min() == sc[C].max()
            if tie:
                assert S[sc[S] == sc[S].min()].max() < C[sc[C] == sc[C].max()].min()


def test_head_score_bounds_every_key_of_its_page():
    wl = make_workload("gqa", prefix_min=100, prefix_max=200, batch=2, block=5, n_heads_q=4,
                       n_heads_kv=2, head_dim=64)
    st = next(wl.steps(1))
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    qf = oracle.to_f64(st.q, "bf16")
    P = wl.prefix.page_size
    for b in range(2):
        for hk in range(2):
            sc = ores.head_page_scores(wl.prefix, st.q, "bf16", b, hk, smin, smax)
            K, _ = oracle.attention.prefix_keys(wl.prefix, b, hk, "bf16")
            rows = qf[b][:, 2 * hk:2 * hk + 2, :].reshape(-1, K.shape[1])
            dots = rows @ K.T  # exact-ish float64 q.k
            for p in range(len(sc)):
                m = dots[:, p * P:(p + 1) * P].max()
                assert sc[p] >= m - 1e-5 * max(1.0, abs(m))


@pytest.mark.parametrize("topk", [1, 4])
def test_pages_partial_of_selection_and_complement_merge_to_dense(topk):
    wl = make_workload("gqa", prefix_min=60, prefix_max=250, batch=2, block=4, n_heads_q=4,
                       n_heads_kv=2, head_dim=64)
    st = next(wl.steps(1))
    smin, smax = olosa.page_summary(wl.prefix, "bf16")
    sel = ores.head_selection(wl.prefix, st.q, "bf16", topk, smin, smax)
    A_s, L_s = ores.pages_partial(wl.prefix, st.q, "bf16", {k: v[0] for k, v in sel.items()})
    A_c, L_c = ores.pages_partial(wl.prefix, st.q, "bf16", {k: v[1] for k, v in sel.items()})
    A, L = oracle.merge(A_s, L_s, A_c, L_c)
    A_d, L_d = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    assert np.max(np.abs(A - A_d)) < 1e-12 and np.max(np.abs(L - L_d)) < 1e-12
