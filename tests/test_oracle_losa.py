"""Pins of the oracle's LoSA steps (locality score, active set, page summary,
QUEST-style page scores, top-k pages, union, sparse partial).

Source: "LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion
Language Models" (gist.science, es), §2 "El Algoritmo LoSA", steps 1-4.
Checks use properties that hold by mathematics (upper bounds, exact top-k at
page size 1, reduction to dense attention, bounds on the union size) and
hand-worked float32 cases that fix the specified summation order.
"""

import numpy as np
import pytest

import oracle
from oracle import losa
from oracle.controllers import LosaController
from workloads import make_workload


def test_tree_sum_order_is_stride_halving():
    # float32: 1e8 + 1 rounds to 1e8, so the pairing order shows in the result.
    x = np.array([1e8, 1.0, -1e8, 1.0], dtype=np.float32)
    # tree: (x0 + x2) + (x1 + x3) = 0 + 2 = 2 ; left-to-right would give 1
    assert losa.tree_sum(x) == np.float32(2.0)
    # non power of two pads with zeros: [a, b, c] -> (a + c) + (b + 0)
    y = np.array([1e8, 1.0, -1e8], dtype=np.float32)
    assert losa.tree_sum(y) == np.float32(1.0)


def test_tree_sum_exact_on_integers_and_close_on_floats():
    rng = np.random.default_rng(0)
    ints = rng.integers(-1000, 1000, size=(7, 4096)).astype(np.float32)
    np.testing.assert_array_equal(losa.tree_sum(ints), ints.astype(np.float64).sum(axis=1))
    x = rng.normal(size=(5, 3000)).astype(np.float32)
    exact = x.astype(np.float64).sum(axis=1)
    bound = 12 * np.finfo(np.float32).eps * np.abs(x).astype(np.float64).sum(axis=1)
    assert np.all(np.abs(losa.tree_sum(x) - exact) <= bound)


def test_locality_score_definition():
    rng = np.random.default_rng(1)
    qc = rng.normal(size=(2, 6, 4, 8)).astype(np.float32)
    qp = qc.copy()
    qp[0, 3] += 0.5
    qp[1, 0, 2, 5] -= 2.0
    s = losa.locality_score(qc, qp, "f32")
    assert s.dtype == np.float32 and s.shape == (2, 6)
    np.testing.assert_allclose(s[0, 3], 0.25 * 32, rtol=1e-6)
    np.testing.assert_allclose(s[1, 0], 4.0, rtol=1e-6)
    assert np.count_nonzero(s) == 2  # unchanged rows score exactly 0


def test_active_rows_ties_and_extremes():
    sc = np.array([[0.5, 2.0, 2.0, 0.0, 2.0, 1.0]], dtype=np.float32)
    np.testing.assert_array_equal(losa.active_rows(sc, 2), [[1, 2]])
    np.testing.assert_array_equal(losa.active_rows(sc, 4), [[1, 2, 4, 5]])
    assert losa.active_rows(sc, 0).shape == (1, 0)
    np.testing.assert_array_equal(losa.active_rows(sc, 99), [[1, 2, 4, 5, 0, 3]])


def _small(page_size=16, **kw):
    args = dict(prefix_min=211, prefix_max=211, block=8, steps=4, n_heads_q=4,
                n_heads_kv=4, page_size=page_size)
    args.update(kw)
    return make_workload("losa", **args)


def test_page_summary_bounds_are_tight():
    wl = _small(page_size=16, prefix_min=100, prefix_max=180, paged=True, batch=2,
                n_heads_q=4, n_heads_kv=2)
    smin, smax = losa.page_summary(wl.prefix, "bf16")
    P = 16
    for b in range(2):
        n = int(wl.prefix.seq_len[b])
        for hk in range(2):
            K, _ = oracle.attention.prefix_keys(wl.prefix, b, hk, "bf16")
            for p in range(-(-n // P)):
                page = K[p * P: min(n, p * P + P)]
                assert np.all(page >= smin[b, p, hk]) and np.all(page <= smax[b, p, hk])
                # each bound is attained by a key of the page, channel by channel
                assert np.all(np.any(page == smin[b, p, hk], axis=0))
                assert np.all(np.any(page == smax[b, p, hk], axis=0))


def test_page_score_is_an_upper_bound_of_every_key():
    wl = _small()
    smin, smax = losa.page_summary(wl.prefix, "bf16")
    st = next(wl.steps())
    q = losa.to_f32(st.q, "bf16")
    n = int(wl.prefix.seq_len[0])
    for h in range(4):
        K, _ = oracle.attention.prefix_keys(wl.prefix, 0, h, "bf16")
        u = losa.page_scores(q[0, :, h], smin[0, :14, h], smax[0, :14, h])  # [B, pages]
        exact = q[0, :, h].astype(np.float64) @ K.T  # [B, n]
        for p in range(14):
            m = exact[:, p * 16: min(n, p * 16 + 16)].max(axis=1)
            # float32 tree rounding is far below this slack
            assert np.all(u[:, p] >= m - 1e-4)


def test_page_size_one_gives_exact_top_k_keys():
    """With one key per page, kmin = kmax = k, the bound is q.k itself, so the
    top-k pages are the k highest-scoring keys."""
    wl = _small(page_size=1, prefix_min=300, prefix_max=300)
    smin, smax = losa.page_summary(wl.prefix, "bf16")
    st = next(wl.steps())
    q = losa.to_f32(st.q, "bf16")
    K, _ = oracle.attention.prefix_keys(wl.prefix, 0, 1, "bf16")
    u = losa.page_scores(q[0, :, 1], smin[0, :, 1], smax[0, :, 1])
    exact = q[0, :, 1].astype(np.float64) @ K.T
    np.testing.assert_allclose(u, exact, rtol=0, atol=1e-5)
    for r in range(q.shape[1]):
        top = losa.top_indices(u[r], 10)
        assert set(top.tolist()) == set(np.argsort(-exact[r])[:10].tolist())


def test_page_score_hand_worked():
    # q = (1, -2). Page 0, kmin = (0, -1), kmax = (3, 1): channel 0 takes q * kmax
    # = 3, channel 1 takes q * kmin = 2, so the bound is 5. Page 1 has kmin = kmax
    # = (0.5, 0.25), so the bound is q.k itself: 0.5 - 0.5 = 0.
    q = np.array([[1.0, -2.0]], dtype=np.float32)
    smin = np.array([[0.0, -1.0], [0.5, 0.25]], dtype=np.float32)
    smax = np.array([[3.0, 1.0], [0.5, 0.25]], dtype=np.float32)
    np.testing.assert_array_equal(losa.page_scores(q, smin, smax), [[5.0, 0.0]])


@pytest.mark.parametrize("paged", [False, True])
def test_select_pages_breaks_ties_by_the_lower_logical_page(paged):
    """Logical pages score (0.5, 2, 0.5, 2) for q = (1, 0): top-1 is page 1 (not
    3), top-3 adds page 0 (not 2). With the pool stored in reverse page order,
    the tie still goes to the lower logical page, not the lower pool page."""
    from workloads.gen import Prefix
    low = [[0.0, 0.0], [0.5, 0.0]]
    high = [[1.0, 0.0], [2.0, 0.0]]
    logical = [low, high, low, high]
    table = np.array([[3, 2, 1, 0]], dtype=np.int32) if paged else None
    store = [None] * 4
    for p in range(4):
        store[table[0, p] if paged else p] = logical[p]
    k = np.array(store, dtype=np.float32).reshape(8, 1, 2)
    kv = Prefix(k, k.copy(), np.array([8], dtype=np.int32), table, 2, 8)
    smin, smax = losa.page_summary(kv, "f32")
    q = np.array([1.0, 0.0], dtype=np.float32).reshape(1, 1, 1, 2)
    act = np.array([[0]])
    for topk, want in ((1, [1]), (2, [1, 3]), (3, [1, 3, 0]), (4, [1, 3, 0, 2])):
        chosen, union = losa.select_pages(kv, q, "f32", act, topk, smin, smax)
        np.testing.assert_array_equal(chosen[(0, 0, 0)], want)
        np.testing.assert_array_equal(union[(0, 0)], sorted(want))


def test_union_size_bounds_and_bitmap():
    wl = _small(prefix_min=1000, prefix_max=1000, block=16)
    smin, smax = losa.page_summary(wl.prefix, "bf16")
    st = next(wl.steps())
    act = np.array([[0, 5, 9]])
    topk = 7
    chosen, union = losa.select_pages(wl.prefix, st.q, "bf16", act, topk, smin, smax)
    npg = -(-1000 // 16)
    for hk in range(4):
        u = union[(0, hk)]
        assert topk <= len(u) <= min(3 * topk, npg)
        assert list(u) == sorted(set(u.tolist()))
        for i in act[0]:
            assert set(chosen[(0, int(i), hk)].tolist()) <= set(u.tolist())
    bm = losa.union_bitmap(union, 1, 4, npg)
    for hk in range(4):
        got = [p for p in range(npg) if (bm[0, hk, p // 32] >> (p % 32)) & 1]
        assert got == list(union[(0, hk)])


def test_sparse_partial_over_all_pages_is_the_prefix_partial():
    wl = _small(prefix_min=150, prefix_max=150)
    st = next(wl.steps())
    npg = -(-150 // 16)
    union = {(0, hk): np.arange(npg) for hk in range(4)}
    act = np.array([[2, 6]])
    out = losa.sparse_partial(wl.prefix, st.q, "bf16", act, union)
    A, L = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    for (b, i, h), (a, l) in out.items():
        np.testing.assert_allclose(a, A[b, i, h], atol=1e-14)
        np.testing.assert_allclose(l, L[b, i, h], atol=1e-13)


def test_losa_with_every_row_active_and_every_page_is_dense():
    """|A| = B and top-k = all pages: each step refreshes every row over the
    whole prefix, so LoSA reduces to dense attention."""
    wl = _small(prefix_min=203, prefix_max=203, block=6)
    ctl = LosaController(wl.prefix, "bf16", n_active=6, topk=1000)
    for st in wl.steps(3):
        out = ctl.step(st.step, st.q, st.k_in, st.v_in)
        A, L = oracle.dense_attention(wl.prefix, st.q, st.k_in, st.v_in, "bf16")
        np.testing.assert_allclose(out["A_full"], A, atol=1e-12)
        np.testing.assert_allclose(out["L_full"], L, atol=1e-12)


def test_losa_with_no_active_rows_reuses_step_zero():
    wl = _small(prefix_min=190, prefix_max=190, block=6)
    ctl = LosaController(wl.prefix, "bf16", n_active=0, topk=4)
    first = None
    for st in wl.steps(4):
        out = ctl.step(st.step, st.q, st.k_in, st.v_in)
        if first is None:
            first = out["A_out"]
        np.testing.assert_array_equal(out["A_out"], first)


def test_stable_rows_keep_their_cache_and_active_rows_refresh():
    wl = _small(prefix_min=400, prefix_max=400, block=8)
    ctl = LosaController(wl.prefix, "bf16", n_active=2, topk=5)
    prev = None
    for st in wl.steps(3):
        out = ctl.step(st.step, st.q, st.k_in, st.v_in)
        if st.step > 0:
            act = set(out["active"][0].tolist())
            for i in range(8):
                same = np.array_equal(out["A_out"][0, i], prev[0, i])
                assert same == (i not in act)
        prev = out["A_out"]


@pytest.mark.parametrize("G", [1, 2])
def test_union_is_per_kv_head_over_its_q_heads(G):
    wl = _small(prefix_min=500, prefix_max=500, n_heads_q=4, n_heads_kv=4 // G)
    smin, smax = losa.page_summary(wl.prefix, "bf16")
    st = next(wl.steps())
    act = np.array([[1, 3]])
    chosen, union = losa.select_pages(wl.prefix, st.q, "bf16", act, 3, smin, smax)
    for hk in range(4 // G):
        want = set()
        for h in range(hk * G, hk * G + G):
            for i in (1, 3):
                want |= set(chosen[(0, i, h)].tolist())
        assert set(union[(0, hk)].tolist()) == want
