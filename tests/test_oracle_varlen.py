"""Pins of the oracle's packed-row (variable-length) functions.

BlockBatch page, "Optimización del Sistema": branches of different block sizes
packed into one variable-length buffer. Packing is a layout: each packed
segment must give exactly what its sequence gives alone. The pins compare the
varlen oracle with the batched one (itself pinned by brute force, closed forms
and the merge identity in test_oracle_attention.py) on one-sequence views, and
with the unsplit dense attention through the threshold controller at tau = 0.
"""

import numpy as np
import pytest

import oracle
from oracle import varlen as ov
from workloads.gen import Prefix
from workloads.varlen import make_varlen_workload


def _alone(pre, b):
    """Sequence b of a cache as a batch of one (same pool, same page table row)."""
    if pre.page_table is None:
        m = pre.max_seq_len
        return Prefix(pre.k[b * m:(b + 1) * m], pre.v[b * m:(b + 1) * m], pre.seq_len[b:b + 1],
                      None, pre.page_size, m)
    return Prefix(pre.k, pre.v, pre.seq_len[b:b + 1], pre.page_table[b:b + 1], pre.page_size,
                  pre.max_seq_len)


CASES = [
    ("gqa", (3, 0, 7, 1, 5), False, dict(prefix_min=20, prefix_max=90, n_heads_q=8, n_heads_kv=2,
                                          head_dim=8, steps=3)),
    ("gqa", (4, 8, 2), True, dict(prefix_min=33, prefix_max=60, n_heads_q=4, n_heads_kv=2,
                                   head_dim=8, steps=3)),
    ("tiny", (2, 6, 3), False, dict(prefix_min=40, prefix_max=40, head_dim=8, steps=3)),
]


@pytest.mark.parametrize("base,rows,shared,ovr", CASES)
def test_packed_segments_equal_each_sequence_alone(base, rows, shared, ovr):
    wl = make_varlen_workload(base, rows, shared_prefix=shared, **ovr)
    dt = wl.spec.dtype
    st = next(wl.steps(1))
    A, L = ov.prefix_partial_varlen(wl.prefix, st.q, wl.cu, dt)
    Ai, Li = ov.block_partial_varlen(st.q, st.k_in, st.v_in, wl.cu, dt)
    assert A.shape == (wl.total, wl.spec.n_heads_q, wl.spec.head_dim)
    assert not np.isnan(A).any() and not np.isnan(Ai).any()
    for b, r0, r1 in ov.segments(wl.cu):
        if r1 == r0:
            continue
        qb = st.q[r0:r1][None]
        a, l = oracle.prefix_partial(_alone(wl.prefix, b), qb, dt)
        # equal up to the order BLAS sums in (rows are grouped differently)
        np.testing.assert_allclose(A[r0:r1], a[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(L[r0:r1], l[0], rtol=0, atol=1e-13)
        a, l = oracle.block_partial(qb, st.k_in[r0:r1][None], st.v_in[r0:r1][None], dt)
        np.testing.assert_allclose(Ai[r0:r1], a[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(Li[r0:r1], l[0], rtol=0, atol=1e-13)


def test_shared_prefix_branches_read_the_same_keys():
    wl = make_varlen_workload("gqa", (2, 2), shared_prefix=True, prefix_min=30, prefix_max=70,
                              n_heads_q=4, n_heads_kv=2, head_dim=8)
    st = next(wl.steps(1))
    q = st.q.copy()
    q[2:4] = q[0:2]  # the second branch asks the same questions
    A, L = ov.prefix_partial_varlen(wl.prefix, q, wl.cu, "bf16")
    np.testing.assert_array_equal(A[0:2], A[2:4])
    np.testing.assert_array_equal(L[0:2], L[2:4])


def test_equal_lengths_equal_the_batched_oracle():
    wl = make_varlen_workload("gqa", (5, 5, 5), prefix_min=20, prefix_max=80, n_heads_q=8,
                              n_heads_kv=2, head_dim=8)
    st = next(wl.base.steps(1))
    pst = next(wl.steps(1))
    A, L = ov.prefix_partial_varlen(wl.prefix, pst.q, wl.cu, "bf16")
    Ab, Lb = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    np.testing.assert_allclose(A, Ab.reshape(A.shape), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, Lb.reshape(L.shape), rtol=0, atol=1e-13)


def test_threshold_varlen_at_tau_zero_is_dense_per_sequence():
    """tau = 0 recomputes every step: every packed row equals the unsplit dense
    attention over [its prefix ; its block] (which never uses the merge)."""
    wl = make_varlen_workload("gqa", (3, 6, 0, 2), prefix_min=25, prefix_max=70, n_heads_q=4,
                              n_heads_kv=2, head_dim=8, steps=3)
    ctl = ov.ThresholdVarlenController(wl.prefix, "bf16", 0)
    for st in wl.steps():
        ref = ctl.step(st.step, st.q, st.k_in, st.v_in, wl.cu, st.m_updated)
        assert ref["recompute"].all()
        for b, r0, r1 in ov.segments(wl.cu):
            if r1 == r0:
                continue
            a, l = oracle.dense_attention(_alone(wl.prefix, b), st.q[r0:r1][None],
                                          st.k_in[r0:r1][None], st.v_in[r0:r1][None], "bf16")
            np.testing.assert_allclose(ref["A_full"][r0:r1], a[0], atol=1e-12)
            np.testing.assert_allclose(ref["L_full"][r0:r1], l[0], atol=1e-12)


def test_threshold_varlen_reuses_per_sequence():
    """A sequence whose update count stays below tau keeps its step-0 partial."""
    wl = make_varlen_workload("gqa", (3, 4), prefix_min=25, prefix_max=50, n_heads_q=4,
                              n_heads_kv=2, head_dim=8, steps=2)
    ctl = ov.ThresholdVarlenController(wl.prefix, "bf16", 10 ** 6)
    it = wl.steps()
    s0 = next(it)
    ctl.step(0, s0.q, s0.k_in, s0.v_in, wl.cu, s0.m_updated)
    A0 = ctl.A_out.copy()
    s1 = next(it)
    ref = ctl.step(1, s1.q, s1.k_in, s1.v_in, wl.cu, s1.m_updated)
    assert not ref["recompute"].any()
    np.testing.assert_array_equal(ctl.A_out, A0)
