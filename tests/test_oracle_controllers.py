"""Pins of the oracle's reuse controllers (threshold tau, per-head gamma).

FlashBlock (gist.science technical summary, §2 "Adaptive reuse strategies"):
reuse when the updated-token count is below tau, recompute otherwise; in video,
only heads whose similarity exceeds gamma reuse. The extremes reduce to things
with a plain definition: always recomputing is dense attention, always reusing
holds the first step's block-external partial for the whole block.
"""

import json
import os

import numpy as np
import pytest

import oracle
from oracle.controllers import PerHeadController, ThresholdController, head_cosine
from workloads import make_workload


def _tiny_small():
    return make_workload("tiny", prefix_min=300, prefix_max=300)


def test_tau_zero_is_dense_every_step():
    wl = _tiny_small()
    ctl = ThresholdController(wl.prefix, "f32", tau=0)
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        assert out["recompute"].all()
        A, L = oracle.dense_attention(wl.prefix, st.q, st.k_in, st.v_in, "f32")
        np.testing.assert_allclose(out["A_full"], A, atol=1e-12)
        np.testing.assert_allclose(out["L_full"], L, atol=1e-12)


def test_tau_infinite_holds_step_zero_partial():
    wl = _tiny_small()
    ctl = ThresholdController(wl.prefix, "f32", tau=10**9)
    A0 = L0 = None
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        if st.step == 0:
            A0, L0 = oracle.prefix_partial(wl.prefix, st.q, "f32")
        else:
            assert not out["recompute"].any()
        np.testing.assert_array_equal(out["A_out"], A0)
        A_in, L_in = oracle.block_partial(st.q, st.k_in, st.v_in, "f32")
        A, L = oracle.merge(A0, L0, A_in, L_in)
        np.testing.assert_array_equal(out["A_full"], A)


def test_tiny_decision_trace(golden_dir):
    """The stored trace lists the seeded update counts of the tiny workload and
    the decisions the rule gives for tau = 3: compute at step 0, then exactly
    when M >= 3."""
    g = json.load(open(os.path.join(golden_dir, "tiny_tau_trace.json")))
    wl = make_workload("tiny")
    ctl = ThresholdController(wl.prefix, "f32", tau=g["tau"])
    ms, dec = [], []
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        ms.append(int(st.m_updated[0]))
        dec.append(bool(out["recompute"][0]))
    assert ms == g["m_updated"]
    assert dec == g["recompute"]


def test_per_sequence_decisions_in_a_batch():
    wl = make_workload("gqa", prefix_min=40, prefix_max=90, block=6, steps=6, batch=3)
    ctl = ThresholdController(wl.prefix, "bf16", tau=2)
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in, st.m_updated)
        want = np.array([st.step == 0 or m >= 2 for m in st.m_updated])
        np.testing.assert_array_equal(out["recompute"], want)


def test_head_cosine_special_values():
    rng = np.random.default_rng(0)
    a = rng.normal(size=(7, 9)).astype(np.float32)
    assert abs(head_cosine(a, a) - 1.0) <= 2e-16
    assert abs(head_cosine(a, -a) + 1.0) <= 2e-16
    assert abs(head_cosine(a, 4 * a) - 1.0) <= 2e-16
    x = np.zeros(10)
    y = np.zeros(10)
    x[:5] = 1.0
    y[5:] = 2.0
    assert head_cosine(x, y) == 0.0
    assert head_cosine(np.zeros(4), a.ravel()[:4]) == 0.0
    b = rng.normal(size=(7, 9)).astype(np.float32)
    ref = float(np.dot(a.ravel().astype(np.float64), b.ravel()) /
                (np.linalg.norm(a.astype(np.float64)) * np.linalg.norm(b.astype(np.float64))))
    assert abs(head_cosine(a, b) - ref) < 1e-14


def _video_small():
    return make_workload("video", prefix_min=120, prefix_max=120, block=10, steps=6,
                         n_heads_q=4, n_heads_kv=4)


def test_gamma_above_one_is_dense_every_step():
    wl = _video_small()
    ctl = PerHeadController(wl.prefix, "bf16", gamma=2.0)
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in)
        assert out["computed"].all()
        A, L = oracle.dense_attention(wl.prefix, st.q, st.k_in, st.v_in, "bf16")
        np.testing.assert_allclose(out["A_full"], A, atol=1e-12)


def test_gamma_minus_one_reuses_from_step_two():
    wl = _video_small()
    ctl = PerHeadController(wl.prefix, "bf16", gamma=-1.0)
    A1 = None
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in)
        assert out["computed"].all() == (st.step <= 1)
        if st.step == 1:
            A1 = out["A_out"]
        if st.step >= 2:
            assert not out["computed"].any()
            np.testing.assert_array_equal(out["A_out"], A1)


def test_gamma_decisions_are_sticky_and_follow_the_cosine():
    wl = _video_small()
    ctl = PerHeadController(wl.prefix, "bf16", gamma=0.9999)
    prev_A = None
    prev_mask = None
    for st in wl.steps():
        out = ctl.step(st.step, st.q, st.k_in, st.v_in)
        if prev_mask is not None:
            # once a head stops computing it never restarts
            assert np.all(out["computed"] <= prev_mask)
        for h in range(4):
            if st.step >= 1 and out["computed"][0, h]:
                c = head_cosine(out["A_out"][0, :, h], prev_A[0, :, h])
                assert c == out["cos"][0, h]
                assert out["next_mask"][0, h] == (c < 0.9999)
        prev_A, prev_mask = out["A_out"], out["computed"]


@pytest.mark.parametrize("name", ["tiny", "dllm", "gqa", "video", "losa"])
def test_workload_shapes_and_determinism(name):
    kw = dict(prefix_min=64, prefix_max=96, steps=3)
    if name == "video":
        kw["block"] = 12
    a = make_workload(name, **kw)
    b = make_workload(name, **kw)
    np.testing.assert_array_equal(a.prefix.k, b.prefix.k)
    sa, sb = list(a.steps()), list(b.steps())
    for x, y in zip(sa, sb):
        np.testing.assert_array_equal(x.q, y.q)
        np.testing.assert_array_equal(x.m_updated, y.m_updated)
    sp = a.spec
    assert sa[0].q.shape == (sp.batch, sp.block, sp.n_heads_q, sp.head_dim)
    assert sa[0].k_in.shape == (sp.batch, sp.block, sp.n_heads_kv, sp.head_dim)
