"""Pins of the oracle's partial, merge and dense attention against mathematics.

The FlashBlock pages state the decomposition (technical summary, §2 "Core
mechanism"): a partial (A, L = log Z) per key set and the log-space merge.
Nothing here compares the oracle with itself: every check is a closed form,
an mpmath brute force, an identity that holds exactly in real arithmetic, or a
hand-derived value from tests/golden/closed_forms.json.
"""

import json
import math
import os

import mpmath
import numpy as np
import pytest

import oracle
from oracle.attention import bf16_bits_to_f64

mpmath.mp.dps = 50


def _mp_partial(q, K, V, scale):
    """Softmax attention straight from its definition, at 50 digits."""
    R, N, d = len(q), len(K), len(q[0])
    A = np.zeros((R, V.shape[1]))
    L = np.zeros(R)
    for r in range(R):
        s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(q[r][c]) * mpmath.mpf(K[j][c])
                                           for c in range(d)) for j in range(N)]
        Z = mpmath.fsum(mpmath.e ** sj for sj in s)
        L[r] = float(mpmath.log(Z))
        for c in range(V.shape[1]):
            A[r, c] = float(mpmath.fsum(mpmath.e ** s[j] * mpmath.mpf(V[j][c]) for j in range(N)) / Z)
    return A, L


@pytest.mark.parametrize("seed", range(6))
def test_partial_matches_mpmath_bruteforce(seed):
    rng = np.random.default_rng(seed)
    R, N, d = rng.integers(1, 5), rng.integers(1, 9), rng.integers(1, 5)
    q = rng.normal(size=(R, d)) * 3
    K = rng.normal(size=(N, d)) * 3
    V = rng.normal(size=(N, d + 1))
    scale = float(rng.uniform(0.1, 2.0))
    A, L = oracle.partial(q, K, V, scale)
    A_ref, L_ref = _mp_partial(q, K, V, scale)
    np.testing.assert_allclose(L, L_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(A, A_ref, rtol=0, atol=1e-13)


def test_partial_large_scores_do_not_overflow():
    # scores around 1000: e^1000 overflows float64, the two-pass form must not
    q = np.array([[1000.0]])
    K = np.array([[1.0], [0.999]])
    V = np.array([[1.0], [0.0]])
    A, L = oracle.partial(q, K, V)
    A_ref, L_ref = _mp_partial(q, K, V, 1.0)
    np.testing.assert_allclose(L, L_ref, atol=1e-12)
    np.testing.assert_allclose(A, A_ref, atol=1e-13)


def test_partial_closed_forms(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "closed_forms.json")))
    for name in ("partial_two_keys", "partial_one_key", "partial_equal_scores"):
        c = g[name]
        A, L = oracle.partial(np.array(c["q"]), np.array(c["K"]), np.array(c["V"]), c["scale"])
        np.testing.assert_allclose(L, [c["L"]], atol=1e-15, err_msg=name)
        np.testing.assert_allclose(A[0], c["A"], atol=1e-15, err_msg=name)


def test_partial_shift_invariance():
    # adding a constant c to every score (via an extra channel) keeps A, moves L by c
    rng = np.random.default_rng(7)
    q = rng.normal(size=(3, 5))
    K = rng.normal(size=(11, 5))
    V = rng.normal(size=(11, 5))
    c = 2.75
    q2 = np.concatenate([q, np.ones((3, 1))], axis=1)
    K2 = np.concatenate([K, np.full((11, 1), c)], axis=1)
    A, L = oracle.partial(q, K, V)
    A2, L2 = oracle.partial(q2, K2, V)
    np.testing.assert_allclose(A2, A, atol=1e-14)
    np.testing.assert_allclose(L2, L + c, atol=1e-13)


def test_partial_empty_key_set():
    A, L = oracle.partial(np.ones((2, 4)), np.zeros((0, 4)), np.zeros((0, 4)))
    assert np.all(A == 0) and np.all(np.isneginf(L))


def test_merge_closed_forms(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "closed_forms.json")))
    for name in ("merge_weights_one_to_three", "merge_one_side_empty"):
        c = g[name]
        f = lambda x: -np.inf if x == "-inf" else x  # noqa: E731
        A, L = oracle.merge(np.array(c["A_out"]), np.array(f(c["L_out"])),
                            np.array(c["A_in"]), np.array(f(c["L_in"])))
        np.testing.assert_allclose(A, c["A"], atol=1e-15, err_msg=name)
        np.testing.assert_allclose(L, c["L"], atol=1e-15, err_msg=name)


def test_merge_both_empty():
    A, L = oracle.merge(np.zeros(3), np.array(-np.inf), np.zeros(3), np.array(-np.inf))
    assert np.all(A == 0) and np.isneginf(L)


@pytest.mark.parametrize("seed", range(8))
def test_split_then_merge_equals_unsplit(seed):
    """The decomposition is exact: merging partials of a split key set gives
    the softmax over the whole set, to float64 rounding (<= 1e-12)."""
    rng = np.random.default_rng(100 + seed)
    R, N, d = 5, int(rng.integers(2, 300)), 16
    q = rng.normal(size=(R, d)) * 2
    K = rng.normal(size=(N, d))
    V = rng.normal(size=(N, d))
    cut = int(rng.integers(0, N + 1))  # may leave one side empty
    perm = rng.permutation(N)
    J1, J2 = perm[:cut], perm[cut:]
    A, L = oracle.partial(q, K, V)
    A1, L1 = oracle.partial(q, K[J1], V[J1])
    A2, L2 = oracle.partial(q, K[J2], V[J2])
    Am, Lm = oracle.merge(A1, L1, A2, L2)
    np.testing.assert_allclose(Am, A, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lm, L, rtol=0, atol=1e-12)
    # order of the two sides does not matter
    Am2, Lm2 = oracle.merge(A2, L2, A1, L1)
    np.testing.assert_allclose(Am2, Am, atol=1e-15)
    np.testing.assert_allclose(Lm2, Lm, atol=1e-15)


def test_merge_is_associative_three_way():
    rng = np.random.default_rng(5)
    q = rng.normal(size=(4, 8))
    K = rng.normal(size=(90, 8))
    V = rng.normal(size=(90, 8))
    parts = [slice(0, 17), slice(17, 60), slice(60, 90)]
    P = [oracle.partial(q, K[s], V[s]) for s in parts]
    left = oracle.merge(*oracle.merge(*P[0], *P[1]), *P[2])
    right = oracle.merge(*P[0], *oracle.merge(*P[1], *P[2]))
    full = oracle.partial(q, K, V)
    for x in (left, right):
        np.testing.assert_allclose(x[0], full[0], atol=1e-12)
        np.testing.assert_allclose(x[1], full[1], atol=1e-12)


def test_bf16_decode_matches_torch():
    torch = pytest.importorskip("torch")
    bits = np.array([0x3F80, 0xC049, 0x0001, 0x7F7F, 0x8000, 0x4780], dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(bf16_bits_to_f64(bits), ref)


class _KV:
    def __init__(self, k, v, seq_len, page_table, page_size, max_seq_len):
        self.k, self.v, self.seq_len = k, v, np.asarray(seq_len, dtype=np.int32)
        self.page_table, self.page_size, self.max_seq_len = page_table, page_size, max_seq_len


def test_paged_lookup_equals_contiguous():
    """A permuted page pool read through its page table gives the same keys
    as the contiguous layout of the same tokens."""
    rng = np.random.default_rng(3)
    L, P, H, d = 45, 4, 2, 3
    K = rng.normal(size=(L, H, d)).astype(np.float32)
    V = rng.normal(size=(L, H, d)).astype(np.float32)
    npg = -(-L // P)
    perm = rng.permutation(npg)
    kp = np.full((npg * P, H, d), np.nan, dtype=np.float32)
    vp = np.full((npg * P, H, d), np.nan, dtype=np.float32)
    for t in range(L):
        kp[perm[t // P] * P + t % P] = K[t]
        vp[perm[t // P] * P + t % P] = V[t]
    cont = _KV(K, V, [L], None, P, L)
    paged = _KV(kp, vp, [L], perm[None, :].astype(np.int32), P, L)
    q = rng.normal(size=(1, 3, H, d)).astype(np.float32)
    A1, L1 = oracle.prefix_partial(cont, q, "f32")
    A2, L2 = oracle.prefix_partial(paged, q, "f32")
    np.testing.assert_array_equal(A1, A2)
    np.testing.assert_array_equal(L1, L2)
    assert not np.isnan(A2).any()


def test_dense_step_equals_unsplit_dense():
    """prefix partial + block partial + merge equals one softmax over
    [prefix; block] (the dense block-diffusion attention) to 1e-12."""
    from oracle.controllers import dense_step
    from workloads import make_workload
    wl = make_workload("gqa", prefix_min=37, prefix_max=70, block=5, steps=1, batch=2)
    st = next(wl.steps())
    A, L = dense_step(wl.prefix, "bf16", st.q, st.k_in, st.v_in)
    A_ref, L_ref = oracle.dense_attention(wl.prefix, st.q, st.k_in, st.v_in, "bf16")
    np.testing.assert_allclose(A, A_ref, atol=1e-12)
    np.testing.assert_allclose(L, L_ref, atol=1e-12)
    assert math.isfinite(float(np.abs(A).max()))
