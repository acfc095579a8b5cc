"""Pins of the oracle's sampled-row helpers, the checkers of every full-size
GPU parity test.

``prefix_partial_samples`` and ``dense_attention(samples=...)`` compute the
block-external partial (FlashBlock technical summary, §2 "Core mechanism") and
the unsplit dense attention for a list of (sequence, block row, q head)
triples only. A slip in their grouping (the wrong kv head of a GQA sample, a
write-back to the wrong position) would shift every full-size expectation, so
they are held here to:
  * a per-row brute force written in this file: the page table walked token
    by token, scores and weights summed with math.fsum, nothing shared with
    the oracle's key-set helpers;
  * the whole-tensor functions (prefix_partial, dense_attention without
    samples) at 1e-12, on a paged, ragged, batched GQA cache (G = 4) with
    samples that are shuffled, repeated and spread over sequences and heads.
"""

import math

import numpy as np
import pytest

import oracle
from oracle.attention import bf16_bits_to_f64
from workloads import make_workload


def _bf16(x):
    return bf16_bits_to_f64(x)


def _row_bruteforce(wl, q, b, i, h, with_block=None):
    """Softmax attention of one q row over sequence b's prefix (and optionally
    the block's own keys), token by token from the page table."""
    pre, sp = wl.prefix, wl.spec
    G = sp.n_heads_q // sp.n_heads_kv
    hk = h // G
    P = pre.page_size
    keys, vals = [], []
    for t in range(int(pre.seq_len[b])):
        if pre.page_table is None:
            slot = b * pre.max_seq_len + t
        else:
            slot = int(pre.page_table[b][t // P]) * P + t % P
        keys.append(_bf16(pre.k[slot, hk]))
        vals.append(_bf16(pre.v[slot, hk]))
    if with_block is not None:
        k_in, v_in = with_block
        for j in range(k_in.shape[1]):
            keys.append(_bf16(k_in[b, j, hk]))
            vals.append(_bf16(v_in[b, j, hk]))
    qv = _bf16(q[b, i, h])
    s = [math.fsum(float(a) * float(c) for a, c in zip(qv, k)) for k in keys]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    Z = math.fsum(w)
    A = np.array([math.fsum(wj * float(v[c]) for wj, v in zip(w, vals)) / Z
                  for c in range(len(qv))])
    return A, m + math.log(Z)


def _small_gqa():
    # paged pool, pages permuted, ragged lengths (not page multiples), batch 3, G = 4
    wl = make_workload("gqa", prefix_min=21, prefix_max=75, block=5, steps=1, batch=3,
                       n_heads_q=8, n_heads_kv=2, head_dim=8)
    return wl, next(wl.steps())


def _samples(sp, n, seed):
    rng = np.random.default_rng(seed)
    s = [(int(rng.integers(sp.batch)), int(rng.integers(sp.block)), int(rng.integers(sp.n_heads_q)))
         for _ in range(n)]
    s += s[:3]  # repeated entries
    rng.shuffle(s)
    return s


def test_workload_is_paged_ragged_gqa():
    wl, _ = _small_gqa()
    assert wl.prefix.page_table is not None
    assert len(set(int(n) for n in wl.prefix.seq_len)) > 1
    assert any(int(n) % wl.prefix.page_size for n in wl.prefix.seq_len)
    assert wl.spec.n_heads_q // wl.spec.n_heads_kv == 4


def test_prefix_partial_samples_matches_bruteforce():
    wl, st = _small_gqa()
    samples = _samples(wl.spec, 9, 1)
    A, L = oracle.prefix_partial_samples(wl.prefix, st.q, "bf16", samples)
    for n, (b, i, h) in enumerate(samples):
        a_ref, l_ref = _row_bruteforce(wl, st.q, b, i, h)
        np.testing.assert_allclose(A[n], a_ref, rtol=0, atol=1e-12)
        assert abs(L[n] - l_ref) <= 1e-12


def test_prefix_partial_samples_matches_whole_tensor():
    wl, st = _small_gqa()
    samples = _samples(wl.spec, 40, 2)
    A, L = oracle.prefix_partial_samples(wl.prefix, st.q, "bf16", samples)
    A_all, L_all = oracle.prefix_partial(wl.prefix, st.q, "bf16")
    for n, s in enumerate(samples):
        np.testing.assert_allclose(A[n], A_all[s], rtol=0, atol=1e-12)
        assert abs(L[n] - L_all[s]) <= 1e-12


def test_dense_attention_samples_matches_bruteforce_and_whole_tensor():
    wl, st = _small_gqa()
    samples = _samples(wl.spec, 12, 3)
    A, L = oracle.dense_attention(wl.prefix, st.q, st.k_in, st.v_in, "bf16", samples=samples)
    A_all, L_all = oracle.dense_attention(wl.prefix, st.q, st.k_in, st.v_in, "bf16")
    for n, (b, i, h) in enumerate(samples):
        np.testing.assert_allclose(A[n], A_all[b, i, h], rtol=0, atol=1e-12)
        assert abs(L[n] - L_all[b, i, h]) <= 1e-12
        if n < 5:
            a_ref, l_ref = _row_bruteforce(wl, st.q, b, i, h, with_block=(st.k_in, st.v_in))
            np.testing.assert_allclose(A[n], a_ref, rtol=0, atol=1e-12)
            assert abs(L[n] - l_ref) <= 1e-12


@pytest.mark.parametrize("wrong", ["kv_head", "order"])
def test_sampled_checker_catches_planted_mistakes(wrong):
    """A checker that read the wrong kv head or wrote rows back out of order
    would differ from the brute force: plant each mistake in a copy of the
    grouping and check that the comparison above would fail."""
    wl, st = _small_gqa()
    sp = wl.spec
    G = sp.n_heads_q // sp.n_heads_kv
    samples = [(0, 1, 0), (1, 2, 5), (2, 0, 7), (0, 4, 3)]
    out = []
    for (b, i, h) in samples:
        hk = (h % sp.n_heads_kv) if wrong == "kv_head" else h // G
        K, V = oracle.attention.prefix_keys(wl.prefix, b, hk, "bf16")
        out.append(oracle.partial(oracle.to_f64(st.q[b, i, h][None], "bf16"), K, V)[0][0])
    if wrong == "order":
        out = out[::-1]
    ref = [_row_bruteforce(wl, st.q, *s)[0] for s in samples]
    assert any(np.abs(o - r).max() > 1e-6 for o, r in zip(out, ref))
