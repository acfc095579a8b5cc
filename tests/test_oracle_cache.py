"""Pins of the oracle's block commit (oracle/cache.py).

Block diffusion is causal between blocks: a finished block's tokens join the
block-external set J_out of every later block (FlashBlock abstract and
technical summary §2). Pins: the grown key sequence is the old one followed by
the block's rows; attention over the grown cache equals the log-space merge of
the old prefix partial with the block partial (the FlashBlock merge identity);
pages wholly before the old end keep their LoSA summaries.
"""

import numpy as np
import pytest

import oracle
from oracle import attention as oatt
from oracle import losa as olosa
from oracle.cache import block_commit
from workloads import make_workload
from workloads.gen import grow_capacity

CASES = {
    "paged_gqa": ("gqa", dict(prefix_min=5, prefix_max=70, batch=3, block=20, n_heads_q=4,
                              n_heads_kv=2, head_dim=64)),
    "contig_dllm": ("dllm", dict(prefix_min=33, prefix_max=33, block=12, n_heads_q=2,
                                 n_heads_kv=2, head_dim=64)),
    "contig_tiny_f32": ("tiny", dict(prefix_min=40, prefix_max=40, block=16)),
}


def _grown(name, ov):
    wl = make_workload(name, **ov)
    st = next(wl.steps(1))
    return wl, st, grow_capacity(wl.prefix, wl.spec.block, seed=5)


@pytest.mark.parametrize("case", sorted(CASES))
def test_grow_capacity_keeps_every_token(case):
    wl, _, big = _grown(*CASES[case])
    dt = wl.spec.dtype
    for b in range(wl.spec.batch):
        for hk in range(wl.spec.n_heads_kv):
            K0, V0 = oatt.prefix_keys(wl.prefix, b, hk, dt)
            K1, V1 = oatt.prefix_keys(big, b, hk, dt)
            assert np.array_equal(K0, K1) and np.array_equal(V0, V1)


@pytest.mark.parametrize("case", sorted(CASES))
def test_commit_appends_block_rows_in_token_order(case):
    wl, st, big = _grown(*CASES[case])
    dt = wl.spec.dtype
    new = block_commit(big, st.k_in, st.v_in)
    assert np.array_equal(new.seq_len, big.seq_len + wl.spec.block)
    for b in range(wl.spec.batch):
        for hk in range(wl.spec.n_heads_kv):
            K0, V0 = oatt.prefix_keys(big, b, hk, dt)
            K1, V1 = oatt.prefix_keys(new, b, hk, dt)
            assert np.array_equal(K1, np.concatenate([K0, oatt.to_f64(st.k_in[b, :, hk], dt)]))
            assert np.array_equal(V1, np.concatenate([V0, oatt.to_f64(st.v_in[b, :, hk], dt)]))
    # the input cache is not modified
    assert np.array_equal(big.seq_len, wl.prefix.seq_len)


@pytest.mark.parametrize("case", sorted(CASES))
def test_attention_after_commit_is_the_merge_of_prefix_and_block_partials(case):
    wl, st, big = _grown(*CASES[case])
    dt = wl.spec.dtype
    new = block_commit(big, st.k_in, st.v_in)
    A1, L1 = oracle.prefix_partial(new, st.q, dt)
    A0, L0 = oracle.prefix_partial(big, st.q, dt)
    Ab, Lb = oracle.block_partial(st.q, st.k_in, st.v_in, dt)
    Am, Lm = oracle.merge(A0, L0, Ab, Lb)
    assert np.max(np.abs(A1 - Am)) < 1e-12
    assert np.max(np.abs(L1 - Lm)) < 1e-12


def test_summaries_of_pages_before_the_old_end_are_unchanged():
    wl, st, big = _grown(*CASES["paged_gqa"])
    new = block_commit(big, st.k_in, st.v_in)
    s0 = olosa.page_summary(big, "bf16")
    s1 = olosa.page_summary(new, "bf16")
    P = big.page_size
    for b in range(wl.spec.batch):
        full = int(big.seq_len[b]) // P
        for a0, a1 in zip(s0, s1):
            assert np.array_equal(a0[b, :full], a1[b, :full])
        # a page that held tokens before keeps min <= its old min, max >= its old max
        if int(big.seq_len[b]) % P:
            assert np.all(s1[0][b, full] <= s0[0][b, full])
            assert np.all(s1[1][b, full] >= s0[1][b, full])


def test_commit_rejects_a_cache_without_room():
    wl = make_workload("dllm", prefix_min=40, prefix_max=40, block=8, n_heads_q=2, n_heads_kv=2,
                       head_dim=64)
    st = next(wl.steps(1))
    with pytest.raises(ValueError):
        block_commit(wl.prefix, st.k_in, st.v_in)  # contiguous, already full
