"""GPU parity at the full workload sizes (the five configurations), on sampled
outputs the oracle computes row by row; integer decisions are checked whole.

The sampled rows are fixed by a seed and span the first and last block rows,
every kv head and, for GQA, every sequence. Steps run through fb_step (or
fb_prefix_attn for the dense partial), exactly as bench.py calls them, over
every denoise step of the block; the prefix is frozen, so the float64 keys of
each sampled (sequence, kv head) are converted once per test.
"""

import numpy as np
import pytest
import torch

import block_diffusion_attention_fb_b200 as fb
import oracle
from block_diffusion_attention_fb_b200.runtime import BlockAttention
from oracle import losa as olosa
from oracle.controllers import head_cosine
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _samples(sp, n, seed):
    rng = np.random.default_rng(seed)
    out = {(0, 0, 0), (sp.batch - 1, sp.block - 1, sp.n_heads_q - 1)}
    for b in range(sp.batch):
        out.add((b, int(rng.integers(sp.block)), int(rng.integers(sp.n_heads_q))))
    while len(out) < n:
        out.add((int(rng.integers(sp.batch)), int(rng.integers(sp.block)),
                 int(rng.integers(sp.n_heads_q))))
    return sorted(out)


def _grouped_samples(sp, groups, rows_per_group, seed):
    """Sampled (b, i, h) rows from a few (sequence, kv head) groups: the first
    and the last group always, then `groups - 2` more (every sequence first)."""
    rng = np.random.default_rng(seed)
    G = sp.n_heads_q // sp.n_heads_kv
    chosen = [(0, 0), (sp.batch - 1, sp.n_heads_kv - 1)]
    for b in range(sp.batch):
        if len(chosen) >= groups:
            break
        g = (b, int(rng.integers(sp.n_heads_kv)))
        if g not in chosen:
            chosen.append(g)
    while len(chosen) < groups:
        g = (int(rng.integers(sp.batch)), int(rng.integers(sp.n_heads_kv)))
        if g not in chosen:
            chosen.append(g)
    out = set()
    for (b, hk) in chosen:
        rows = [0, sp.block - 1] + [int(x) for x in rng.integers(sp.block, size=rows_per_group)]
        for i in rows[:rows_per_group]:
            out.add((b, i, hk * G + int(rng.integers(G))))
    return sorted(out)


class SampledOracle:
    """Oracle partials of sampled rows. Each sampled (sequence, kv head)'s
    prefix keys and values are converted to float64 once: the prefix is frozen
    for the whole block."""

    def __init__(self, prefix, dtype, samples, G):
        self.dtype, self.G = dtype, G
        self.kv = {}
        for (b, _, h) in samples:
            key = (b, h // G)
            if key not in self.kv:
                self.kv[key] = oracle.attention.prefix_keys(prefix, b, h // G, dtype)

    def prefix_rows(self, q, samples):
        A = np.zeros((len(samples), q.shape[-1]))
        L = np.zeros(len(samples))
        for n, (b, i, h) in enumerate(samples):
            K, V = self.kv[(b, h // self.G)]
            a, l = oracle.partial(oracle.to_f64(q[b, i, h][None], self.dtype), K, V)
            A[n], L[n] = a[0], l[0]
        return A, L

    def full_rows(self, st, samples, A_out_rows, L_out_rows):
        """A_full of the sampled rows: the cached prefix rows merged with the
        sampled rows' block partials."""
        ai = np.zeros_like(A_out_rows)
        li = np.zeros_like(L_out_rows)
        for n, (b, i, h) in enumerate(samples):
            hk = h // self.G
            a, l = oracle.partial(oracle.to_f64(st.q[b, i, h][None], self.dtype),
                                  oracle.to_f64(st.k_in[b, :, hk], self.dtype),
                                  oracle.to_f64(st.v_in[b, :, hk], self.dtype))
            ai[n], li[n] = a[0], l[0]
        return oracle.merge(A_out_rows, L_out_rows, ai, li)


def _check_rows(A, L, samples, A_ref, L_ref, dtype, what):
    got_A = np.stack([A[s] for s in samples])
    got_L = np.array([L[s] for s in samples])
    assert_close_A(got_A, A_ref, dtype, what)
    assert_close_L(got_L, L_ref, what)


def _oracle_full_rows(wl, st, samples, A_out_rows, L_out_rows):
    """A_full of the sampled rows: cached prefix rows merged with the block partial."""
    A_in, L_in = oracle.block_partial(st.q, st.k_in, st.v_in, wl.spec.dtype)
    ai = np.stack([A_in[s] for s in samples])
    li = np.array([L_in[s] for s in samples])
    return oracle.merge(A_out_rows, L_out_rows, ai, li)


@pytest.mark.parametrize("name", ["dllm", "gqa", "video", "losa"])
def test_dense_prefix_partial_full_size(name):
    wl = make_workload(name)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    st = next(wl.steps(1))
    q = dev(st.q, sp.dtype)
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, sp.block, sp.n_heads_q), dtype=torch.uint8,
                     device="cuda")
    fb.fb_prefix_attn(q, kv, A, L, ws)
    sync()
    A, L = cpu(A), cpu(L)
    assert np.isfinite(A).all() and np.isfinite(L).all()
    samples = _samples(sp, 48, 7)
    A_ref, L_ref = oracle.prefix_partial_samples(wl.prefix, st.q, sp.dtype, samples)
    _check_rows(A, L, samples, A_ref, L_ref, sp.dtype, name)


@pytest.mark.parametrize("name", ["dllm", "gqa"])
def test_threshold_block_full_size(name):
    """tau controller over every step of the block: per-sequence decisions
    exact, sampled A_full within tolerance (oracle rows cached at recompute
    steps, as the controller caches them)."""
    wl = make_workload(name)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "threshold", tau=sp.tau)
    samples = _grouped_samples(sp, min(sp.batch * sp.n_heads_kv, 8), 3, 11)
    orc = SampledOracle(wl.prefix, sp.dtype, samples, sp.n_heads_q // sp.n_heads_kv)
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    A_out_rows = np.full((len(samples), sp.head_dim), np.nan)
    L_out_rows = np.full(len(samples), np.nan)
    n_steps = 0
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        sync()
        rec = [st.step == 0 or int(m) >= sp.tau for m in st.m_updated]
        assert blk.recomputed == sum(rec)
        fresh = [n for n, s in enumerate(samples) if rec[s[0]]]
        if fresh:
            a, l = orc.prefix_rows(st.q, [samples[n] for n in fresh])
            A_out_rows[fresh], L_out_rows[fresh] = a, l
        A_ref, L_ref = orc.full_rows(st, samples, A_out_rows, L_out_rows)
        _check_rows(cpu(A), cpu(L), samples, A_ref, L_ref, sp.dtype, f"{name} step {st.step}")
        n_steps += 1
    assert n_steps == sp.steps


def test_per_head_video_full_size():
    """gamma controller over all 50 steps at full video size: the GPU's cosine
    equals the oracle's cosine on the GPU's own tiles bit for bit, masks follow
    it, and sampled A_full rows match the oracle with the GPU's decisions
    (teacher forcing)."""
    wl = make_workload("video")
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "per_head", gamma=sp.gamma)
    samples = _grouped_samples(sp, 6, 4, 13)
    orc = SampledOracle(wl.prefix, sp.dtype, samples, 1)
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    A_out_rows = np.full((len(samples), sp.head_dim), np.nan)
    L_out_rows = np.full(len(samples), np.nan)
    reused = n_steps = 0
    for st in wl.steps():
        mask = cpu(blk.t["head_mask"]).astype(bool)
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L)
        sync()
        nxt = cpu(blk.t["head_mask"]).astype(bool)
        if st.step >= 1 and mask.any():
            cur, prev = cpu(blk.a_out), cpu(blk.t["a_out_prev"])
            cos = cpu(blk.t["head_cos"])
            for h in range(sp.n_heads_q):
                if mask[0, h]:
                    c = head_cosine(cur[0, :, h], prev[0, :, h])
                    assert cos[0, h] == c, (st.step, h)
                    assert nxt[0, h] == (c < sp.gamma)
                else:
                    assert not nxt[0, h]
        elif st.step >= 1:
            assert not nxt.any()
        reused += int((~mask).sum())
        fresh = [n for n, s in enumerate(samples) if mask[s[0], s[2]]]
        if fresh:
            a, l = orc.prefix_rows(st.q, [samples[n] for n in fresh])
            A_out_rows[fresh], L_out_rows[fresh] = a, l
        A_ref, L_ref = orc.full_rows(st, samples, A_out_rows, L_out_rows)
        _check_rows(cpu(A), cpu(L), samples, A_ref, L_ref, sp.dtype, f"video step {st.step}")
        n_steps += 1
    assert n_steps == sp.steps
    assert reused > 0, "at gamma = 0.95 some heads reuse within the block"


def test_losa_full_size():
    """LoSA over all 32 steps at full size: step 0 dense; every later step's
    active rows and page unions equal the oracle's exactly, and the refreshed
    rows match its sparse partial."""
    wl = make_workload("losa")
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "losa", n_active=sp.n_active,
                         topk_pages=sp.topk_pages)
    smin, smax = olosa.page_summary(wl.prefix, sp.dtype)
    gmin = cpu(blk.page_min.float())
    gmax = cpu(blk.page_max.float())
    np.testing.assert_array_equal(gmin[0], smin[0])
    np.testing.assert_array_equal(gmax[0], smax[0])
    samples = _grouped_samples(sp, 4, 4, 17)
    orc = SampledOracle(wl.prefix, sp.dtype, samples, 1)
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    q_prev = None
    A_out_rows = L_out_rows = None
    n_steps = 0
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L)
        sync()
        if st.step == 0:
            A_out_rows, L_out_rows = orc.prefix_rows(st.q, samples)
        else:
            score = olosa.locality_score(st.q, q_prev, sp.dtype)
            act = olosa.active_rows(score, sp.n_active)
            np.testing.assert_array_equal(cpu(blk.t["active_rows"]), act)
            _, union = olosa.select_pages(wl.prefix, st.q, sp.dtype, act, sp.topk_pages, smin,
                                          smax)
            ul, uc = cpu(blk.t["union_list"]), cpu(blk.t["union_count"])
            for (b, hk), pages in union.items():
                assert int(uc[b, hk]) == len(pages)
                np.testing.assert_array_equal(ul[b, hk, :len(pages)], pages)
            fresh = olosa.sparse_partial(wl.prefix, st.q, sp.dtype, act, union)
            a_gpu, l_gpu = cpu(blk.a_out), cpu(blk.l_out)
            keys = list(fresh)
            assert_close_A(np.stack([a_gpu[k] for k in keys]),
                           np.stack([fresh[k][0] for k in keys]), sp.dtype, f"step {st.step}")
            assert_close_L(np.array([l_gpu[k] for k in keys]),
                           np.array([fresh[k][1] for k in keys]), f"step {st.step}")
            for j, s in enumerate(samples):
                if s in fresh:
                    A_out_rows[j], L_out_rows[j] = fresh[s]
        A_ref, L_ref = orc.full_rows(st, samples, A_out_rows, L_out_rows)
        _check_rows(cpu(A), cpu(L), samples, A_ref, L_ref, sp.dtype, f"losa step {st.step}")
        q_prev = st.q
        n_steps += 1
    assert n_steps == sp.steps


def test_long_context_prefix_partial_sampled():
    """A 262144-token prefix (the long-context sweep's lengths run to 819200):
    sampled rows of two kv heads against the oracle on CPU copies of those heads."""
    from oracle.attention import partial, to_f64
    from workloads.long_context import long_prefix
    n_tok = 262144
    k, v, _ = long_prefix(n_tok, 32, 128, seed=2262144)
    wl = make_workload("dllm", prefix_min=16, prefix_max=16)
    sp = wl.spec
    st = next(wl.steps(1))
    seq_len = torch.tensor([n_tok], dtype=torch.int32, device="cuda")
    kv = fb.KV(k, v, seq_len=seq_len, page_table=None, page_size=16, max_seq_len=n_tok)
    q = dev(st.q, sp.dtype)
    A = torch.zeros(1, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(1, sp.block, sp.n_heads_q, device="cuda")
    ws = torch.empty(fb.fb_workspace_size(kv, sp.block, sp.n_heads_q), dtype=torch.uint8,
                     device="cuda")
    fb.fb_prefix_attn(q, kv, A, L, ws)
    sync()
    A, L = cpu(A), cpu(L)
    for h in (0, 31):
        K = to_f64(cpu(k[:, h].contiguous().view(torch.int16)).view(np.uint16), "bf16")
        V = to_f64(cpu(v[:, h].contiguous().view(torch.int16)).view(np.uint16), "bf16")
        rows = [0, 13, sp.block - 1]
        a_ref, l_ref = partial(to_f64(st.q[0, rows, h], "bf16"), K, V)
        assert_close_A(A[0, rows, h], a_ref, "bf16", f"head {h}")
        assert_close_L(L[0, rows, h], l_ref, f"head {h}")


def test_sparse_residual_full_size_dllm():
    """FlashBlock + sparse residual over the dllm block (20 % of the 2048 pages per
    kv head): the selection at every refresh bit-exact, sampled A_full rows within
    tolerance of the oracle's fresh-sparse + cached-residual merge."""
    from oracle import residual as ores
    wl = make_workload("dllm", steps=5)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)
    topk = 410
    blk = BlockAttention(kv, sp.block, sp.n_heads_q, "sparse_residual", tau=sp.tau,
                         topk_pages=topk)
    smin, smax = olosa.page_summary(wl.prefix, sp.dtype)
    samples = _samples(sp, 12, 11)
    heads = sorted({h for _, _, h in samples})
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    res = None
    for st in wl.steps():
        blk.step(dev(st.q, sp.dtype), dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), A, L,
                 m_updated=st.m_updated)
        sync()
        refresh = st.step == 0 or int(st.m_updated[0]) >= sp.tau
        assert blk.recomputed == (1 if refresh else 0)
        if refresh:  # oracle selection of the sampled heads, bit-exact against the GPU's
            ul, uc = cpu(blk.t["union_list"]), cpu(blk.t["union_count"])
            res = {}
            for h in heads:
                sc = ores.head_page_scores(wl.prefix, st.q, sp.dtype, 0, h, smin, smax)
                S_sel = np.sort(olosa.top_indices(sc, topk)).astype(np.int32)
                assert uc[0, h] == len(S_sel) and np.array_equal(ul[0, h, :len(S_sel)], S_sel)
                C = np.setdiff1d(np.arange(len(sc), dtype=np.int32), S_sel)
                res[h] = (S_sel, C, st.q)
        A_ref, L_ref = [], []
        for (b, i, h) in samples:
            S_sel, C, q_ref = res[h]
            P = wl.prefix.page_size
            toks = lambda pages: np.asarray([t for p in pages for t in range(p * P, (p + 1) * P)],
                                            dtype=np.int64)
            Ks, Vs = oracle.attention.prefix_keys(wl.prefix, 0, h, sp.dtype, tokens=toks(S_sel))
            Kc, Vc = oracle.attention.prefix_keys(wl.prefix, 0, h, sp.dtype, tokens=toks(C))
            a_s, l_s = oracle.partial(oracle.to_f64(st.q[0, [i], h], sp.dtype), Ks, Vs)
            a_c, l_c = oracle.partial(oracle.to_f64(q_ref[0, [i], h], sp.dtype), Kc, Vc)
            a_o, l_o = oracle.merge(a_s, l_s, a_c, l_c)
            A_ref.append(a_o[0])
            L_ref.append(l_o[0])
        A_full, L_full = _oracle_full_rows(wl, st, samples, np.stack(A_ref), np.array(L_ref))
        _check_rows(cpu(A), cpu(L), samples, A_full, L_full, sp.dtype, f"step {st.step}")
