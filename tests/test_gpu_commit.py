"""GPU parity of fb_block_commit against the oracle's block commit.

Block diffusion is causal between blocks (FlashBlock abstract and technical
summary §2): a finished block's keys and values join J_out of the next block,
and the LoSA page summaries (LoSA §2 step 3) must cover them. Checked bit for
bit: the whole K/V pool (appended slots and every untouched slot), the device
lengths, and the incrementally updated summaries against a from-scratch
summary of the grown cache; then attention over the grown cache.
"""

import numpy as np
import pytest
import torch

import block_diffusion_attention_fb_b200 as fb
import oracle
from oracle import losa as olosa
from oracle.cache import block_commit
from tests.gpu_util import assert_close_A, assert_close_L, cpu, dev, make_kv, sync
from workloads import make_workload
from workloads.gen import grow_capacity

pytestmark = pytest.mark.gpu

CASES = {
    # paged, ragged lengths (pages part-filled), GQA, one and two blocks
    "gqa_paged": ("gqa", dict(prefix_min=100, prefix_max=700, batch=3, block=20, n_heads_q=8,
                              n_heads_kv=2), 2),
    "gqa_paged_block64": ("gqa", dict(prefix_min=17, prefix_max=300, batch=4, block=64,
                                      n_heads_q=8, n_heads_kv=2), 1),
    # contiguous caches: bf16 head_dim 128 and f32 head_dim 64
    "dllm_contig": ("dllm", dict(prefix_min=1000, prefix_max=1000, block=32, n_heads_q=4,
                                 n_heads_kv=4), 2),
    "tiny_contig_f32": ("tiny", dict(prefix_min=1001, prefix_max=1001, block=13), 1),
}


def _bits(a, dtype):
    return np.asarray(a).view(np.uint16 if dtype == "bf16" else np.uint32)


def _summaries(kv, sp):
    tdt = torch.bfloat16 if sp.dtype == "bf16" else torch.float32
    pmin = torch.empty(kv.batch, kv.n_pages, sp.n_heads_kv, sp.head_dim, dtype=tdt, device="cuda")
    pmax = torch.empty_like(pmin)
    fb.fb_page_summary(kv, pmin, pmax)
    return pmin, pmax


@pytest.mark.parametrize("case", sorted(CASES))
def test_block_commit_matches_oracle(case):
    name, ov, n_blocks = CASES[case]
    wl = make_workload(name, **ov)
    sp = wl.spec
    ref = grow_capacity(wl.prefix, n_blocks * sp.block, seed=7)
    kv = make_kv(ref, sp.dtype)
    pmin, pmax = _summaries(kv, sp)
    steps = list(wl.steps(n_blocks))  # one step's block per committed block
    for st in steps:
        lens = ref.seq_len.copy()
        fb.fb_block_commit(kv, lens, dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype), pmin, pmax)
        ref = block_commit(ref, st.k_in, st.v_in)
    sync()
    fb.fb_device_status()
    np.testing.assert_array_equal(_bits(cpu(kv.k.view(torch.int16) if sp.dtype == "bf16"
                                            else kv.k), sp.dtype), _bits(ref.k, sp.dtype))
    np.testing.assert_array_equal(_bits(cpu(kv.v.view(torch.int16) if sp.dtype == "bf16"
                                            else kv.v), sp.dtype), _bits(ref.v, sp.dtype))
    np.testing.assert_array_equal(cpu(kv.seq_len), ref.seq_len)
    smin, smax = olosa.page_summary(ref, sp.dtype)
    gmin, gmax = cpu(pmin.float()), cpu(pmax.float())
    for b in range(sp.batch):
        n = -(-int(ref.seq_len[b]) // ref.page_size)
        np.testing.assert_array_equal(gmin[b, :n], smin[b, :n])
        np.testing.assert_array_equal(gmax[b, :n], smax[b, :n])
    # the next block attends the grown cache: every appended token is seen
    q = steps[-1].q
    ws = torch.empty(fb.fb_workspace_size(kv, sp.block, sp.n_heads_q), dtype=torch.uint8,
                     device="cuda")
    A = torch.zeros(sp.batch, sp.block, sp.n_heads_q, sp.head_dim, device="cuda")
    L = torch.zeros(sp.batch, sp.block, sp.n_heads_q, device="cuda")
    fb.fb_prefix_attn(dev(q, sp.dtype), kv, A, L, ws)
    sync()
    A_ref, L_ref = oracle.prefix_partial(ref, q, sp.dtype)
    assert_close_A(cpu(A), A_ref, sp.dtype, case)
    assert_close_L(cpu(L), L_ref, case)


def test_block_commit_without_summaries_and_empty_block():
    wl = make_workload("dllm", prefix_min=300, prefix_max=300, block=8, n_heads_q=2, n_heads_kv=2)
    sp = wl.spec
    ref = grow_capacity(wl.prefix, sp.block)
    kv = make_kv(ref, sp.dtype)
    st = next(wl.steps(1))
    k0 = cpu(kv.k.view(torch.int16)).copy()
    fb.fb_block_commit(kv, ref.seq_len, dev(st.k_in[:, :0], sp.dtype),
                       dev(st.v_in[:, :0], sp.dtype))  # B = 0: nothing changes
    sync()
    assert np.array_equal(cpu(kv.k.view(torch.int16)), k0)
    assert np.array_equal(cpu(kv.seq_len), ref.seq_len)
    fb.fb_block_commit(kv, ref.seq_len, dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype))
    ref = block_commit(ref, st.k_in, st.v_in)
    sync()
    np.testing.assert_array_equal(cpu(kv.k.view(torch.int16)).view(np.uint16), ref.k)
    np.testing.assert_array_equal(cpu(kv.seq_len), ref.seq_len)


def test_block_commit_rejects_a_cache_without_room():
    wl = make_workload("dllm", prefix_min=300, prefix_max=300, block=8, n_heads_q=2, n_heads_kv=2)
    sp = wl.spec
    kv = make_kv(wl.prefix, sp.dtype)  # contiguous and already full
    st = next(wl.steps(1))
    with pytest.raises(fb.FbError) as e:
        fb.fb_block_commit(kv, wl.prefix.seq_len, dev(st.k_in, sp.dtype), dev(st.v_in, sp.dtype))
    assert e.value.code == fb.FB_ERR_ARG
    fb.fb_device_status()
