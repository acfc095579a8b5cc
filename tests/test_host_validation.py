"""Host-side argument checks of every C-ABI entry point, run without a GPU.

Each case is rejected by the library's own validation before any launch, with
the FB_ERR_* code include/fb.h documents for it. Device pointers here are fake
(aligned or deliberately misaligned integers), so the module is skipped where a
GPU is visible: a case that slipped past validation must never reach a kernel.
"""

import ctypes
import math

import pytest

import block_diffusion_attention_fb_b200 as fb

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake device pointers: CPU-only checks")

DEV = 1 << 20   # an aligned fake device address
DEV2 = 2 << 20
MISALIGNED = DEV + 4


@pytest.fixture(scope="module")
def lib():
    from block_diffusion_attention_fb_b200 import build as _build
    _build.build()
    return fb.load_library()


def make_kv(**ov):
    kv = fb.fb_kv()
    kv.k, kv.v = DEV, DEV2
    kv.page_table = None
    kv.seq_len = None
    kv.batch, kv.n_heads_kv, kv.head_dim, kv.page_size = 1, 2, 128, 16
    kv.max_seq_len, kv.n_slots, kv.max_pages_per_seq = 64, 64, 4
    kv.dtype = fb.FB_BF16
    for k, v in ov.items():
        setattr(kv, k, v)
    return kv


def err(lib):
    return lib.fb_last_error().decode()


def prefix(lib, kv, q=DEV, B=4, Hq=4, scale=1.0, a_out=DEV, l_out=DEV):
    return lib.fb_prefix_attn(q, B, Hq, scale, ctypes.byref(kv), None, a_out, l_out, DEV,
                              1 << 30, None)


# -------------------------------------------------------------- fb_prefix_attn
@pytest.mark.parametrize("scale", [0.0, -1.0, math.nan, math.inf])
def test_prefix_rejects_a_non_positive_or_non_finite_scale(lib, scale):
    assert prefix(lib, make_kv(), scale=scale) == fb.FB_ERR_ARG
    assert "scale" in err(lib)


@pytest.mark.parametrize("ov,code", [
    (dict(head_dim=96), fb.FB_ERR_SHAPE),
    (dict(page_size=24), fb.FB_ERR_SHAPE),
    (dict(page_size=8), fb.FB_ERR_SHAPE),
    (dict(batch=0), fb.FB_ERR_ARG),
    (dict(batch=257), fb.FB_ERR_ARG),
    (dict(n_slots=1 << 31, max_seq_len=64), fb.FB_ERR_SHAPE),
    (dict(max_seq_len=65), fb.FB_ERR_ARG),           # contiguous: batch * L > n_slots
    (dict(page_table=DEV, max_pages_per_seq=3), fb.FB_ERR_ARG),  # 3 pages < 64 tokens
    (dict(k=MISALIGNED), fb.FB_ERR_ALIGN),
    (dict(v=None), fb.FB_ERR_ARG),
    (dict(dtype=7), fb.FB_ERR_ARG),
])
def test_prefix_rejects_bad_caches(lib, ov, code):
    assert prefix(lib, make_kv(**ov)) == code, err(lib)


def test_prefix_rejects_bad_queries_and_outputs(lib):
    kv = make_kv()
    assert prefix(lib, kv, Hq=3) == fb.FB_ERR_SHAPE          # 3 % 2 q heads per kv head
    assert prefix(lib, kv, B=0) == fb.FB_ERR_ARG
    assert prefix(lib, kv, q=MISALIGNED) == fb.FB_ERR_ALIGN
    assert prefix(lib, kv, q=None) == fb.FB_ERR_ARG
    assert prefix(lib, kv, l_out=None) == fb.FB_ERR_ARG


def test_noalloc_checks_the_scale_and_its_static_scratch_before_the_device(lib):
    kv = make_kv()
    rc = lib.fb_prefix_attn_noalloc(DEV, 4, 4, -1.0, ctypes.byref(kv), None, DEV, DEV, None)
    assert rc == fb.FB_ERR_ARG and "scale" in err(lib)
    # 3 sequences of up to 2M tokens, 256 stacked rows: at least one split per 128
    # key tiles of a sequence, i.e. 128 splits x 3 x 256 rows of float32 partials
    # (50 MB), beyond the 32 MiB static scratch
    big = make_kv(batch=3, n_heads_kv=1, max_seq_len=1 << 21, n_slots=3 << 21)
    rc = lib.fb_prefix_attn_noalloc(DEV, 256, 1, 1.0, ctypes.byref(big), None, DEV, DEV, None)
    assert rc == fb.FB_ERR_WORKSPACE and "static" in err(lib)


# ------------------------------------------------------- fb_block_attn, fb_merge
def test_block_attn_checks(lib):
    def call(q=DEV, B=16, Hq=4, Hkv=2, d=128, scale=1.0, dt=fb.FB_BF16, a=DEV, l=DEV):
        return lib.fb_block_attn(q, DEV, DEV2, 1, B, Hq, Hkv, d, scale, dt, a, l, None)
    for dt in (fb.FB_BF16, fb.FB_F32):
        for B in (16, 100):   # the short-block kernels and the general one
            assert call(B=B, dt=dt, scale=0.0) == fb.FB_ERR_ARG, (dt, B)
    assert call(d=96) == fb.FB_ERR_SHAPE
    assert call(Hq=5) == fb.FB_ERR_SHAPE
    assert call(a=None) == fb.FB_ERR_ARG
    assert call(q=MISALIGNED) == fb.FB_ERR_ALIGN


def test_merge_checks(lib):
    assert lib.fb_merge(DEV, DEV, DEV, None, 8, 128, DEV, DEV, None) == fb.FB_ERR_ARG
    assert lib.fb_merge(DEV, DEV, DEV, DEV, -1, 128, DEV, DEV, None) == fb.FB_ERR_ARG
    assert lib.fb_merge(DEV, DEV, DEV, DEV, 8, 96, DEV, DEV, None) == fb.FB_ERR_SHAPE
    # zero rows is a valid no-op that never touches the device
    assert lib.fb_merge(DEV, DEV, DEV, DEV, 0, 128, DEV, DEV, None) == fb.FB_OK


# ------------------------------------------------------------------ LoSA calls
def test_page_summary_checks(lib):
    kv = make_kv()
    assert lib.fb_page_summary(ctypes.byref(kv), None, DEV, None) == fb.FB_ERR_ARG
    bad = make_kv(head_dim=96)
    assert lib.fb_page_summary(ctypes.byref(bad), DEV, DEV, None) == fb.FB_ERR_SHAPE


def select(lib, kv, Hq=4, n_active=2, topk=4, page_min=DEV, q_prev=DEV):
    return lib.losa_select(DEV, q_prev, 4, Hq, page_min, DEV2, ctypes.byref(kv), n_active, topk,
                           DEV, None, DEV, DEV, DEV, DEV, 1 << 30, None)


def test_losa_select_checks(lib):
    kv = make_kv()
    assert select(lib, kv, n_active=-1) == fb.FB_ERR_ARG
    assert select(lib, kv, topk=-1) == fb.FB_ERR_ARG
    assert select(lib, kv, page_min=MISALIGNED) == fb.FB_ERR_ALIGN
    assert select(lib, kv, q_prev=None) == fb.FB_ERR_ARG
    assert select(lib, kv, Hq=256) == fb.FB_ERR_SHAPE      # n_heads_q * d > 16384
    long_kv = make_kv(max_seq_len=16 * 40000, n_slots=16 * 40000)   # 40000 pages
    assert select(lib, long_kv) == fb.FB_ERR_SHAPE
    assert "32768 pages" in err(lib)


def test_losa_gather_checks(lib):
    kv = make_kv()

    def call(n_active=2, union_list=DEV, scale=1.0):
        return lib.losa_gather(DEV, 4, 4, DEV, n_active, union_list, DEV, 0, ctypes.byref(kv),
                               scale, DEV, DEV, DEV, 1 << 30, None)
    assert call(union_list=None) == fb.FB_ERR_ARG
    assert call(scale=math.nan) == fb.FB_ERR_ARG
    assert call(n_active=0) == fb.FB_OK   # nothing active: a no-op


# --------------------------------------------------------------------- fb_step
def step(lib, policy, cache, kv, ws_bytes=1 << 40):
    return lib.fb_step(ctypes.byref(policy) if policy is not None else None,
                       ctypes.byref(cache), DEV, DEV, DEV2, 4, 4, ctypes.byref(kv), None, None,
                       None, DEV, DEV, DEV, ws_bytes, None)


def test_step_checks(lib):
    kv = make_kv()
    cache = fb.fb_cache()
    cache.a_out, cache.l_out = DEV, DEV
    pol = fb.fb_policy()
    pol.mode, pol.tau, pol.scale = fb.FB_THRESHOLD, 2, 1.0
    assert step(lib, None, cache, kv) == fb.FB_ERR_ARG
    assert step(lib, pol, cache, kv, ws_bytes=16) == fb.FB_ERR_WORKSPACE
    pol.scale = -2.0      # step 0 recomputes: the prefix launcher rejects it
    assert step(lib, pol, cache, kv) == fb.FB_ERR_ARG
    pol.scale = 1.0
    pol.mode = fb.FB_PER_HEAD
    assert step(lib, pol, cache, kv) == fb.FB_ERR_ARG   # no head_mask / a_out_prev / head_cos
    assert "PER_HEAD" in err(lib)
    cache.l_out = None
    pol.mode = fb.FB_THRESHOLD
    assert step(lib, pol, cache, kv) == fb.FB_ERR_ARG


# ------------------------------------------------------------- fb_block_commit
def test_block_commit_checks(lib):
    lens = (ctypes.c_int32 * 1)(40)
    kv = make_kv(seq_len=DEV)

    def call(kv=kv, lens=lens, k_in=DEV, v_in=DEV2, B=16, pmin=None, pmax=None):
        return lib.fb_block_commit(ctypes.byref(kv), lens, k_in, v_in, B, pmin, pmax, None)
    assert call(kv=make_kv()) == fb.FB_ERR_ARG            # no device lengths to update
    assert call(lens=None) == fb.FB_ERR_ARG
    assert call(B=-1) == fb.FB_ERR_ARG
    assert call(k_in=None) == fb.FB_ERR_ARG
    assert call(pmin=DEV) == fb.FB_ERR_ARG                # min without max
    assert call(v_in=MISALIGNED) == fb.FB_ERR_ALIGN
    assert call(B=25) == fb.FB_ERR_ARG                    # 40 + 25 > max_seq_len 64
    assert "exceed max_seq_len" in err(lib)
    assert call(B=0) == fb.FB_OK                          # an empty block: nothing to do


# ---------------------------------------------------------- fb_workspace_size
def test_workspace_size_is_zero_for_shapes_no_call_accepts(lib):
    for ov in (dict(head_dim=96), dict(page_size=24), dict(page_size=8), dict(dtype=7),
               dict(batch=0)):
        kv = make_kv(**ov)
        assert lib.fb_workspace_size(ctypes.byref(kv), 4, 4, 0, 0, 148) == 0, ov
    kv = make_kv()
    assert lib.fb_workspace_size(ctypes.byref(kv), 4, 3, 0, 0, 148) == 0
    assert lib.fb_workspace_size(ctypes.byref(kv), 4, 4, -1, 4, 148) == 0


def test_workspace_size_covers_the_split_partials_of_a_dllm_prefix(lib):
    # 32 heads, 32 block rows, 32768 prefix tokens on 148 SMs: the plan splits each
    # head's keys nine ways (two CTAs per SM over 32 heads), and each split keeps a
    # float32 partial of every row
    kv = make_kv(n_heads_kv=32, max_seq_len=32768, n_slots=32768)
    ws = lib.fb_workspace_size(ctypes.byref(kv), 32, 32, 0, 0, 148)
    assert ws >= 9 * 32 * 32 * 128 * 4
    short = make_kv(n_heads_kv=32, max_seq_len=64, n_slots=64)   # one tile: no split
    ws_short = lib.fb_workspace_size(ctypes.byref(short), 32, 32, 0, 0, 148)
    assert 0 < ws_short < ws
    # LoSA adds page scores for every active row and head over the prefix's pages
    ws_losa = lib.fb_workspace_size(ctypes.byref(kv), 32, 32, 4, 256, 148)
    assert ws_losa >= ws + 4 * 32 * (32768 // 16) * 4


def test_page_score_offset_lies_inside_the_losa_workspace(lib):
    # the page scores sit after the split partials, 256-byte aligned, with room
    # for one float32 per (active row, q head, logical page) before the end
    kv = make_kv(n_heads_kv=32, max_seq_len=32768, n_slots=32768)
    args = (ctypes.byref(kv), 32, 32, 4, 256, 148)
    off = lib.fb_workspace_page_scores(*args)
    total = lib.fb_workspace_size(*args)
    assert off > 0 and off % 256 == 0
    assert off >= 9 * 32 * 32 * 128 * 4                   # after the nine-way split partials
    assert off + 4 * 32 * (32768 // 16) * 4 <= total
    # n_active caps at the block rows; a paged cache counts its page-table width
    paged = make_kv(page_table=3 << 20,
                    max_pages_per_seq=10, max_seq_len=160, n_slots=160)
    pargs = (ctypes.byref(paged), 4, 4, 9, 3, 148)
    off = lib.fb_workspace_page_scores(*pargs)
    assert off > 0 and off + 4 * 4 * 10 * 4 <= lib.fb_workspace_size(*pargs)


def test_page_score_offset_is_zero_without_a_selection_or_for_bad_shapes(lib):
    kv = make_kv()
    assert lib.fb_workspace_page_scores(ctypes.byref(kv), 4, 4, 0, 4, 148) == 0
    assert lib.fb_workspace_page_scores(ctypes.byref(kv), 4, 4, 4, 0, 148) == 0
    assert lib.fb_workspace_page_scores(ctypes.byref(kv), 4, 3, 4, 4, 148) == 0  # Hq % Hkv
    bad = make_kv(head_dim=96)
    assert lib.fb_workspace_page_scores(ctypes.byref(bad), 4, 4, 4, 4, 148) == 0


def test_step_binding_rejects_too_few_update_counts():
    # the library reads m_updated[b] for every sequence b: a short host array is
    # refused before any pointer is taken
    import types
    kv = types.SimpleNamespace(batch=3, c=make_kv())
    q = torch.zeros(3, 4, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="3 sequences"):
        fb.fb_step(fb.fb_policy(), fb.fb_cache(), q, q, q, kv, q, m_updated=[1, 2])


# ------------------------------------------------------ packed-row entry points
def test_varlen_entry_points_reject_bad_row_arguments(lib):
    kv = make_kv()
    # cu_rows NULL, max_rows <= 0, total_rows < 0
    for cu, mx, tot in ((None, 4, 8), (DEV, 0, 8), (DEV, 4, -1)):
        rc = lib.fb_prefix_attn_varlen(DEV, cu, mx, tot, 4, 1.0, ctypes.byref(kv), DEV, DEV, DEV,
                                       1 << 30, None)
        assert rc == fb.FB_ERR_ARG, err(lib)
        rc = lib.fb_block_attn_varlen(DEV, DEV, DEV, cu, 1, mx, tot, 4, 2, 128, 1.0, fb.FB_BF16,
                                      DEV, DEV, None)
        assert rc == fb.FB_ERR_ARG, err(lib)
    # misaligned block keys
    rc = lib.fb_block_attn_varlen(DEV, MISALIGNED, DEV, DEV, 1, 4, 8, 4, 2, 128, 1.0, fb.FB_BF16,
                                  DEV, DEV, None)
    assert rc == fb.FB_ERR_ALIGN, err(lib)
    # a bad cache is still a bad cache
    rc = lib.fb_prefix_attn_varlen(DEV, DEV, 4, 8, 4, 1.0, ctypes.byref(make_kv(head_dim=96)), DEV,
                                   DEV, DEV, 1 << 30, None)
    assert rc == fb.FB_ERR_SHAPE


@pytest.mark.parametrize("mode", [fb.FB_PER_HEAD, fb.FB_LOSA, fb.FB_SPARSE_RESIDUAL])
def test_step_varlen_takes_the_threshold_controller_only(lib, mode):
    kv = make_kv()
    pol = fb.fb_policy(mode, 2, 0.9, 2, 4, 1.0)
    cache = fb.fb_cache()
    cache.a_out = cache.l_out = DEV
    rc = lib.fb_step_varlen(ctypes.byref(pol), ctypes.byref(cache), DEV, DEV, DEV, DEV, 4, 8, 4,
                            ctypes.byref(kv), None, DEV, DEV, DEV, 1 << 30, None)
    assert rc == fb.FB_ERR_ARG
    assert "threshold" in err(lib)
