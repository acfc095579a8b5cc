"""Pins of the oracle's small helpers that the larger pins use only indirectly.

bf16_bits_to_f32 (the bf16 storage read as float32): bf16 is the top half of
a float32, so known bit patterns have known values, and converting the top 16
bits of any float32 gives that float32 with its low 16 bits cleared.

token_slots (token order -> pool rows, FlashBlock technical summary §2: J_out
is the whole prefix of the sequence, read through the cache's layout): a
paged pool built by scattering known per-token rows through a permuted page
table must give the tokens back in their original order, and a contiguous
pool is the identity on each sequence's stretch.
"""

import numpy as np

from oracle.attention import token_slots
from oracle.losa import bf16_bits_to_f32
from workloads.gen import Prefix


def test_bf16_bits_known_values():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x7F80, 0xFF80, 0x4049, 0x0001, 0x7F7F],
                    dtype=np.uint16)
    got = bf16_bits_to_f32(bits)
    assert got[0] == 1.0 and got[1] == -2.0
    assert got[2] == 0.0 and not np.signbit(got[2])
    assert got[3] == 0.0 and np.signbit(got[3])
    assert np.isposinf(got[4]) and np.isneginf(got[5])
    assert got[6] == np.float32(3.140625)             # 0x4049: 1.5703125 * 2
    assert got[7] == np.float32(2.0) ** -133          # smallest subnormal bf16
    assert got[8] == np.float32((2 - 2 ** -7) * 2.0 ** 127)  # largest finite bf16
    assert np.isnan(bf16_bits_to_f32(np.array([0x7FC0], dtype=np.uint16))[0])


def test_bf16_bits_are_the_top_half_of_float32():
    x = np.random.default_rng(3).standard_normal(4096).astype(np.float32) * 1e3
    top = (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    want = (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    np.testing.assert_array_equal(bf16_bits_to_f32(top), want)


def _rows(n_tok, batch):
    """Per-token rows that name their token: [batch, n_tok, 1, 2] (b, t)."""
    r = np.zeros((batch, n_tok, 1, 2), dtype=np.float32)
    r[..., 0, 0] = np.arange(batch)[:, None]
    r[..., 0, 1] = np.arange(n_tok)[None, :]
    return r


def test_token_slots_paged_pool_recovers_token_order():
    P, batch, max_pages = 16, 3, 9
    lens = np.array([130, 0, 97], dtype=np.int32)
    rng = np.random.default_rng(7)
    perm = rng.permutation(batch * max_pages).astype(np.int32)
    table = perm.reshape(batch, max_pages)
    rows = _rows(max_pages * P, batch)
    pool = np.full((batch * max_pages * P, 1, 2), -1.0, dtype=np.float32)
    for b in range(batch):
        for t in range(int(lens[b])):
            pool[table[b, t // P] * P + t % P] = rows[b, t]
    kv = Prefix(pool, pool, lens, table, P, max_pages * P)
    for b in range(batch):
        s = token_slots(kv, b)
        assert s.shape == (int(lens[b]),)
        np.testing.assert_array_equal(pool[s, 0, 0], np.full(int(lens[b]), b))
        np.testing.assert_array_equal(pool[s, 0, 1], np.arange(int(lens[b])))
        assert len(np.unique(s)) == len(s)


def test_token_slots_contiguous_pool_is_each_sequences_stretch():
    batch, m = 4, 50
    lens = np.array([50, 1, 0, 23], dtype=np.int32)
    pool = np.zeros((batch * m, 1, 2), dtype=np.float32)
    kv = Prefix(pool, pool, lens, None, 16, m)
    for b in range(batch):
        np.testing.assert_array_equal(token_slots(kv, b), b * m + np.arange(int(lens[b])))
