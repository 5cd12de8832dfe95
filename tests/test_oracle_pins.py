"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one part of the oracle to something other than itself: a worked
example printed on a page (tests/golden), a closed form, an invariant, or a
library routine (numpy's fp16 decoding, torch's float64 scaled-dot-product
attention).  Together they fail on a dropped term, a wrong sign or index, a
swapped layout axis, a wrong GQA head mapping or a missing max subtraction.
"""
import math

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

from conftest import read_golden


def _place(dense_k, dense_v, table, N, bs, fill=np.float16(0.0)):
    """Pools [N][Hk][bs][D] holding dense rows [L][Hk][D] at the blocks of `table`
    (test-side setup, written with plain slicing)."""
    L, Hk, D = dense_k.shape
    kc = np.full((N, Hk, bs, D), fill, np.float16)
    vc = np.full((N, Hk, bs, D), fill, np.float16)
    for j in range(-(-L // bs)):
        rows = slice(j * bs, min((j + 1) * bs, L))
        n = rows.stop - rows.start
        kc[table[j], :, :n, :] = dense_k[rows].transpose(1, 0, 2)
        vc[table[j], :, :n, :] = dense_v[rows].transpose(1, 0, 2)
    return kc, vc


def _nan_fill():
    return np.array([0x7E5A], np.uint16).view(np.float16)[0]


# -- fp16 decoding -------------------------------------------------------------

def test_half_decoding_matches_numpy_for_every_bit_pattern(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32)
    ref = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([oracle_mod.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_half_decoding_known_values(oracle_mod):
    assert oracle_mod.half_to_double(0x3C00) == 1.0
    assert oracle_mod.half_to_double(0xC000) == -2.0
    assert oracle_mod.half_to_double(0x7BFF) == 65504.0
    assert oracle_mod.half_to_double(0x0001) == 2.0 ** -24
    assert oracle_mod.half_to_double(0x0400) == 2.0 ** -14
    assert oracle_mod.half_to_double(0x3555) == 0.333251953125


# -- gather through the block table --------------------------------------------

def test_gather_follows_the_block_table_figure(oracle_mod):
    g = dict((r[0], r[1:]) for r in read_golden("block_table_figure.txt"))
    bs = int(g["block_size"][0])
    L = int(g["seq_len"][0])
    table = [int(x) for x in g["table"]]
    N, Hk, D = 10, 2, 8
    # token i's row carries the marker i (+ 100*kv head) in every element
    dense_k = np.zeros((L, Hk, D), np.float16)
    for i in range(L):
        for h in range(Hk):
            dense_k[i, h, :] = i + 100 * h
    dense_v = -dense_k
    kc, vc = _place(dense_k, dense_v, table, N, bs, fill=_nan_fill())
    # the blocks the page marks free or owned by others are never read
    for blk in [int(x) for x in g["free"] + g["other"]]:
        assert np.isnan(kc[blk].astype(np.float64)).all()
    for kvh in range(Hk):
        k, v = oracle_mod.gather_kv(kc, vc, table, L, kvh, bs)
        assert np.array_equal(k[:, 0], np.arange(L) + 100.0 * kvh)
        assert np.array_equal(v[:, 0], -(np.arange(L) + 100.0 * kvh))
    # token i lives at row i % bs of physical block table[i // bs]: logical 0,1,2 -> 7,3,1
    assert [table[i // bs] for i in (0, 4, 8)] == [7, 3, 1]
    assert kc[7, 0, 0, 0] == 0 and kc[3, 0, 0, 0] == 4 and kc[1, 0, 3, 0] == 11


def test_gather_rejects_out_of_range_block(oracle_mod):
    kc = np.zeros((4, 1, 4, 8), np.float16)
    with pytest.raises(ValueError):
        oracle_mod.gather_kv(kc, kc, [0, 9], 6, 0, 4)
    with pytest.raises(ValueError):
        oracle_mod.gather_kv(kc, kc, [0, -1], 6, 0, 4)


# -- attention -----------------------------------------------------------------

def _random_case(seed, lens, H, Hk, D, bs, N):
    rng = np.random.default_rng(seed)
    B = len(lens)
    maxblk = max(-(-L // bs) for L in lens)
    perm = rng.permutation(N)
    tables = np.full((B, maxblk), -1, np.int32)
    denses = []
    kc = np.full((N, Hk, bs, D), _nan_fill(), np.float16)
    vc = kc.copy()
    pos = 0
    for b, L in enumerate(lens):
        nb = -(-L // bs)
        tables[b, :nb] = perm[pos:pos + nb]
        pos += nb
        dk = rng.standard_normal((L, Hk, D)).astype(np.float16)
        dv = rng.standard_normal((L, Hk, D)).astype(np.float16)
        denses.append((dk, dv))
        k1, v1 = _place(dk, dv, tables[b], N, bs, fill=_nan_fill())
        for j in range(nb):
            kc[tables[b, j]] = k1[tables[b, j]]
            vc[tables[b, j]] = v1[tables[b, j]]
    q = rng.standard_normal((B, H, D)).astype(np.float16)
    return q, kc, vc, tables, np.asarray(lens, np.int32), denses


@pytest.mark.parametrize("H,Hk", [(4, 4), (4, 2), (8, 1)])
def test_attention_equals_torch_sdpa_on_the_dense_sequence(oracle_mod, H, Hk):
    D, bs, N = 16, 4, 40
    lens = [1, 7, 13, 16]
    q, kc, vc, tables, cl, denses = _random_case(5, lens, H, Hk, D, bs, N)
    scale = 1.0 / math.sqrt(D)
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, scale, bs, Hk)
    for b, (dk, dv) in enumerate(denses):
        qt = torch.from_numpy(q[b].astype(np.float64)).view(1, H, 1, D)
        kt = torch.from_numpy(dk.astype(np.float64)).permute(1, 0, 2).unsqueeze(0)
        vt = torch.from_numpy(dv.astype(np.float64)).permute(1, 0, 2).unsqueeze(0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, scale=scale, enable_gqa=(H != Hk)).view(H, D).numpy()
        np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-13)


def test_context_of_one_returns_v_exactly(oracle_mod):
    q, kc, vc, tables, cl, denses = _random_case(6, [1, 1], 4, 4, 16, 8, 8)
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.25, 8, 4)
    for b in range(2):
        assert np.array_equal(out[b], denses[b][1][0].astype(np.float64))


def test_identical_keys_give_the_mean_of_v(oracle_mod):
    q, kc, vc, tables, cl, denses = _random_case(7, [9, 30], 2, 2, 8, 4, 16)
    kc[...] = np.float16(0.75)          # every key row identical
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.35, 4, 2)
    for b, (_, dv) in enumerate(denses):
        mean = dv.astype(np.float64).mean(axis=0)        # [Hk][D]
        np.testing.assert_allclose(out[b], mean, rtol=1e-13, atol=1e-14)


def test_zero_scale_gives_the_mean_of_v(oracle_mod):
    q, kc, vc, tables, cl, denses = _random_case(8, [5, 17], 2, 2, 8, 4, 16)
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.0, 4, 2)
    for b, (_, dv) in enumerate(denses):
        np.testing.assert_allclose(out[b], dv.astype(np.float64).mean(axis=0),
                                   rtol=1e-13, atol=1e-14)


def test_two_token_closed_form(oracle_mod):
    # q = e0, K0 = e0, K1 = 0, scale 1: weights e/(e+1) and 1/(e+1)
    D, bs = 4, 4
    kc = np.zeros((2, 1, bs, D), np.float16)
    vc = np.zeros((2, 1, bs, D), np.float16)
    kc[1, 0, 0, 0] = 1.0
    vc[1, 0, 0] = [1, 2, 3, 4]
    vc[1, 0, 1] = [-4, 0.5, 0, 8]
    q = np.zeros((1, 1, D), np.float16)
    q[0, 0, 0] = 1.0
    out = oracle_mod.paged_attention(q, kc, vc, [[1]], [2], 1.0, bs, 1)
    e = math.e
    ref = (e * np.array([1, 2, 3, 4.0]) + np.array([-4, 0.5, 0, 8.0])) / (e + 1)
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-15, atol=1e-15)


def test_scale_multiplies_the_scores(oracle_mod):
    # scores (2, 0) with scale 0.5 equal scores (1, 0) with scale 1
    D, bs = 4, 4
    kc = np.zeros((1, 1, bs, D), np.float16)
    vc = np.zeros((1, 1, bs, D), np.float16)
    kc[0, 0, 0, 0] = 2.0
    vc[0, 0, 0, 1] = 1.0
    q = np.zeros((1, 1, D), np.float16)
    q[0, 0, 0] = 1.0
    out = oracle_mod.paged_attention(q, kc, vc, [[0]], [2], 0.5, bs, 1)
    assert out[0, 0, 1] == pytest.approx(math.e / (math.e + 1), rel=1e-15)


def test_physical_placement_does_not_change_the_result(oracle_mod):
    H, Hk, D, bs, N = 4, 2, 16, 4, 64
    lens = [3, 11, 20, 33]
    q, kc, vc, tables, cl, _ = _random_case(9, lens, H, Hk, D, bs, N)
    base = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.25, bs, Hk)
    rng = np.random.default_rng(1)
    for _ in range(3):
        relabel = rng.permutation(N)        # physical id p moves to relabel[p]
        kc2 = np.empty_like(kc)
        vc2 = np.empty_like(vc)
        kc2[relabel] = kc
        vc2[relabel] = vc
        t2 = np.where(tables >= 0, relabel[np.maximum(tables, 0)], -1).astype(np.int32)
        out = oracle_mod.paged_attention(q, kc2, vc2, t2, cl, 0.25, bs, Hk)
        assert np.array_equal(out, base)


def test_gqa_groups_are_contiguous_query_heads(oracle_mod):
    # kv head j holds V == j + 1 everywhere: query head h must read kv head h // G
    H, Hk, D, bs, N = 8, 2, 8, 4, 8
    q, kc, vc, tables, cl, _ = _random_case(10, [6, 9], H, Hk, D, bs, N)
    for j in range(Hk):
        vc[:, j] = np.float16(j + 1)
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.3, bs, Hk)
    G = H // Hk
    for h in range(H):
        np.testing.assert_allclose(out[:, h], h // G + 1, rtol=1e-14)


def test_huge_scores_need_the_max_subtraction(oracle_mod):
    # scores near 2000 overflow exp() without max subtraction; the softmax is one-hot
    D, bs = 8, 4
    kc = np.zeros((2, 1, bs, D), np.float16)
    vc = np.zeros((2, 1, bs, D), np.float16)
    kc[0, 0, 1, :] = 16.0                  # token 1: score 8 * 16 * 16 = 2048
    kc[0, 0, 0, :] = 15.0                  # token 0: score 1920
    vc[0, 0, 0, :] = 3.0
    vc[0, 0, 1, :] = -5.0
    q = np.full((1, 1, D), 16.0, np.float16)
    out = oracle_mod.paged_attention(q, kc, vc, [[0]], [2], 1.0, bs, 1)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out[0, 0], -5.0, rtol=1e-15)


def test_shared_shift_of_all_keys(oracle_mod):
    # adding one vector c to every key adds scale * q.c to every score: softmax ignores it
    H, Hk, D, bs, N = 2, 2, 8, 4, 12
    q, kc, vc, tables, cl, _ = _random_case(11, [7, 10], H, Hk, D, bs, N)
    rng = np.random.default_rng(2)
    kc = (rng.integers(-16, 16, kc.shape) / 8).astype(np.float16)      # a grid where +c is exact
    c = (rng.integers(-4, 4, (Hk, 1, D)) / 8).astype(np.float16)
    kc2 = (kc.astype(np.float32) + c.astype(np.float32)).astype(np.float16)
    assert np.array_equal(kc2.astype(np.float32) - c.astype(np.float32), kc.astype(np.float32))
    base = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.4, bs, Hk)
    out = oracle_mod.paged_attention(q, kc2, vc, tables, cl, 0.4, bs, Hk)
    np.testing.assert_allclose(out, base, rtol=1e-11, atol=1e-12)


def test_linear_in_v(oracle_mod):
    H, Hk, D, bs, N = 2, 1, 8, 4, 12
    q, kc, vc, tables, cl, _ = _random_case(12, [5, 12], H, Hk, D, bs, N)
    rng = np.random.default_rng(3)
    v1 = rng.integers(-8, 8, vc.shape).astype(np.float16)
    v2 = rng.integers(-8, 8, vc.shape).astype(np.float16)
    o1 = oracle_mod.paged_attention(q, kc, v1, tables, cl, 0.3, bs, Hk)
    o2 = oracle_mod.paged_attention(q, kc, v2, tables, cl, 0.3, bs, Hk)
    o12 = oracle_mod.paged_attention(q, kc, (v1 + v2).astype(np.float16), tables, cl, 0.3, bs, Hk)
    np.testing.assert_allclose(o12, o1 + o2, rtol=1e-12, atol=1e-12)


def test_unwritten_slots_and_table_padding_are_never_read(oracle_mod):
    H, Hk, D, bs, N = 2, 2, 8, 4, 16
    q, kc, vc, tables, cl, denses = _random_case(13, [6, 9], H, Hk, D, bs, N)
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.3, bs, Hk)
    assert np.isfinite(out).all()           # NaN rows after each tail and in free blocks
    assert (tables[0, 2:] == -1).all()      # padding entries of the short sequence


def test_attention_rejects_bad_arguments(oracle_mod):
    kc = np.zeros((4, 1, 4, 8), np.float16)
    q = np.zeros((1, 1, 8), np.float16)
    with pytest.raises(ValueError):
        oracle_mod.paged_attention(q, kc, kc, [[0]], [0], 1.0, 4, 1)      # empty context
    with pytest.raises(ValueError):
        oracle_mod.paged_attention(q, kc, kc, [[0]], [5], 1.0, 4, 1)      # beyond the table
    with pytest.raises(ValueError):
        oracle_mod.paged_attention(q, kc, kc, [[7]], [2], 1.0, 4, 1)      # block out of range


def test_threaded_oracle_is_identical_to_serial(oracle_mod):
    q, kc, vc, tables, cl, _ = _random_case(14, [3, 17, 29, 8, 40], 4, 2, 16, 4, 64)
    a = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.25, 4, 2, nthreads=1)
    b = oracle_mod.paged_attention(q, kc, vc, tables, cl, 0.25, 4, 2, nthreads=3)
    assert np.array_equal(a, b)


# -- cache writes and copies ------------------------------------------------------

def test_reshape_and_cache_writes_the_slot_the_table_reads(oracle_mod):
    g = dict((r[0], r[1:]) for r in read_golden("block_table_figure.txt"))
    bs = int(g["block_size"][0])
    table = [int(x) for x in g["table"]] + [int(g["next_block"][0])]
    N, Hk, D = 10, 2, 8
    kc = np.full((N, Hk, bs, D), _nan_fill(), np.float16)
    vc = kc.copy()
    L = 13                                             # the 13th token lands in block 2, row 0
    dense_k = np.arange(L * Hk * D, dtype=np.float16).reshape(L, Hk, D) / np.float16(64)
    dense_v = -dense_k
    slots = [table[i // bs] * bs + i % bs for i in range(L)]
    assert slots[12] == 8
    kc2, vc2 = oracle_mod.reshape_and_cache(kc, vc, dense_k, dense_v, slots, bs)
    for kvh in range(Hk):
        k, v = oracle_mod.gather_kv(kc2, vc2, table, L, kvh, bs)
        assert np.array_equal(k, dense_k[:, kvh].astype(np.float64))
        assert np.array_equal(v, dense_v[:, kvh].astype(np.float64))
    # nothing else was touched: the NaN sentinel survives in every other slot
    written = np.zeros((N, bs), bool)
    for s in slots:
        written[s // bs, s % bs] = True
    untouched = kc2.view(np.uint16).transpose(0, 2, 1, 3)[~written]
    assert (untouched == 0x7E5A).all()


def test_reshape_and_cache_skips_padding_slots(oracle_mod):
    kc = np.zeros((4, 1, 4, 8), np.float16)
    k = np.ones((2, 1, 8), np.float16)
    kc2, vc2 = oracle_mod.reshape_and_cache(kc, kc, k, k, [-1, 5], 4)
    assert kc2[1, 0, 1].tolist() == [1.0] * 8
    kc2[1, 0, 1] = 0
    assert not kc2.any()


def test_copy_blocks_copies_whole_blocks_in_every_layer(oracle_mod):
    rng = np.random.default_rng(4)
    layers = [rng.standard_normal((6, 2, 4, 8)).astype(np.float16) for _ in range(3)]
    vals = [rng.standard_normal((6, 2, 4, 8)).astype(np.float16) for _ in range(3)]
    k2, v2 = oracle_mod.copy_blocks(layers, vals, [(1, 4), (2, 5)])
    for li in range(3):
        assert np.array_equal(k2[li][4], layers[li][1]) and np.array_equal(k2[li][5], layers[li][2])
        assert np.array_equal(v2[li][4], vals[li][1]) and np.array_equal(v2[li][5], vals[li][2])
        for blk in (0, 1, 2, 3):
            assert np.array_equal(k2[li][blk], layers[li][blk])


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2 ** 20), hk=st.sampled_from([1, 2, 3]), g=st.sampled_from([1, 2, 4]),
       d=st.sampled_from([8, 16, 24]), bs=st.sampled_from([1, 2, 4, 8]),
       lens=st.lists(st.integers(1, 40), min_size=1, max_size=4),
       scale=st.floats(0.0, 2.0))
def test_attention_equals_torch_sdpa_on_random_shapes(oracle_mod, seed, hk, g, d, bs, lens,
                                                      scale):
    # any head grouping, head size, block size, lengths, scale and physical placement
    H = hk * g
    N = sum(-(-L // bs) for L in lens) + 3
    q, kc, vc, tables, cl, denses = _random_case(seed, lens, H, hk, d, bs, N)
    out = oracle_mod.paged_attention(q, kc, vc, tables, cl, scale, bs, hk)
    for b, (dk, dv) in enumerate(denses):
        qt = torch.from_numpy(q[b].astype(np.float64)).view(1, H, 1, d)
        kt = torch.from_numpy(dk.astype(np.float64)).permute(1, 0, 2).unsqueeze(0)
        vt = torch.from_numpy(dv.astype(np.float64)).permute(1, 0, 2).unsqueeze(0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, scale=scale, enable_gqa=(H != hk)).view(H, d).numpy()
        np.testing.assert_allclose(out[b], ref, rtol=1e-11, atol=1e-12)
