"""The seeded input generators: byte accounting pins, ranges, determinism."""
import math

import numpy as np
import pytest

import workloads as wl
from conftest import read_golden


@pytest.mark.parametrize("row", read_golden("kv_bytes.txt"))
def test_kv_cache_bytes_match_the_pages(row):
    layers, heads, head_dim, seq_len, batch, dtype_bytes = map(int, row[:6])
    printed_gb = float(row[6])
    total = wl.kv_cache_bytes(layers, heads, head_dim, seq_len, batch, dtype_bytes)
    assert round(total / 1e9, 2) == printed_gb


def test_bytes_per_token_of_the_llama7b_layer():
    # 8.59e9 bytes over 32 layers x 2048 tokens x 8 sequences = 16384 bytes per token and layer
    assert wl.kv_bytes_per_token(32, 128) == 16384
    assert wl.kv_cache_bytes(32, 32, 128, 2048, 8, 2) == 32 * 2048 * 8 * 16384


def test_context_length_recipes():
    tiny = wl.context_lens(wl.get("tiny"))
    assert tiny.tolist() == [12, 50, 1]
    l7 = wl.context_lens(wl.get("llama7b"))
    assert l7.shape == (256,) and l7.min() >= 500 and l7.max() <= 1524
    assert abs(l7.mean() - 1012) < 40
    g = wl.context_lens(wl.get("gqa"))
    assert g.shape == (128,) and g.min() >= 64 and g.max() <= 16384
    assert 600 < np.median(g) < 1700
    cow = wl.context_lens(wl.get("cow"))
    assert (cow == 1001).all()
    for bs in wl.SWEEP_BLOCK_SIZES:
        w = wl.bs_sweep(bs)
        assert w.num_blocks * bs == wl.SWEEP_POOL_TOKENS
        assert np.array_equal(wl.context_lens(w), l7)


def test_pool_fits_every_workload():
    for name in ("tiny", "llama7b", "gqa", "llama7b_small", "gqa_small"):
        w = wl.get(name)
        need = sum(-(-int(L) // w.block_size) for L in wl.context_lens(w))
        assert need <= w.num_blocks, name
    for bs in wl.SWEEP_BLOCK_SIZES:
        w = wl.bs_sweep(bs)
        need = sum(-(-int(L) // bs) for L in wl.context_lens(w))
        assert need <= w.num_blocks
    for name in ("cow", "cow_small", "cow_compact"):
        # prompts written once; every sample then owns its copied tail block and the
        # blocks its 200 steps grow into
        w = wl.get(name)
        prefix = w.prompts * -(-w.prompt_len // w.block_size)
        grown = w.num_seqs * (-(-(w.prompt_len + w.decode_steps) // w.block_size)
                              - w.prompt_len // w.block_size)
        assert prefix + grown <= w.num_blocks, name


def test_generators_are_deterministic_and_length_independent():
    k1, v1 = wl.sequence_kv(1002, 5, 40, 2, 8)
    k2, v2 = wl.sequence_kv(1002, 5, 100, 2, 8)
    assert np.array_equal(k1, k2[:40]) and np.array_equal(v1, v2[:40])
    assert not np.array_equal(k1, v1)
    assert k1.dtype == np.float16
    a = wl.decode_q(1, 3, 4, 2, 8)
    b = wl.decode_q(1, 3, 4, 2, 8)
    assert np.array_equal(a, b) and not np.array_equal(a, wl.decode_q(1, 4, 4, 2, 8))
    order = wl.free_order(100, 7)
    assert sorted(order.tolist()) == list(range(100))
    many = wl.sequences_kv(1002, [5, 6], [40, 10], 2, 8)
    assert np.array_equal(many[0][0], k1)


def test_values_are_standard_normal():
    k, _ = wl.sequence_kv(3, 0, 2000, 4, 64)
    x = k.astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01


def test_sentinel_is_a_nan():
    p = wl.sentinel_pool(2, 1, 4, 8)
    assert np.isnan(p.astype(np.float32)).all()
    assert (p.view(np.uint16) == wl.SENTINEL_BITS).all()


def test_scale():
    assert wl.get("llama7b").scale == 1 / math.sqrt(128)
    assert wl.get("gqa").group == 8
