"""GPU parity of the fused append + attend call against the CPU oracle.

paged_attention_decode_append writes each sequence's new K/V row at position
L_b - 1 through its block table and attends over the updated cache in one
launch.  Expected results: the oracle's reshape_and_cache of the new rows at
the slots the block-manager model hands out (bit for bit, sentinels included),
then the oracle's attention (|gpu - oracle| <= 2e-3 + 1e-2 |oracle|).
"""
import numpy as np
import pytest
import torch

from test_gpu_parity import DEV, SMALL, _bits, _fixed, _run_and_compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from paged_kv_cache_393_b200 import build
    build.build()
    import paged_kv_cache_393_b200 as m
    m.device_errors(clear=True)
    yield m
    torch.cuda.empty_cache()


@pytest.mark.parametrize("w,part", SMALL, ids=[c[0].name for c in SMALL])
def test_small_cases_fused(pkv, w, part):
    _run_and_compare(pkv, w, partition_size=part, fused=True)


def test_query_groups_split_over_ctas_write_one_row(pkv):
    # 32 query heads on 1 kv head: several CTAs cover the kv head and all store its row
    _run_and_compare(pkv, _fixed("mqa32", 32, 1, 64, 16, [3, 16, 17, 200]), fused=True)
    _run_and_compare(pkv, _fixed("mqa32_split", 32, 1, 128, 16, [3, 16, 17, 200]),
                     partition_size=32, fused=True)


def _edge_batch(H=4, Hk=4):
    from batches import PagedBatch
    return PagedBatch(_fixed("edge_fused", H, Hk, 64, 16, [5, 40, 17]), DEV)


@pytest.mark.parametrize("H", [4, 8])  # CUDA-core and tensor-core kernels
def test_rejected_lengths_and_bad_blocks_write_nothing(pkv, H):
    gb = _edge_batch(H=H, Hk=4 if H == 4 else 2)
    tables = gb.block_tables.clone()
    tables[2, 1] = gb.w.num_blocks + 7          # sequence 2's new token lives in block 1
    lens = gb.context_lens.clone()
    lens[0] = 0                                 # no context
    lens[1] = 10_000                            # beyond max_context_len
    kc, vc = _bits(gb.key_cache), _bits(gb.value_cache)
    pkv.paged_attention_decode_append(gb.out, gb.q, gb.k_new, gb.v_new, gb.key_cache,
                                      gb.value_cache, tables, lens, 0.125, gb.max_context_len)
    flags = pkv.device_errors()
    assert flags & pkv.DEVERR_CONTEXT_LEN and flags & pkv.DEVERR_BLOCK_ID
    assert np.array_equal(kc, _bits(gb.key_cache)) and np.array_equal(vc, _bits(gb.value_cache))


def test_fused_arguments_are_checked(pkv):
    from paged_kv_cache_393_b200 import PagedKVError
    gb = _edge_batch()
    with pytest.raises(ValueError):
        pkv.paged_attention_decode_append(gb.out, gb.q, gb.k_new[:2], gb.v_new, gb.key_cache,
                                          gb.value_cache, gb.block_tables, gb.context_lens, 0.125,
                                          gb.max_context_len)
    lib = pkv.load_library()
    st = lib.paged_attention_decode_append(
        gb.out.data_ptr(), gb.q.data_ptr(), None, gb.v_new.data_ptr(), gb.key_cache.data_ptr(),
        gb.value_cache.data_ptr(), gb.block_tables.data_ptr(), gb.context_lens.data_ptr(), 0.125,
        16, 4, 3, 4, 64, gb.block_tables.shape[1], gb.w.num_blocks, gb.max_context_len, 0, None, 0,
        None)
    assert st == -1                              # PAGEDKV_EINVAL, nothing enqueued
    with pytest.raises(PagedKVError):
        pkv.paged_attention_decode_append(gb.out, gb.q, gb.k_new, gb.v_new, gb.key_cache,
                                          gb.value_cache, gb.block_tables, gb.context_lens, 0.125,
                                          gb.max_context_len, partition_size=24)  # not a multiple of 16


