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

import oracle
import workloads as wl
from oracle_side import assert_attention_close
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


def test_llama7b_full_size_fused(pkv):
    w = wl.get("llama7b")
    lens = wl.context_lens(w)
    _run_and_compare(pkv, w, sample=sorted({0, int(np.argmax(lens)), int(np.argmin(lens)), 255}),
                     fused=True)


def test_gqa_full_size_fused(pkv):
    w = wl.get("gqa")
    lens = wl.context_lens(w)
    _run_and_compare(pkv, w, partition_size=w.partition_size,
                     sample=sorted({0, int(np.argmax(lens)), int(np.argmin(lens)), 127}), fused=True)


@pytest.mark.parametrize("bs", [8, 64])
def test_block_size_sweep_fused(pkv, bs):
    _run_and_compare(pkv, wl.bs_sweep(bs), sample=[0, 255], fused=True)


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


def test_cow_workload_fused(pkv):
    # copy-on-write step then the fused call, for all decode steps; afterwards the cache
    # rows of chosen samples and their attention match the oracle
    from batches import CowBatch
    from oracle_side import compact_pools
    w = wl.get("cow")
    Hk, D, bs, N = w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks
    gb = CowBatch(w, DEV)
    model = oracle.BlockManagerModel(N, bs, free_order=wl.free_order(N, w.seed))
    samples, prompt_of = [], {}
    for p in range(w.prompts):
        s = model.add_seq(w.prompt_len)
        for x in [s] + model.fork(s, w.samples - 1):
            samples.append(x)
            prompt_of[x] = p
    assert samples == gb.samples
    news = []
    for step in range(w.decode_steps):
        host = gb.prepare_step()
        assert host["slots"].tolist() == [model.append_token(s) for s in samples]
        assert host["pairs"].tolist() == [list(x) for x in model.take_copies()]
        dev = {k: torch.from_numpy(host[k]).to(DEV) for k in ("tables", "lens", "q", "k", "v")}
        if len(host["pairs"]):
            pkv.copy_blocks([gb.key_cache], [gb.value_cache],
                            torch.from_numpy(host["pairs"]).to(DEV))
        out = torch.empty_like(dev["q"])
        pkv.paged_attention_decode_append(out, dev["q"], dev["k"], dev["v"], gb.key_cache,
                                          gb.value_cache, dev["tables"], dev["lens"], w.scale,
                                          gb.max_context_len)
        news.append((host["k"], host["v"]))
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    chosen = [0, 7, 8, 100, 255]
    entries = []
    for i in chosen:
        s = samples[i]
        k0, v0 = wl.sequence_kv(w.seed, prompt_of[s], w.prompt_len, Hk, D)
        entries.append((model.block_table(s), np.concatenate([k0, np.stack([k[i] for k, _ in news])]),
                        np.concatenate([v0, np.stack([v[i] for _, v in news])])))
    kc_o, vc_o, t_o, l_o, relabel = compact_pools(entries, bs, Hk, D)
    # every block these samples use holds exactly the oracle's bytes
    idx = torch.tensor(list(relabel), dtype=torch.long, device=DEV)
    assert np.array_equal(_bits(gb.key_cache[idx]), kc_o.view(np.uint16))
    assert np.array_equal(_bits(gb.value_cache[idx]), vc_o.view(np.uint16))
    ref = oracle.paged_attention(host["q"][chosen], kc_o, vc_o, t_o, l_o, w.scale, bs, Hk,
                                 nthreads=8)
    assert_attention_close(out.cpu().numpy()[chosen], ref)
