"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Cache writes and block copies must match bit for bit (compared as raw fp16 bit
patterns, NaN sentinels included); attention outputs must satisfy
|gpu - oracle| <= 2e-3 + 1e-2 |oracle| element by element.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle_side import OracleBatch, assert_attention_close, compact_pools

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


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


def _fixed(name, H, Hk, D, bs, lens, seed=2000, slack=16):
    N = sum(-(-L // bs) for L in lens) + slack
    return wl.Workload(name, len(lens), H, Hk, D, bs, N, seed, "fixed", fixed_lens=tuple(lens))


def _bits(t):
    return t.detach().cpu().numpy().view(np.uint16)


def _run_and_compare(pkv, w, partition_size=0, sample=None, check_pool=True, fused=False):
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    ob = OracleBatch(w, sample)
    # the product block manager and the oracle's model agree exactly
    assert [gb.bm.block_table(s) for s in gb.seqs] == ob.tables
    assert np.array_equal(gb.slots_host, ob.new_slots)
    if fused:
        # one call writes the new token at position L-1 through the table, then attends
        pkv.paged_attention_decode_append(gb.out, gb.q, gb.k_new, gb.v_new, gb.key_cache,
                                          gb.value_cache, gb.block_tables, gb.context_lens,
                                          w.scale, gb.max_context_len, partition_size)
    else:
        # one decode step: scatter the new token, then attend
        pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len, partition_size)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    if fused:
        # the same kernels over the same (now updated) cache give the same outputs bit for
        # bit: every kernel fixes which warp sums which chunk, whatever the work order
        fused_out = gb.out.clone()
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len, partition_size)
        assert np.array_equal(_bits(fused_out), _bits(gb.out))
    if check_pool:
        idx = torch.tensor(ob.blocks, dtype=torch.long, device=DEV)
        assert np.array_equal(_bits(gb.key_cache[idx]), ob.key_cache.view(np.uint16))
        assert np.array_equal(_bits(gb.value_cache[idx]), ob.value_cache.view(np.uint16))
        if sample is None:
            # the whole pool: every block outside the tables still holds the sentinel
            used = {b for t in ob.tables for b in t}
            free = torch.tensor([b for b in range(w.num_blocks) if b not in used],
                                dtype=torch.long, device=DEV)
            if len(free):
                for pool in (gb.key_cache, gb.value_cache):
                    assert (_bits(pool[free]) == wl.SENTINEL_BITS).all()
    got = gb.out.cpu().numpy().astype(np.float64)[ob.sample]
    err = assert_attention_close(got, ob.attention())
    del gb
    torch.cuda.empty_cache()
    return err


# ---- small cases: every kernel variant, ragged tails, several tiles ----------------

SMALL = [
    # (workload, partition_size)
    (wl.get("tiny"), 0),                                                    # 4=4 heads, D64, bs4
    (_fixed("mha128_bs16", 8, 8, 128, 16, [1, 15, 16, 17, 100, 257, 700]), 0),
    (_fixed("mha128_bs16_split", 8, 8, 128, 16, [1, 15, 16, 17, 100, 257, 700]), 32),
    (_fixed("mha64_bs8", 4, 4, 64, 8, [3, 8, 9, 64, 65, 333]), 0),
    (_fixed("mha64_bs32_split", 4, 4, 64, 32, [5, 31, 32, 33, 600]), 64),
    (_fixed("mha128_bs64", 4, 4, 128, 64, [1, 63, 64, 65, 500]), 0),
    (_fixed("mha128_bs4", 6, 6, 128, 4, [2, 4, 5, 77]), 0),
    (_fixed("gqa8_d128_bs16", 16, 2, 128, 16, [1, 16, 17, 300, 1030]), 0),
    (_fixed("gqa8_d128_bs16_split", 16, 2, 128, 16, [1, 16, 17, 300, 1030]), 64),
    (_fixed("gqa4_d64_bs8", 8, 2, 64, 8, [3, 8, 9, 33, 200]), 0),
    (_fixed("gqa4_d64_bs8_split", 8, 2, 64, 8, [3, 8, 9, 33, 200]), 16),
    (_fixed("gqa2_d128_bs32", 4, 2, 128, 32, [1, 31, 32, 33, 410]), 0),
    (_fixed("gqa2_d128_bs64_split", 4, 2, 128, 64, [1, 63, 64, 65, 410]), 128),
    (_fixed("gqa3_d64_bs16", 6, 2, 64, 16, [7, 40, 129]), 0),
    (_fixed("gqa4_d64_bs32", 8, 2, 64, 32, [1, 31, 32, 33, 500]), 0),
    (_fixed("gqa8_d64_bs64_split", 16, 2, 64, 64, [1, 63, 64, 65, 700]), 128),
    (_fixed("gqa8_bs4_cuda_cores", 16, 2, 64, 4, [1, 4, 5, 90]), 0),
    (_fixed("gqa16_cuda_cores", 32, 2, 64, 16, [2, 17, 250]), 0),
    (_fixed("gqa16_cuda_cores_split", 32, 2, 64, 16, [2, 17, 250]), 32),
    # CUDA-core CTAs of 2 and 4 query heads over one kv head (G = 2 at bs 4; G = 10, 12)
    (_fixed("gqa2_bs4_cuda_cores", 4, 2, 128, 4, [1, 4, 5, 63]), 0),
    (_fixed("gqa10_cuda_cores_split", 20, 2, 128, 16, [3, 16, 17, 300]), 64),
    (_fixed("gqa12_cuda_cores", 24, 2, 64, 16, [2, 33, 190]), 0),
    # long single passes: every stage of the ring is refilled many times
    (_fixed("gqa8_d128_bs64_long", 16, 2, 128, 64, [700, 1500]), -1),
    (_fixed("gqa4_d128_bs32_long", 8, 2, 128, 32, [999, 1800]), -1),
    (_fixed("gqa8_d64_bs8_long", 16, 2, 64, 8, [1500, 33]), -1),
    (_fixed("mha128_bs64_long", 4, 4, 128, 64, [1000, 1777]), -1),
    (_fixed("mha64_bs32_long", 8, 8, 64, 32, [1300, 7]), -1),
    # many small partitions into one merge
    (_fixed("gqa8_d128_250_parts", 16, 2, 128, 16, [4000, 33]), 16),
    # more sequences than the persistent tensor-core grid takes: one CTA per item
    (_fixed("gqa8_1030_seqs_split", 16, 2, 64, 16, [1 + (7 * i) % 97 for i in range(1030)]), 32),
]


@pytest.mark.parametrize("w,part", SMALL, ids=[c[0].name for c in SMALL])
def test_small_cases(pkv, w, part):
    _run_and_compare(pkv, w, partition_size=part)


def test_single_pass_and_split_agree(pkv):
    w = _fixed("agree", 8, 2, 128, 16, [100, 1000, 2049])
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    outs = []
    for part in (-1, 512, 64):
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len, part)
        outs.append(gb.out.float().cpu().numpy())
    assert np.isfinite(outs[0]).all()
    assert np.abs(outs[0] - outs[1]).max() < 2e-3 and np.abs(outs[0] - outs[2]).max() < 2e-3


def test_deterministic(pkv):
    w = _fixed("det", 8, 8, 128, 16, [33, 400])
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    res = []
    for _ in range(3):
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len)
        res.append(_bits(gb.out))
    assert np.isfinite(gb.out.float().cpu().numpy()).all()
    assert np.array_equal(res[0], res[1]) and np.array_equal(res[0], res[2])


@pytest.mark.parametrize("part", [512, 0, -1])
def test_gqa_full_size_is_reproducible(pkv, part):
    # the persistent tensor-core kernel hands out work items at run time; chunk j of an item
    # always goes to consumer warp j mod 2, so three runs agree bit for bit
    from batches import PagedBatch
    w = wl.get("gqa")
    gb = PagedBatch(w, DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    res = []
    for _ in range(3):
        gb.out.fill_(float("nan"))
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len, part)
        res.append(_bits(gb.out))
    assert pkv.device_errors() == 0
    assert np.isfinite(gb.out.float().cpu().numpy()).all()
    assert np.array_equal(res[0], res[1]) and np.array_equal(res[0], res[2])
    del gb
    torch.cuda.empty_cache()


@pytest.mark.parametrize("part", [64, -1])
def test_work_counters_are_left_zero_and_a_dirty_start_is_flagged(pkv, part):
    # grouped queries take their work from counters at the start of the workspace: every
    # launch leaves them zero (no reset between launches); a workspace whose counters do
    # not start at zero is flagged, and the launch still leaves them zero
    from batches import PagedBatch
    w = _fixed("counters", 16, 2, 128, 16, [1, 300, 1030, 77])
    gb = PagedBatch(w, DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    need = pkv.paged_attention_workspace_bytes(4, 16, 2, 128, 16, gb.max_context_len, part)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)

    def run():
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len, part, ws)
        torch.cuda.synchronize()

    run()
    assert pkv.device_errors() == 0 and (ws[:32] == 0).all()
    ref = _bits(gb.out)
    run()
    assert pkv.device_errors() == 0 and np.array_equal(ref, _bits(gb.out))
    ws[0] = 5                                      # a ticket count left by someone else
    run()
    assert pkv.device_errors() & pkv.DEVERR_INTERNAL
    assert (ws[:32] == 0).all()
    run()
    assert pkv.device_errors() == 0 and np.array_equal(ref, _bits(gb.out))


def test_block_table_figure_on_the_gpu(pkv):
    # the pages' example: 12 tokens at block_size 4 in physical blocks 7, 3, 1
    D, bs, N = 64, 4, 10
    rng = np.random.default_rng(5)
    k = rng.standard_normal((12, 1, D)).astype(np.float16)
    v = rng.standard_normal((12, 1, D)).astype(np.float16)
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    table = [7, 3, 1]
    slots = np.array([table[i // bs] * bs + i % bs for i in range(12)], np.int64)
    kc_h, vc_h = oracle.reshape_and_cache(wl.sentinel_pool(N, 1, bs, D), wl.sentinel_pool(N, 1, bs, D),
                                          k, v, slots, bs)
    ref = oracle.paged_attention(q, kc_h, vc_h, [table], [12], 0.125, bs, 1)
    from batches import sentinel_pools
    kc, vc = sentinel_pools(N, 1, bs, D, DEV)
    pkv.reshape_and_cache(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), kc, vc,
                          torch.from_numpy(slots).to(DEV))
    out = torch.empty((1, 1, D), dtype=torch.float16, device=DEV)
    pkv.paged_attention_decode(out, torch.from_numpy(q).to(DEV), kc, vc,
                               torch.tensor([table], dtype=torch.int32, device=DEV),
                               torch.tensor([12], dtype=torch.int32, device=DEV), 0.125, 12)
    assert np.array_equal(_bits(kc), kc_h.view(np.uint16))
    assert_attention_close(out.cpu().numpy(), ref)


def test_context_of_one_is_exactly_v(pkv):
    w = _fixed("len1", 8, 2, 128, 16, [1, 1, 1])
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                               gb.context_lens, w.scale, 1)
    out = _bits(gb.out)
    vnew = gb.v_new_host.view(np.uint16)
    for h in range(8):
        assert np.array_equal(out[:, h], vnew[:, h // 4])


# (the full-size workloads, whole batches: test_gpu_full_size.py)

# ---- edge cases and device-side checks ----------------------------------------------

def _tiny_batch():
    from batches import PagedBatch
    import paged_kv_cache_393_b200 as m
    gb = PagedBatch(_fixed("edge", 4, 4, 64, 16, [5, 40, 17]), DEV)
    m.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    return gb


def test_empty_batch_is_a_no_op(pkv):
    gb = _tiny_batch()
    before = _bits(gb.out)
    pkv.paged_attention_decode(gb.out[:0], gb.q[:0], gb.key_cache, gb.value_cache,
                               gb.block_tables[:0], gb.context_lens[:0], 0.125, 40)
    pkv.reshape_and_cache(gb.k_new[:0], gb.v_new[:0], gb.key_cache, gb.value_cache, gb.slots[:0])
    torch.cuda.synchronize()
    assert np.array_equal(before, _bits(gb.out))
    assert pkv.device_errors() == 0


def test_zero_context_length_gives_zeros_and_a_flag(pkv):
    gb = _tiny_batch()
    for part in (-1, 16):
        lens = gb.context_lens.clone()
        lens[1] = 0
        gb.out.fill_(1.0)
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   lens, 0.125, gb.max_context_len, part)
        flags = pkv.device_errors()
        assert flags & pkv.DEVERR_CONTEXT_LEN
        assert (gb.out[1] == 0).all()
        assert torch.isfinite(gb.out).all()


def test_bad_block_id_is_flagged_not_faulted(pkv):
    gb = _tiny_batch()
    tables = gb.block_tables.clone()
    tables[1, 1] = gb.w.num_blocks + 5
    tables[2, 0] = -3
    pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, tables,
                               gb.context_lens, 0.125, gb.max_context_len)
    assert pkv.device_errors() & pkv.DEVERR_BLOCK_ID
    # the mma kernel's producer checks the same way
    from batches import PagedBatch
    g2 = PagedBatch(_fixed("edge_gqa", 8, 2, 64, 16, [20, 40]), DEV)
    t2 = g2.block_tables.clone()
    t2[0, 1] = 1 << 30
    pkv.paged_attention_decode(g2.out, g2.q, g2.key_cache, g2.value_cache, t2, g2.context_lens,
                               0.125, g2.max_context_len)
    assert pkv.device_errors() & pkv.DEVERR_BLOCK_ID


def test_context_beyond_max_is_clamped_and_flagged(pkv):
    gb = _tiny_batch()
    lens = gb.context_lens.clone()
    lens[0] = 10_000
    pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                               lens, 0.125, gb.max_context_len)
    assert pkv.device_errors() & pkv.DEVERR_CONTEXT_LEN


def test_bad_slot_is_flagged_and_skipped(pkv):
    gb = _tiny_batch()
    before = _bits(gb.key_cache)
    slots = torch.tensor([-1, gb.w.num_blocks * 16 + 3, -1], dtype=torch.int64, device=DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, slots)
    assert pkv.device_errors() & pkv.DEVERR_SLOT
    assert np.array_equal(before, _bits(gb.key_cache))


def test_copy_blocks_multi_layer_and_bad_ids(pkv):
    rng = np.random.default_rng(3)
    N, Hk, bs, D = 12, 2, 16, 64
    layers_k = [rng.standard_normal((N, Hk, bs, D)).astype(np.float16) for _ in range(3)]
    layers_v = [rng.standard_normal((N, Hk, bs, D)).astype(np.float16) for _ in range(3)]
    pairs = [(1, 7), (2, 9), (4, 0)]
    ek, ev = oracle.copy_blocks(layers_k, layers_v, pairs)
    dk = [torch.from_numpy(x).to(DEV) for x in layers_k]
    dv = [torch.from_numpy(x).to(DEV) for x in layers_v]
    pkv.copy_blocks(dk, dv, torch.tensor(pairs, dtype=torch.int64, device=DEV))
    torch.cuda.synchronize()
    for i in range(3):
        assert np.array_equal(_bits(dk[i]), ek[i].view(np.uint16))
        assert np.array_equal(_bits(dv[i]), ev[i].view(np.uint16))
    assert pkv.device_errors() == 0
    before = _bits(dk[0])
    pkv.copy_blocks(dk, dv, torch.tensor([(3, N), (-1, 2)], dtype=torch.int64, device=DEV))
    assert pkv.device_errors() & pkv.DEVERR_BLOCK_ID
    assert np.array_equal(before, _bits(dk[0]))


def test_max_context_at_the_table_limit(pkv):
    # the longest context the table allows, split and unsplit
    w = _fixed("maxctx", 2, 2, 128, 16, [4096], slack=0)
    for part in (-1, 512):
        _run_and_compare(pkv, w, partition_size=part)
