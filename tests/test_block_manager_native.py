"""The C++ block manager (product) against the oracle's concept model: identical
tables, slots, reference counts, free lists and copy-on-write pairs, bit for bit."""
import threading

import numpy as np
import pytest

from conftest import read_golden

from paged_kv_cache_393_b200 import BlockManager, PagedKVError


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_393_b200 import build
    build.build()


def _same_state(native, model, ids):
    for s in ids:
        assert native.block_table(s) == model.block_table(s)
        assert native.seq_len(s) == model.lens[s]
    assert native.free_list() == model.free
    assert [native.refcount(b) for b in range(model.num_blocks)] == model.refcount
    assert native.stats() == model.stats()


def test_block_table_figure():
    g = dict((r[0], r[1:]) for r in read_golden("block_table_figure.txt"))
    bm = BlockManager(10, 4, free_order=[0, 9, 6, 4, 2, 1, 3, 7, 5, 8])
    other = bm.add_seq(8)
    seq = bm.add_seq(12)
    assert sorted(bm.block_table(other)) == [5, 8]
    assert bm.block_table(seq) == [int(x) for x in g["table"]]
    assert bm.append_token(seq) == 8            # token 13 -> physical block 2, row 0
    assert bm.block_table(seq)[3] == int(g["next_block"][0])


@pytest.mark.parametrize("row", read_golden("block_counts.txt"))
def test_block_counts(row):
    tokens, bs, blocks = map(int, row[:3])
    bm = BlockManager(300, bs)
    assert len(bm.block_table(bm.add_seq(tokens))) == blocks


def test_matches_the_model_on_random_operations(oracle_mod):
    rng = np.random.default_rng(7)
    N, bs = 96, 4
    order = rng.permutation(N)
    native = BlockManager(N, bs, free_order=order)
    model = oracle_mod.BlockManagerModel(N, bs, free_order=order)
    live = []
    for step in range(4000):
        op = int(rng.integers(0, 10))
        if op == 0 or not live:
            n = int(rng.integers(0, 14))
            a, b = native.add_seq(n), model.add_seq(n)
            assert a == b
            if a is not None:
                live.append(a)
        elif op == 1:
            s = live[int(rng.integers(len(live)))]
            k = int(rng.integers(1, 4))
            a, b = native.fork(s, k), model.fork(s, k)
            assert a == b
            live += a
        elif op == 2:
            s = live.pop(int(rng.integers(len(live))))
            native.free_seq(s)
            model.free_seq(s)
        elif op == 3:
            batch = [live[int(i)] for i in rng.integers(0, len(live), size=int(rng.integers(1, 6)))]
            slots = native.append_tokens(batch)
            ref = []
            for s in batch:
                r = model.append_token(s)
                if r is None:
                    break
                ref.append(r)
            assert slots.tolist() == ref
        else:
            s = live[int(rng.integers(len(live)))]
            assert native.append_token(s) == model.append_token(s)
        assert native.take_copies().tolist() == [list(p) for p in model.take_copies()]
        if step % 50 == 0:
            _same_state(native, model, live)
    _same_state(native, model, live)


def test_cow_workload_shape(oracle_mod):
    # 32 prompts of 1000 tokens, 8 samples each, first append: 7 copies per prompt
    order = np.random.default_rng(1).permutation(32768)
    native = BlockManager(32768, 16, free_order=order)
    model = oracle_mod.BlockManagerModel(32768, 16, free_order=order)
    samples = []
    for _ in range(32):
        p = native.add_seq(1000)
        assert model.add_seq(1000) == p
        kids = native.fork(p, 7)
        assert model.fork(p, 7) == kids
        samples += [p] + kids
    slots = native.append_tokens(samples)
    ref = [model.append_token(s) for s in samples]
    assert slots.tolist() == ref
    pairs = native.take_copies()
    assert pairs.tolist() == [list(p) for p in model.take_copies()]
    assert pairs.shape == (224, 2)
    tails = {native.block_table(s)[-1] for s in samples}
    assert len(tails) == 256                    # every sample now owns its tail block
    tables, lens = native.build_batch(samples, 80)
    assert (lens == 1001).all() and (tables[:, 63:] == -1).all()


def test_errors():
    bm = BlockManager(4, 4)
    s = bm.add_seq(16)
    assert bm.append_token(s) is None           # pool exhausted
    assert bm.add_seq(1) is None
    with pytest.raises(PagedKVError):
        bm.free_seq(99)
    with pytest.raises(PagedKVError):
        bm.append_token(99)
    with pytest.raises(PagedKVError):
        bm.refcount(4)
    with pytest.raises(PagedKVError):
        bm.build_batch([s], 3)                  # table of 4 does not fit
    with pytest.raises(PagedKVError):
        BlockManager(4, 4, free_order=[0, 1, 1, 2])


def test_concurrent_callers_keep_counts_consistent():
    # Several threads fork, append to and free sequences of one manager at once; the
    # manager locks every call, so reference counts must still equal table references.
    N, bs = 4096, 4
    bm = BlockManager(N, bs)
    roots = [bm.add_seq(6) for _ in range(8)]

    def worker(seed):
        rng = np.random.default_rng(seed)
        mine = []
        for _ in range(1500):
            op = rng.integers(0, 4)
            if op == 0 or not mine:
                mine += bm.fork(roots[int(rng.integers(len(roots)))], 1)
            elif op == 1 and len(mine) > 2:
                bm.free_seq(mine.pop(int(rng.integers(len(mine)))))
            else:
                bm.append_token(mine[int(rng.integers(len(mine)))])
        return mine

    results = [None] * 8
    threads = [threading.Thread(target=lambda i=i: results.__setitem__(i, worker(i))) for i in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    bm.take_copies()
    live = roots + [s for r in results for s in r]
    refs = np.zeros(N, int)
    for s in live:
        for b in bm.block_table(s):
            refs[b] += 1
    assert [bm.refcount(b) for b in range(N)] == refs.tolist()
    assert sorted(bm.free_list()) == [b for b in range(N) if refs[b] == 0]
    for s in live:
        bm.free_seq(s)
    assert bm.num_free() == N


def test_block_size_trade_off_on_the_llama7b_batch():
    # smaller blocks: less tail waste, longer tables, more allocations per append
    import bm_bench
    r = {bs: bm_bench.run(bs, steps=20) for bs in (8, 16, 32, 64)}
    waste = [r[bs]["tail_waste"] for bs in (8, 16, 32, 64)]
    entries = [r[bs]["table_entries"] for bs in (8, 16, 32, 64)]
    allocs = [r[bs]["blocks_allocated_per_1000_appends"] for bs in (8, 16, 32, 64)]
    assert waste == sorted(waste) and entries == sorted(entries, reverse=True)
    assert allocs == sorted(allocs, reverse=True)
    # a uniform tail wastes about (bs - 1) / 2 slots per sequence
    for bs in (8, 16, 32, 64):
        st = r[bs]["stats"]
        per_seq = (st["allocated_slots"] - st["filled_slots"]) / st["num_seqs"]
        assert abs(per_seq - (bs - 1) / 2) < 0.25 * bs


def test_queued_copy_blocks_stay_allocated_until_taken(oracle_mod):
    # the ordering that used to hand a queued copy's source out again: a write into a
    # shared tail queues (T -> F), the other sharer is released, and another
    # copy-on-write follows before the pairs are taken
    native = BlockManager(8, 4, free_order=list(range(8)))
    model = oracle_mod.BlockManagerModel(8, 4, free_order=list(range(8)))
    ids = []
    for bm in (native, model):
        a = bm.add_seq(2)
        (b,) = bm.fork(a, 1)
        u = bm.add_seq(3)
        (u2,) = bm.fork(u, 1)
        bm.append_token(a)
        bm.free_seq(b)
        bm.append_token(u)
        ids.append((a, u, u2))
    assert ids[0] == ids[1]
    t = native.block_table(ids[0][0])
    assert native.stats() == model.stats() and native.stats()["held_blocks"] == 1
    assert native.free_list() == model.free
    pairs = native.take_copies().tolist()
    assert pairs == [list(p) for p in model.take_copies()]
    assert len(pairs) == 2 and pairs[1][1] != pairs[0][0]
    assert native.free_list() == model.free and native.stats()["held_blocks"] == 0
    assert t == model.block_table(ids[1][0])


def test_seq_slots_match_the_model(oracle_mod):
    order = np.random.default_rng(2).permutation(64)
    native = BlockManager(64, 4, free_order=order)
    model = oracle_mod.BlockManagerModel(64, 4, free_order=order)
    s = native.add_seq(13)
    assert model.add_seq(13) == s
    for _ in range(6):
        native.append_token(s)
        model.append_token(s)
    assert native.seq_slots(s).tolist() == model.slots_of(s)
    assert native.seq_slots(s, 5, 7).tolist() == model.slots_of(s)[5:12]
    with pytest.raises(PagedKVError):
        native.seq_slots(s, 10, 10)               # beyond the sequence


def test_released_ids_are_reused_so_memory_stays_bounded():
    # 1e6 add / release cycles with at most 3 sequences alive: ids stay below 3, so the
    # manager's per-sequence storage stays at 3 entries
    lib = __import__("paged_kv_cache_393_b200._native", fromlist=["x"]).load_library()
    bm = BlockManager(16, 4)
    h = bm._h
    live = [bm.add_seq(5), bm.add_seq(1)]
    top = max(live)
    for i in range(1_000_000):
        s = lib.bm_add_seq(h, 3)
        assert s >= 0
        top = max(top, s)
        assert lib.bm_free_seq(h, s) == 0
    assert top == 2
    assert bm.stats()["num_seqs"] == 2 and bm.num_free() == 16 - 2 - 1
