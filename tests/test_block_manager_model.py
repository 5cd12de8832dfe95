"""Pins of the oracle's block-manager concept model against the pages' examples and rules."""
import numpy as np
import pytest

from conftest import read_golden


def _model(oracle_mod, *a, **k):
    return oracle_mod.BlockManagerModel(*a, **k)


def test_block_table_figure(oracle_mod):
    g = dict((r[0], r[1:]) for r in read_golden("block_table_figure.txt"))
    bs = int(g["block_size"][0])
    # free list popped from its end: another request takes 8 and 5, then our 12 tokens
    # take 7, 3, 1; the next block handed out is 2 (block 0 is outside the figure)
    m = _model(oracle_mod, 10, bs, free_order=[0, 9, 6, 4, 2, 1, 3, 7, 5, 8])
    other = m.add_seq(8)
    seq = m.add_seq(int(g["seq_len"][0]))
    assert sorted(m.block_table(other)) == sorted(int(x) for x in g["other"])
    assert m.block_table(seq) == [int(x) for x in g["table"]]
    assert set(int(x) for x in g["free"]) <= set(m.free)
    slot = m.append_token(seq)                       # token 13: logical block 3 is mapped now
    assert m.block_table(seq)[3] == int(g["next_block"][0])
    assert slot == int(g["next_block"][0]) * bs
    assert m.take_copies() == []


@pytest.mark.parametrize("row", read_golden("block_counts.txt"))
def test_block_counts_and_tail_waste(oracle_mod, row):
    tokens, bs, blocks, tail, capacity, wasted = map(int, row)
    m = _model(oracle_mod, 300, bs)
    s = m.add_seq(tokens)
    assert len(m.block_table(s)) == blocks
    assert tokens - (blocks - 1) * bs == tail
    assert blocks * bs == capacity and capacity - tokens == wasted
    st = m.stats()
    assert st["allocated_slots"] == capacity and st["filled_slots"] == tokens
    assert st["allocated_slots"] - st["filled_slots"] == wasted


def test_stats_count_shared_blocks_once(oracle_mod):
    m = _model(oracle_mod, 64, 16)
    p = m.add_seq(1000)                        # 62 full blocks and a tail of 8
    m.fork(p, 7)
    st = m.stats()
    assert st["used_blocks"] == 63 and st["allocated_slots"] == 63 * 16
    assert st["filled_slots"] == 1000          # one copy of the shared prefix
    assert st["logical_tokens"] == 8 * 1000 and st["table_entries"] == 8 * 63
    assert st["num_seqs"] == 8 and st["free_blocks"] == 1


def test_block_counts_grow_on_demand(oracle_mod):
    # appending one token at a time allocates exactly when the last block is full
    m = _model(oracle_mod, 8, 16)
    s = m.add_seq(0)
    assert m.block_table(s) == []
    counts = []
    for _ in range(50):
        m.append_token(s)
        counts.append(len(m.block_table(s)))
    assert counts[0] == 1 and counts[15] == 1 and counts[16] == 2 and counts[49] == 4
    assert m.num_free() == 4


def test_slots_are_block_and_offset(oracle_mod):
    m = _model(oracle_mod, 6, 4, free_order=[5, 4, 3, 2, 1, 0])
    s = m.add_seq(0)
    slots = [m.append_token(s) for _ in range(6)]
    # pops 0 then 1: tokens 0-3 in block 0, tokens 4-5 in block 1
    assert slots == [0, 1, 2, 3, 4, 5]
    m2 = _model(oracle_mod, 6, 4, free_order=[0, 1, 2, 3, 4, 5])
    s2 = m2.add_seq(0)
    assert [m2.append_token(s2) for _ in range(5)] == [20, 21, 22, 23, 16]
    assert m2.slots_of(s2) == [20, 21, 22, 23, 16]


def test_exhausted_pool_fails_and_leaves_state_unchanged(oracle_mod):
    m = _model(oracle_mod, 2, 4)
    s = m.add_seq(8)                              # both blocks
    before = (m.block_table(s), m.lens[s], list(m.free), list(m.refcount))
    assert m.append_token(s) is None
    assert (m.block_table(s), m.lens[s], list(m.free), list(m.refcount)) == before
    assert m.add_seq(1) is None
    assert m.add_seq(0) is not None               # no block needed


def test_refcount_lifecycle(oracle_mod):
    m = _model(oracle_mod, 8, 4)
    a = m.add_seq(6)
    blocks = m.block_table(a)
    assert [m.refcount[b] for b in blocks] == [1, 1]
    kids = m.fork(a, 2)
    assert [m.refcount[b] for b in blocks] == [3, 3]
    assert all(m.block_table(k) == blocks for k in kids)
    m.free_seq(a)
    assert [m.refcount[b] for b in blocks] == [2, 2] and not set(blocks) & set(m.free)
    m.free_seq(kids[0])
    m.free_seq(kids[1])
    assert [m.refcount[b] for b in blocks] == [0, 0] and set(blocks) <= set(m.free)
    assert m.num_free() == 8


def test_copy_on_write_of_a_shared_partial_block(oracle_mod):
    # cow workload shape: 1000 tokens at block_size 16, 8 samples share the prefix
    m = _model(oracle_mod, 200, 16)
    p = m.add_seq(1000)
    table = m.block_table(p)
    tail = table[-1]
    assert 1000 % 16 == 8 and len(table) == 63
    kids = m.fork(p, 7)
    assert m.refcount[tail] == 8
    samples = [p] + kids
    for i, s in enumerate(samples):
        slot = m.append_token(s)
        copies = m.take_copies()
        if i < 7:                                  # refcount > 1: copy first
            assert len(copies) == 1 and copies[0][0] == tail
            new = copies[0][1]
            assert m.block_table(s)[-1] == new and m.refcount[new] == 1
            assert m.refcount[tail] == 8 - (i + 1)
            assert slot == new * 16 + 8
        else:                                      # the last sharer writes in place
            assert copies == [] and m.block_table(s)[-1] == tail and slot == tail * 16 + 8
    # the prefix blocks stay shared by all eight samples
    assert all(m.refcount[b] == 8 for b in table[:-1])


def test_shared_full_block_needs_no_copy(oracle_mod):
    m = _model(oracle_mod, 16, 4)
    p = m.add_seq(8)                               # two full blocks
    kids = m.fork(p, 3)
    for s in [p] + kids:
        m.append_token(s)
    assert m.take_copies() == []
    last = [m.block_table(s)[-1] for s in [p] + kids]
    assert len(set(last)) == 4                     # each got a fresh block of its own
    assert all(m.refcount[b] == 1 for b in last)
    assert all(m.refcount[b] == 4 for b in m.block_table(p)[:2])


def test_failed_copy_on_write_leaves_state_unchanged(oracle_mod):
    m = _model(oracle_mod, 2, 4)
    p = m.add_seq(2)
    (k,) = m.fork(p, 1)
    m.add_seq(1)                                   # takes the last free block
    before = (m.block_table(p), m.block_table(k), list(m.refcount), list(m.free))
    assert m.append_token(k) is None
    assert m.take_copies() == []
    assert (m.block_table(p), m.block_table(k), list(m.refcount), list(m.free)) == before


def test_random_operations_keep_the_invariants(oracle_mod):
    rng = np.random.default_rng(0)
    N, bs = 64, 4
    m = _model(oracle_mod, N, bs, free_order=rng.permutation(N))
    live = []
    for _ in range(3000):
        op = rng.integers(0, 10)
        if op == 0 or not live:
            s = m.add_seq(int(rng.integers(0, 12)))
            if s is not None:
                live.append(s)
        elif op == 1:
            live += m.fork(live[rng.integers(len(live))], int(rng.integers(1, 3)))
        elif op == 2:
            m.free_seq(live.pop(rng.integers(len(live))))
        else:
            m.append_token(live[rng.integers(len(live))])
        m.take_copies()
        refs = np.zeros(N, int)
        for s in live:
            assert len(m.block_table(s)) == -(-m.lens[s] // bs)
            for b in m.block_table(s):
                refs[b] += 1
        assert list(refs) == list(m.refcount)
        assert sorted(m.free) == [b for b in range(N) if refs[b] == 0]
    for s in live:
        m.free_seq(s)
    assert m.num_free() == N and not any(m.refcount)


def test_appended_slot_is_the_table_position_of_the_last_token(oracle_mod):
    # the fused append writes token L-1 at row (L-1) % bs of block table[(L-1) // bs]; that
    # must be the slot append_token hands out, through growth, forks and copy-on-write
    rng = np.random.default_rng(5)
    N, bs = 128, 4
    m = _model(oracle_mod, N, bs, free_order=rng.permutation(N))
    live = [m.add_seq(int(rng.integers(0, 9))) for _ in range(4)]
    for _ in range(2000):
        op = rng.integers(0, 6)
        if op == 0 and len(live) < 30:
            live += m.fork(live[rng.integers(len(live))], 1)
        elif op == 1 and len(live) > 2:
            m.free_seq(live.pop(rng.integers(len(live))))
        else:
            s = live[rng.integers(len(live))]
            slot = m.append_token(s)
            if slot is None:
                continue
            L = m.lens[s]
            table = m.block_table(s)
            assert slot == table[(L - 1) // bs] * bs + (L - 1) % bs
        m.take_copies()


def _disjoint(pairs):
    """No destination repeats and no destination is also a source: copy_blocks may then
    apply the pairs in any order, or all at once, with the same result."""
    dsts = [d for _, d in pairs]
    return len(set(dsts)) == len(dsts) and not set(dsts) & {s for s, _ in pairs}


def test_queued_copy_source_is_not_reclaimed_before_the_copy(oracle_mod):
    # A and B share a partial tail T; A's write queues (T -> F); B is released before the
    # copy is taken.  T must not go back to the free list yet: another copy-on-write in
    # the same batch would otherwise take T as its destination (pages: the shared block
    # is copied before its count drops, and an early-reclaimed block gets overwritten,
    # lpnh.cn/news/2758356 §4.2-§4.3).
    m = _model(oracle_mod, 8, 4, free_order=list(range(8)))
    a = m.add_seq(2)
    (b,) = m.fork(a, 1)
    t = m.block_table(a)[0]
    u_owner = m.add_seq(3)
    (u_sib,) = m.fork(u_owner, 1)
    m.append_token(a)                              # queues (t, f1)
    m.free_seq(b)                                  # t now has no reader but the copy
    assert m.refcount[t] == 0 and t not in m.free
    assert m.stats()["held_blocks"] == 1
    m.append_token(u_owner)                        # queues (u, f2) with f2 != t
    pairs = m.take_copies()
    assert len(pairs) == 2 and pairs[0][0] == t and pairs[1][1] != t
    assert _disjoint(pairs)
    assert t in m.free                             # released once its copy is handed out
    m.free_seq(u_sib)


def test_copy_of_a_block_still_waiting_for_its_copy_reads_the_original(oracle_mod):
    # A writes into shared T (queues T -> F1); then A is forked and the child writes
    # into F1 before the copies are taken: its copy comes from T (F1 does not hold
    # T's rows yet), so the batch is (T -> F1), (T -> F2) and has no overlap
    m = _model(oracle_mod, 8, 4, free_order=list(range(8)))
    a = m.add_seq(1)
    m.fork(a, 1)
    t = m.block_table(a)[0]
    m.append_token(a)
    f1 = m.block_table(a)[0]
    (c,) = m.fork(a, 1)
    m.append_token(c)
    f2 = m.block_table(c)[0]
    assert m.take_copies() == [(t, f1), (t, f2)]


def test_ids_of_released_sequences_are_reused(oracle_mod):
    m = _model(oracle_mod, 16, 4)
    ids = [m.add_seq(1) for _ in range(4)]
    assert ids == [0, 1, 2, 3]
    m.free_seq(1)
    m.free_seq(3)
    assert m.add_seq(1) == 3 and m.add_seq(1) == 1 and m.add_seq(1) == 4


def test_every_sequence_reads_back_its_own_tokens(oracle_mod):
    # A simulated device pool, run step by step the way a decode loop drives the block
    # manager: appends (with releases and new prompts in between), then the step's
    # copy-on-write pairs are taken and copied, then the step's new rows are written.
    # Forks happen between steps.  After every step each live sequence, gathered through
    # its table, must read exactly its own token history (each fork shares its parent's
    # history, then diverges); every batch of pairs must be free of overlaps.
    rng = np.random.default_rng(11)
    for trial in range(40):
        N, bs = int(rng.integers(6, 30)), int(rng.choice([1, 2, 4]))
        m = _model(oracle_mod, N, bs, free_order=rng.permutation(N))
        pool = [[None] * bs for _ in range(N)]
        history = {}
        token = [0]

        def fresh():
            token[0] += 1
            return token[0]

        def write(slot, tok):
            pool[slot // bs][slot % bs] = tok

        for step in range(60):
            if history and rng.random() < 0.3:     # fork between steps
                parent = list(history)[int(rng.integers(len(history)))]
                for kid in m.fork(parent, int(rng.integers(1, 3))):
                    history[kid] = list(history[parent])
            pending = {}
            for _ in range(int(rng.integers(1, 6))):
                op = rng.random()
                if op < 0.15 or not history:
                    n = int(rng.integers(0, 3 * bs + 1))
                    s = m.add_seq(n)
                    if s is not None:
                        history[s] = [fresh() for _ in range(n)]
                        for i, slot in enumerate(m.slots_of(s)):
                            write(slot, history[s][i])
                elif op < 0.3:
                    s = list(history)[int(rng.integers(len(history)))]
                    m.free_seq(s)
                    del history[s]
                    pending.pop(s, None)
                else:
                    s = list(history)[int(rng.integers(len(history)))]
                    slot = m.append_token(s)
                    if slot is not None:
                        tok = fresh()
                        history[s].append(tok)
                        pending.setdefault(s, []).append((slot, tok))
            pairs = m.take_copies()
            assert _disjoint(pairs), (trial, step, pairs)
            snapshot = {s: list(pool[s]) for s, _ in pairs}
            for src, dst in pairs:                 # all at once, as one copy_blocks launch
                pool[dst] = list(snapshot[src])
            for writes in pending.values():
                for slot, tok in writes:
                    write(slot, tok)
            for s, hist in history.items():
                assert [pool[x // bs][x % bs] for x in m.slots_of(s)] == hist, (trial, step, s)
