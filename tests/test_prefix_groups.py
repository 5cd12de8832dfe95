"""pagedkv_prefix_groups (host): grouping a decode batch by shared table prefixes.

The grouping is checked against what the block tables themselves fix: members of
a group reference the same physical blocks for the group's prefix, the prefix is
whole blocks before every member's last token, and a sequence is in at most one
group.  The copy-on-write workload's fork structure (32 prompts of 1000 tokens,
8 samples each) pins the expected groups exactly.
"""
import ctypes

import numpy as np
import pytest

import workloads as wl
from paged_kv_cache_393_b200 import BlockManager, PagedKVError, prefix_groups
from paged_kv_cache_393_b200 import _native as nat


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_393_b200 import build
    build.build()


def _check_invariants(tables, lens, bs, max_members, pre, groups, refcount=None):
    seen = set()
    for g in groups:
        blocks, members = int(g[0]), [int(m) for m in g[1:] if m >= 0]
        assert 2 <= len(members) <= max_members and len(set(members)) == len(members)
        assert all(m == -1 for m in g[1 + len(members):])      # padding after the members
        assert not seen & set(members)
        seen |= set(members)
        assert blocks >= 1
        for m in members:
            assert blocks <= (lens[m] - 1) // bs                 # whole blocks before the last token
            assert list(tables[m][:blocks]) == list(tables[members[0]][:blocks])
            assert pre[m] == blocks * bs
        if refcount is not None:                                 # shared blocks are referenced
            assert all(refcount(b) >= len(members) for b in tables[members[0]][:blocks])
    assert all(pre[b] == 0 for b in range(len(lens)) if b not in seen)


def _cow_batch(prompts=32, samples=8, prompt_len=1000, bs=16):
    bm = BlockManager(32768, bs, free_order=wl.free_order(32768, 1004))
    seqs = []
    for _ in range(prompts):
        s = bm.add_seq(prompt_len)
        seqs += [s] + bm.fork(s, samples - 1)
    bm.append_tokens(seqs)
    bm.take_copies()
    tables, lens = bm.build_batch(seqs, 80)
    return bm, tables, lens


def test_cow_workload_groups_are_the_forks():
    bm, tables, lens = _cow_batch()
    pre, groups = prefix_groups(tables, lens, 16, 8)
    assert groups.shape == (32, nat.GROUP_WIDTH)
    assert (groups[:, 0] == 62).all()                    # 1000 tokens: 62 whole blocks + 8 rows
    assert sorted(groups[:, 1:].ravel().tolist()) == list(range(256))
    assert (pre == 992).all()
    _check_invariants(tables, lens, 16, 8, pre, groups, bm.refcount)


@pytest.mark.parametrize("max_members", [1, 2, 4, 8])
def test_group_size_limit(max_members):
    bm, tables, lens = _cow_batch(prompts=4)
    pre, groups = prefix_groups(tables, lens, 16, max_members)
    if max_members == 1:
        assert len(groups) == 0 and not pre.any()
    else:
        assert len(groups) == 4 * 8 // max_members
    _check_invariants(tables, lens, 16, max_members, pre, groups, bm.refcount)


def test_random_fork_trees():
    rng = np.random.default_rng(11)
    bs = 8
    bm = BlockManager(20000, bs, free_order=rng.permutation(20000))
    live = []
    for _ in range(40):
        s = bm.add_seq(int(rng.integers(1, 200)))
        live.append(s)
        for _ in range(int(rng.integers(0, 3))):          # forks of forks
            kids = bm.fork(live[int(rng.integers(len(live)))], int(rng.integers(1, 5)))
            live += kids
            for k in kids:
                for _ in range(int(rng.integers(0, 30))):
                    bm.append_token(k)
    bm.take_copies()
    bm.append_tokens(live)
    bm.take_copies()
    tables, lens = bm.build_batch(live, max(len(bm.block_table(s)) for s in live))
    for mm in (2, 3, 8):
        pre, groups = prefix_groups(tables, lens, bs, mm)
        assert len(groups) > 0
        _check_invariants(tables, lens, bs, mm, pre, groups, bm.refcount)


def test_no_sharing_no_groups():
    bm = BlockManager(1000, 16)
    seqs = [bm.add_seq(100 + i) for i in range(10)]
    tables, lens = bm.build_batch(seqs, 8)
    pre, groups = prefix_groups(tables, lens, 16, 8)
    assert len(groups) == 0 and not pre.any()


def test_prefix_never_covers_the_last_token():
    # 32 tokens = 2 full blocks: the block with token 31 stays out of the prefix
    tables = np.array([[5, 6, -1], [5, 6, -1]], np.int32)
    lens = np.array([32, 32], np.int32)
    pre, groups = prefix_groups(tables, lens, 16, 8)
    assert groups.tolist() == [[1, 0, 1, -1, -1, -1, -1, -1, -1]] and pre.tolist() == [16, 16]
    pre, groups = prefix_groups(tables, np.array([17, 16], np.int32), 16, 8)
    assert len(groups) == 0                              # 16 tokens: no whole block before the last


def test_errors_and_capacity():
    lib = nat.load_library()
    t = np.array([[1, 2], [1, 2], [3, 4], [3, 4]], np.int32)
    lens = np.array([30, 30, 30, 30], np.int32)
    pre = np.full(4, 7, np.int32)
    groups = np.zeros((1, nat.GROUP_WIDTH), np.int32)
    P = ctypes.c_void_p
    st = lib.pagedkv_prefix_groups(t.ctypes.data, lens.ctypes.data, 4, 2, 16, 8, pre.ctypes.data,
                                   groups.ctypes.data, 1)
    assert st == nat.ERANGE and not pre.any()
    assert lib.pagedkv_prefix_groups(t.ctypes.data, lens.ctypes.data, 4, 2, 16, 9, pre.ctypes.data,
                                     groups.ctypes.data, 1) == nat.EINVAL
    assert lib.pagedkv_prefix_groups(None, lens.ctypes.data, 4, 2, 16, 8, pre.ctypes.data,
                                     groups.ctypes.data, 1) == nat.EINVAL
    assert lib.pagedkv_prefix_groups(None, None, 0, 2, 16, 8, None, None, 0) == 0
    with pytest.raises(ValueError):
        prefix_groups(t, lens[:3], 16, 8)
    del P


from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(seed=st.integers(0, 2 ** 20), bs=st.sampled_from([1, 2, 4, 8, 16]),
       prompts=st.integers(1, 6), max_members=st.integers(1, 8))
def test_random_forests_keep_the_grouping_rules(seed, bs, prompts, max_members):
    rng = np.random.default_rng(seed)
    N = 4000
    bm = BlockManager(N, bs, free_order=rng.permutation(N))
    live = []
    for _ in range(prompts):
        live.append(bm.add_seq(int(rng.integers(0, 60))))
        for _ in range(int(rng.integers(0, 4))):
            kids = bm.fork(live[int(rng.integers(len(live)))], int(rng.integers(1, 4)))
            for k in kids:
                for _ in range(int(rng.integers(0, 2 * bs + 2))):
                    bm.append_token(k)
            live += kids
    bm.append_tokens(live)
    bm.take_copies()
    maxblk = max(1, max(len(bm.block_table(s)) for s in live))
    tables, lens = bm.build_batch(live, maxblk)
    pre, groups = prefix_groups(tables, lens, bs, max_members)
    _check_invariants(tables, lens, bs, max_members, pre, groups, bm.refcount)
