"""Stateful property test: the C++ block manager against the oracle's concept model.

Hypothesis drives both through random sequences of every operation -- add a
sequence, fork it, free it, append one token, append a batch, take the
copy-on-write pairs -- on small pools where exhaustion is common, and after
every step requires identical results, tables, lengths, reference counts, free
lists and utilisation counts.  The model follows the pages' rules (free list
popped from its end, refcounts, copy-on-write of a shared partial block:
n1n.ai "实现逻辑代码示例"; lpnh.cn/news/2758356 §3.1-§4.2).
"""
import numpy as np
import pytest
from hypothesis import HealthCheck, settings
from hypothesis import strategies as st
from hypothesis.stateful import RuleBasedStateMachine, initialize, invariant, precondition, rule

import oracle
from paged_kv_cache_393_b200 import BlockManager


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_393_b200 import build
    build.build()


class BlockManagerMachine(RuleBasedStateMachine):
    @initialize(num_blocks=st.integers(1, 24), block_size=st.sampled_from([1, 2, 4, 16]),
                seed=st.integers(0, 2 ** 16))
    def setup(self, num_blocks, block_size, seed):
        order = np.random.default_rng(seed).permutation(num_blocks)
        self.native = BlockManager(num_blocks, block_size, free_order=order)
        self.model = oracle.BlockManagerModel(num_blocks, block_size, free_order=order)
        self.live = []

    @rule(n=st.integers(0, 40))
    def add_seq(self, n):
        a, b = self.native.add_seq(n), self.model.add_seq(n)
        assert a == b
        if a is not None:
            self.live.append(a)

    @precondition(lambda self: self.live)
    @rule(i=st.integers(0, 1000), k=st.integers(1, 3))
    def fork(self, i, k):
        s = self.live[i % len(self.live)]
        a, b = self.native.fork(s, k), self.model.fork(s, k)
        assert a == b
        self.live += a

    @precondition(lambda self: self.live)
    @rule(i=st.integers(0, 1000))
    def free_seq(self, i):
        s = self.live.pop(i % len(self.live))
        self.native.free_seq(s)
        self.model.free_seq(s)

    @precondition(lambda self: self.live)
    @rule(i=st.integers(0, 1000))
    def append_token(self, i):
        s = self.live[i % len(self.live)]
        assert self.native.append_token(s) == self.model.append_token(s)

    @precondition(lambda self: self.live)
    @rule(idx=st.lists(st.integers(0, 1000), min_size=1, max_size=6))
    def append_tokens(self, idx):
        batch = [self.live[i % len(self.live)] for i in idx]
        got = self.native.append_tokens(batch).tolist()
        want = []
        for s in batch:              # the batch stops at the first sequence that cannot grow
            r = self.model.append_token(s)
            if r is None:
                break
            want.append(r)
        assert got == want

    @rule()
    def take_copies(self):
        pairs = self.native.take_copies().tolist()
        assert pairs == [list(p) for p in self.model.take_copies()]
        # one batch is safe for a single copy_blocks launch: no destination repeats and
        # none is also a source
        dsts = [d for _, d in pairs]
        assert len(set(dsts)) == len(dsts) and not set(dsts) & {s for s, _ in pairs}

    @invariant()
    def same_state(self):
        if not hasattr(self, "native"):
            return
        for s in self.live:
            assert self.native.block_table(s) == self.model.block_table(s)
            assert self.native.seq_len(s) == self.model.lens[s]
        assert self.native.free_list() == self.model.free
        assert [self.native.refcount(b) for b in range(self.model.num_blocks)] == \
            self.model.refcount
        assert self.native.stats() == self.model.stats()


BlockManagerMachine.TestCase.settings = settings(
    max_examples=60, stateful_step_count=40, deadline=None,
    suppress_health_check=[HealthCheck.too_slow])
test_block_manager_state_machine = BlockManagerMachine.TestCase
