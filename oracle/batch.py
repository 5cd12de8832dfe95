"""Oracle-side construction of a decode batch -- TEST INFRASTRUCTURE ONLY.

Built from the same seeded generators as the GPU side, using only this package
and workloads.py.  The oracle's block-manager model, seeded
with the workload's free list, gives the block tables and slots; oracle
reshape_and_cache writes every token's K/V into host pools; oracle attention
computes the expected outputs.  For full-size workloads only a sample of
sequences is built: their blocks are relabeled into a compact host pool, which
leaves the attention unchanged (placement invariance is pinned in
test_oracle_pins.py) and keeps host memory small.
"""
from __future__ import annotations

import numpy as np

import workloads as wl

from . import BlockManagerModel, paged_attention, reshape_and_cache


class OracleBatch:
    def __init__(self, w: wl.Workload, sample=None):
        B, H, Hk, D, bs, N = (w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                              w.num_blocks)
        self.w = w
        lens = wl.context_lens(w)
        model = BlockManagerModel(N, bs, free_order=wl.free_order(N, w.seed))
        seqs = [model.add_seq(int(L) - 1) for L in lens]
        self.new_slots = np.array([model.append_token(s) for s in seqs], np.int64)
        self.tables = [model.block_table(s) for s in seqs]        # physical, full batch
        self.sample = list(range(B)) if sample is None else list(sample)
        self.lens = lens[self.sample]
        # compact pools holding only the sampled sequences' blocks, relabeled in order
        self.blocks = []
        relabel = {}
        for b in self.sample:
            for blk in self.tables[b]:
                if blk not in relabel:
                    relabel[blk] = len(self.blocks)
                    self.blocks.append(blk)
        M = len(self.blocks)
        kc = wl.sentinel_pool(M, Hk, bs, D)
        vc = wl.sentinel_pool(M, Hk, bs, D)
        maxblk = max(len(self.tables[b]) for b in self.sample)
        self.compact_tables = np.full((len(self.sample), maxblk), -1, np.int32)
        ks, vs, slots = [], [], []
        for j, b in enumerate(self.sample):
            t = [relabel[x] for x in self.tables[b]]
            self.compact_tables[j, :len(t)] = t
            L = int(lens[b])
            k, v = wl.sequence_kv(w.seed, b, L, Hk, D)
            i = np.arange(L)
            ks.append(k)
            vs.append(v)
            slots.append(np.asarray(t, np.int64)[i // bs] * bs + i % bs)
        self.key_cache, self.value_cache = reshape_and_cache(
            kc, vc, np.concatenate(ks), np.concatenate(vs), np.concatenate(slots), bs)
        self.q = wl.decode_q(w.seed, 0, B, H, D)[self.sample]

    def attention(self, nthreads=8):
        w = self.w
        return paged_attention(self.q, self.key_cache, self.value_cache, self.compact_tables,
                                      self.lens, w.scale, w.block_size, w.num_kv_heads,
                                      nthreads=nthreads)


def compact_pools(entries, block_size, num_kv_heads, head_dim):
    """Host pools holding the given sequences only.

    entries: list of (physical table, K [L][Hk][D], V [L][Hk][D]).  Physical ids
    are relabeled in order of first appearance; returns (key_cache, value_cache,
    compact tables [n][max blocks] padded with -1, lengths, relabel dict).
    """
    relabel = {}
    for table, _, _ in entries:
        for blk in table:
            relabel.setdefault(blk, len(relabel))
    M = max(len(relabel), 1)
    kc = wl.sentinel_pool(M, num_kv_heads, block_size, head_dim)
    vc = wl.sentinel_pool(M, num_kv_heads, block_size, head_dim)
    maxblk = max(len(t) for t, _, _ in entries)
    tables = np.full((len(entries), maxblk), -1, np.int32)
    ks, vs, slots, lens = [], [], [], []
    for j, (table, k, v) in enumerate(entries):
        t = [relabel[x] for x in table]
        tables[j, :len(t)] = t
        L = k.shape[0]
        i = np.arange(L)
        ks.append(k)
        vs.append(v)
        slots.append(np.asarray(t, np.int64)[i // block_size] * block_size + i % block_size)
        lens.append(L)
    kc, vc = reshape_and_cache(kc, vc, np.concatenate(ks), np.concatenate(vs),
                                      np.concatenate(slots), block_size)
    return kc, vc, tables, np.asarray(lens, np.int32), relabel
