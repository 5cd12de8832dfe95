"""GPU-side set-up of the seeded decode batches, for the tests, the smoke check and
the bench (a fixture, not part of the library).

A batch is: K/V pools on the device (every slot pre-filled with a NaN sentinel),
a host BlockManager seeded with the workload's shuffled free list, one sequence
per row whose prompt (all tokens but the last) is written through
reshape_and_cache, and the inputs of one decode step: q, the new token's K/V,
its slot (from BlockManager.append_tokens), the block tables and context lengths.

CowBatch follows the copy-on-write workload: prompts are prefilled, forked into
samples, and every step appends one token per sample, copying shared partial
blocks first (copy_blocks) when the block manager asks for it.
"""
from __future__ import annotations

import numpy as np
import torch

import workloads as wl

from paged_kv_cache_393_b200 import BlockManager, copy_blocks, reshape_and_cache


def sentinel_pools(num_blocks, num_kv_heads, block_size, head_dim, device):
    shape = (num_blocks, num_kv_heads, block_size, head_dim)
    bits = np.array([wl.SENTINEL_BITS], np.uint16).view(np.int16)[0]
    kc = torch.full(shape, int(bits), dtype=torch.int16, device=device).view(torch.float16)
    vc = torch.full(shape, int(bits), dtype=torch.int16, device=device).view(torch.float16)
    return kc, vc


def _write_tokens(kc, vc, k, v, slots, device):
    if len(slots) == 0:
        return
    reshape_and_cache(torch.from_numpy(k).to(device), torch.from_numpy(v).to(device), kc, vc,
                      torch.from_numpy(np.ascontiguousarray(slots, np.int64)).to(device))


class PagedBatch:
    """One decode step of a fixed-length workload (tiny, llama7b, bs_sweep_*, gqa)."""

    def __init__(self, w: wl.Workload, device, prefill_chunk_tokens: int = 1 << 17, _defer=False):
        self.w = w
        self.device = torch.device(device)
        B, Hk, D, bs, N = w.num_seqs, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks
        self.lens_host = wl.context_lens(w)
        self.max_context_len = int(self.lens_host.max())
        self.max_blocks = -(-self.max_context_len // bs)
        self.key_cache, self.value_cache = sentinel_pools(N, Hk, bs, D, self.device)
        self.bm = BlockManager(N, bs, free_order=wl.free_order(N, w.seed))
        self.seqs = []
        for L in self.lens_host:
            s = self.bm.add_seq(int(L) - 1)
            if s is None:
                raise MemoryError("pool of %d blocks too small for the workload" % N)
            self.seqs.append(s)
        self.k_new_host = np.empty((B, Hk, D), np.float16)
        self.v_new_host = np.empty((B, Hk, D), np.float16)
        if not _defer:
            _prefill([self], prefill_chunk_tokens)
            self._finish()

    def _write_prompts(self, b0, kvs):
        """Writes every token but the last of sequences b0, b0+1, ... (K/V rows kvs)."""
        ks, vs, slots = [], [], []
        for j, (k, v) in enumerate(kvs):
            b = b0 + j
            L = int(self.lens_host[b])
            ks.append(k[:L - 1])
            vs.append(v[:L - 1])
            slots.append(self.bm.seq_slots(self.seqs[b], 0, L - 1))
            self.k_new_host[b], self.v_new_host[b] = k[L - 1], v[L - 1]
        _write_tokens(self.key_cache, self.value_cache, np.concatenate(ks), np.concatenate(vs),
                      np.concatenate(slots), self.device)

    def _finish(self):
        """The decode step: one new token per sequence."""
        w, dev = self.w, self.device
        B = w.num_seqs
        self.slots_host = self.bm.append_tokens(self.seqs)
        assert len(self.slots_host) == B
        self.tables_host, lens = self.bm.build_batch(self.seqs, self.max_blocks)
        assert np.array_equal(lens, self.lens_host)
        self.q_host = wl.decode_q(w.seed, 0, B, w.num_heads, w.head_dim)
        self.q = torch.from_numpy(self.q_host).to(dev)
        self.k_new = torch.from_numpy(self.k_new_host).to(dev)
        self.v_new = torch.from_numpy(self.v_new_host).to(dev)
        self.slots = torch.from_numpy(self.slots_host).to(dev)
        self.block_tables = torch.from_numpy(self.tables_host).to(dev)
        self.context_lens = torch.from_numpy(self.lens_host).to(dev)
        self.out = torch.empty((B, w.num_heads, w.head_dim), dtype=torch.float16, device=dev)


    @property
    def scale(self) -> float:
        return self.w.scale

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one attention pass reads."""
        return int(self.lens_host.astype(np.int64).sum()) * wl.kv_bytes_per_token(
            self.w.num_kv_heads, self.w.head_dim)

def _prefill(batches, chunk_tokens):
    """Writes the prompts of every batch, drawing each sequence's K/V values once (the
    batches differ only in block size and pool)."""
    w = batches[0].w
    lens = batches[0].lens_host
    B = w.num_seqs
    b0 = 0
    while b0 < B:
        b1, tok = b0, 0
        while b1 < B and (b1 == b0 or tok + int(lens[b1]) <= chunk_tokens):
            tok += int(lens[b1])
            b1 += 1
        kvs = wl.sequences_kv(w.seed, range(b0, b1), lens[b0:b1], w.num_kv_heads, w.head_dim)
        for gb in batches:
            gb._write_prompts(b0, kvs)
        b0 = b1


def paged_batches(ws, device, prefill_chunk_tokens: int = 1 << 17):
    """PagedBatch of several workloads that differ only in block size and pool size (the
    block-size sweep: the same tokens, K/V values and lengths), from one draw of the values."""
    ref = ws[0]
    for w in ws:
        if (w.seed, w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.lens, w.len_lo,
                w.len_hi) != (ref.seed, ref.num_seqs, ref.num_heads, ref.num_kv_heads,
                              ref.head_dim, ref.lens, ref.len_lo, ref.len_hi):
            raise ValueError("paged_batches needs workloads that differ only in block size")
    out = [PagedBatch(w, device, _defer=True) for w in ws]
    _prefill(out, prefill_chunk_tokens)
    for gb in out:
        gb._finish()
    return out


class CowBatch:
    """The copy-on-write workload: prompts forked into samples, then decode steps."""

    def __init__(self, w: wl.Workload, device):
        assert w.lens == "cow"
        self.w = w
        self.device = torch.device(device)
        Hk, D, bs, N = w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks
        self.key_cache, self.value_cache = sentinel_pools(N, Hk, bs, D, self.device)
        self.bm = BlockManager(N, bs, free_order=wl.free_order(N, w.seed))
        self.samples = []
        for p in range(w.prompts):
            s = self.bm.add_seq(w.prompt_len)
            k, v = wl.sequence_kv(w.seed, p, w.prompt_len, Hk, D)
            _write_tokens(self.key_cache, self.value_cache, k, v, self.bm.seq_slots(s),
                          self.device)
            self.samples += [s] + self.bm.fork(s, w.samples - 1)
        self.step_index = 0
        self.max_context_len = w.prompt_len + w.decode_steps
        self.max_blocks = -(-self.max_context_len // bs)

    def prepare_step(self):
        """Host side of the next step: slots (may queue copy-on-write pairs), pairs,
        block tables, lengths, q and the new K/V.  Returns a dict of host arrays."""
        w = self.w
        slots = self.bm.append_tokens(self.samples)
        assert len(slots) == len(self.samples)
        pairs = self.bm.take_copies()
        tables, lens = self.bm.build_batch(self.samples, self.max_blocks)
        q = wl.decode_q(w.seed, self.step_index, w.num_seqs, w.num_heads, w.head_dim)
        k, v = wl.decode_kv(w.seed, self.step_index, w.num_seqs, w.num_kv_heads, w.head_dim)
        self.step_index += 1
        return dict(slots=slots, pairs=pairs, tables=tables, lens=lens, q=q, k=k, v=v)

    def run_cache_updates(self, host):
        """Device side of a step's cache updates: copy_blocks, then reshape_and_cache."""
        dev = self.device
        if len(host["pairs"]):
            copy_blocks([self.key_cache], [self.value_cache], torch.from_numpy(host["pairs"]).to(dev))
        _write_tokens(self.key_cache, self.value_cache, host["k"], host["v"], host["slots"], dev)
