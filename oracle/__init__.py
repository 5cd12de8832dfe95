"""CPU oracle for the paged-KV decode path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference arm may import this package.  It shares no code with the CUDA
library (``paged_kv_cache_393_b200``) and neither imports the other; both take
their inputs from the seeded generators in ``workloads.py``.

Contents
--------
* ``paged_attention``      -- fp64 paged decode attention (C, ``paged_attention_oracle.c``).
* ``gather_kv``            -- the block-table gather step alone.
* ``reshape_and_cache``    -- byte-level expectation of the slot-mapping scatter.
* ``copy_blocks``          -- byte-level expectation of the copy-on-write block copy.
* ``BlockManagerModel``    -- concept model of the block manager (free list,
  refcounts, append-token allocation, fork, copy-on-write, release).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
and ``tests/test_block_manager_model.py`` against what the pages and the
mathematics fix (worked examples, closed forms, invariants, a library routine).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "paged_attention_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with plain gcc -O2 (no fast-math) into liboracle.so."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i = ctypes.c_int
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_gather_kv.argtypes = [P, P, P, P, P, i, i, i, i, i, i, i]
            lib.oracle_gather_kv.restype = i
            lib.oracle_paged_attention.argtypes = [
                P, P, P, P, P, P, ctypes.c_double, i, i, i, i, i, i, i, i]
            lib.oracle_paged_attention.restype = i
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _as_half_bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    if a.dtype == np.uint16:
        return a
    raise TypeError("expected float16 (or its uint16 bit pattern), got %s" % a.dtype)


def half_to_double(bits: int) -> float:
    """Decode one IEEE binary16 bit pattern exactly (the C oracle's decoder)."""
    return _load().oracle_half_to_double(int(bits) & 0xFFFF)


def gather_kv(key_cache, value_cache, table_row, L, kvh, block_size):
    """K_b, V_b [L][D] float64 of one sequence and kv head, gathered through its table row."""
    kc = _as_half_bits(key_cache)
    vc = _as_half_bits(value_cache)
    N, Hk, bs, D = kc.shape
    assert bs == block_size and vc.shape == kc.shape
    row = np.ascontiguousarray(table_row, dtype=np.int32)
    k_out = np.empty((max(L, 1), D), np.float64)
    v_out = np.empty((max(L, 1), D), np.float64)
    st = _load().oracle_gather_kv(_ptr(k_out), _ptr(v_out), _ptr(kc), _ptr(vc), _ptr(row),
                                  int(L), int(kvh), Hk, bs, D, row.shape[0], N)
    if st != 0:
        raise ValueError("oracle_gather_kv rejected its arguments (status %d)" % st)
    return k_out[:L], v_out[:L]


def paged_attention(q, key_cache, value_cache, block_tables, context_lens, scale,
                    block_size, num_kv_heads, nthreads: int = 1) -> np.ndarray:
    """fp64 paged decode attention.

    q: [B][H][D] fp16; key_cache/value_cache: [N][Hk][bs][D] fp16;
    block_tables: [B][max_blocks] int32; context_lens: [B] int32.
    Returns out [B][H][D] float64.
    """
    qb = _as_half_bits(q)
    kc = _as_half_bits(key_cache)
    vc = _as_half_bits(value_cache)
    B, H, D = qb.shape
    N, Hk, bs, D2 = kc.shape
    assert D2 == D and bs == block_size and Hk == num_kv_heads and vc.shape == kc.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    assert bt.ndim == 2 and bt.shape[0] == B and cl.shape == (B,)
    out = np.zeros((B, H, D), np.float64)
    st = _load().oracle_paged_attention(
        _ptr(out), _ptr(qb), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cl), float(scale),
        bs, Hk, B, H, D, bt.shape[1], N, int(nthreads))
    if st != 0:
        raise ValueError("oracle_paged_attention rejected its arguments (status %d)" % st)
    return out


def reshape_and_cache(key_cache, value_cache, k, v, slot_mapping, block_size):
    """Expected pools after writing token t's K/V rows to slot s = slot_mapping[t].

    Slot s addresses row s % bs of physical block s // bs (the new rows are scattered into
    their blocks: lpnh.cn/news/1824136 §3.1).  A slot of -1 is padding and is skipped.  Tokens are
    applied in order, so a later token wins if two share a slot.  Returns new arrays.
    """
    kc = np.array(key_cache, copy=True)
    vc = np.array(value_cache, copy=True)
    N, Hk, bs, D = kc.shape
    assert bs == block_size
    slots = np.asarray(slot_mapping, dtype=np.int64)
    for t in range(slots.shape[0]):
        s = int(slots[t])
        if s < 0:
            continue
        if s >= N * bs:
            raise ValueError("slot %d beyond the pool of %d blocks x %d" % (s, N, bs))
        blk, off = s // bs, s % bs
        kc[blk, :, off, :] = k[t]
        vc[blk, :, off, :] = v[t]
    return kc, vc


def copy_blocks(key_caches, value_caches, pairs):
    """Expected pools after copying whole blocks src -> dst for every (src, dst) pair,
    in every layer, applied in pair order (the copy step of copy-on-write, where a fresh
    block receives the shared block's contents: lpnh.cn/news/2758356 §4.2).  Returns new
    lists."""
    out_k = [np.array(x, copy=True) for x in key_caches]
    out_v = [np.array(x, copy=True) for x in value_caches]
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        for layer in range(len(out_k)):
            out_k[layer][dst] = out_k[layer][src]
            out_v[layer][dst] = out_v[layer][src]
    return out_k, out_v


class BlockManagerModel:
    """Concept model of the paged KV block manager, in the pages' terms.

    * Free list: a list of physical ids; allocation pops from its END
      (the ``PagedKVManager.allocate_block`` concept model of n1n.ai
      "PagedAttention 对比传统 KV 缓存", section "实现逻辑代码示例").  The caller
      passes the initial order (the seeded shuffle is an input).
    * Allocation sets refcount 1; release walks the table, decrements, and returns
      blocks that reach 0 to the end of the free list (lpnh.cn/news/2758356 §3.2).
    * append_token: when the sequence has no block or its last block is full,
      allocate a new block and append it to the table; an empty pool is an error
      that leaves all state unchanged (same concept model; lpnh.cn/news/2758356 §3.1).
    * fork: children share every block of the parent; each block's refcount grows
      by the number of children (lpnh.cn/news/2758356 §4.2 step 1).
    * copy-on-write: a write into a shared (refcount > 1) block that is NOT full
      allocates a new block, records (src, dst) for the copy, decrements the old
      block's refcount and repoints the writer's table entry.  A shared FULL block
      needs no copy: the next token goes to a fresh block (lpnh.cn/news/2758356 §4.2).
    * Fill of the last block is derived from the sequence length (the concept
      model's per-block token_count is ambiguous once blocks are shared).
    * A queued copy has not happened yet: the pages copy the shared block's
      contents first and only then drop its count (lpnh.cn/news/2758356 §4.2),
      and a block reclaimed too early gets handed out again and overwritten
      (§4.3).  So both ends of a queued pair stay out of the free list until
      the pair is taken (take_copies), even when their count reaches 0 first;
      take_copies then returns them in pair order (source, then destination).
      A write into a block that is itself still waiting for its copy is copied
      from that block's source, so the pairs of one take name no block twice as
      destination and no destination as a source: applied all at once they give
      what applying them one after another gives.
    * Released sequence ids are reused, the most recently released first.
    """

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        if free_order is None:
            self.free = list(range(num_blocks))
        else:
            self.free = [int(x) for x in free_order]
            if sorted(self.free) != list(range(num_blocks)):
                raise ValueError("free_order must be a permutation of 0..num_blocks-1")
        self.refcount = [0] * num_blocks
        self.pinned = [0] * num_blocks      # queued copy pairs naming the block
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.copies: list[tuple[int, int]] = []
        self.copy_source: dict[int, int] = {}   # destination -> source of a queued pair
        self._next_id = 0
        self._free_ids: list[int] = []

    # -- allocation ---------------------------------------------------------
    def allocate_block(self):
        if not self.free:
            return None
        blk = self.free.pop()
        self.refcount[blk] = 1
        return blk

    def _new_seq(self, table, length):
        if self._free_ids:
            sid = self._free_ids.pop()
        else:
            sid = self._next_id
            self._next_id += 1
        self.tables[sid] = table
        self.lens[sid] = length
        return sid

    def add_seq(self, num_tokens: int):
        """New sequence holding num_tokens tokens (its prompt).  None on OOM."""
        if num_tokens < 0:
            raise ValueError("num_tokens must be >= 0")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            return None
        table = [self.allocate_block() for _ in range(need)]
        return self._new_seq(table, num_tokens)

    def append_token(self, seq: int):
        """Reserve the slot of the sequence's next token; returns the flat slot
        phys * block_size + offset, or None when the pool is exhausted."""
        table = self.tables[seq]
        L = self.lens[seq]
        bs = self.block_size
        if L % bs == 0:
            blk = self.allocate_block()
            if blk is None:
                return None
            table.append(blk)
        else:
            last = table[-1]
            if self.refcount[last] > 1:
                new = self.allocate_block()
                if new is None:
                    return None
                src = self.copy_source.get(last, last)
                self.copies.append((src, new))
                self.copy_source[new] = src
                self.pinned[src] += 1
                self.pinned[new] += 1
                self.refcount[last] -= 1
                table[-1] = new
        slot = table[L // bs] * bs + L % bs
        self.lens[seq] = L + 1
        return slot

    def fork(self, seq: int, n: int):
        """n children sharing every block of seq; returns their ids."""
        if n < 0:
            raise ValueError("n must be >= 0")
        ids = []
        for _ in range(n):
            for blk in self.tables[seq]:
                self.refcount[blk] += 1
            ids.append(self._new_seq(list(self.tables[seq]), self.lens[seq]))
        return ids

    def free_seq(self, seq: int):
        for blk in self.tables.pop(seq):
            self.refcount[blk] -= 1
            if self.refcount[blk] == 0 and self.pinned[blk] == 0:
                self.free.append(blk)
        del self.lens[seq]
        self._free_ids.append(seq)

    def take_copies(self):
        """The queued (source, destination) pairs, in queue order; their blocks are
        released from the queue (and freed if no table references them)."""
        out, self.copies = self.copies, []
        self.copy_source = {}
        for pair in out:
            for blk in pair:
                self.pinned[blk] -= 1
                if self.pinned[blk] == 0 and self.refcount[blk] == 0:
                    self.free.append(blk)
        return out

    # -- views ----------------------------------------------------------------
    def block_table(self, seq: int):
        return list(self.tables[seq])

    def num_free(self) -> int:
        return len(self.free)

    def stats(self):
        """Pool occupancy.  A physical block's filled slots are the most tokens any
        sequence referencing it keeps in it; allocated slots are whole used blocks."""
        bs = self.block_size
        fill = {}
        for seq, table in self.tables.items():
            L = self.lens[seq]
            for j, blk in enumerate(table):
                fill[blk] = max(fill.get(blk, 0), min(bs, L - j * bs))
        used = sum(1 for r in self.refcount if r > 0)
        held = sum(1 for r, p in zip(self.refcount, self.pinned) if r == 0 and p > 0)
        return {"num_blocks": self.num_blocks, "free_blocks": len(self.free),
                "used_blocks": used, "num_seqs": len(self.tables),
                "logical_tokens": sum(self.lens.values()), "filled_slots": sum(fill.values()),
                "allocated_slots": used * bs,
                "table_entries": sum(len(t) for t in self.tables.values()),
                "held_blocks": held}

    def slots_of(self, seq: int):
        """Flat slots of every token of the sequence, in logical order."""
        bs = self.block_size
        t = self.tables[seq]
        return [t[i // bs] * bs + i % bs for i in range(self.lens[seq])]
