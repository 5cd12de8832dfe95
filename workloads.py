"""Seeded synthetic inputs for the paged-KV decode path.

This module is shared by the CUDA side (tests, bench, smoke) and the CPU oracle
side.  It holds no arithmetic of the method itself: no block-table translation,
no slot computation, no attention.  It only draws the inputs -- context
lengths, the shuffled free-list order, fp16 q/K/V values -- and describes the
workload shapes.

Workloads (shapes of the pages' Llama-2-7B / 70B-like decode batches):

* ``tiny``      3 sequences (context 12, 50, 1), 4 = 4 heads, head_dim 64,
                block_size 4, pool of 64 blocks.
* ``llama7b``   256 sequences, 32 = 32 heads, head_dim 128, block_size 16,
                context lengths uniform in [500, 1524], pool of 32768 blocks.
* ``bs_sweep``  ``llama7b`` at block_size 8/16/32/64 with pool bytes held fixed
                (num_blocks = 524288 / block_size) and the same K/V per token.
* ``cow``       32 prompts of 1000 tokens, each forked into 8 samples (256
                sequences), then 200 decode steps; 32 = 32 heads, head_dim 128,
                block_size 16, pool of 32768 blocks.
* ``llama7b_small`` / ``gqa_small``  32- and 16-sequence cuts of those batches
                (pools of about 1 GB) for profiler captures; ``cow_small`` an
                8-prompt cut of ``cow``, ``cow_compact`` the whole ``cow`` batch in
                a 6144-block pool.
* ``gqa``       128 sequences, 64 query heads over 8 kv heads, head_dim 128,
                block_size 16, context lengths round(LogNormal(ln 1024, 1))
                clipped to [64, 16384], split into 512-token partitions,
                pool of 131072 blocks.

Value recipe: every fp16 value is a float32 draw of numpy's PCG64
``standard_normal`` rounded to fp16.  K and V of sequence ``b`` come from two
streams keyed by ``(seed, b, 0)`` and ``(seed, b, 1)``, one row of Hk x D
values per token in token order, so token i's values do not depend on the
sequence length or on the block size.  Decode-step inputs (q and the new
token's K/V of a step) are keyed by ``(seed, 1_000_000 + step, j)``.  Pool
slots that no token ever wrote hold the fp16 NaN bit pattern ``SENTINEL_BITS``.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

#: fp16 bit pattern left in every pool slot that no token wrote (a quiet NaN
#: with a payload, so any read of an unwritten slot poisons the result).
SENTINEL_BITS = 0x7E5A


@dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    seed: int
    lens: str                    # "fixed", "uniform", "lognormal", "cow"
    fixed_lens: tuple = ()
    len_lo: int = 0
    len_hi: int = 0
    lognormal_median: float = 0.0
    lognormal_sigma: float = 0.0
    partition_size: int = 0      # 0 = single pass
    prompts: int = 0             # cow only
    prompt_len: int = 0          # cow only
    samples: int = 0             # cow only
    decode_steps: int = 0        # cow only

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads


WORKLOADS = {
    "tiny": Workload("tiny", 3, 4, 4, 64, 4, 64, 1001, "fixed", fixed_lens=(12, 50, 1)),
    "llama7b": Workload("llama7b", 256, 32, 32, 128, 16, 32768, 1002, "uniform",
                        len_lo=500, len_hi=1524),
    # a 32-sequence cut of llama7b (0.5 GB of K/V, pools of 1 GB) for profiler captures
    "llama7b_small": Workload("llama7b_small", 32, 32, 32, 128, 16, 4096, 1002, "uniform",
                              len_lo=500, len_hi=1524),
    "gqa_small": Workload("gqa_small", 16, 64, 8, 128, 16, 16384, 1005, "lognormal",
                          lognormal_median=1024.0, lognormal_sigma=1.0, len_lo=64, len_hi=16384,
                          partition_size=512),
    "cow": Workload("cow", 256, 32, 32, 128, 16, 32768, 1004, "cow",
                    prompts=32, prompt_len=1000, samples=8, decode_steps=200),
    # an 8-prompt cut of cow (64 samples) for profiler captures of the shared-prefix pass
    "cow_small": Workload("cow_small", 64, 32, 32, 128, 16, 8192, 1004, "cow",
                          prompts=8, prompt_len=1000, samples=8, decode_steps=200),
    # the whole cow batch in a pool of 6144 blocks (1.6 GB; 200 steps need 5344): the
    # prefix pass's full item count, for multi-pass profiler captures
    "cow_compact": Workload("cow_compact", 256, 32, 32, 128, 16, 6144, 1004, "cow",
                            prompts=32, prompt_len=1000, samples=8, decode_steps=200),
    "gqa": Workload("gqa", 128, 64, 8, 128, 16, 131072, 1005, "lognormal",
                    lognormal_median=1024.0, lognormal_sigma=1.0, len_lo=64, len_hi=16384,
                    partition_size=512),
}

#: block sizes of the block-size sweep; pool bytes are held fixed
SWEEP_BLOCK_SIZES = (8, 16, 32, 64)
SWEEP_POOL_TOKENS = 524288


def bs_sweep(block_size: int) -> Workload:
    """The llama7b batch at another block size, same lengths and K/V per token."""
    if block_size not in SWEEP_BLOCK_SIZES:
        raise ValueError("block size sweep covers %s" % (SWEEP_BLOCK_SIZES,))
    base = WORKLOADS["llama7b"]
    return replace(base, name="bs_sweep_%d" % block_size, block_size=block_size,
                   num_blocks=SWEEP_POOL_TOKENS // block_size)


def get(name: str) -> Workload:
    if name.startswith("bs_sweep_"):
        return bs_sweep(int(name.split("_")[-1]))
    return WORKLOADS[name]


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(k) for k in key]))


def context_lens(w: Workload) -> np.ndarray:
    """Context length of every sequence (including the token written this step)."""
    if w.lens == "fixed":
        return np.asarray(w.fixed_lens, dtype=np.int32)
    if w.lens == "uniform":
        return _rng(w.seed, 7).integers(w.len_lo, w.len_hi + 1, size=w.num_seqs).astype(np.int32)
    if w.lens == "lognormal":
        x = _rng(w.seed, 7).lognormal(math.log(w.lognormal_median), w.lognormal_sigma,
                                      size=w.num_seqs)
        return np.clip(np.rint(x), w.len_lo, w.len_hi).astype(np.int32)
    if w.lens == "cow":
        return np.full(w.num_seqs, w.prompt_len + 1, dtype=np.int32)
    raise ValueError(w.lens)


def free_order(num_blocks: int, seed: int) -> np.ndarray:
    """Seeded shuffle of the physical block ids; the block manager pops from its end."""
    return _rng(seed, 11).permutation(num_blocks).astype(np.int32)


def sequence_kv(seed: int, seq: int, length: int, num_kv_heads: int, head_dim: int):
    """fp16 K and V rows [length][Hk][D] of every token of one sequence."""
    shape = (length, num_kv_heads, head_dim)
    k = _rng(seed, seq, 0).standard_normal(shape, dtype=np.float32).astype(np.float16)
    v = _rng(seed, seq, 1).standard_normal(shape, dtype=np.float32).astype(np.float16)
    return k, v


def sequences_kv(seed: int, seqs, lengths, num_kv_heads: int, head_dim: int, threads: int = 8):
    """sequence_kv for many sequences, drawn on a thread pool (order preserved)."""
    def one(args):
        s, n = args
        return sequence_kv(seed, s, int(n), num_kv_heads, head_dim)
    with ThreadPoolExecutor(max(1, threads)) as ex:
        return list(ex.map(one, zip(list(seqs), list(lengths))))


def decode_q(seed: int, step: int, num_seqs: int, num_heads: int, head_dim: int) -> np.ndarray:
    """fp16 query [B][H][D] of one decode step."""
    return _rng(seed, 1_000_000 + step, 2).standard_normal(
        (num_seqs, num_heads, head_dim), dtype=np.float32).astype(np.float16)


def decode_kv(seed: int, step: int, num_seqs: int, num_kv_heads: int, head_dim: int):
    """fp16 K and V [B][Hk][D] of the token each sequence appends at a decode step."""
    shape = (num_seqs, num_kv_heads, head_dim)
    k = _rng(seed, 1_000_000 + step, 0).standard_normal(shape, dtype=np.float32).astype(np.float16)
    v = _rng(seed, 1_000_000 + step, 1).standard_normal(shape, dtype=np.float32).astype(np.float16)
    return k, v


def sentinel_pool(num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int) -> np.ndarray:
    """A host pool [N][Hk][bs][D] of fp16 whose every element is the sentinel NaN."""
    return np.full((num_blocks, num_kv_heads, block_size, head_dim), SENTINEL_BITS,
                   dtype=np.uint16).view(np.float16)


# -- byte accounting (measurement, not the method) -----------------------------

def kv_bytes_per_token(num_kv_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """Bytes of K plus V of one token in one layer."""
    return 2 * num_kv_heads * head_dim * elem_bytes


def kv_cache_bytes(num_layers: int, num_heads: int, head_dim: int, seq_len: int,
                   batch: int, dtype_bytes: int) -> int:
    """Total KV-cache bytes: K and V of every layer, head, token and sequence."""
    return 2 * num_layers * num_heads * head_dim * seq_len * batch * dtype_bytes
