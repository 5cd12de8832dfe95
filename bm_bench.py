"""Host block-manager benchmark: allocation cost and tail waste per block size.

The pages weigh block size as a trade-off: smaller blocks waste less of each
sequence's last block but make tables longer and allocation more frequent
(5688vip ch. 4 "PagedAttention：显存管理、分页机制、块大小选择", section "块大小选择"
and its table; lpnh.cn/news/2758356 §5.1-§5.2).  For every block size this
runs a decode batch through the host block manager -- prompts of the llama7b
lengths, then one appended token per sequence per step -- and reports appended
tokens per second, blocks allocated per 1000 appends, and the pool's tail waste
(1 - filled / allocated slots) and table entries at the end.

    python bm_bench.py [--steps 200] [--block-sizes 8 16 32 64]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

_ROOT = os.path.dirname(os.path.abspath(__file__))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import workloads as wl  # noqa: E402

from paged_kv_cache_393_b200 import BlockManager  # noqa: E402


def run(block_size: int, steps: int, workload: str = "llama7b", pool_tokens: int = None) -> dict:
    w = wl.get(workload)
    lens = wl.context_lens(w)
    pool_tokens = pool_tokens or wl.SWEEP_POOL_TOKENS * 2
    n_blocks = pool_tokens // block_size
    bm = BlockManager(n_blocks, block_size, free_order=wl.free_order(n_blocks, w.seed))
    seqs = [bm.add_seq(int(L) - 1) for L in lens]
    assert all(s is not None for s in seqs)
    seqs = np.asarray(seqs, np.int32)
    free0 = bm.num_free()
    t = time.perf_counter()
    for _ in range(steps):
        out = bm.append_tokens(seqs)
        assert len(out) == len(seqs)
    dt = time.perf_counter() - t
    st = bm.stats()
    appends = steps * len(seqs)
    return {"block_size": block_size, "sequences": len(seqs), "steps": steps,
            "appends_per_s": round(appends / dt, 1),
            "blocks_allocated_per_1000_appends": round(1000 * (free0 - bm.num_free()) / appends, 2),
            "tail_waste": round(1 - st["filled_slots"] / st["allocated_slots"], 5),
            "table_entries": st["table_entries"], "stats": st}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--block-sizes", type=int, nargs="+", default=list(wl.SWEEP_BLOCK_SIZES))
    ap.add_argument("--workload", default="llama7b")
    a = ap.parse_args(argv)
    for bs in a.block_sizes:
        print(json.dumps(run(bs, a.steps, a.workload)), flush=True)


if __name__ == "__main__":
    main()
