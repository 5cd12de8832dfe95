"""GPU parity at the full workload sizes, on the whole batch.

Every (sequence, head) output of the decode step is compared with the fp64
oracle -- elementwise |gpu - oracle| <= 2e-3 + 1e-2 |oracle|, and the max abs
error <= 2e-3 read literally -- and every pool block the tables use is compared
bit for bit (the new rows included); blocks outside the tables must still hold
the sentinel.  The max abs / rel errors of every configuration are printed at
the end of the session.  The oracle's expected values of a workload are
computed once and shared by its runs (separate launches, fused append, shared
prefix), which must all give the same outputs.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle_side import OracleBatch, assert_attention_close, compact_pools
from test_gpu_parity import DEV, _bits

pytestmark = pytest.mark.gpu
CORES = len(os.sched_getaffinity(0))
CHUNK_BLOCKS = 2048


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


_cache = {}


def _oracle(w):
    """(OracleBatch of the whole batch, its fp64 attention), one workload at a time."""
    if w.name not in _cache:
        _cache.clear()
        ob = OracleBatch(w)
        _cache[w.name] = (ob, ob.attention(nthreads=CORES))
    return _cache[w.name]


def _compare_blocks(pool, blocks, expected):
    """pool[blocks[i]] == expected[i] bit for bit, in chunks of blocks."""
    for i in range(0, len(blocks), CHUNK_BLOCKS):
        idx = torch.tensor(blocks[i:i + CHUNK_BLOCKS], dtype=torch.long, device=DEV)
        assert np.array_equal(_bits(pool[idx]), expected[i:i + CHUNK_BLOCKS].view(np.uint16)), \
            "pool blocks %d.. differ from the oracle" % i


def _compare_sentinel(pool, blocks):
    for i in range(0, len(blocks), CHUNK_BLOCKS):
        idx = torch.tensor(blocks[i:i + CHUNK_BLOCKS], dtype=torch.long, device=DEV)
        assert (_bits(pool[idx]) == wl.SENTINEL_BITS).all(), "an unused block was written"


FULL = [
    ("llama7b", 0, "separate"), ("llama7b", 0, "fused"),
    ("bs_sweep_8", 0, "separate"), ("bs_sweep_8", 0, "fused"),
    ("bs_sweep_16", 0, "fused"),
    ("bs_sweep_32", 0, "separate"), ("bs_sweep_32", 0, "fused"),
    ("bs_sweep_64", 0, "separate"), ("bs_sweep_64", 0, "fused"),
    ("gqa", 512, "separate"), ("gqa", 512, "fused"), ("gqa", 0, "separate"), ("gqa", 0, "fused"),
]


@pytest.mark.parametrize("name,part,step", FULL, ids=["%s-%s-%s" % c for c in FULL])
def test_whole_batch(pkv, name, part, step):
    from batches import PagedBatch
    w = wl.get(name)
    gb = PagedBatch(w, DEV)
    ob, ref = _oracle(w)
    assert [gb.bm.block_table(s) for s in gb.seqs] == ob.tables
    assert np.array_equal(gb.slots_host, ob.new_slots)
    if step == "fused":
        pkv.paged_attention_decode_append(gb.out, gb.q, gb.k_new, gb.v_new, gb.key_cache,
                                          gb.value_cache, gb.block_tables, gb.context_lens,
                                          w.scale, gb.max_context_len, part)
    else:
        pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
        pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                                   gb.context_lens, w.scale, gb.max_context_len, part)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    # every block of the batch (the new row of every sequence included), bit for bit
    _compare_blocks(gb.key_cache, ob.blocks, ob.key_cache)
    _compare_blocks(gb.value_cache, ob.blocks, ob.value_cache)
    used = set(ob.blocks)
    unused = [b for b in range(w.num_blocks) if b not in used]
    _compare_sentinel(gb.key_cache, unused)
    _compare_sentinel(gb.value_cache, unused)
    assert_attention_close(gb.out.cpu().numpy(), ref, record="%s %s part=%d" % (name, step, part),
                           literal=True)
    del gb
    torch.cuda.empty_cache()


# ---- the copy-on-write workload: every sample after the first and the last step ----------

_cow = {}


def _cow_expected():
    """The oracle side of the cow workload: its block-manager model run through all decode
    steps (slots, pairs, tables), and every sample's expected output after step 1 and after
    the last step, from the oracle's own pools."""
    if _cow:
        return _cow
    w = wl.get("cow")
    Hk, D, bs, N = w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks
    model = oracle.BlockManagerModel(N, bs, free_order=wl.free_order(N, w.seed))
    samples, prompt_of = [], {}
    for p in range(w.prompts):
        s = model.add_seq(w.prompt_len)
        for x in [s] + model.fork(s, w.samples - 1):
            samples.append(x)
            prompt_of[x] = p
    prompt_kv = [wl.sequence_kv(w.seed, p, w.prompt_len, Hk, D) for p in range(w.prompts)]
    steps = []
    news = []
    refs = {}
    for step in range(w.decode_steps):
        slots = [model.append_token(s) for s in samples]
        pairs = model.take_copies()
        k, v = wl.decode_kv(w.seed, step, w.num_seqs, Hk, D)
        news.append((k, v))
        steps.append((slots, pairs))
        if step in (0, w.decode_steps - 1):
            entries = []
            for i, s in enumerate(samples):
                k0, v0 = prompt_kv[prompt_of[s]]
                entries.append((model.block_table(s),
                                np.concatenate([k0, np.stack([x[0][i] for x in news])]),
                                np.concatenate([v0, np.stack([x[1][i] for x in news])])))
            kc, vc, t, lens, relabel = compact_pools(entries, bs, Hk, D)
            q = wl.decode_q(w.seed, step, w.num_seqs, w.num_heads, D)
            ref = oracle.paged_attention(q, kc, vc, t, lens, w.scale, bs, Hk, nthreads=CORES)
            if step == w.decode_steps - 1:
                _cow["pools"] = (list(relabel), kc, vc)
            refs[step] = ref
            del entries
    _cow.update(samples=samples, steps=steps, refs=refs)
    return _cow


@pytest.mark.parametrize("step_kind", ["separate", "fused", "shared"])
def test_cow_whole_batch(pkv, step_kind):
    from batches import CowBatch
    w = wl.get("cow")
    exp = _cow_expected()
    gb = CowBatch(w, DEV)
    assert gb.samples == exp["samples"]
    last = w.decode_steps - 1
    for step in range(w.decode_steps):
        host = gb.prepare_step()
        slots, pairs = exp["steps"][step]
        assert host["slots"].tolist() == slots
        assert host["pairs"].tolist() == [list(x) for x in pairs]
        if step == 0:
            assert len(pairs) == w.prompts * (w.samples - 1)
        dev = {k: torch.from_numpy(host[k]).to(DEV) for k in ("tables", "lens", "q", "k", "v")}
        out = torch.empty_like(dev["q"])
        if step_kind == "separate":
            gb.run_cache_updates(host)
            pkv.paged_attention_decode(out, dev["q"], gb.key_cache, gb.value_cache, dev["tables"],
                                       dev["lens"], w.scale, gb.max_context_len)
        else:
            if len(host["pairs"]):
                pkv.copy_blocks([gb.key_cache], [gb.value_cache],
                                torch.from_numpy(host["pairs"]).to(DEV))
            if step_kind == "fused":
                pkv.paged_attention_decode_append(out, dev["q"], dev["k"], dev["v"],
                                                  gb.key_cache, gb.value_cache, dev["tables"],
                                                  dev["lens"], w.scale, gb.max_context_len)
            else:
                pre, groups = pkv.prefix_groups(host["tables"], host["lens"], w.block_size, 8)
                assert len(groups) == w.prompts
                pkv.paged_attention_decode_shared_prefix(
                    out, dev["q"], gb.key_cache, gb.value_cache, dev["tables"], dev["lens"],
                    torch.from_numpy(pre).to(DEV), torch.from_numpy(groups).to(DEV), w.scale,
                    gb.max_context_len, k_new=dev["k"], v_new=dev["v"],
                    max_prefix_tokens=int(groups[:, 0].max()) * w.block_size,
                    max_suffix_tokens=int((host["lens"] - pre).max()))
        if step in (0, last):
            torch.cuda.synchronize()
            assert pkv.device_errors() == 0
            assert_attention_close(out.cpu().numpy(), exp["refs"][step],
                                   record="cow %s after step %d" % (step_kind, step + 1),
                                   literal=True)
    blocks, kc, vc = exp["pools"]
    _compare_blocks(gb.key_cache, blocks, kc)
    _compare_blocks(gb.value_cache, blocks, vc)
    del gb
    torch.cuda.empty_cache()
