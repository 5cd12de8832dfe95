"""GPU parity of paged_decode_step_host: one decode step driven from host buffers.

The inputs are host arrays (pinned and pageable); the call uploads them, runs the
copy-on-write copies, writes each new token at position L-1 through the tables,
attends, and downloads the output.  Expected: the oracle's cache bytes (bit for
bit) and the oracle's attention (|gpu - oracle| <= 2e-3 + 1e-2 |oracle|).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle_side import OracleBatch, assert_attention_close, compact_pools
from test_gpu_parity import DEV, _bits, _fixed

pytestmark = pytest.mark.gpu


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


def _host(a, pinned):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.pin_memory() if pinned else t


CASES = [
    (_fixed("host_mha", 8, 8, 128, 16, [1, 15, 16, 17, 300, 700]), 0),
    (_fixed("host_mha_split", 8, 8, 128, 16, [1, 15, 16, 17, 300, 700]), 64),
    (_fixed("host_gqa", 16, 2, 128, 16, [1, 16, 17, 300, 1030]), 0),
    (_fixed("host_gqa_bs8_split", 8, 2, 64, 8, [3, 8, 9, 200]), 16),
]


def _ragged(n, hi, seed):
    """n context lengths in [1, hi], with block-edge lengths at the chunks' first and last
    sequences (whatever the chunking) and at the batch's ends."""
    lens = np.random.default_rng(seed).integers(1, hi + 1, n)
    edges = [1, 15, 16, 17, 31, 32, 33, 2]
    for i, j in enumerate([0, n - 1, n // 6, n // 6 - 1, n // 2, n // 2 - 1, 5 * n // 6,
                           5 * n // 6 - 1]):
        lens[j] = edges[i]
    return [int(x) for x in lens]


# at least 128 sequences: the host step splits the batch into chunks (3 or 4 here) pipelined
# over two copy streams and two compute streams
CASES += [
    (_fixed("host_chunked_mha", 8, 8, 64, 16, _ragged(200, 400, 1)), 0),
    (_fixed("host_chunked_mha_split", 8, 8, 128, 16, _ragged(256, 700, 2)), 64),
    (_fixed("host_chunked_gqa", 16, 2, 128, 16, _ragged(256, 900, 3)), 0),
]


@pytest.mark.parametrize("pinned", [True, False], ids=["pinned", "pageable"])
@pytest.mark.parametrize("w,part", CASES, ids=[c[0].name for c in CASES])
def test_host_step_matches_the_oracle(pkv, w, part, pinned):
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    ob = OracleBatch(w)
    B, H, D = w.num_seqs, w.num_heads, w.head_dim
    sess = pkv.DecodeSession(gb.key_cache, gb.value_cache, B, H, gb.max_blocks,
                             gb.max_context_len, w.scale, part)
    out = _host(np.full((B, H, D), np.nan, np.float16), pinned)
    stream = torch.cuda.Stream()
    sess.step(_host(gb.q_host, pinned), _host(gb.k_new_host, pinned),
              _host(gb.v_new_host, pinned), _host(gb.tables_host, pinned),
              _host(gb.lens_host, pinned), out, stream=stream)
    stream.synchronize()
    assert pkv.device_errors() == 0
    idx = torch.tensor(ob.blocks, dtype=torch.long, device=DEV)
    assert np.array_equal(_bits(gb.key_cache[idx]), ob.key_cache.view(np.uint16))
    assert np.array_equal(_bits(gb.value_cache[idx]), ob.value_cache.view(np.uint16))
    assert_attention_close(out.numpy().astype(np.float64), ob.attention())


CHUNKED = [c for c in CASES if c[0].num_seqs >= 128]


@pytest.mark.parametrize("w,part", CHUNKED, ids=[c[0].name for c in CHUNKED])
def test_chunked_step_equals_one_call(pkv, w, part):
    # every chunk is split as the whole batch is, so the pipelined step computes each
    # (sequence, head) exactly as one fused call over the batch does: the outputs agree
    # bit for bit
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    B, H, D = w.num_seqs, w.num_heads, w.head_dim
    sess = pkv.DecodeSession(gb.key_cache, gb.value_cache, B, H, gb.max_blocks,
                             gb.max_context_len, w.scale, part)
    out = _host(np.full((B, H, D), np.nan, np.float16), True)
    stream = torch.cuda.Stream()
    sess.step(_host(gb.q_host, True), _host(gb.k_new_host, True), _host(gb.v_new_host, True),
              _host(gb.tables_host, True), _host(gb.lens_host, True), out, stream=stream)
    stream.synchronize()
    # one call over the whole batch (it stores the same new rows again)
    need = pkv.paged_attention_workspace_bytes(B, H, w.num_kv_heads, D, w.block_size,
                                               gb.max_context_len, part)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=DEV)
    one = torch.full((B, H, D), float("nan"), dtype=torch.float16, device=DEV)
    pkv.paged_attention_decode_append(one, gb.q, gb.k_new, gb.v_new, gb.key_cache,
                                      gb.value_cache, gb.block_tables, gb.context_lens, w.scale,
                                      gb.max_context_len, part, ws)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    assert np.array_equal(out.numpy().view(np.uint16), _bits(one))


# the copy-on-write workload's shape at 8 prompts (64 samples, one chunk), and 16 prompts of
# 100 tokens (128 samples: two chunks, the copies ahead of both)
COW = {"cow_small": lambda: wl.get("cow_small"),
       "cow_128_chunked": lambda: wl.Workload("cow_128_chunked", 128, 8, 8, 64, 16, 2048, 1004,
                                              "cow", prompts=16, prompt_len=100, samples=8,
                                              decode_steps=3)}


@pytest.mark.parametrize("cow", list(COW))
@pytest.mark.parametrize("shared", [False, True], ids=["plain", "shared_prefix"])
def test_host_step_copy_on_write_steps(pkv, shared, cow):
    # step 0 copies the shared partial tails (7 per prompt), then two more steps; every
    # step goes through the host call
    from batches import CowBatch
    w = COW[cow]()
    B, H, Hk, D, bs, N = w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, \
        w.num_blocks
    gb = CowBatch(w, DEV)
    model = oracle.BlockManagerModel(N, bs, free_order=wl.free_order(N, w.seed))
    samples, prompt_of = [], {}
    for p in range(w.prompts):
        s = model.add_seq(w.prompt_len)
        for x in [s] + model.fork(s, w.samples - 1):
            samples.append(x)
            prompt_of[x] = p
    assert samples == gb.samples
    sess = pkv.DecodeSession(gb.key_cache, gb.value_cache, B, H, gb.max_blocks,
                             gb.max_context_len, w.scale, max_pairs=B, shared_prefix=shared)
    out = torch.empty((B, H, D), dtype=torch.float16).pin_memory()
    news = []
    for step in range(3):
        host = gb.prepare_step()
        assert host["slots"].tolist() == [model.append_token(s) for s in samples]
        pairs = model.take_copies()
        assert host["pairs"].tolist() == [list(x) for x in pairs]
        assert len(pairs) == (w.prompts * (w.samples - 1) if step == 0 else 0)
        sess.step(*[_host(host[k], True) for k in ("q", "k", "v", "tables", "lens")], out,
                  pairs=_host(host["pairs"], True) if len(pairs) else None)
        torch.cuda.synchronize()
        news.append((host["k"], host["v"]))
        if shared:
            assert sess._last_groups == w.prompts
    assert pkv.device_errors() == 0
    entries = []
    for i, s in enumerate(samples):
        k0, v0 = wl.sequence_kv(w.seed, prompt_of[s], w.prompt_len, Hk, D)
        entries.append((model.block_table(s), np.concatenate([k0, np.stack([k[i] for k, _ in news])]),
                        np.concatenate([v0, np.stack([v[i] for _, v in news])])))
    kc_o, vc_o, t_o, l_o, relabel = compact_pools(entries, bs, Hk, D)
    idx = torch.tensor(list(relabel), dtype=torch.long, device=DEV)
    assert np.array_equal(_bits(gb.key_cache[idx]), kc_o.view(np.uint16))
    assert np.array_equal(_bits(gb.value_cache[idx]), vc_o.view(np.uint16))
    ref = oracle.paged_attention(host["q"], kc_o, vc_o, t_o, l_o, w.scale, bs, Hk, nthreads=16)
    assert_attention_close(out.numpy().astype(np.float64), ref)


def test_host_step_refuses_overlapping_pairs_before_enqueueing(pkv):
    from paged_kv_cache_393_b200 import PagedKVError
    from batches import PagedBatch
    w = _fixed("host_refuse", 4, 4, 64, 16, [5, 40])
    gb = PagedBatch(w, DEV)
    before = _bits(gb.key_cache)
    sess = pkv.DecodeSession(gb.key_cache, gb.value_cache, 2, 4, gb.max_blocks,
                             gb.max_context_len, w.scale, max_pairs=2)
    out = torch.empty((2, 4, 64), dtype=torch.float16)
    bad = np.array([[1, 2], [2, 3]], np.int64)     # block 2 is written and read
    with pytest.raises(PagedKVError):
        sess.step(gb.q_host, gb.k_new_host, gb.v_new_host, gb.tables_host, gb.lens_host, out,
                  pairs=bad)
    torch.cuda.synchronize()
    assert np.array_equal(before, _bits(gb.key_cache))
