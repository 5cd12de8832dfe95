"""GPU parity of the multi-layer decode step (LayeredDecodeStep, one CUDA graph).

Every layer has its own pools and contents (K/V drawn from a per-layer seed) but
the same block tables; after the graph replays, each layer's output must match
the oracle's attention over that layer's K/V and each layer's pools must hold
the oracle's bytes, new rows included.  Copy-on-write copies reach every layer.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle_side import assert_attention_close, compact_pools
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


def _layer_seed(w, l):
    return w.seed + 7919 * l


def _build(pkv, w, layers):
    from batches import PagedBatch, sentinel_pools
    gb = PagedBatch(w, DEV)                       # tables, lengths and layer 0's pools
    lens = gb.lens_host
    kcs, vcs = [gb.key_cache], [gb.value_cache]
    for l in range(1, layers):
        kc, vc = sentinel_pools(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, DEV)
        kvs = wl.sequences_kv(_layer_seed(w, l), range(w.num_seqs), lens, w.num_kv_heads,
                              w.head_dim)
        ks, vs, slots = [], [], []
        for b, (k, v) in enumerate(kvs):
            L = int(lens[b])
            t = np.asarray(gb.tables_host[b][:-(-L // w.block_size)], np.int64)
            i = np.arange(L - 1)
            ks.append(k[:L - 1])
            vs.append(v[:L - 1])
            slots.append(t[i // w.block_size] * w.block_size + i % w.block_size)
        pkv.reshape_and_cache(torch.from_numpy(np.concatenate(ks)).to(DEV),
                              torch.from_numpy(np.concatenate(vs)).to(DEV), kc, vc,
                              torch.from_numpy(np.concatenate(slots)).to(DEV))
        kcs.append(kc)
        vcs.append(vc)
    return gb, kcs, vcs


def _layer_inputs(w, gb, l):
    if l == 0:
        return gb.q_host, gb.k_new_host, gb.v_new_host
    s = _layer_seed(w, l)
    kvs = wl.sequences_kv(s, range(w.num_seqs), gb.lens_host, w.num_kv_heads, w.head_dim)
    kn = np.stack([k[int(L) - 1] for (k, _), L in zip(kvs, gb.lens_host)])
    vn = np.stack([v[int(L) - 1] for (_, v), L in zip(kvs, gb.lens_host)])
    return wl.decode_q(s, 0, w.num_seqs, w.num_heads, w.head_dim), kn, vn


@pytest.mark.parametrize("w,part", [
    (_fixed("layers_mha", 8, 8, 128, 16, [5, 300, 1030]), 0),
    (_fixed("layers_gqa", 16, 2, 128, 16, [17, 600, 1500]), 256),
], ids=["mha", "gqa_split"])
def test_layered_step_matches_the_oracle_per_layer(pkv, w, part):
    layers = 3
    gb, kcs, vcs = _build(pkv, w, layers)
    step = pkv.LayeredDecodeStep(kcs, vcs, w.num_seqs, w.num_heads, gb.max_blocks,
                                 gb.max_context_len, w.scale, part)
    ins = [_layer_inputs(w, gb, l) for l in range(layers)]
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)  # noqa: E731
    step.set_inputs(q=up(np.stack([x[0] for x in ins])), k_new=up(np.stack([x[1] for x in ins])),
                    v_new=up(np.stack([x[2] for x in ins])), block_tables=gb.block_tables,
                    context_lens=gb.context_lens)
    step.capture()
    step.out.zero_()
    step.replay()
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    model_tables = [list(gb.tables_host[b][:-(-int(L) // w.block_size)])
                    for b, L in enumerate(gb.lens_host)]
    for l in range(layers):
        s = w.seed if l == 0 else _layer_seed(w, l)
        kvs = wl.sequences_kv(s, range(w.num_seqs), gb.lens_host, w.num_kv_heads, w.head_dim)
        kc, vc, t, lens, relabel = compact_pools(
            [(model_tables[b],) + kvs[b] for b in range(w.num_seqs)], w.block_size,
            w.num_kv_heads, w.head_dim)
        idx = torch.tensor(list(relabel), dtype=torch.long, device=DEV)
        assert np.array_equal(_bits(kcs[l][idx]), kc.view(np.uint16))
        assert np.array_equal(_bits(vcs[l][idx]), vc.view(np.uint16))
        ref = oracle.paged_attention(ins[l][0], kc, vc, t, lens, w.scale, w.block_size,
                                     w.num_kv_heads)
        assert_attention_close(step.out[l].cpu().numpy(), ref)


def test_copy_on_write_pairs_reach_every_layer(pkv):
    w = _fixed("layers_cow", 4, 4, 64, 16, [40, 70], slack=8)
    gb, kcs, vcs = _build(pkv, w, 2)
    step = pkv.LayeredDecodeStep(kcs, vcs, w.num_seqs, w.num_heads, gb.max_blocks,
                                 gb.max_context_len, w.scale)
    step.set_inputs(block_tables=gb.block_tables, context_lens=gb.context_lens)
    src = int(gb.tables_host[1][0])
    dst = int(gb.bm.free_list()[-1])
    before = [(_bits(k), _bits(v)) for k, v in zip(kcs, vcs)]
    step.replay(pairs=torch.tensor([[src, dst]], dtype=torch.int64, device=DEV))
    torch.cuda.synchronize()
    for l in range(2):
        ek, ev = oracle.copy_blocks([before[l][0].view(np.float16)], [before[l][1].view(np.float16)],
                                    [(src, dst)])
        got_k, got_v = _bits(kcs[l]), _bits(vcs[l])
        # the copied block equals the oracle's; the step's new rows are written elsewhere
        assert np.array_equal(got_k[dst], ek[0].view(np.uint16)[dst])
        assert np.array_equal(got_v[dst], ev[0].view(np.uint16)[dst])


def test_capture_needs_the_inputs_first(pkv):
    # the capture's set-up run reads the tables: with the placeholders it would raise
    # device error bits the caller never caused, so capture() refuses instead
    w = _fixed("layers_capture", 4, 4, 64, 16, [40, 70], slack=8)
    gb, kcs, vcs = _build(pkv, w, 2)
    step = pkv.LayeredDecodeStep(kcs, vcs, w.num_seqs, w.num_heads, gb.max_blocks,
                                 gb.max_context_len, w.scale)
    with pytest.raises(RuntimeError, match="set_inputs"):
        step.capture()
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
