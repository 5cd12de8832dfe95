"""GPU parity of the shared-prefix decode against the CPU oracle.

Batches of forked sequences: prompts written once, forked into samples that
share the prompt's blocks, each sample then appends private tokens (copy-on-write
copies first where the block manager asks for them), and one decode step.  The
expected output of every sequence is the oracle's attention over that
sequence's own K/V gathered through its own table -- sharing is invisible in the
result.  Cache bytes must match the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from oracle_side import assert_attention_close, compact_pools
from test_gpu_parity import DEV, _bits

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


class ForkBatch:
    """Prompts forked into samples with private tokens, then one decode step."""

    def __init__(self, pkv, H, Hk, D, bs, prompts, samples, extra, seed=3000):
        from paged_kv_cache_393_b200 import BlockManager
        from batches import sentinel_pools
        self.H, self.Hk, self.D, self.bs = H, Hk, D, bs
        total = len(prompts) * samples
        N = sum(-(-L // bs) for L in prompts) + total * (max(extra(i) for i in range(total)) // bs + 3)
        self.N = N
        self.bm = BlockManager(N, bs, free_order=wl.free_order(N, seed))
        self.model = oracle.BlockManagerModel(N, bs, free_order=wl.free_order(N, seed))
        self.kc, self.vc = sentinel_pools(N, Hk, bs, D, DEV)
        self.seqs, kv = [], []
        for pi, L in enumerate(prompts):
            s = self.bm.add_seq(L)
            assert self.model.add_seq(L) == s
            k, v = wl.sequence_kv(seed, pi, L, Hk, D)
            self._write(k, v, self.model.slots_of(s))
            kids = self.bm.fork(s, samples - 1)
            assert self.model.fork(s, samples - 1) == kids
            for x in [s] + kids:
                self.seqs.append(x)
                kv.append((k, v))
        self.new = []
        for i, x in enumerate(self.seqs):
            n = extra(i)
            kp, vp = wl.sequence_kv(seed, 100_000 + i, n + 1, Hk, D)
            slots = []
            for _ in range(n):
                slot = self.bm.append_token(x)
                assert self.model.append_token(x) == slot
                slots.append(slot)
            self._copies()
            if n:
                self._write(kp[:n], vp[:n], slots)
            kv[i] = (np.concatenate([kv[i][0], kp[:n]]), np.concatenate([kv[i][1], vp[:n]]))
            self.new.append((kp[n], vp[n]))
        # the decode step: one new token per sequence
        self.slots = self.bm.append_tokens(self.seqs)
        assert self.slots.tolist() == [self.model.append_token(x) for x in self.seqs]
        self._copies()
        self.kv = [(np.concatenate([k, nk[None]]), np.concatenate([v, nv[None]]))
                   for (k, v), (nk, nv) in zip(kv, self.new)]
        self.lens_host = np.array([k.shape[0] for k, _ in self.kv], np.int32)
        self.max_blocks = int(max(len(self.bm.block_table(x)) for x in self.seqs))
        self.tables_host, lens = self.bm.build_batch(self.seqs, self.max_blocks)
        assert lens.tolist() == self.lens_host.tolist()
        B = len(self.seqs)
        self.q_host = wl.decode_q(seed, 0, B, H, D)
        self.q = torch.from_numpy(self.q_host).to(DEV)
        self.k_new = torch.from_numpy(np.stack([a for a, _ in self.new])).to(DEV)
        self.v_new = torch.from_numpy(np.stack([b for _, b in self.new])).to(DEV)
        self.tables = torch.from_numpy(self.tables_host).to(DEV)
        self.lens = torch.from_numpy(self.lens_host).to(DEV)
        self.out = torch.empty((B, H, D), dtype=torch.float16, device=DEV)
        self.max_context_len = int(self.lens_host.max())

    def _write(self, k, v, slots):
        import paged_kv_cache_393_b200 as m
        m.reshape_and_cache(torch.from_numpy(np.ascontiguousarray(k)).to(DEV),
                            torch.from_numpy(np.ascontiguousarray(v)).to(DEV), self.kc, self.vc,
                            torch.tensor(np.asarray(slots, np.int64), device=DEV))

    def _copies(self):
        import paged_kv_cache_393_b200 as m
        pairs = self.bm.take_copies()
        assert pairs.tolist() == [list(p) for p in self.model.take_copies()]
        if len(pairs):
            m.copy_blocks([self.kc], [self.vc], torch.from_numpy(pairs).to(DEV))

    def write_new_tokens(self):
        import paged_kv_cache_393_b200 as m
        m.reshape_and_cache(self.k_new, self.v_new, self.kc, self.vc,
                            torch.from_numpy(self.slots).to(DEV))

    def groups(self, max_members=None):
        import paged_kv_cache_393_b200 as m
        mm = max_members or max(1, 8 // (self.H // self.Hk))
        pre, groups = m.prefix_groups(self.tables_host, self.lens_host, self.bs, mm)
        return pre, groups

    def expected(self, sample):
        entries = [(self.model.block_table(self.seqs[i]),) + self.kv[i] for i in sample]
        kc, vc, t, l, relabel = compact_pools(entries, self.bs, self.Hk, self.D)
        assert l.tolist() == self.lens_host[sample].tolist()
        ref = oracle.paged_attention(self.q_host[sample], kc, vc, t, l, 1.0 / self.D ** 0.5,
                                     self.bs, self.Hk, nthreads=8)
        return ref, kc, vc, relabel


def _bounds(fb, pre, groups):
    """Host upper bounds of the prefix and suffix lengths (they size the grids)."""
    mp = int(groups[:, 0].max()) * fb.bs if len(groups) else 0
    return mp, int((fb.lens_host - pre).max())


def _run(pkv, fb, fused, partition_size=0, sample=None, max_members=None, expect_groups=True,
         bounds=True):
    pre, groups = fb.groups(max_members)
    mp, ms = _bounds(fb, pre, groups) if bounds else (0, 0)
    if expect_groups:
        assert len(groups) > 0
    pre_d = torch.from_numpy(pre).to(DEV)
    groups_d = torch.from_numpy(groups).to(DEV) if len(groups) else \
        torch.zeros((0, 9), dtype=torch.int32, device=DEV)
    if not fused:
        fb.write_new_tokens()
    pkv.paged_attention_decode_shared_prefix(
        fb.out, fb.q, fb.kc, fb.vc, fb.tables, fb.lens, pre_d, groups_d, 1.0 / fb.D ** 0.5,
        fb.max_context_len, partition_size, k_new=fb.k_new if fused else None,
        v_new=fb.v_new if fused else None, max_prefix_tokens=mp, max_suffix_tokens=ms)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    sample = list(range(len(fb.seqs))) if sample is None else sample
    ref, kc, vc, relabel = fb.expected(sample)
    idx = torch.tensor(list(relabel), dtype=torch.long, device=DEV)
    assert np.array_equal(_bits(fb.kc[idx]), kc.view(np.uint16))
    assert np.array_equal(_bits(fb.vc[idx]), vc.view(np.uint16))
    # blocks no sequence references were never written
    used = {b for x in fb.seqs for b in fb.model.block_table(x)}
    free = [b for b in range(fb.N) if b not in used]
    if free:
        fi = torch.tensor(free, dtype=torch.long, device=DEV)
        assert (_bits(fb.kc[fi]) == wl.SENTINEL_BITS).all()
        assert (_bits(fb.vc[fi]) == wl.SENTINEL_BITS).all()
    err = assert_attention_close(fb.out.cpu().numpy()[sample], ref)
    # the plain decode over the same cache agrees too
    plain = torch.empty_like(fb.out)
    pkv.paged_attention_decode(plain, fb.q, fb.kc, fb.vc, fb.tables, fb.lens, 1.0 / fb.D ** 0.5,
                               fb.max_context_len, partition_size if partition_size > 0 else 0)
    assert_attention_close(fb.out.cpu().numpy(), plain.cpu().numpy())
    return err


CASES = [
    # (name, H, Hk, D, bs, prompts, samples, extra(i), partition_size)
    ("mha128_bs16", 8, 8, 128, 16, [1000, 37, 300], 8, lambda i: (7 * i) % 23, 0),
    ("mha128_bs16_p64", 8, 8, 128, 16, [1000, 37, 300], 8, lambda i: (7 * i) % 23, 64),
    ("mha64_bs8_p32", 4, 4, 64, 8, [200, 9], 5, lambda i: i % 4, 32),
    ("mha128_bs64", 4, 4, 128, 64, [700, 130], 3, lambda i: 40 * i, 0),
    ("gqa2_d128_bs32", 8, 4, 128, 32, [900, 100], 6, lambda i: (5 * i) % 40, 0),
    ("gqa4_d64_bs16_p128", 16, 4, 64, 16, [600], 4, lambda i: i, 128),
    ("gqa8_no_groups", 16, 2, 128, 16, [300], 3, lambda i: i, 0),
    ("mha64_bs32", 4, 4, 64, 32, [500, 70], 4, lambda i: (9 * i) % 50, 0),
    ("mha64_bs64_p128", 4, 4, 64, 64, [600, 130], 3, lambda i: 30 * i, 128),
    ("gqa2_d128_bs8", 8, 4, 128, 8, [400, 45], 4, lambda i: (3 * i) % 20, 0),
    ("single_samples", 4, 4, 128, 16, [50, 60, 70], 1, lambda i: 0, 0),
]


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_forked_batches(pkv, case, fused):
    name, H, Hk, D, bs, prompts, samples, extra, part = case
    fb = ForkBatch(pkv, H, Hk, D, bs, prompts, samples, extra)
    # the separate runs size the grids from max_context_len, the fused ones from host bounds
    _run(pkv, fb, fused, part, expect_groups=samples > 1 and H // Hk < 8, bounds=fused)


@pytest.mark.parametrize("H,Hk", [(8, 8), (8, 2)], ids=["mha", "gqa"])
def test_bounds_below_the_real_lengths(pkv, H, Hk):
    fb = ForkBatch(pkv, H, Hk, 128, 16, [1000, 300], 4, lambda i: 100 * i)
    pre, groups = fb.groups()
    mp, ms = _bounds(fb, pre, groups)
    fb.write_new_tokens()
    ref, _, _, _ = fb.expected(list(range(len(fb.seqs))))

    def run(mp_, ms_):
        fb.out.fill_(float("nan"))
        pkv.paged_attention_decode_shared_prefix(
            fb.out, fb.q, fb.kc, fb.vc, fb.tables, fb.lens, torch.from_numpy(pre).to(DEV),
            torch.from_numpy(groups).to(DEV), 1.0 / fb.D ** 0.5, fb.max_context_len, 64,
            max_prefix_tokens=mp_, max_suffix_tokens=ms_)
        return pkv.device_errors()

    # the persistent prefix pass takes every group's items from its queue: a prefix bound
    # one partition short only sizes its grid, and the result is still complete
    assert run(mp - 512, ms) == 0
    assert_attention_close(fb.out.cpu().numpy(), ref)
    # a suffix bound one partition short leaves work undone and says so
    assert run(mp, 16) & pkv.DEVERR_PREFIX


def test_more_sequences_than_the_persistent_grid(pkv):
    # 1040 grouped-query sequences: the suffix pass runs one CTA per item
    fb = ForkBatch(pkv, 4, 2, 64, 16, [40 + 3 * i for i in range(260)], 4, lambda i: i % 5)
    assert len(fb.seqs) > 1024
    _run(pkv, fb, True, 32, sample=[0, 1, 2, 3, 517, 1039])


@pytest.mark.parametrize("part", [0, 64])
def test_many_short_suffixes(pkv, part):
    # 320 sequences x 16 head pairs: several waves of suffix CTAs, every suffix within one
    # partition (folded in place, no merge), over 40 groups whose prefixes end at assorted
    # block counts.  The 9-token prompts share no whole block, so their samples have no
    # prefix and sit among the grouped ones.
    prompts = [9 + 53 * (i % 13) for i in range(40)]
    fb = ForkBatch(pkv, 32, 32, 128, 16, prompts, 8, lambda i: (11 * i) % 41)
    assert len(fb.seqs) == 320
    pre, _ = fb.groups()
    assert (pre == 0).sum() >= 8 and (pre > 0).sum() >= 200
    _run(pkv, fb, True, part)


def test_more_groups_than_the_persistent_grid(pkv):
    # 1100 prompts of 16-55 tokens, 2 samples each: 1100 groups, so the prefix pass runs
    # one CTA per item (the persistent grid takes up to 1024 groups)
    fb = ForkBatch(pkv, 4, 4, 64, 16, [16 + i % 40 for i in range(1100)], 2, lambda i: i % 3)
    pre, groups = fb.groups()
    assert len(groups) == 1100
    _run(pkv, fb, True, 0)


def test_inconsistent_groups_are_flagged_not_faulted(pkv):
    fb = ForkBatch(pkv, 8, 8, 128, 16, [300, 200], 4, lambda i: i)
    pre, groups = fb.groups()
    assert len(groups) == 2
    bad = groups.copy()
    bad[0, 2] = int(bad[1, 1])                       # a member of the other prompt
    pre_bad = pre.copy()
    pre_bad[5] = 7                                   # not a whole number of blocks
    fb.write_new_tokens()
    for p_host, g_host in ((pre, bad), (pre_bad, groups)):
        pkv.paged_attention_decode_shared_prefix(
            fb.out, fb.q, fb.kc, fb.vc, fb.tables, fb.lens, torch.from_numpy(p_host).to(DEV),
            torch.from_numpy(g_host).to(DEV), 1.0 / fb.D ** 0.5, fb.max_context_len)
        assert pkv.device_errors() & pkv.DEVERR_PREFIX
    # a group naming a sequence outside the batch, or a prefix longer than the table
    g2 = groups.copy()
    g2[0, 3] = 10_000
    g3 = groups.copy()
    g3[1, 0] = 10_000
    for g_host in (g2, g3):
        pkv.paged_attention_decode_shared_prefix(
            fb.out, fb.q, fb.kc, fb.vc, fb.tables, fb.lens, torch.from_numpy(pre).to(DEV),
            torch.from_numpy(g_host).to(DEV), 1.0 / fb.D ** 0.5, fb.max_context_len)
        assert pkv.device_errors() & pkv.DEVERR_PREFIX
    # (the outputs of the flagged members are unspecified)
    # the consistent groups still give the oracle's result afterwards
    pkv.paged_attention_decode_shared_prefix(
        fb.out, fb.q, fb.kc, fb.vc, fb.tables, fb.lens, torch.from_numpy(pre).to(DEV),
        torch.from_numpy(groups).to(DEV), 1.0 / fb.D ** 0.5, fb.max_context_len)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    ref, _, _, _ = fb.expected(list(range(len(fb.seqs))))
    assert_attention_close(fb.out.cpu().numpy(), ref)


@pytest.mark.parametrize("H,Hk", [(8, 8), (8, 2)], ids=["mha", "gqa"])
def test_decode_session_with_shared_prefixes(pkv, H, Hk):
    # the host-buffer call: inputs from pinned host memory, groups built on the host per step
    fb = ForkBatch(pkv, H, Hk, 128, 16, [700, 90], 4, lambda i: (11 * i) % 30)
    sess = pkv.DecodeSession(fb.kc, fb.vc, len(fb.seqs), H, fb.max_blocks, fb.max_context_len,
                             scale=1.0 / 128 ** 0.5, shared_prefix=True)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()  # noqa: E731
    out = torch.empty((len(fb.seqs), H, 128), dtype=torch.float16).pin_memory()
    kn = np.stack([a for a, _ in fb.new])
    vn = np.stack([b for _, b in fb.new])
    sess.step(pin(fb.q_host), pin(kn), pin(vn), pin(fb.tables_host), pin(fb.lens_host), out)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    # 4 samples per prompt: one group each with MHA, two of 2 members with 4 heads per kv head
    assert sess._last_groups == (2 if H == Hk else 4)
    ref, kc, vc, relabel = fb.expected(list(range(len(fb.seqs))))
    idx = torch.tensor(list(relabel), dtype=torch.long, device=DEV)
    assert np.array_equal(_bits(fb.kc[idx]), kc.view(np.uint16))
    assert_attention_close(out.numpy(), ref)
