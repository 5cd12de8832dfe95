"""paged_attention_decode_noalloc: the decode call for callers that cannot allocate.

Engines that reserve nearly all GPU memory for their block pool, plugins inside
a runtime that owns the allocator, and latency-bound loops that cannot afford
cudaMalloc cannot pass a workspace; this entry point takes its scratch
from an array built into the library instead.  The test calls it through the C
ABI, twice in a row on the same inputs, and checks each result against the
regular paged_attention_decode with a caller-owned workspace, within the
attention tolerance of the other parity tests.  It runs last so that a failure
here cannot hide the other GPU tests, and it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from paged_kv_cache_393_b200 import _native, build
    build.build()
    lib = _native.load_library()
    fn = lib.paged_attention_decode_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [P, P, P, P, P, P, ctypes.c_float] + [I] * 9 + [P]
    fn.restype = I
    return lib


def _workload(name, H, Hk, D, bs, lens):
    N = sum(-(-L // bs) for L in lens) + 8
    return wl.Workload(name, len(lens), H, Hk, D, bs, N, 3000, "fixed", fixed_lens=tuple(lens))


CASES = [
    (_workload("gqa_split", 16, 2, 128, 16, [1, 300, 1030]), 64),      # tensor-core kernel + merge
    (_workload("mha_split", 8, 8, 64, 8, [5, 129, 700]), 32),          # CUDA-core kernel + merge
    (_workload("auto", 8, 8, 128, 16, [17, 2500]), 0),                 # library's choice (splits)
    (_workload("single", 4, 4, 128, 16, [40, 90]), -1),                # no scratch needed
    (_workload("gqa_single", 16, 2, 128, 16, [40, 900]), -1),          # only the work counter
    # the library's split would need ~19 MB of scratch (128 x 32 heads x 9 partitions of 1024
    # tokens): more than the built-in 16 MiB, so the call falls back to a single pass
    (_workload("auto_fallback", 32, 32, 128, 16, [8200] + [5 + i % 40 for i in range(127)]), 0),
]


@pytest.mark.parametrize("w,part", CASES, ids=[c[0].name for c in CASES])
def test_matches_the_regular_entry_point_twice(lib, w, part):
    import paged_kv_cache_393_b200 as pkv
    from batches import PagedBatch
    gb = PagedBatch(w, DEV)
    pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots)
    ref = torch.empty_like(gb.out)
    pkv.paged_attention_decode(ref, gb.q, gb.key_cache, gb.value_cache, gb.block_tables,
                               gb.context_lens, w.scale, gb.max_context_len, part)
    torch.cuda.synchronize()
    ref = ref.double().cpu().numpy()
    assert np.isfinite(ref).all()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out = torch.full_like(gb.out, float("nan"))
        st = lib.paged_attention_decode_noalloc(
            out.data_ptr(), gb.q.data_ptr(), gb.key_cache.data_ptr(), gb.value_cache.data_ptr(),
            gb.block_tables.data_ptr(), gb.context_lens.data_ptr(), w.scale, w.block_size,
            w.num_kv_heads, w.num_seqs, w.num_heads, w.head_dim, gb.max_blocks, w.num_blocks,
            gb.max_context_len, part, stream)
        assert st == 0, lib.pagedkv_last_error()
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert (np.abs(got - ref) <= 2e-3 + 1e-2 * np.abs(ref)).all()
    assert pkv.device_errors() == 0


def test_rejects_a_split_larger_than_its_scratch(lib):
    # 256 sequences x 64 heads x 32 partitions of 512 tokens need ~273 MB of scratch
    B, H, Hk, D, bs, maxlen = 256, 64, 8, 128, 16, 16384
    need = lib.paged_attention_workspace_bytes(B, H, Hk, D, bs, maxlen, 512)
    assert need > (16 << 20)
    fake = 1 << 20          # never dereferenced: the call is rejected before any launch
    st = lib.paged_attention_decode_noalloc(fake, fake, fake, fake, fake, fake, 0.1, bs, Hk, B, H,
                                            D, maxlen // bs, 4096, maxlen, 512, None)
    assert st == -4         # PAGEDKV_EWORKSPACE
    assert b"built-in scratch" in lib.pagedkv_last_error()
