"""The C ABI: the library loads, exports every symbol the headers declare, and
rejects bad arguments on the host before touching a GPU (no compute call here)."""
import ctypes
import glob
import os
import re

import pytest

from conftest import ROOT

import paged_kv_cache_393_b200 as pkv
from paged_kv_cache_393_b200 import _native as nat


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_393_b200 import build
    build.build()
    return nat.load_library()


def _declared_functions():
    """Every function the headers declare (each declaration starts with PAGEDKV_API)."""
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(path, encoding="utf-8").read(), flags=re.S)
        for m in re.finditer(r"^PAGEDKV_API\s+[^;(]*?\b([A-Za-z_][A-Za-z0-9_]*)\s*\(", text, re.M):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"paged_attention_decode", "reshape_and_cache", "copy_blocks", "bm_create",
            "bm_append_token", "pagedkv_last_error"} <= names
    for name in sorted(names):
        assert hasattr(lib, name), name


def test_exports_are_limited_to_the_abi(lib):
    # the library is built with hidden visibility except for the extern "C" entry points
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", nat.library_path()], capture_output=True,
                         text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert _declared_functions() <= exported


FAKE = 1 << 20      # 16-byte aligned addresses never dereferenced: rejected before any launch


def _decode(lib, **over):
    a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, scale=0.125, bs=16, hk=4, b=2,
             h=8, d=128, maxblk=8, n=64, maxlen=100, part=0, ws=None, wsb=0)
    a.update(over)
    return lib.paged_attention_decode(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["cl"],
                                      a["scale"], a["bs"], a["hk"], a["b"], a["h"], a["d"],
                                      a["maxblk"], a["n"], a["maxlen"], a["part"], a["ws"],
                                      a["wsb"], None)


@pytest.mark.parametrize("over,code", [
    (dict(q=None), nat.EINVAL),
    (dict(out=FAKE + 8), nat.EINVAL),                 # misaligned
    (dict(d=96), nat.EUNSUPPORTED),
    (dict(bs=12, maxlen=90), nat.EUNSUPPORTED),
    (dict(h=6), nat.EINVAL),                          # not a multiple of the kv heads
    (dict(maxlen=200), nat.EINVAL),                   # beyond 8 blocks of 16
    (dict(maxlen=0), nat.EINVAL),
    (dict(part=24), nat.EINVAL),                      # not a multiple of 16
    (dict(part=-2), nat.EINVAL),
    (dict(part=32), nat.EWORKSPACE),                  # split without a workspace
    (dict(scale=float("nan")), nat.EINVAL),
    (dict(b=70000), nat.EUNSUPPORTED),
    (dict(part=16, maxlen=100000, maxblk=6250), nat.EUNSUPPORTED),   # > 4096 partitions
])
def test_decode_rejects_bad_arguments_on_the_host(lib, over, code):
    assert _decode(lib, **over) == code
    assert lib.pagedkv_last_error().decode()


def _decode_append(lib, kn=FAKE, vn=FAKE, **over):
    a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, scale=0.1, bs=16, hk=8, b=4,
             h=8, d=128, maxblk=8, n=64, maxlen=100, part=0, ws=None, wsb=0)
    a.update(over)
    return lib.paged_attention_decode_append(a["out"], a["q"], kn, vn, a["kc"], a["vc"], a["bt"],
                                             a["cl"], a["scale"], a["bs"], a["hk"], a["b"], a["h"],
                                             a["d"], a["maxblk"], a["n"], a["maxlen"], a["part"],
                                             a["ws"], a["wsb"], None)


@pytest.mark.parametrize("over,code", [
    (dict(kn=None), nat.EINVAL),
    (dict(vn=None), nat.EINVAL),
    (dict(kn=FAKE + 8), nat.EINVAL),                  # misaligned
    (dict(q=None), nat.EINVAL),
    (dict(d=96), nat.EUNSUPPORTED),
    (dict(part=32), nat.EWORKSPACE),
])
def test_fused_append_rejects_bad_arguments_on_the_host(lib, over, code):
    assert _decode_append(lib, **over) == code
    assert lib.pagedkv_last_error().decode()
    assert _decode_append(lib, b=0, kn=None, q=None) == nat.OK   # empty batch: no-op


def _decode_shared(lib, pre=FAKE, groups=FAKE, ng=1, kn=None, vn=None, **over):
    a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, cl=FAKE, scale=0.1, bs=16, hk=8, b=4,
             h=8, d=128, maxblk=8, n=64, maxlen=100, part=0, ws=None, wsb=0)
    a.update(over)
    return lib.paged_attention_decode_shared_prefix(
        a["out"], a["q"], kn, vn, a["kc"], a["vc"], a["bt"], a["cl"], pre, groups, ng,
        a.get("mp", 0), a.get("ms", 0), a["scale"],
        a["bs"], a["hk"], a["b"], a["h"], a["d"], a["maxblk"], a["n"], a["maxlen"], a["part"],
        a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(pre=None), nat.EINVAL),
    (dict(groups=None), nat.EINVAL),                  # groups required when num_groups > 0
    (dict(ng=-1), nat.EINVAL),
    (dict(ng=70000), nat.EINVAL),
    (dict(mp=-1), nat.EINVAL),
    (dict(ms=-5), nat.EINVAL),
    (dict(kn=FAKE), nat.EINVAL),                      # k_new without v_new
    (dict(kn=FAKE + 8, vn=FAKE), nat.EINVAL),         # misaligned
    (dict(bs=4, maxblk=32), nat.EUNSUPPORTED),        # the prefix pass runs on the tensor cores
    (dict(h=72, hk=4), nat.EUNSUPPORTED),             # more than 8 query heads per kv head
    (dict(), nat.EWORKSPACE),                         # always split: needs a workspace
])
def test_shared_prefix_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert _decode_shared(lib, **kw) == code
    assert lib.pagedkv_last_error().decode()


def test_shared_prefix_workspace_bytes(lib):
    # 32 bytes of work counters, then the partials: always split at 512 tokens (or the given
    # size), with one extra slot per (sequence, head): a prefix can end inside a partition
    f = lib.paged_attention_shared_prefix_workspace_bytes
    assert f(4, 8, 8, 128, 16, 1200, 0) == 32 + 4 * 8 * (3 + 1) * 130 * 4
    assert f(4, 8, 8, 128, 16, 1200, -1) == 32 + 4 * 8 * (3 + 1) * 130 * 4
    assert f(4, 8, 8, 64, 16, 1200, 256) == 32 + 4 * 8 * (5 + 1) * 66 * 4
    assert f(4, 16, 8, 128, 16, 1200, 0) == 32 + 4 * 16 * 4 * 130 * 4
    assert f(4, 8, 8, 128, 4, 1200, 0) == 0            # rejected: block_size 4


def test_self_test_rejects_bad_timeouts_on_the_host(lib):
    assert lib.pagedkv_selftest_wait_timeout(0, None) == nat.EINVAL
    assert lib.pagedkv_selftest_wait_timeout(1_000_001, None) == nat.EINVAL


def test_empty_batch_is_a_no_op(lib):
    assert _decode(lib, b=0, q=None) == nat.OK


def test_workspace_bytes(lib):
    # every workspace starts with 32 bytes of work counters, then the split-K partials
    # single pass over one kv head per query head: no workspace
    assert pkv.paged_attention_workspace_bytes(256, 32, 32, 128, 16, 1524, -1) == 0
    assert pkv.paged_attention_workspace_bytes(256, 32, 32, 128, 16, 512, 0) == 0
    # CUDA-core kernel, automatic: 1024-token partitions for the 256-sequence batch, halved to
    # 128 for 32 sequences (2 kv heads per CTA: 512 CTAs per partition, ~4 waves wanted)
    assert pkv.paged_attention_workspace_bytes(256, 32, 32, 128, 16, 1524, 0) == \
        32 + 256 * 32 * 2 * 130 * 4
    assert pkv.paged_attention_workspace_bytes(32, 32, 32, 128, 16, 1524, 0) == \
        32 + 32 * 32 * 12 * 130 * 4
    # explicit split: B * H * P * (D + 2) floats (CUDA-core kernel, MHA)
    assert pkv.paged_attention_workspace_bytes(4, 8, 8, 64, 16, 1000, 256) == 32 + 4 * 8 * 4 * 66 * 4
    # tensor-core split-K (persistent CTAs fed by the work counter)
    assert pkv.paged_attention_workspace_bytes(4, 8, 2, 64, 16, 1000, 256) == 32 + 4 * 8 * 4 * 66 * 4
    # long GQA contexts split automatically into 512-token partitions
    assert pkv.paged_attention_workspace_bytes(128, 64, 8, 128, 16, 16384, 0) == \
        32 + 128 * 64 * 32 * 130 * 4
    # grouped queries in a single pass still take their work from the counter
    assert pkv.paged_attention_workspace_bytes(128, 64, 8, 128, 16, 2048, -1) == 32
    # beyond 1024 sequences the tensor-core split runs one CTA per item (the counters unused)
    assert pkv.paged_attention_workspace_bytes(1100, 16, 2, 64, 16, 1000, 512) == \
        32 + 1100 * 16 * 2 * 66 * 4
    assert pkv.paged_attention_workspace_bytes(1, 8, 3, 64, 16, 100, 0) == 0     # rejected shape


def test_noalloc_falls_back_to_a_single_pass_for_the_automatic_plan(lib):
    # 256 MHA sequences up to 4000 tokens: the automatic 1024-token split needs ~17 MB, more
    # than the 16 MiB built-in scratch, so the call runs a single pass instead of refusing.
    # Without a GPU here it then fails on the device lookup, never with EWORKSPACE.
    B, H, D, bs, maxlen = 256, 32, 128, 16, 4000
    assert lib.paged_attention_workspace_bytes(B, H, H, D, bs, maxlen, 0) > (16 << 20)
    fn = lib.paged_attention_decode_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [P, P, P, P, P, P, ctypes.c_float] + [I] * 9 + [P]
    fn.restype = I
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, bs, H, B, H, D, 256, 65536, maxlen)
    st = fn(*args, 0, None)
    assert st != nat.EWORKSPACE
    assert fn(*args, 512, None) == nat.EWORKSPACE     # an explicit split is kept, and refused


def test_partition_tokens(lib):
    f = pkv.paged_attention_partition_tokens
    assert f(256, 32, 32, 128, 16, 1524, -1) == 0          # single pass asked for
    assert f(256, 32, 32, 128, 16, 1524, 0) == 1024        # automatic split
    assert f(32, 32, 32, 128, 16, 1524, 0) == 128          # small batch: smaller partitions
    assert f(128, 64, 8, 128, 16, 16384, 0) == 512         # long grouped-query contexts
    assert f(256, 32, 32, 128, 16, 1524, 256) == 256
    assert lib.paged_attention_partition_tokens(1, 8, 3, 64, 16, 100, 0) == nat.EINVAL


def test_cache_ops_reject_bad_arguments_on_the_host(lib):
    assert lib.reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 64, 16, 8, None) == nat.OK
    assert lib.reshape_and_cache(None, FAKE, FAKE, FAKE, FAKE, 3, 4, 64, 16, 8, None) == nat.EINVAL
    assert lib.reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 3, 4, 60, 16, 8, None) == nat.EINVAL
    assert lib.reshape_and_cache(FAKE + 4, FAKE, FAKE, FAKE, FAKE, 3, 4, 64, 16, 8, None) == nat.EINVAL
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert lib.copy_blocks(arr, arr, FAKE, 0, 2, 1024, 8, None) == nat.OK
    assert lib.copy_blocks(arr, arr, FAKE, 3, 0, 1024, 8, None) == nat.EINVAL
    assert lib.copy_blocks(arr, arr, FAKE, 3, 129, 1024, 8, None) == nat.EINVAL
    assert lib.copy_blocks(arr, arr, FAKE, 3, 2, 1020, 8, None) == nat.EINVAL
    bad = (ctypes.c_void_p * 2)(FAKE, FAKE + 2)
    assert lib.copy_blocks(bad, arr, FAKE, 3, 2, 1024, 8, None) == nat.EINVAL


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(nat, "_lib", None)
    monkeypatch.setattr(nat, "library_path", lambda: str(tmp_path / "libpagedkv.so"))
    with pytest.raises(nat.PagedKVError, match="no CPU fallback"):
        nat.load_library()


def _host_step(lib, lens, pairs=None, staging_bytes=None, staging=FAKE, maxlen=100, max_pairs=4,
               pre=None, groups=None, ng=0, B=None):
    """paged_decode_step_host with real host arrays and fake device pointers: every refusal
    below happens on the host, before any CUDA call."""
    import numpy as np
    lens = np.ascontiguousarray(lens, np.int32)
    B = len(lens) if B is None else B
    H, Hk, D, bs, maxblk, N = 8, 8, 64, 16, 8, 64
    tables = np.zeros((max(B, 1), maxblk), np.int32)
    pr = np.ascontiguousarray(pairs if pairs is not None else np.zeros((0, 2)), np.int64)
    need = lib.paged_decode_step_staging_bytes(B, H, Hk, D, bs, maxblk, maxlen, 0, max_pairs,
                                               int(pre is not None))
    return lib.paged_decode_step_host(
        FAKE, FAKE, FAKE, FAKE, tables.ctypes.data, lens.ctypes.data,
        pr.ctypes.data if len(pr) else None, len(pr),
        None if pre is None else np.ascontiguousarray(pre, np.int32).ctypes.data,
        None if groups is None else np.ascontiguousarray(groups, np.int32).ctypes.data, ng,
        FAKE, FAKE, 0.125, bs, Hk, B, H, D, maxblk, N, maxlen, 0, max_pairs, staging,
        need if staging_bytes is None else staging_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(lens=[5, 0]), nat.EINVAL),                          # a context length below 1
    (dict(lens=[5, 101]), nat.EINVAL),                        # beyond max_context_len
    (dict(lens=[5, 7], pairs=[[1, 2], [3, 1]]), nat.EINVAL),  # a destination used as a source
    (dict(lens=[5, 7], pairs=[[1, 2], [3, 2]]), nat.EINVAL),  # a destination repeated
    (dict(lens=[5, 7], pairs=[[1, 64]]), nat.EINVAL),         # outside the pool
    (dict(lens=[5, 7], pairs=[[1, 2]] * 5), nat.EINVAL),      # more than max_pairs
    (dict(lens=[5, 7], staging_bytes=1024), nat.EWORKSPACE),
    (dict(lens=[5, 7], staging=FAKE + 16), nat.EINVAL),       # staging not 256-byte aligned
    (dict(lens=[5, 7], pre=[0, 0], ng=3), nat.EINVAL),        # more groups than num_seqs / 2
])
def test_host_step_rejects_bad_host_inputs(lib, kw, code):
    assert _host_step(lib, **kw) == code
    assert lib.pagedkv_last_error().decode()


def test_host_step_staging_bytes(lib):
    f = lib.paged_decode_step_staging_bytes
    r = lambda n: (n + 255) // 256 * 256  # noqa: E731
    B, H, Hk, D, bs, maxblk, maxlen = 256, 32, 32, 128, 16, 96, 1524
    ws = lib.paged_attention_workspace_bytes(B, H, Hk, D, bs, maxlen, 0)
    # the plain step pipelines 4 chunks over two compute streams: two workspaces
    want = (r(B * H * D * 2) * 2 + r(B * Hk * D * 2) * 2 + r(B * maxblk * 4) + r(B * 4) +
            r(224 * 16) + 2 * r(ws))
    assert f(B, H, Hk, D, bs, maxblk, maxlen, 0, 224, 0) == want
    ws2 = lib.paged_attention_shared_prefix_workspace_bytes(B, H, Hk, D, bs, maxlen, 0)
    assert f(B, H, Hk, D, bs, maxblk, maxlen, 0, 224, 1) == \
        want - 2 * r(ws) + r(B * 4) + r(B // 2 * 9 * 4) + r(ws2)
    assert f(B, H, Hk, 96, bs, maxblk, maxlen, 0, 0, 0) == 0    # rejected head_dim


def test_host_step_refuses_a_prefix_no_group_lists(lib):
    import numpy as np
    # sequence 1 claims 16 prefix tokens, but the only group lists sequences 0 and 2
    groups = np.array([[1, 0, 2, -1, -1, -1, -1, -1, -1]], np.int32)
    assert _host_step(lib, lens=[40, 40, 40, 40], pre=[16, 16, 16, 0], groups=groups, ng=1) == \
        nat.EINVAL
    assert b"no group" in lib.pagedkv_last_error()
