"""The Python binding's own checks, which run before anything reaches the library.

Every GPU call refuses host tensors, wrong dtypes and mismatched shapes with a
Python error; there is no silent CPU path.  None of these calls touches a GPU.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_393_b200 as pkv


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_393_b200 import build
    build.build()


def _decode_args(B=2, H=4, Hk=4, D=64, N=8, bs=16, maxblk=2):
    q = torch.zeros((B, H, D), dtype=torch.float16)
    out = torch.empty_like(q)
    kc = torch.zeros((N, Hk, bs, D), dtype=torch.float16)
    vc = torch.zeros_like(kc)
    tables = torch.zeros((B, maxblk), dtype=torch.int32)
    lens = torch.ones(B, dtype=torch.int32)
    return out, q, kc, vc, tables, lens


def test_host_tensors_are_refused():
    out, q, kc, vc, tables, lens = _decode_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.paged_attention_decode(out, q, kc, vc, tables, lens, 0.125, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.paged_attention_decode_append(out, q, q[:, :4], q[:, :4], kc, vc, tables, lens,
                                          0.125, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.reshape_and_cache(q, q, kc, vc, torch.zeros(2, dtype=torch.int64))


def test_shape_mismatches_are_refused():
    out, q, kc, vc, tables, lens = _decode_args()
    with pytest.raises(ValueError, match="shape mismatch"):
        pkv.paged_attention_decode(out[:1], q, kc, vc, tables, lens, 0.125, 16)
    with pytest.raises(ValueError, match="shape mismatch"):
        pkv.paged_attention_decode(out, q, kc, vc[:4], tables, lens, 0.125, 16)
    with pytest.raises(ValueError, match="block_tables"):
        pkv.paged_attention_decode(out, q, kc, vc, tables[:1], lens, 0.125, 16)
    with pytest.raises(ValueError, match="k_new and v_new"):
        pkv.paged_attention_decode_append(out, q, q[:, :2], q[:, :2], kc, vc, tables, lens,
                                          0.125, 16)
    with pytest.raises(ValueError, match="shape mismatch"):
        pkv.reshape_and_cache(q[:, :2], q[:, :2], kc, vc, torch.zeros(2, dtype=torch.int64))


def test_shared_prefix_arguments_are_checked():
    out, q, kc, vc, tables, lens = _decode_args()
    pre = torch.zeros(2, dtype=torch.int32)
    groups = torch.zeros((1, 9), dtype=torch.int32)
    with pytest.raises(ValueError, match="seq_prefix_tokens"):
        pkv.paged_attention_decode_shared_prefix(out, q, kc, vc, tables, lens, pre[:1], groups,
                                                 0.125, 16)
    with pytest.raises(ValueError, match="groups"):
        pkv.paged_attention_decode_shared_prefix(out, q, kc, vc, tables, lens, pre,
                                                 groups[:, :8], 0.125, 16)
    with pytest.raises(ValueError, match="both"):
        pkv.paged_attention_decode_shared_prefix(out, q, kc, vc, tables, lens, pre, groups, 0.125,
                                                 16, k_new=q)


def test_copy_blocks_checks_its_pools():
    kc = torch.zeros((8, 2, 16, 64), dtype=torch.float16)
    with pytest.raises(ValueError, match="one K and one V pool"):
        pkv.copy_blocks([kc], [], torch.zeros((1, 2), dtype=torch.int64))
    with pytest.raises(ValueError, match="every pool"):
        pkv.copy_blocks([kc, kc[:4]], [kc, kc], torch.zeros((1, 2), dtype=torch.int64))


def test_prefix_groups_output_shapes():
    tables = np.array([[3, 4, -1], [3, 4, -1], [7, -1, -1]], np.int32)
    lens = np.array([40, 35, 10], np.int32)
    pre, groups = pkv.prefix_groups(tables, lens, 16, 8)
    assert pre.dtype == np.int32 and pre.shape == (3,)
    assert groups.dtype == np.int32 and groups.shape == (1, pkv.GROUP_WIDTH)
    assert groups[0].tolist() == [2, 0, 1, -1, -1, -1, -1, -1, -1]
    assert pre.tolist() == [32, 32, 0]
