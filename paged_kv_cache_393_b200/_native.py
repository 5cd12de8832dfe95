"""ctypes binding of libpagedkv.so (argument marshalling only).

Each function checks its tensors (device, dtype, shape, contiguity), takes the
current CUDA stream unless one is given, calls the C entry point of the same
name and raises PagedKVError on a non-zero status.  Nothing here computes any
part of the path.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None
_lock = threading.Lock()

OK, EINVAL, EUNSUPPORTED, ECUDA, EWORKSPACE, ENOMEM, ENOENT, ERANGE = 0, -1, -2, -3, -4, -5, -6, -7
DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, DEVERR_SLOT, DEVERR_TIMEOUT, DEVERR_INTERNAL = 1, 2, 4, 8, 16
DEVERR_PREFIX = 32
GROUP_WIDTH, GROUP_MAX_MEMBERS = 9, 8


class PagedKVError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__("%s (status %d)" % (message, code))
        self.code = code


def library_path() -> str:
    return os.path.join(_HERE, "libpagedkv.so")


def load_library():
    """Loads libpagedkv.so; raises if it has not been built (there is no fallback)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise PagedKVError(ECUDA, "libpagedkv.so is missing: build it with "
                               "`python -m paged_kv_cache_393_b200.build`; this package has no "
                               "CPU fallback")
        lib = ctypes.CDLL(path)
        P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        sig = {
            "pagedkv_last_error": ([], ctypes.c_char_p),
            "pagedkv_device_errors": ([ctypes.POINTER(ctypes.c_uint), I], I),
            "pagedkv_selftest_wait_timeout": ([ctypes.c_uint, P], I),
            "paged_attention_decode": ([P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, P, Z, P], I),
            "paged_attention_decode_append": (
                [P, P, P, P, P, P, P, P, F, I, I, I, I, I, I, I, I, I, P, Z, P], I),
            "paged_attention_workspace_bytes": ([I, I, I, I, I, I, I], Z),
            "paged_attention_partition_tokens": ([I, I, I, I, I, I, I], I),
            "paged_attention_decode_shared_prefix": (
                [P, P, P, P, P, P, P, P, P, P, I, I, I, F, I, I, I, I, I, I, I, I, I, P, Z, P], I),
            "paged_attention_shared_prefix_workspace_bytes": ([I, I, I, I, I, I, I], Z),
            "pagedkv_prefix_groups": ([P, P, I, I, I, I, P, P, I], I),
            "paged_decode_step_host": (
                [P, P, P, P, P, P, P, I, P, P, I, P, P, F, I, I, I, I, I, I, I, I, I, I, P, Z, P],
                I),
            "paged_decode_step_staging_bytes": ([I, I, I, I, I, I, I, I, I, I], Z),
            "reshape_and_cache": ([P, P, P, P, P, I, I, I, I, I, P], I),
            "copy_blocks": ([P, P, P, I, I, Z, I, P], I),
            "bm_create": ([I, I, P], P),
            "bm_destroy": ([P], None),
            "bm_add_seq": ([P, I], I),
            "bm_append_token": ([P, I, P], I),
            "bm_append_tokens": ([P, P, I, P], I),
            "bm_fork": ([P, I, I, P], I),
            "bm_free_seq": ([P, I], I),
            "bm_block_table": ([P, I, P, I], I),
            "bm_seq_len": ([P, I], I),
            "bm_seq_slots": ([P, I, I, I, P], I),
            "bm_build_batch": ([P, P, I, P, I, P], I),
            "bm_take_copies": ([P, P, I], I),
            "bm_refcount": ([P, I], I),
            "bm_num_free": ([P], I),
            "bm_free_list": ([P, P, I], I),
            "bm_last_error": ([], ctypes.c_char_p),
            "bm_stats": ([P, P], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return _lib


def _check(status: int, what: str, err_fn: str = "pagedkv_last_error"):
    if status < 0:
        lib = load_library()
        msg = getattr(lib, err_fn)().decode(errors="replace")
        raise PagedKVError(status, "%s: %s" % (what, msg))
    return status


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cuda(t: torch.Tensor, name: str, dtype, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got shape %s" % (name, ndim, tuple(t.shape)))
    return t.data_ptr()


# ---- GPU operations ------------------------------------------------------------

def paged_attention_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                    max_context_len, partition_size=0) -> int:
    return int(load_library().paged_attention_workspace_bytes(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size))


def paged_attention_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                     max_context_len, partition_size=0) -> int:
    """Tokens per split-K partition the library uses (0 = single pass)."""
    n = load_library().paged_attention_partition_tokens(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size)
    return _check(n, "paged_attention_partition_tokens")


def paged_attention_decode(out, q, key_cache, value_cache, block_tables, context_lens, scale,
                           max_context_len, partition_size=0, workspace=None, stream=None):
    """out[B][H][D] = paged decode attention of q over the pools; see include/pagedkv.h."""
    return _decode("paged_attention_decode", out, q, None, None, key_cache, value_cache,
                   block_tables, context_lens, scale, max_context_len, partition_size, workspace,
                   stream)


def paged_attention_decode_append(out, q, k_new, v_new, key_cache, value_cache, block_tables,
                                  context_lens, scale, max_context_len, partition_size=0,
                                  workspace=None, stream=None):
    """One fused step: k_new/v_new ([B][Hk][D]) are written at position L_b - 1 through the
    block tables, then out = paged decode attention over the updated pools."""
    return _decode("paged_attention_decode_append", out, q, k_new, v_new, key_cache, value_cache,
                   block_tables, context_lens, scale, max_context_len, partition_size, workspace,
                   stream)


def _decode(name, out, q, k_new, v_new, key_cache, value_cache, block_tables, context_lens, scale,
            max_context_len, partition_size, workspace, stream):
    lib = load_library()
    B, H, D = q.shape
    N, Hk, bs, D2 = key_cache.shape
    if D2 != D or tuple(value_cache.shape) != tuple(key_cache.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch: q %s, pools %s/%s, out %s" % (
            tuple(q.shape), tuple(key_cache.shape), tuple(value_cache.shape), tuple(out.shape)))
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("block_tables must be [B][max_blocks] and context_lens [B]")
    if k_new is not None and (tuple(k_new.shape) != (B, Hk, D) or tuple(v_new.shape) != (B, Hk, D)):
        raise ValueError("k_new and v_new must be [B][Hk][D]")
    ptrs = [_cuda(out, "out", torch.float16, 3), _cuda(q, "q", torch.float16, 3)]
    if k_new is not None:
        ptrs += [_cuda(k_new, "k_new", torch.float16, 3), _cuda(v_new, "v_new", torch.float16, 3)]
    ptrs += [_cuda(key_cache, "key_cache", torch.float16, 4),
             _cuda(value_cache, "value_cache", torch.float16, 4),
             _cuda(block_tables, "block_tables", torch.int32, 2),
             _cuda(context_lens, "context_lens", torch.int32, 1)]
    need = paged_attention_workspace_bytes(B, H, Hk, D, bs, max_context_len, partition_size)
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None:
            workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
        _cuda(workspace, "workspace", workspace.dtype)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = getattr(lib, name)(*ptrs, float(scale), bs, Hk, B, H, D, block_tables.shape[1], N,
                            int(max_context_len), int(partition_size), ws_ptr, ws_bytes,
                            _stream(stream, q.device))
    _check(st, name)
    return out


def paged_attention_shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                                  block_size, max_context_len,
                                                  partition_size=0) -> int:
    return int(load_library().paged_attention_shared_prefix_workspace_bytes(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size))


def prefix_groups(block_tables, context_lens, block_size, max_members):
    """Host grouping of a batch by shared table prefixes (pagedkv_prefix_groups).

    block_tables: int32 [B][max_blocks] (-1 padded), context_lens: int32 [B] (numpy).
    Returns (seq_prefix_tokens int32 [B], groups int32 [n][GROUP_WIDTH])."""
    lib = load_library()
    t = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    B = t.shape[0]
    if t.ndim != 2 or lens.shape != (B,):
        raise ValueError("block_tables must be [B][max_blocks] and context_lens [B]")
    pre = np.zeros(B, np.int32)
    cap = max(B // 2, 1)
    groups = np.zeros((cap, GROUP_WIDTH), np.int32)
    n = lib.pagedkv_prefix_groups(_np_ptr(t), _np_ptr(lens), B, t.shape[1], int(block_size),
                                  int(max_members), _np_ptr(pre), _np_ptr(groups), cap)
    _check(n, "pagedkv_prefix_groups")
    return pre, groups[:n].copy()


def paged_attention_decode_shared_prefix(out, q, key_cache, value_cache, block_tables,
                                         context_lens, seq_prefix_tokens, groups, scale,
                                         max_context_len, partition_size=0, workspace=None,
                                         k_new=None, v_new=None, stream=None,
                                         max_prefix_tokens=0, max_suffix_tokens=0):
    """Paged decode attention that reads each group's shared prefix once (device tensors:
    seq_prefix_tokens int32 [B], groups int32 [n][GROUP_WIDTH]); with k_new/v_new the new
    rows are written first, as paged_attention_decode_append does.  max_prefix_tokens /
    max_suffix_tokens: host upper bounds that size the grids (0 = max_context_len)."""
    lib = load_library()
    B, H, D = q.shape
    N, Hk, bs, D2 = key_cache.shape
    if D2 != D or tuple(value_cache.shape) != tuple(key_cache.shape) or tuple(out.shape) != (B, H, D):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("block_tables must be [B][max_blocks] and context_lens [B]")
    if tuple(seq_prefix_tokens.shape) != (B,) or groups.dim() != 2 or groups.shape[1] != GROUP_WIDTH:
        raise ValueError("seq_prefix_tokens must be [B] and groups [n][%d]" % GROUP_WIDTH)
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    kn = vn = None
    if k_new is not None:
        if tuple(k_new.shape) != (B, Hk, D) or tuple(v_new.shape) != (B, Hk, D):
            raise ValueError("k_new and v_new must be [B][Hk][D]")
        kn, vn = _cuda(k_new, "k_new", torch.float16, 3), _cuda(v_new, "v_new", torch.float16, 3)
    ng = groups.shape[0]
    gptr = _cuda(groups, "groups", torch.int32, 2) if ng else None
    need = paged_attention_shared_prefix_workspace_bytes(B, H, Hk, D, bs, max_context_len,
                                                         partition_size)
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None:
            workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
        _cuda(workspace, "workspace", workspace.dtype)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = lib.paged_attention_decode_shared_prefix(
        _cuda(out, "out", torch.float16, 3), _cuda(q, "q", torch.float16, 3), kn, vn,
        _cuda(key_cache, "key_cache", torch.float16, 4),
        _cuda(value_cache, "value_cache", torch.float16, 4),
        _cuda(block_tables, "block_tables", torch.int32, 2),
        _cuda(context_lens, "context_lens", torch.int32, 1),
        _cuda(seq_prefix_tokens, "seq_prefix_tokens", torch.int32, 1), gptr, ng,
        int(max_prefix_tokens), int(max_suffix_tokens), float(scale),
        bs, Hk, B, H, D, block_tables.shape[1], N, int(max_context_len), int(partition_size),
        ws_ptr, ws_bytes, _stream(stream, q.device))
    _check(st, "paged_attention_decode_shared_prefix")
    return out


def reshape_and_cache(k, v, key_cache, value_cache, slot_mapping, stream=None):
    """Writes k[t], v[t] ([T][Hk][D]) into slot slot_mapping[t] of the pools (bit-exact)."""
    lib = load_library()
    T, Hk, D = k.shape
    N, Hk2, bs, D2 = key_cache.shape
    if (Hk2, D2) != (Hk, D) or tuple(v.shape) != tuple(k.shape) or \
            tuple(value_cache.shape) != tuple(key_cache.shape) or tuple(slot_mapping.shape) != (T,):
        raise ValueError("shape mismatch")
    st = lib.reshape_and_cache(_cuda(k, "k", torch.float16, 3), _cuda(v, "v", torch.float16, 3),
                               _cuda(key_cache, "key_cache", torch.float16, 4),
                               _cuda(value_cache, "value_cache", torch.float16, 4),
                               _cuda(slot_mapping, "slot_mapping", torch.int64, 1),
                               T, Hk, D, bs, N, _stream(stream, k.device))
    _check(st, "reshape_and_cache")


def copy_blocks(key_caches, value_caches, pairs, stream=None):
    """Copies block src -> dst for every row (src, dst) of pairs ([n][2] int64, device), in
    every layer's K and V pool."""
    lib = load_library()
    if len(key_caches) != len(value_caches) or not key_caches:
        raise ValueError("need one K and one V pool per layer")
    shape = tuple(key_caches[0].shape)
    for t in list(key_caches) + list(value_caches):
        if tuple(t.shape) != shape:
            raise ValueError("every pool must have shape %s" % (shape,))
    for t in list(key_caches) + list(value_caches):
        _cuda(t, "pool", torch.float16, 4)
    n = 0 if pairs is None else pairs.shape[0]
    if n == 0:
        return
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n][2]")
    L = len(key_caches)
    karr = (ctypes.c_void_p * L)(*[t.data_ptr() for t in key_caches])
    varr = (ctypes.c_void_p * L)(*[t.data_ptr() for t in value_caches])
    N = shape[0]
    block_elems = shape[1] * shape[2] * shape[3]
    st = lib.copy_blocks(karr, varr, _cuda(pairs, "pairs", torch.int64, 2), n, L, block_elems, N,
                         _stream(stream, key_caches[0].device))
    _check(st, "copy_blocks")


def selftest_wait_timeout(timeout_us: int, stream=None):
    """Enqueues the bounded-wait self-test (see include/pagedkv.h)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib.pagedkv_selftest_wait_timeout(int(timeout_us), _stream(stream, dev)),
           "pagedkv_selftest_wait_timeout")


def device_errors(clear: bool = True) -> int:
    """Error bits the kernels raised on the current device (synchronizes the device)."""
    flags = ctypes.c_uint(0)
    _check(load_library().pagedkv_device_errors(ctypes.byref(flags), int(bool(clear))),
           "pagedkv_device_errors")
    return int(flags.value)


def _host(a, name, dtype, shape):
    """Pointer of a contiguous host array (torch CPU tensor, pinned or not, or numpy)."""
    if isinstance(a, torch.Tensor):
        if a.is_cuda:
            raise ValueError("%s must be in host memory" % name)
        if a.dtype != dtype:
            raise TypeError("%s must be %s, got %s" % (name, dtype, a.dtype))
        if not a.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
        got, ptr = tuple(a.shape), a.data_ptr()
    else:
        npd = {torch.float16: np.float16, torch.int32: np.int32, torch.int64: np.int64}[dtype]
        if not isinstance(a, np.ndarray) or a.dtype != npd or not a.flags.c_contiguous:
            raise TypeError("%s must be a contiguous %s array" % (name, np.dtype(npd).name))
        got, ptr = a.shape, a.ctypes.data
    if tuple(got) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(got)))
    return ptr


def paged_decode_step_staging_bytes(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                    max_blocks_per_seq, max_context_len, partition_size=0,
                                    max_pairs=0, shared_prefix=False) -> int:
    return int(load_library().paged_decode_step_staging_bytes(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
        max_context_len, partition_size, max_pairs, int(bool(shared_prefix))))


def paged_decode_step_host(out_host, q, k_new, v_new, block_tables, context_lens, key_cache,
                           value_cache, scale, max_context_len, staging, partition_size=0,
                           pairs=None, max_pairs=0, seq_prefix_tokens=None, groups=None,
                           stream=None):
    """One decode step from host buffers (paged_decode_step_host in include/pagedkv.h): the
    inputs are uploaded into ``staging`` (a device uint8 tensor of
    paged_decode_step_staging_bytes), copy-on-write pairs are copied, the fused append +
    attention (or the shared-prefix form, given seq_prefix_tokens and groups) runs, and the
    output is copied into out_host.  Returns out_host; it is valid once the stream
    synchronizes."""
    lib = load_library()
    N, Hk, bs, D = key_cache.shape
    B, H = q.shape[0], q.shape[1]
    maxblk = block_tables.shape[1]
    npairs = 0 if pairs is None else int(pairs.shape[0])
    shared = seq_prefix_tokens is not None
    ng = 0 if groups is None else int(groups.shape[0])
    if tuple(value_cache.shape) != tuple(key_cache.shape):
        raise ValueError("the pools must have the same shape")
    ptrs = [_host(out_host, "out_host", torch.float16, (B, H, D)),
            _host(q, "q", torch.float16, (B, H, D)),
            _host(k_new, "k_new", torch.float16, (B, Hk, D)),
            _host(v_new, "v_new", torch.float16, (B, Hk, D)),
            _host(block_tables, "block_tables", torch.int32, (B, maxblk)),
            _host(context_lens, "context_lens", torch.int32, (B,)),
            _host(pairs, "pairs", torch.int64, (npairs, 2)) if npairs else None, npairs,
            _host(seq_prefix_tokens, "seq_prefix_tokens", torch.int32, (B,)) if shared else None,
            _host(groups, "groups", torch.int32, (ng, GROUP_WIDTH)) if ng else None, ng]
    st = lib.paged_decode_step_host(
        *ptrs, _cuda(key_cache, "key_cache", torch.float16, 4),
        _cuda(value_cache, "value_cache", torch.float16, 4), float(scale), bs, Hk, B, H, D,
        maxblk, N, int(max_context_len), int(partition_size), int(max_pairs),
        _cuda(staging, "staging", torch.uint8), staging.numel(), _stream(stream, key_cache.device))
    _check(st, "paged_decode_step_host")
    return out_host


class DecodeSession:
    """A decode step driven from host buffers: the call a serving loop makes.

    Holds the device staging buffer for one batch shape.  ``step`` hands the step's
    host inputs to paged_decode_step_host, which uploads them, runs copy_blocks for
    pending copy-on-write pairs, writes every sequence's new token at position L-1
    through the tables and attends (paged_attention_decode_append), and copies the
    output back into a host tensor.  With shared_prefix=True the batch is grouped
    by shared table prefixes on the host each step (pagedkv_prefix_groups) and the
    shared-prefix call runs instead.
    """

    def __init__(self, key_cache, value_cache, num_seqs, num_heads, max_blocks, max_context_len,
                 scale=None, partition_size=0, max_pairs=0, shared_prefix=False):
        N, Hk, bs, D = key_cache.shape
        self.key_cache, self.value_cache = key_cache, value_cache
        self.num_seqs, self.num_heads, self.max_blocks = num_seqs, num_heads, max_blocks
        self.max_context_len = int(max_context_len)
        self.scale = 1.0 / D ** 0.5 if scale is None else float(scale)
        self.partition_size = partition_size
        self.max_pairs = int(max_pairs)
        self.shared_prefix = bool(shared_prefix)
        self.block_size = bs
        self.max_members = max(1, 8 // (num_heads // Hk))
        need = paged_decode_step_staging_bytes(num_seqs, num_heads, Hk, D, bs, max_blocks,
                                               max_context_len, partition_size, max_pairs,
                                               shared_prefix)
        if need == 0:
            _check(EINVAL, "paged_decode_step_staging_bytes")
        self.staging = torch.zeros(need, dtype=torch.uint8, device=key_cache.device)
        self._last_groups = 0
        self._last_pairs = 0

    def h2d_bytes(self) -> int:
        """Host-to-device bytes of the last step."""
        B, H, D = self.num_seqs, self.num_heads, self.key_cache.shape[3]
        Hk = self.key_cache.shape[1]
        n = B * H * D * 2 + 2 * B * Hk * D * 2 + B * self.max_blocks * 4 + B * 4
        n += self._last_pairs * 16
        if self.shared_prefix:
            n += B * 4 + self._last_groups * GROUP_WIDTH * 4
        return n

    def d2h_bytes(self) -> int:
        return self.num_seqs * self.num_heads * self.key_cache.shape[3] * 2

    def step(self, q, k, v, tables, lens, out_host, pairs=None, stream=None):
        """q [B][H][D], k/v [B][Hk][D] fp16, tables [B][max_blocks] and lens [B] int32, pairs
        [n][2] int64 or None: host arrays (pinned for asynchronous copies).  Returns out_host
        (valid once the stream synchronizes)."""
        pre = groups = None
        if self.shared_prefix:
            t_host = tables.numpy() if isinstance(tables, torch.Tensor) else np.asarray(tables)
            l_host = lens.numpy() if isinstance(lens, torch.Tensor) else np.asarray(lens)
            pre, groups = prefix_groups(t_host, l_host, self.block_size, self.max_members)
            self._last_groups = groups.shape[0]
        self._last_pairs = 0 if pairs is None else int(pairs.shape[0])
        return paged_decode_step_host(
            out_host, q, k, v, tables, lens, self.key_cache, self.value_cache, self.scale,
            self.max_context_len, self.staging, self.partition_size,
            pairs if self._last_pairs else None, self.max_pairs, pre, groups, stream)


def decode_step(session: DecodeSession, *args, **kwargs):
    """Functional alias of DecodeSession.step."""
    return session.step(*args, **kwargs)


# ---- host block manager --------------------------------------------------------

def _np_ptr(a: np.ndarray) -> int:
    return a.ctypes.data


class BlockManager:
    """Host block manager (bm_* in include/pagedkv.h).  add_seq / append_token return
    None when the pool is exhausted; other failures raise PagedKVError."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self._lib = load_library()
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
            if order.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        self._h = self._lib.bm_create(num_blocks, block_size,
                                      None if order is None else _np_ptr(order))
        if not self._h:
            raise PagedKVError(EINVAL, "bm_create rejected its arguments")

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and self._lib is not None:
            self._lib.bm_destroy(h)

    def _chk(self, st, what):
        return _check(st, what, "bm_last_error")

    def add_seq(self, num_tokens: int):
        st = self._lib.bm_add_seq(self._h, int(num_tokens))
        if st == ENOMEM:
            return None
        return self._chk(st, "bm_add_seq")

    def append_token(self, seq: int):
        slot = ctypes.c_int64(0)
        st = self._lib.bm_append_token(self._h, int(seq), ctypes.byref(slot))
        if st == ENOMEM:
            return None
        self._chk(st, "bm_append_token")
        return int(slot.value)

    def append_tokens(self, seqs) -> np.ndarray:
        """Appends one token to each sequence in order; returns the slots of those that
        succeeded (fewer than len(seqs) when the pool ran out)."""
        s = np.ascontiguousarray(seqs, dtype=np.int32)
        out = np.empty(s.shape[0], np.int64)
        n = self._chk(self._lib.bm_append_tokens(self._h, _np_ptr(s), s.shape[0], _np_ptr(out)),
                      "bm_append_tokens")
        return out[:n]

    def fork(self, seq: int, n: int):
        ids = np.empty(max(n, 1), np.int32)
        self._chk(self._lib.bm_fork(self._h, int(seq), int(n), _np_ptr(ids)), "bm_fork")
        return ids[:n].tolist()

    def free_seq(self, seq: int):
        self._chk(self._lib.bm_free_seq(self._h, int(seq)), "bm_free_seq")

    def block_table(self, seq: int):
        n = self._chk(self._lib.bm_block_table(self._h, int(seq), None, 0), "bm_block_table")
        out = np.empty(max(n, 1), np.int32)
        self._chk(self._lib.bm_block_table(self._h, int(seq), _np_ptr(out), n), "bm_block_table")
        return out[:n].tolist()

    def seq_len(self, seq: int) -> int:
        return self._chk(self._lib.bm_seq_len(self._h, int(seq)), "bm_seq_len")

    def seq_slots(self, seq: int, first: int = 0, count: int = None) -> np.ndarray:
        """Slots of the sequence's tokens first .. first+count-1 (default: to its end)."""
        if count is None:
            count = self.seq_len(seq) - first
        out = np.empty(max(count, 1), np.int64)
        self._chk(self._lib.bm_seq_slots(self._h, int(seq), int(first), int(count),
                                         _np_ptr(out)), "bm_seq_slots")
        return out[:count]

    def build_batch(self, seqs, max_blocks: int):
        s = np.ascontiguousarray(seqs, dtype=np.int32)
        tables = np.empty((s.shape[0], max_blocks), np.int32)
        lens = np.empty(s.shape[0], np.int32)
        self._chk(self._lib.bm_build_batch(self._h, _np_ptr(s), s.shape[0], _np_ptr(tables),
                                           int(max_blocks), _np_ptr(lens)), "bm_build_batch")
        return tables, lens

    def take_copies(self) -> np.ndarray:
        n = self._chk(self._lib.bm_take_copies(self._h, None, 0), "bm_take_copies")
        out = np.empty((max(n, 1), 2), np.int64)
        n = self._chk(self._lib.bm_take_copies(self._h, _np_ptr(out), n), "bm_take_copies")
        return out[:n]

    def refcount(self, block: int) -> int:
        return self._chk(self._lib.bm_refcount(self._h, int(block)), "bm_refcount")

    def num_free(self) -> int:
        return self._chk(self._lib.bm_num_free(self._h), "bm_num_free")

    def stats(self) -> dict:
        """Pool occupancy: see pagedkv_bm_stats in include/pagedkv.h."""
        keys = ("num_blocks", "free_blocks", "used_blocks", "num_seqs", "logical_tokens",
                "filled_slots", "allocated_slots", "table_entries", "held_blocks")
        out = (ctypes.c_int64 * len(keys))()
        self._chk(self._lib.bm_stats(self._h, out), "bm_stats")
        return dict(zip(keys, [int(x) for x in out]))

    def free_list(self):
        n = self._chk(self._lib.bm_free_list(self._h, None, 0), "bm_free_list")
        out = np.empty(max(n, 1), np.int32)
        self._chk(self._lib.bm_free_list(self._h, _np_ptr(out), n), "bm_free_list")
        return out[:n].tolist()
