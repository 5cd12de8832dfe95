"""A decode step over every attention layer of a model, replayed as one CUDA graph.

Each layer has its own K/V pools but the same sequences, so all layers share one
block table and one set of context lengths (the block manager's), while the
query, the new K/V rows and the output are per layer.  Layers run one after
another in a model (layer l+1's query depends on layer l's output), so the step
is a chain of per-layer launches; capturing the chain once as a CUDA graph
removes the per-launch host cost when the step is replayed.  Copy-on-write
copies of a step are one copy_blocks launch over all layers' pools, issued
before the graph on the same stream.

All tensors are device tensors whose addresses stay fixed: callers write each
step's inputs into them in place (or with ``set_inputs``) and call ``replay``.
"""
from __future__ import annotations

import torch

from ._native import (copy_blocks, paged_attention_decode_append,
                      paged_attention_workspace_bytes)


class LayeredDecodeStep:
    def __init__(self, key_caches, value_caches, num_seqs, num_heads, max_blocks,
                 max_context_len, scale=None, partition_size=0, stream=None, max_pairs=0):
        if len(key_caches) != len(value_caches) or not key_caches:
            raise ValueError("need one K and one V pool per layer")
        self.key_caches, self.value_caches = list(key_caches), list(value_caches)
        dev = key_caches[0].device
        N, Hk, bs, D = key_caches[0].shape
        L, B, H = len(key_caches), num_seqs, num_heads
        self.num_layers = L
        self.scale = 1.0 / D ** 0.5 if scale is None else float(scale)
        self.max_context_len = int(max_context_len)
        self.partition_size = partition_size
        self.stream = stream if stream is not None else torch.cuda.Stream(dev)
        self.q = torch.zeros((L, B, H, D), dtype=torch.float16, device=dev)
        self.k_new = torch.zeros((L, B, Hk, D), dtype=torch.float16, device=dev)
        self.v_new = torch.zeros_like(self.k_new)
        self.out = torch.empty((L, B, H, D), dtype=torch.float16, device=dev)
        self.block_tables = torch.full((B, max_blocks), -1, dtype=torch.int32, device=dev)
        self.context_lens = torch.ones(B, dtype=torch.int32, device=dev)
        self.pairs = torch.empty((max(max_pairs, 1), 2), dtype=torch.int64, device=dev)
        need = paged_attention_workspace_bytes(B, H, Hk, D, bs, max_context_len, partition_size)
        # the layers run in order on one stream, so they share one workspace (zeroed: its
        # work counters must start at zero)
        self.workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
        self.graph = None
        self._inputs_set = False

    def _layers(self):
        for l in range(self.num_layers):
            paged_attention_decode_append(
                self.out[l], self.q[l], self.k_new[l], self.v_new[l], self.key_caches[l],
                self.value_caches[l], self.block_tables, self.context_lens, self.scale,
                self.max_context_len, self.partition_size, self.workspace, stream=self.stream)

    def capture(self):
        """Captures the per-layer launches (after one eager run that sets up the kernels).
        The eager run writes the current inputs' new rows, as a replay would, so the
        inputs must be set first (set_inputs): the placeholder tables hold no blocks."""
        if not self._inputs_set:
            raise RuntimeError("set_inputs() before capture(): the set-up run reads the tables")
        self._layers()
        self.stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self._layers()
        self.graph = g
        return self

    def set_inputs(self, q=None, k_new=None, v_new=None, block_tables=None, context_lens=None):
        with torch.cuda.stream(self.stream):
            for dst, src in ((self.q, q), (self.k_new, k_new), (self.v_new, v_new),
                             (self.block_tables, block_tables), (self.context_lens, context_lens)):
                if src is not None:
                    dst.copy_(src, non_blocking=True)
        if block_tables is not None and context_lens is not None:
            self._inputs_set = True

    def replay(self, pairs=None):
        """One decode step: copy-on-write copies (pairs [n][2] int64, device or None) over every
        layer, then every layer's fused append + attention."""
        if pairs is not None and len(pairs):
            copy_blocks(self.key_caches, self.value_caches, pairs, stream=self.stream)
        if self.graph is None:
            self._layers()
        else:
            with torch.cuda.stream(self.stream):   # a graph launches on the current stream
                self.graph.replay()
        return self.out
