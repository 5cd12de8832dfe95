// Internal interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace pkv {

// Arguments of one paged decode-attention launch (both passes of split-K).
struct DecodeParams {
  __half* out;                 // [B][H][D]
  const __half* q;             // [B][H][D]
  const __half* k_cache;       // [N][Hk][bs][D]
  const __half* v_cache;       // [N][Hk][bs][D]
  const int32_t* block_tables; // [B][max_blocks]
  const int32_t* context_lens; // [B]
  float* ws_o;                 // split only: [B][H][num_parts][D] unnormalised partial outputs
  float* ws_ml;                // split only: [B][H][num_parts][2] (running max in log2 units, sum)
  unsigned* err;               // per-device error word
  float scale_log2;            // scale * log2(e): scores are kept in log2 units
  int num_seqs, num_heads, num_kv_heads, head_dim, block_size;
  int max_blocks, num_blocks, max_context_len;
  int part_tokens;             // tokens per partition (a multiple of 16 and of bs)
  int prefix_part_tokens;      // tokens per partition of a shared prefix (its slots come first)
  int num_parts;               // partial-result slots per (sequence, head)
  int grid_parts;              // partitions in the launch grid (<= num_parts)
  int no_merge;                // no merge kernel follows: a partial result here is an error
  int after_prefix;            // launched as a programmatic dependent of the shared-prefix pass:
                               // wait for it (griddepcontrol.wait) before reading its partials
  int fold_prefix;             // a suffix within one partition folds the prefix partials into
                               // the output itself; 0: it leaves a partial, the merge combines
  int stages;                  // depth of the shared-memory ring
  // Fused append (NULL = none): this step's new K/V rows, [B][Hk][D], which the
  // kernel writes to position L_b - 1 through the block table before reading it.
  const __half* k_new;
  const __half* v_new;
  // Shared-prefix (cascade) decode (NULL = none).  seq_prefix_tokens[b] tokens of
  // sequence b are covered by its group's prefix pass; the rest by the suffix
  // pass.  Partial slots of (b, h): prefix partitions first, then suffix ones.
  const int32_t* seq_prefix_tokens;  // [B]
  const int32_t* groups;             // [num_groups][GROUP_WIDTH]: prefix blocks, members
  int num_groups;
};

// A shared-prefix group: its prefix length in blocks, then up to 8 member
// sequences (-1 = unused).
constexpr int GROUP_WIDTH = 9;
constexpr int GROUP_MAX_MEMBERS = 8;

// kernel<<<grid, block, smem, stream>>>(args...), as a programmatic dependent launch
// (it may start while the previous kernel on the stream finishes) when pdl is set.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                 size_t smem, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Consumer warps of the grouped-query (tensor-core) kernel; plus one producer warp
// (fixed at build time; 2 measured best).
#ifndef PAGEDKV_TUNE_MMA_WARPS
#define PAGEDKV_TUNE_MMA_WARPS 2
#endif
constexpr int MMA_CONSUMER_WARPS = PAGEDKV_TUNE_MMA_WARPS;

// Shared-memory bytes of one ring stage / the whole launch.
size_t simt_stage_bytes(int head_dim, int block_size, int kvc);
size_t simt_smem_bytes(int head_dim, int block_size, int kvc, int stages);
size_t mma_stage_bytes(int head_dim, int block_size);
size_t mma_smem_bytes(int head_dim, int block_size, int stages);

// CUDA-core kernel: CTA = (b, group of hpc query heads, partition); the group
// reads kvc consecutive kv heads.  Returns cudaErrorInvalidValue for an
// uncompiled (head_dim, block_size, hpc, kvc) combination.
cudaError_t launch_simt_decode(const DecodeParams& p, int hpc, int kvc, bool split,
                               cudaStream_t stream);

// Tensor-core kernel for query groups of 2..8 heads: CTA = (b, kv head, partition).
cudaError_t launch_mma_decode(const DecodeParams& p, const CUtensorMap& k_map,
                              const CUtensorMap& v_map, bool split, cudaStream_t stream);

// Work counters at the start of every workspace, 16 bytes per persistent pass
// (the decode pass, then the shared-prefix pass): a 32-bit ticket, 4 unused
// bytes, and a 64-bit word of finished CTAs (high half) and items they
// processed (low half); the last CTA of a launch zeroes its pass's counters.
// They must be zero before a workspace's first use and every launch leaves
// them zero.
constexpr size_t WORK_COUNTER_BYTES = 32;

// Persistent tensor-core kernel: a few CTAs per SM take (b, kv head, partition)
// work items from the decode pass's ticket (counters[0]).  Without a split every item is a
// whole context.
cudaError_t launch_mma_decode_persistent(const DecodeParams& p, const CUtensorMap& k_map,
                                         const CUtensorMap& v_map, unsigned int* counters,
                                         bool split, cudaStream_t stream);
// Shared-prefix pass on the same persistent grid: work items (group, kv head,
// prefix partition) from the prefix pass's ticket (counters[4]); the columns of an item's tile
// are the group's usable members' query heads of that kv head.
cudaError_t launch_mma_prefix_persistent(const DecodeParams& p, const CUtensorMap& k_map,
                                         const CUtensorMap& v_map, unsigned int* counters,
                                         int prefix_parts, cudaStream_t stream);
size_t mma_persistent_smem_bytes(int head_dim, int stages, int num_rows, bool prefix = false);
constexpr int PERSISTENT_MAX_SEQS = 1024;

// Shared-prefix pass: CTA = (kv head, group, prefix partition); the members'
// query rows for that kv head are the columns of one tensor-core tile.
cudaError_t launch_mma_prefix(const DecodeParams& p, const CUtensorMap& k_map,
                              const CUtensorMap& v_map, int prefix_parts, cudaStream_t stream);

// Merges the partitions of a split launch into `out` (a programmatic dependent
// launch after the partition pass on the same stream).
cudaError_t launch_split_reduce(const DecodeParams& p, cudaStream_t stream);
size_t split_merge_smem_bytes(int num_parts);
constexpr int MAX_PARTITIONS = 4096;

// Slot-mapping scatter of new K/V rows into the pools.
cudaError_t launch_reshape_and_cache(const __half* k, const __half* v, __half* key_cache,
                                     __half* value_cache, const int64_t* slot_mapping,
                                     int num_tokens, int num_kv_heads, int head_dim,
                                     int block_size, int num_blocks, unsigned* err,
                                     cudaStream_t stream);

constexpr int MAX_COPY_LAYERS = 128;

// Copy-on-write block copies over every layer's K and V pool.
cudaError_t launch_copy_blocks(void* const* key_caches, void* const* value_caches,
                               const int64_t* pairs, int num_pairs, int num_layers,
                               size_t block_elems, int num_blocks, unsigned* err,
                               cudaStream_t stream);

}  // namespace pkv
