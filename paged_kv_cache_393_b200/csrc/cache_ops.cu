// Data-movement kernels of the paged KV cache (sm_100a): the slot-mapping
// scatter of new K/V rows and the copy-on-write block copy.  Both are plain
// bit-exact copies with 16-byte vector loads and stores; they are bound by HBM
// bandwidth (or by launch latency at small sizes).
#include "common.cuh"
#include "kernels.h"

namespace pkv {
namespace {

// Streaming 16-byte load of data no thread of this launch writes (the new rows).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Streaming 16-byte load through the coherent path: copy_blocks reads the pools
// it writes in the same launch (another pair's destination), so the read-only
// path is not allowed there.
__device__ __forceinline__ uint4 ld_coherent_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p)
               : "memory");
  return r;
}

// Token t's row of kv head h goes to row s % bs of block s / bs, s = slot_mapping[t]
// (the scatter of new K/V into their blocks: lpnh.cn/news/1824136 §3.1).
// One thread per 16-byte vector of a (token, head) row; grid-stride.
__global__ void reshape_and_cache_kernel(const __half* __restrict__ k, const __half* __restrict__ v,
                                         __half* __restrict__ kc, __half* __restrict__ vc,
                                         const int64_t* __restrict__ slots, int num_tokens,
                                         int num_kv_heads, int head_dim, int block_size,
                                         long long pool_slots, unsigned* err) {
  const int vecs_per_row = head_dim / 8;
  const long long vecs_per_tok = (long long)num_kv_heads * vecs_per_row;
  const long long total = (long long)num_tokens * vecs_per_tok;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long tok = idx / vecs_per_tok;
    const long long rem = idx - tok * vecs_per_tok;
    const int h = (int)(rem / vecs_per_row);
    const int c = (int)(rem - (long long)h * vecs_per_row);
    const long long s = slots[tok];
    if (s < 0) continue;  // padding
    if (s >= pool_slots) {
      if (rem == 0) flag_error(err, ERR_SLOT);
      continue;
    }
    const long long blk = s / block_size;
    const int off = (int)(s - blk * block_size);
    const size_t src = ((size_t)tok * num_kv_heads + h) * head_dim + (size_t)c * 8;
    const size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * head_dim + (size_t)c * 8;
    const uint4 kk = ld_stream(k + src);
    const uint4 vv = ld_stream(v + src);
    *reinterpret_cast<uint4*>(kc + dst) = kk;
    *reinterpret_cast<uint4*>(vc + dst) = vv;
  }
}

struct LayerPointers {
  __half* k[MAX_COPY_LAYERS];
  __half* v[MAX_COPY_LAYERS];
};

constexpr int COPY_THREADS = 256;
constexpr int COPY_VPT = 4;  // 16-byte vectors per thread in flight

// grid = (chunks of one block, pair, layer * 2 + {K, V}).  Copies whole blocks
// src -> dst (the copy step of copy-on-write: lpnh.cn/news/2758356 §4.2).
__global__ void __launch_bounds__(COPY_THREADS)
    copy_blocks_kernel(const LayerPointers ptrs, const int64_t* __restrict__ pairs,
                       long long block_vecs, int num_blocks, unsigned* err) {
  const int pair = blockIdx.y;
  const int layer = blockIdx.z >> 1;
  const bool is_v = blockIdx.z & 1;
  const long long src = pairs[2 * pair];
  const long long dst = pairs[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(err, ERR_BLOCK_ID);
    return;
  }
  const __half* base = is_v ? ptrs.v[layer] : ptrs.k[layer];
  const uint4* s = reinterpret_cast<const uint4*>(base) + src * block_vecs;
  uint4* d = reinterpret_cast<uint4*>(const_cast<__half*>(base)) + dst * block_vecs;
  const long long chunk = (long long)COPY_THREADS * COPY_VPT;
  for (long long i0 = (long long)blockIdx.x * chunk; i0 < block_vecs; i0 += (long long)gridDim.x * chunk) {
    uint4 r[COPY_VPT];
#pragma unroll
    for (int j = 0; j < COPY_VPT; ++j) {
      const long long i = i0 + j * COPY_THREADS + threadIdx.x;
      if (i < block_vecs) r[j] = ld_coherent_stream(s + i);
    }
#pragma unroll
    for (int j = 0; j < COPY_VPT; ++j) {
      const long long i = i0 + j * COPY_THREADS + threadIdx.x;
      if (i < block_vecs) d[i] = r[j];
    }
  }
}

}  // namespace

cudaError_t launch_reshape_and_cache(const __half* k, const __half* v, __half* key_cache,
                                     __half* value_cache, const int64_t* slot_mapping,
                                     int num_tokens, int num_kv_heads, int head_dim,
                                     int block_size, int num_blocks, unsigned* err,
                                     cudaStream_t stream) {
  const long long total = (long long)num_tokens * num_kv_heads * (head_dim / 8);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  reshape_and_cache_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
      k, v, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
      (long long)num_blocks * block_size, err);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* const* key_caches, void* const* value_caches,
                               const int64_t* pairs, int num_pairs, int num_layers,
                               size_t block_elems, int num_blocks, unsigned* err,
                               cudaStream_t stream) {
  if (num_pairs == 0 || num_layers == 0) return cudaSuccess;
  LayerPointers ptrs = {};
  for (int l = 0; l < num_layers; ++l) {
    ptrs.k[l] = static_cast<__half*>(key_caches[l]);
    ptrs.v[l] = static_cast<__half*>(value_caches[l]);
  }
  const long long block_vecs = (long long)(block_elems / 8);
  const long long chunk = (long long)COPY_THREADS * COPY_VPT;
  long long chunks = (block_vecs + chunk - 1) / chunk;
  if (chunks > 1024) chunks = 1024;
  const dim3 grid((unsigned)chunks, (unsigned)num_pairs, (unsigned)(2 * num_layers));
  copy_blocks_kernel<<<grid, COPY_THREADS, 0, stream>>>(ptrs, pairs, block_vecs, num_blocks, err);
  return cudaGetLastError();
}

}  // namespace pkv
