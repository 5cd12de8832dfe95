// paged_attention_decode_noalloc: paged decode attention that allocates nothing.
//
// Some callers cannot hand this library a workspace.  A serving engine that
// reserves almost all of HBM for its KV block pool at start-up leaves no room
// for, and often no path to, a further device allocation; a plugin running
// inside a host runtime that owns the device allocator may have no way to ask
// for memory at all; and a decode loop with a tight latency budget cannot
// afford cudaMalloc/cudaFree, which may synchronize the whole device.  For
// them this entry point takes its scratch -- the split-K partial maxima, sums
// and outputs merged by the second kernel, and the work counter of the
// grouped-query kernel -- from one fixed array compiled into the library
// instead of from a caller's buffer.
//
// The array lives in device memory of every GPU that loads the library, for
// the life of the process, and holds PAGEDKV_NOALLOC_SCRATCH_BYTES.  Calls
// needing more are rejected.  All calls on a device share it, and each call
// leaves its partial results behind: calls that may run on the GPU at the same
// time (different streams, or different host threads) corrupt each other's
// results, so serialize them.  Its first 32 bytes are the work counters of the
// grouped-query kernel, which must start at zero: they are cleared once, when a
// device's address is looked up, and every call leaves them at zero.  Every
// partial result a call reads was written earlier in that same call.
#include "../../include/pagedkv.h"

#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

namespace pkv {
int record_error(int code, const char* message);
}

namespace {

constexpr size_t kScratchBytes = PAGEDKV_NOALLOC_SCRATCH_BYTES;
constexpr size_t kCounterBytes = 32;  // the work counters at the start of every workspace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_address[kMaxDevices];

int report(int code, const char* fmt, size_t a = 0, size_t b = 0) {
  char msg[400];
  snprintf(msg, sizeof(msg), fmt, a, b);
  return pkv::record_error(code, msg);
}

// Device address of the scratch array on the current device.  In host code the
// array's name only stands for it; the address is looked up once per device,
// with that device current, and cached; the work counters at its start are
// cleared then, on the caller's stream, ahead of the first kernel that uses them.
int scratch_address(void** out, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return report(PAGEDKV_ECUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return report(PAGEDKV_ECUDA, "device id out of range");
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_address[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return report(PAGEDKV_ECUDA, "cudaGetSymbolAddress of the built-in scratch failed");
    e = cudaMemsetAsync(p, 0, kCounterBytes, stream);
    if (e != cudaSuccess) return report(PAGEDKV_ECUDA, "clearing the built-in scratch failed");
    g_scratch_address[dev] = p;
  }
  *out = g_scratch_address[dev];
  return PAGEDKV_OK;
}

}  // namespace

extern "C" int paged_attention_decode_noalloc(
    void* out, const void* q, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, const int32_t* context_lens, float scale, int block_size,
    int num_kv_heads, int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
    int num_blocks, int max_context_len, int partition_size, void* stream) {
  if (num_seqs == 0) return PAGEDKV_OK;
  size_t need = paged_attention_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim,
                                                block_size, max_context_len, partition_size);
  if (need > kScratchBytes && partition_size == 0) {
    // the library's own split does not fit: a single pass needs (almost) no scratch
    const size_t single = paged_attention_workspace_bytes(
        num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len, -1);
    if (single <= kScratchBytes) {
      partition_size = -1;
      need = single;
    }
  }
  if (need > kScratchBytes)
    return report(PAGEDKV_EWORKSPACE,
                  "this call needs %zu bytes of scratch but the built-in scratch holds "
                  "%zu; use longer partitions or fewer sequences per call, or "
                  "paged_attention_decode with a workspace of your own",
                  need, kScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    const int st = scratch_address(&scratch, static_cast<cudaStream_t>(stream));
    if (st != PAGEDKV_OK) return st;
  }
  return paged_attention_decode(out, q, key_cache, value_cache, block_tables, context_lens, scale,
                                block_size, num_kv_heads, num_seqs, num_heads, head_dim,
                                max_blocks_per_seq, num_blocks, max_context_len, partition_size,
                                scratch, need > 0 ? kScratchBytes : 0, stream);
}
