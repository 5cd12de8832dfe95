// C ABI of libpagedkv.so: argument checks, launch planning and dispatch.
// Declarations and the contract of every entry point: include/pagedkv.h.
#include "../../include/pagedkv.h"
#include "common.cuh"
#include "kernels.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>
#include <algorithm>

namespace pkv {
namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(PAGEDKV_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- per-device error word -----------------------------------------------------

__device__ unsigned int g_error_word;

constexpr int MAX_DEVICES = 64;
std::mutex g_err_mutex;
unsigned* g_err_ptr[MAX_DEVICES];

// Device address of the current device's error word (looked up once per device).
int error_word(unsigned** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= MAX_DEVICES) return fail(PAGEDKV_ECUDA, "device id %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_err_mutex);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_error_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_err_ptr[dev];
  return PAGEDKV_OK;
}

// ---- tensor maps for the tensor-core kernel -------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// The pool [N][Hk][bs][D] viewed as a [N*Hk*bs][D] fp16 matrix; box = min(bs, 16)
// rows x 64 columns (128 bytes, the 128-byte swizzle span).
int encode_pool_map(CUtensorMap* map, const void* pool, int rows, int head_dim, int block_size) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(PAGEDKV_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)(block_size < 16 ? block_size : 16)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(pool), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PAGEDKV_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return PAGEDKV_OK;
}

// ---- launch plan -------------------------------------------------------------------

constexpr int NUM_SMS_HINT = 148;
constexpr int AUTO_PARTITION = 512;
constexpr int SIMT_CTAS_PER_SM = 6;  // resident CUDA-core CTAs per SM at the usual 2-stage ring
constexpr size_t MAX_SMEM = 227 * 1024;

// Tuning choices, fixed at build time (measured defaults; a sweep rebuilds the
// library with -D overrides instead of reading the environment at run time).
#ifndef PAGEDKV_TUNE_SIMT_KVC
#define PAGEDKV_TUNE_SIMT_KVC 0          // 0: widest of 4/2/1 kv heads within a 16 KB stage
#endif
#ifndef PAGEDKV_TUNE_SIMT_RING_BYTES
#define PAGEDKV_TUNE_SIMT_RING_BYTES 32768
#endif
#ifndef PAGEDKV_TUNE_MMA_STAGES
#define PAGEDKV_TUNE_MMA_STAGES 4
#endif
#ifndef PAGEDKV_TUNE_PERSISTENT
#define PAGEDKV_TUNE_PERSISTENT 1
#endif
#ifndef PAGEDKV_TUNE_MHA_SUFFIX_MMA
#define PAGEDKV_TUNE_MHA_SUFFIX_MMA 0       // 1: a shared-prefix call's MHA suffix pass on the
                                            // persistent tensor-core kernel, not folding
#endif
#ifndef PAGEDKV_TUNE_PREFIX_HALF
#define PAGEDKV_TUNE_PREFIX_HALF 0          // 1: shared prefixes in half-size partitions
#endif

struct Plan {
  bool mma = false;
  bool persistent = false;   // tensor-core kernel on a ticket-fed persistent grid
  int hpc = 1, kvc = 1;      // CUDA-core kernel: query heads / kv heads per CTA
  bool split = false;
  int part_tokens = 0;
  int prefix_part_tokens = 0;  // shared-prefix decode: tokens per prefix partition
  int num_parts = 1;
  int stages = 2;
  size_t smem = 0;
  size_t ws_bytes = 0;
  bool cascade = false;      // shared-prefix decode: prefix pass + suffix pass + merge
  bool fold_prefix = true;   // the suffix pass folds the prefix partials (single-partition suffixes)
  int prefix_stages = 0;     // ring depth of the prefix pass
};

bool valid_block_size(int bs) { return bs == 4 || bs == 8 || bs == 16 || bs == 32 || bs == 64; }

int largest_divisor_of(int n, const int* choices, int count) {
  for (int i = 0; i < count; ++i)
    if (n % choices[i] == 0) return choices[i];
  return 1;
}

int make_plan(Plan* plan, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
              int block_size, int max_context_len, int partition_size, bool cascade = false) {
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
    return fail(PAGEDKV_EINVAL, "num_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                num_heads, num_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return fail(PAGEDKV_EUNSUPPORTED, "head_dim %d unsupported (64 or 128)", head_dim);
  if (!valid_block_size(block_size))
    return fail(PAGEDKV_EUNSUPPORTED, "block_size %d unsupported (4, 8, 16, 32 or 64)", block_size);
  if (max_context_len <= 0) return fail(PAGEDKV_EINVAL, "max_context_len must be positive");
  if (num_seqs < 0 || num_seqs > 65535)
    return fail(PAGEDKV_EUNSUPPORTED, "num_seqs %d outside [0, 65535]", num_seqs);
  const int G = num_heads / num_kv_heads;
  if (cascade && (G > 8 || block_size < 8))
    return fail(PAGEDKV_EUNSUPPORTED,
                "shared-prefix decode needs block_size >= 8 and at most 8 query heads per kv "
                "head (block_size %d, %d)", block_size, G);
  Plan p;
  p.cascade = cascade;
  // tensor cores for query groups (running the suffix pass of a shared-prefix call for one kv
  // head per query head on them too was measured slower: every suffix item folds the prefix
  // partials, so the persistent suffix CTAs wait for the whole prefix pass)
  p.mma = (G >= 2 || (cascade && PAGEDKV_TUNE_MHA_SUFFIX_MMA)) && G <= 8 && block_size >= 8;
  p.fold_prefix = !(cascade && G == 1 && PAGEDKV_TUNE_MHA_SUFFIX_MMA);
  if (!p.mma) {
    if (G == 1) {
      // widest contiguous kv-head group whose stage stays within 16 KB
      const int choices[3] = {4, 2, 1};
      p.kvc = 1;
      for (int c : choices) {
        if (num_heads % c == 0 && simt_stage_bytes(head_dim, block_size, c) <= 16384) {
          p.kvc = c;
          break;
        }
      }
      if (PAGEDKV_TUNE_SIMT_KVC == 1 || PAGEDKV_TUNE_SIMT_KVC == 2 || PAGEDKV_TUNE_SIMT_KVC == 4) {
        if (num_heads % PAGEDKV_TUNE_SIMT_KVC == 0) p.kvc = PAGEDKV_TUNE_SIMT_KVC;
      }
      p.hpc = p.kvc;
    } else {
      const int choices[4] = {8, 4, 2, 1};
      p.hpc = largest_divisor_of(G, choices, 4);
      p.kvc = 1;
    }
  }
  // split-K: explicit, or automatic for long contexts / too few CTAs to fill the GPU
  const int unit = p.mma ? 16 : block_size;
  const int align = block_size > 16 ? block_size : 16;
  if (cascade && partition_size <= 0) {
    // always split: the prefix and suffix passes each leave partial results
    p.split = true;
    p.part_tokens = AUTO_PARTITION % align == 0 ? AUTO_PARTITION : align;
  } else if (partition_size > 0) {
    if (partition_size % align != 0)
      return fail(PAGEDKV_EINVAL, "partition_size %d must be a multiple of 16 and of block_size",
                  partition_size);
    p.split = true;
    p.part_tokens = partition_size;
  } else if (partition_size == 0) {
    const int auto_part = AUTO_PARTITION % align == 0 ? AUTO_PARTITION : align;
    if (!p.mma) {
      // CUDA-core kernel: split every context longer than a partition -- smaller, more uniform
      // CTAs balance the end of the launch (measured faster at 256 and at 32 sequences) --
      // starting from 1024 tokens and halving (down to 128) until there are ~4 waves of CTAs.
      // (256 sequences of 500..1524 tokens: 1024 beat 512, 1280, 2048 and a single pass.)
      const long long groups = (long long)num_seqs * (num_heads / p.hpc);
      int pt = 2 * auto_part;
      while (pt > 128 && pt / 2 % align == 0 &&
             groups * ((max_context_len + pt - 1) / pt) < 4LL * NUM_SMS_HINT * SIMT_CTAS_PER_SM)
        pt /= 2;
      if (max_context_len > pt) {
        p.split = true;
        p.part_tokens = pt;
      }
    } else {
      const long long ctas = (long long)num_seqs * num_kv_heads;
      if (max_context_len > auto_part &&
          (max_context_len > 4 * auto_part || ctas < 2LL * NUM_SMS_HINT)) {
        p.split = true;
        p.part_tokens = auto_part;
      }
    }
  } else if (partition_size != -1) {
    return fail(PAGEDKV_EINVAL, "partition_size %d invalid (-1, 0 or a positive size)",
                partition_size);
  }
  (void)unit;
  // A shared prefix can be split into partitions of its own size (finer prefix items
  // balance the persistent grid better, but measured slower overall: more prefix partials
  // to write and to fold in).
  p.prefix_part_tokens = p.part_tokens;
  if (PAGEDKV_TUNE_PREFIX_HALF && cascade && partition_size <= 0 &&
      (p.part_tokens / 2) % align == 0)
    p.prefix_part_tokens = p.part_tokens / 2;
  if (p.split) {
    // slots: the prefix partitions, then the rest's; a shared prefix can end inside a
    // partition, so one more slot per (sequence, head)
    p.num_parts = cascade ? (max_context_len + p.prefix_part_tokens - 1) / p.prefix_part_tokens + 1
                          : (max_context_len + p.part_tokens - 1) / p.part_tokens;
    if (p.num_parts > MAX_PARTITIONS)
      return fail(PAGEDKV_EUNSUPPORTED, "%d partitions exceed %d: use a larger partition_size",
                  p.num_parts, MAX_PARTITIONS);
    p.ws_bytes = (size_t)num_seqs * num_heads * p.num_parts * (head_dim + 2) * sizeof(float);
  } else {
    p.part_tokens = ((max_context_len + block_size - 1) / block_size) * block_size;
    p.num_parts = 1;
  }
  // the tensor-core path runs persistent CTAs fed by a work counter; the counters take the
  // first WORK_COUNTER_BYTES of every workspace, the partials follow
  p.persistent = p.mma && num_seqs <= PERSISTENT_MAX_SEQS && PAGEDKV_TUNE_PERSISTENT;
  if (p.persistent || p.ws_bytes > 0) p.ws_bytes += WORK_COUNTER_BYTES;
  // ring depth: few stages and many CTAs per SM stream best (measured)
  if (p.mma) {
    // a multiple of the consumer warps, so every warp owns the same number of stages
    int st = PAGEDKV_TUNE_MMA_STAGES;
    st = ((st + MMA_CONSUMER_WARPS - 1) / MMA_CONSUMER_WARPS) * MMA_CONSUMER_WARPS;
    st = st > 16 ? 16 : st;
    auto smem_of = [&](int n) {
      return p.persistent ? mma_persistent_smem_bytes(head_dim, n, num_seqs)
                          : mma_smem_bytes(head_dim, block_size, n);
    };
    while (st > MMA_CONSUMER_WARPS && smem_of(st) > MAX_SMEM) st -= MMA_CONSUMER_WARPS;
    p.stages = st;
    p.smem = smem_of(st);
  } else {
    const size_t stage = simt_stage_bytes(head_dim, block_size, p.kvc);
    const size_t target = PAGEDKV_TUNE_SIMT_RING_BYTES;
    int st = (int)(target / stage);
    st = st < 2 ? 2 : (st > 16 ? 16 : st);
    while (st > 2 && simt_smem_bytes(head_dim, block_size, p.kvc, st) > MAX_SMEM) --st;
    p.stages = st;
    p.smem = simt_smem_bytes(head_dim, block_size, p.kvc, st);
  }
  if (cascade) {
    int st = PAGEDKV_TUNE_MMA_STAGES;
    st = ((st + MMA_CONSUMER_WARPS - 1) / MMA_CONSUMER_WARPS) * MMA_CONSUMER_WARPS;
    st = st > 16 ? 16 : st;
    while (st > MMA_CONSUMER_WARPS && mma_smem_bytes(head_dim, block_size, st) > MAX_SMEM)
      st -= MMA_CONSUMER_WARPS;
    p.prefix_stages = st;
  }
  if (p.smem > MAX_SMEM) return fail(PAGEDKV_EUNSUPPORTED, "shared memory plan too large");
  *plan = p;
  return PAGEDKV_OK;
}

// The bounded wait every pipeline uses, on an mbarrier that nothing completes:
// after timeout_ns the wait gives up, the error word gets ERR_TIMEOUT, and the
// kernel completes the phase itself and returns.
__global__ void selftest_wait_kernel(unsigned long long timeout_ns, unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t a = smem_u32(&bar);
  mbar_init(a, 1);
  fence_barrier_init();
  if (!mbar_wait(a, 0, timeout_ns)) flag_error(err, ERR_TIMEOUT);
  mbar_arrive(a);  // leave the barrier's phase complete
}

}  // namespace

// Records a failure for pagedkv_last_error() from another translation unit.
int record_error(int code, const char* message) { return fail(code, "%s", message); }

}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pagedkv_last_error(void) { return g_last_error.c_str(); }

int pagedkv_device_errors(unsigned int* flags, int clear) {
  if (!flags) return fail(PAGEDKV_EINVAL, "flags is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpyFromSymbol(flags, g_error_word, sizeof(unsigned));
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (clear) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(unsigned));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  }
  return PAGEDKV_OK;
}

int pagedkv_selftest_wait_timeout(unsigned int timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 1000000u)
    return fail(PAGEDKV_EINVAL, "timeout_us must be in [1, 1000000]");
  unsigned* err = nullptr;
  int st = error_word(&err);
  if (st != PAGEDKV_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)timeout_us * 1000ull, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return PAGEDKV_OK;
}

size_t paged_attention_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                       int block_size, int max_context_len, int partition_size) {
  Plan plan;
  if (make_plan(&plan, num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                partition_size) != PAGEDKV_OK)
    return 0;
  return plan.ws_bytes;
}

int paged_attention_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                     int block_size, int max_context_len, int partition_size) {
  Plan plan;
  const int st = make_plan(&plan, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                           max_context_len, partition_size);
  if (st != PAGEDKV_OK) return st;
  return plan.split ? plan.part_tokens : 0;
}

}  // extern "C"

namespace pkv {
namespace {

// Every decode entry point.  k_new / v_new are NULL without a fused append;
// cascade selects the shared-prefix form (seq_prefix_tokens, groups).
int decode(void* out, const void* q, const void* k_new, const void* v_new, const void* key_cache,
           const void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
           float scale, int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
           int max_blocks_per_seq, int num_blocks, int max_context_len, int partition_size,
           void* workspace, size_t workspace_bytes, void* stream, bool cascade = false,
           const int32_t* seq_prefix_tokens = nullptr, const int32_t* groups = nullptr,
           int num_groups = 0, int max_prefix_tokens = 0, int max_suffix_tokens = 0) {
  if (num_seqs == 0) return PAGEDKV_OK;
  if (cascade) {
    if (!seq_prefix_tokens) return fail(PAGEDKV_EINVAL, "seq_prefix_tokens is required");
    if (num_groups < 0 || num_groups > 65535)
      return fail(PAGEDKV_EINVAL, "num_groups %d outside [0, 65535]", num_groups);
    if (num_groups > 0 && !groups) return fail(PAGEDKV_EINVAL, "groups is NULL");
    if (max_prefix_tokens < 0 || max_suffix_tokens < 0)
      return fail(PAGEDKV_EINVAL, "max_prefix_tokens and max_suffix_tokens must be >= 0");
  }
  if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens)
    return fail(PAGEDKV_EINVAL, "a required pointer is NULL");
  if (!aligned16(out) || !aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache))
    return fail(PAGEDKV_EINVAL, "out, q and the pools must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(PAGEDKV_EINVAL, "scale must be finite");
  if (max_blocks_per_seq <= 0 || num_blocks <= 0)
    return fail(PAGEDKV_EINVAL, "max_blocks_per_seq and num_blocks must be positive");
  if ((long long)max_context_len > (long long)max_blocks_per_seq * block_size)
    return fail(PAGEDKV_EINVAL, "max_context_len %d exceeds the table (%d blocks of %d)",
                max_context_len, max_blocks_per_seq, block_size);
  Plan plan;
  int st = make_plan(&plan, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                     max_context_len, partition_size, cascade);
  if (st != PAGEDKV_OK) return st;
  const bool maps = plan.mma || (cascade && num_groups > 0);  // tensor-core passes need tensor maps
  if (maps && (long long)num_blocks * num_kv_heads * block_size > 0x7fffffffLL)
    return fail(PAGEDKV_EUNSUPPORTED, "pool of %lld rows exceeds the tensor-map range",
                (long long)num_blocks * num_kv_heads * block_size);
  if (plan.ws_bytes > 0) {
    if (!workspace || workspace_bytes < plan.ws_bytes)
      return fail(PAGEDKV_EWORKSPACE, "workspace of %zu bytes required, %zu given", plan.ws_bytes,
                  workspace ? workspace_bytes : (size_t)0);
    if (!aligned16(workspace)) return fail(PAGEDKV_EINVAL, "workspace must be 16-byte aligned");
  }
  unsigned* err = nullptr;
  st = error_word(&err);
  if (st != PAGEDKV_OK) return st;

  DecodeParams p = {};
  p.out = static_cast<__half*>(out);
  p.q = static_cast<const __half*>(q);
  p.k_cache = static_cast<const __half*>(key_cache);
  p.v_cache = static_cast<const __half*>(value_cache);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  if (plan.split) {
    p.ws_o = reinterpret_cast<float*>(static_cast<char*>(workspace) + WORK_COUNTER_BYTES);
    p.ws_ml = p.ws_o + (size_t)num_seqs * num_heads * plan.num_parts * head_dim;
  }
  p.err = err;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_seqs = num_seqs;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.head_dim = head_dim;
  p.block_size = block_size;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.max_context_len = max_context_len;
  p.part_tokens = plan.part_tokens;
  p.prefix_part_tokens = plan.prefix_part_tokens;
  p.num_parts = plan.num_parts;
  p.grid_parts = plan.num_parts;
  if (cascade && max_suffix_tokens > 0) {
    const int need = (max_suffix_tokens + plan.part_tokens - 1) / plan.part_tokens;
    if (need < p.grid_parts) p.grid_parts = need;
  }
  // With a shared prefix and every suffix within one partition, the partition
  // pass finishes every output itself: no merge.
  const bool merged = cascade && plan.fold_prefix && max_suffix_tokens > 0 &&
                      max_suffix_tokens <= plan.part_tokens;
  p.fold_prefix = plan.fold_prefix ? 1 : 0;
  p.no_merge = merged ? 1 : 0;
  p.stages = plan.stages;
  p.k_new = static_cast<const __half*>(k_new);
  p.v_new = static_cast<const __half*>(v_new);
  p.seq_prefix_tokens = cascade ? seq_prefix_tokens : nullptr;
  p.groups = cascade ? groups : nullptr;
  p.num_groups = cascade ? num_groups : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e;
  CUtensorMap km, vm;
  if (maps) {
    const int rows = num_blocks * num_kv_heads * block_size;
    st = encode_pool_map(&km, key_cache, rows, head_dim, block_size);
    if (st != PAGEDKV_OK) return st;
    st = encode_pool_map(&vm, value_cache, rows, head_dim, block_size);
    if (st != PAGEDKV_OK) return st;
  }
  // work counters (self-resetting: the last CTA of a persistent launch zeroes its pass's
  // 16 bytes): the decode pass's first, then the prefix pass's
  unsigned int* counters =
      plan.ws_bytes > 0 ? reinterpret_cast<unsigned int*>(workspace) : nullptr;
  const bool prefix_pass = cascade && num_groups > 0;
  if (prefix_pass) {
    // Prefix pass first.  The suffix pass is its programmatic dependent: it may
    // start on the SMs the prefix pass frees and waits for it only before it
    // reads the prefix partials; the merge follows the suffix pass.
    DecodeParams pp = p;
    pp.stages = plan.prefix_stages;
    pp.k_new = pp.v_new = nullptr;
    pp.no_merge = 0;  // its partial results are always folded in later
    const int ppt = plan.prefix_part_tokens;
    int prefix_parts = (max_context_len + ppt - 1) / ppt;
    if (max_prefix_tokens > 0) {
      const int need = (max_prefix_tokens + ppt - 1) / ppt;
      if (need < prefix_parts) prefix_parts = need;
    }
    // persistent CTAs stream the prefix items from a ticket queue; beyond the
    // persistent grid's row limit, one CTA per item
    if (num_groups <= PERSISTENT_MAX_SEQS)
      e = launch_mma_prefix_persistent(pp, km, vm, counters, prefix_parts, s);
    else
      e = launch_mma_prefix(pp, km, vm, prefix_parts, s);
    if (e != cudaSuccess) return cuda_fail(e, "shared-prefix pass launch");
    p.after_prefix = 1;
  }
  if (plan.mma) {
    if (plan.persistent) {
      e = launch_mma_decode_persistent(p, km, vm, counters, plan.split, s);
    } else {
      e = launch_mma_decode(p, km, vm, plan.split, s);
    }
  } else {
    e = launch_simt_decode(p, plan.hpc, plan.kvc, plan.split, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  if (plan.split && !merged) {
    e = launch_split_reduce(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "split-K merge launch");
  }
  return PAGEDKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" {

int paged_attention_decode(void* out, const void* q, const void* key_cache, const void* value_cache,
                           const int32_t* block_tables, const int32_t* context_lens, float scale,
                           int block_size, int num_kv_heads, int num_seqs, int num_heads,
                           int head_dim, int max_blocks_per_seq, int num_blocks,
                           int max_context_len, int partition_size, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return decode(out, q, nullptr, nullptr, key_cache, value_cache, block_tables, context_lens,
                scale, block_size, num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq,
                num_blocks, max_context_len, partition_size, workspace, workspace_bytes, stream);
}

int paged_attention_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                                  void* key_cache, void* value_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, float scale, int block_size,
                                  int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                  int max_blocks_per_seq, int num_blocks, int max_context_len,
                                  int partition_size, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (num_seqs == 0) return PAGEDKV_OK;
  if (!k_new || !v_new) return fail(PAGEDKV_EINVAL, "k_new and v_new are required");
  if (!aligned16(k_new) || !aligned16(v_new))
    return fail(PAGEDKV_EINVAL, "k_new and v_new must be 16-byte aligned");
  return decode(out, q, k_new, v_new, key_cache, value_cache, block_tables, context_lens, scale,
                block_size, num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq,
                num_blocks, max_context_len, partition_size, workspace, workspace_bytes, stream);
}

int paged_attention_decode_shared_prefix(
    void* out, const void* q, const void* k_new, const void* v_new, void* key_cache,
    void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
    const int32_t* seq_prefix_tokens, const int32_t* groups, int num_groups,
    int max_prefix_tokens, int max_suffix_tokens, float scale,
    int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
    int max_blocks_per_seq, int num_blocks, int max_context_len, int partition_size,
    void* workspace, size_t workspace_bytes, void* stream) {
  if (num_seqs == 0) return PAGEDKV_OK;
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(PAGEDKV_EINVAL, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned16(k_new) || !aligned16(v_new)))
    return fail(PAGEDKV_EINVAL, "k_new and v_new must be 16-byte aligned");
  return decode(out, q, k_new, v_new, key_cache, value_cache, block_tables, context_lens, scale,
                block_size, num_kv_heads, num_seqs, num_heads, head_dim, max_blocks_per_seq,
                num_blocks, max_context_len, partition_size, workspace, workspace_bytes, stream,
                true, seq_prefix_tokens, groups, num_groups, max_prefix_tokens,
                max_suffix_tokens);
}

size_t paged_attention_shared_prefix_workspace_bytes(int num_seqs, int num_heads,
                                                     int num_kv_heads, int head_dim,
                                                     int block_size, int max_context_len,
                                                     int partition_size) {
  Plan plan;
  if (make_plan(&plan, num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                partition_size, true) != PAGEDKV_OK)
    return 0;
  return plan.ws_bytes;
}

int reshape_and_cache(const void* k, const void* v, void* key_cache, void* value_cache,
                      const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                      int block_size, int num_blocks, void* stream) {
  if (num_tokens == 0) return PAGEDKV_OK;
  if (num_tokens < 0) return fail(PAGEDKV_EINVAL, "num_tokens must be >= 0");
  if (!k || !v || !key_cache || !value_cache || !slot_mapping)
    return fail(PAGEDKV_EINVAL, "a required pointer is NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(key_cache) || !aligned16(value_cache))
    return fail(PAGEDKV_EINVAL, "k, v and the pools must be 16-byte aligned");
  if (num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 != 0 || block_size <= 0 || num_blocks <= 0)
    return fail(PAGEDKV_EINVAL, "bad shape (kv heads %d, head_dim %d, block_size %d, blocks %d)",
                num_kv_heads, head_dim, block_size, num_blocks);
  unsigned* err = nullptr;
  int st = error_word(&err);
  if (st != PAGEDKV_OK) return st;
  cudaError_t e = launch_reshape_and_cache(
      static_cast<const __half*>(k), static_cast<const __half*>(v), static_cast<__half*>(key_cache),
      static_cast<__half*>(value_cache), slot_mapping, num_tokens, num_kv_heads, head_dim,
      block_size, num_blocks, err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reshape_and_cache launch");
  return PAGEDKV_OK;
}

int copy_blocks(void* const* key_caches, void* const* value_caches, const int64_t* src_dst_pairs,
                int num_pairs, int num_layers, size_t block_elems, int num_blocks, void* stream) {
  if (num_pairs == 0) return PAGEDKV_OK;
  if (num_pairs < 0 || num_pairs > 65535)
    return fail(PAGEDKV_EINVAL, "num_pairs %d outside [0, 65535]", num_pairs);
  if (num_layers <= 0 || num_layers > MAX_COPY_LAYERS)
    return fail(PAGEDKV_EINVAL, "num_layers %d outside [1, %d]", num_layers, MAX_COPY_LAYERS);
  if (!key_caches || !value_caches || !src_dst_pairs)
    return fail(PAGEDKV_EINVAL, "a required pointer is NULL");
  if (block_elems == 0 || block_elems % 8 != 0 || num_blocks <= 0)
    return fail(PAGEDKV_EINVAL, "block_elems must be a positive multiple of 8");
  for (int l = 0; l < num_layers; ++l) {
    if (!key_caches[l] || !value_caches[l] || !aligned16(key_caches[l]) || !aligned16(value_caches[l]))
      return fail(PAGEDKV_EINVAL, "layer %d pool pointer NULL or not 16-byte aligned", l);
  }
  unsigned* err = nullptr;
  int st = error_word(&err);
  if (st != PAGEDKV_OK) return st;
  cudaError_t e = launch_copy_blocks(key_caches, value_caches, src_dst_pairs, num_pairs, num_layers,
                                     block_elems, num_blocks, err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "copy_blocks launch");
  return PAGEDKV_OK;
}

}  // extern "C"

// ---- one decode step from host buffers ---------------------------------------------

namespace pkv {
namespace {

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Offsets of the regions of the caller's staging buffer (each 256-byte aligned).
struct StepLayout {
  size_t q, k, v, tables, lens, pairs, out, prefix, groups, ws, ws2;
  size_t ws_bytes, total;
  int chunk_part;  // partition_size of every chunk's call: the whole batch's partitioning
};

// The plain host step splits a batch into chunks of sequences so that uploading
// chunk c + 1 and downloading chunk c - 1 overlap the attention of chunk c: up to
// STEP_MAX_CHUNKS chunks of at least STEP_CHUNK_SEQS sequences, alternating over
// two compute streams (each with its own workspace) so that one chunk's last
// CTAs and merge overlap the next chunk's start.  The shared-prefix step runs
// whole (its groups span the batch).
#ifndef PAGEDKV_TUNE_STEP_CHUNKS
#define PAGEDKV_TUNE_STEP_CHUNKS 4
#endif
#ifndef PAGEDKV_TUNE_STEP_CHUNK_SEQS
#define PAGEDKV_TUNE_STEP_CHUNK_SEQS 64
#endif
#ifndef PAGEDKV_TUNE_STEP_END_QUARTERS
#define PAGEDKV_TUNE_STEP_END_QUARTERS 2  // half-size end chunks (measured faster than equal)
#endif
constexpr size_t STEP_SMALL_COPY = 65536;  // host copies below this are staged by the CPU
constexpr int STEP_MAX_CHUNKS = PAGEDKV_TUNE_STEP_CHUNKS;
constexpr int STEP_CHUNK_SEQS = PAGEDKV_TUNE_STEP_CHUNK_SEQS;

int step_chunks(int num_seqs, bool shared_prefix) {
  if (shared_prefix) return 1;
  const int c = num_seqs / STEP_CHUNK_SEQS;
  return c < 1 ? 1 : (c > STEP_MAX_CHUNKS ? STEP_MAX_CHUNKS : c);
}

// Sequences [first, first + count) of chunk i of n.  The first and last chunks weigh
// E = PAGEDKV_TUNE_STEP_END_QUARTERS quarters of a middle chunk: smaller end chunks
// shrink the first upload and the last download, which nothing overlaps.
void chunk_range(int num_seqs, int n, int i, int* first, int* count) {
  const long long E = PAGEDKV_TUNE_STEP_END_QUARTERS;
  const long long total = n < 2 ? 1 : 2 * E + 4LL * (n - 2);
  auto edge = [&](int k) -> int {  // first sequence of chunk k
    if (k <= 0) return 0;
    if (k >= n) return num_seqs;
    return (int)((long long)num_seqs * (E + 4LL * (k - 1)) / total);
  };
  *first = edge(i);
  *count = edge(i + 1) - *first;
}

int step_layout(StepLayout* lay, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                int block_size, int max_blocks_per_seq, int max_context_len, int partition_size,
                int max_pairs, bool shared_prefix) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || max_pairs < 0)
    return fail(PAGEDKV_EINVAL, "num_seqs, max_blocks_per_seq and max_pairs must be >= 0 (> 0)");
  Plan plan;
  const int st = make_plan(&plan, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                           max_context_len, partition_size, shared_prefix);
  if (st != PAGEDKV_OK) return st;
  const size_t B = (size_t)num_seqs, H = (size_t)num_heads, Hk = (size_t)num_kv_heads,
               D = (size_t)head_dim;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  lay->q = take(B * H * D * 2);
  lay->k = take(B * Hk * D * 2);
  lay->v = take(B * Hk * D * 2);
  lay->tables = take(B * (size_t)max_blocks_per_seq * 4);
  lay->lens = take(B * 4);
  lay->pairs = take((size_t)max_pairs * 16);
  lay->out = take(B * H * D * 2);
  lay->prefix = shared_prefix ? take(B * 4) : 0;
  lay->groups = shared_prefix ? take((B / 2 > 0 ? B / 2 : 1) * GROUP_WIDTH * 4) : 0;
  // Every chunk is split as the whole batch would be (its partition size, or a single
  // pass), so that each (sequence, head) is computed exactly as by one call over the
  // batch.  The chunks share two workspaces: size them for the largest chunk plan.
  lay->chunk_part = partition_size != 0 ? partition_size : (plan.split ? plan.part_tokens : -1);
  size_t ws = plan.ws_bytes;
  const int n = step_chunks(num_seqs, shared_prefix);
  for (int i = 0; i < n && n > 1; ++i) {
    int first = 0, count = 0;
    chunk_range(num_seqs, n, i, &first, &count);
    Plan cp;
    if (make_plan(&cp, count, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                  lay->chunk_part, false) == PAGEDKV_OK && cp.ws_bytes > ws)
      ws = cp.ws_bytes;
  }
  lay->ws = take(ws);
  lay->ws2 = n > 1 ? take(ws) : lay->ws;  // the second compute stream's workspace
  lay->ws_bytes = ws;
  lay->total = off;
  return PAGEDKV_OK;
}

// Copy-on-write pairs that one copy_blocks launch may apply in any order: ids in
// range, no destination repeated, no destination also a source.
int check_pairs(const int64_t* pairs, int n, int num_blocks) {
  std::vector<char> role((size_t)num_blocks, 0);  // 1 = source, 2 = destination
  for (int i = 0; i < n; ++i) {
    const int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks)
      return fail(PAGEDKV_EINVAL, "copy pair %d (%lld, %lld) outside the pool", i, (long long)s,
                  (long long)d);
    if (role[(size_t)s] == 2 || role[(size_t)d] != 0)
      return fail(PAGEDKV_EINVAL, "copy pair %d (%lld, %lld) overlaps an earlier pair", i,
                  (long long)s, (long long)d);
    role[(size_t)s] = 1;
    role[(size_t)d] = 2;
  }
  return PAGEDKV_OK;
}

int h2d(void* dst, const void* src, size_t bytes, cudaStream_t s, const char* what) {
  if (bytes == 0) return PAGEDKV_OK;
  const cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, s);
  return e == cudaSuccess ? PAGEDKV_OK : cuda_fail(e, what);
}

// Copy streams and events of the pipelined host step, per host thread and device,
// created at the first chunked call and kept until the process exits.
struct StepAux {
  cudaStream_t up, down, comp;  // uploads, downloads, the second compute stream
  cudaEvent_t start, copied, done, in[STEP_MAX_CHUNKS], out[STEP_MAX_CHUNKS];
  bool ready;
};
thread_local StepAux tl_step_aux[MAX_DEVICES];

int step_aux(StepAux** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= MAX_DEVICES) return fail(PAGEDKV_ECUDA, "device id %d out of range", dev);
  StepAux& a = tl_step_aux[dev];
  if (!a.ready) {
    if ((e = cudaStreamCreateWithFlags(&a.up, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&a.down, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&a.comp, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "creating the step's streams");
    cudaEvent_t* evs[3 + 2 * STEP_MAX_CHUNKS] = {&a.start, &a.copied, &a.done};
    for (int i = 0; i < STEP_MAX_CHUNKS; ++i) {
      evs[3 + i] = &a.in[i];
      evs[3 + STEP_MAX_CHUNKS + i] = &a.out[i];
    }
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
        return cuda_fail(e, "creating the step's events");
    a.ready = true;
  }
  *out = &a;
  return PAGEDKV_OK;
}

#define PKV_CHECK_CUDA(call, what)                 \
  do {                                             \
    const cudaError_t e_ = (call);                 \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

}  // namespace
}  // namespace pkv

extern "C" {

size_t paged_decode_step_staging_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int block_size, int max_blocks_per_seq,
                                       int max_context_len, int partition_size, int max_pairs,
                                       int shared_prefix) {
  StepLayout lay;
  if (step_layout(&lay, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                  max_blocks_per_seq, max_context_len, partition_size, max_pairs,
                  shared_prefix != 0) != PAGEDKV_OK)
    return 0;
  return lay.total;
}

int paged_decode_step_host(void* out_host, const void* q_host, const void* k_new_host,
                           const void* v_new_host, const int32_t* block_tables_host,
                           const int32_t* context_lens_host, const int64_t* copy_pairs_host,
                           int num_pairs, const int32_t* seq_prefix_tokens_host,
                           const int32_t* groups_host, int num_groups, void* key_cache,
                           void* value_cache, float scale, int block_size, int num_kv_heads,
                           int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                           int num_blocks, int max_context_len, int partition_size, int max_pairs,
                           void* staging, size_t staging_bytes, void* stream) {
  if (num_seqs < 0) return fail(PAGEDKV_EINVAL, "num_seqs must be >= 0");
  if (num_pairs < 0 || num_pairs > max_pairs)
    return fail(PAGEDKV_EINVAL, "num_pairs %d outside [0, max_pairs = %d]", num_pairs, max_pairs);
  if (num_seqs == 0 && num_pairs == 0) return PAGEDKV_OK;
  const bool shared = seq_prefix_tokens_host != nullptr;
  if (!key_cache || !value_cache || !staging ||
      (num_seqs > 0 && (!out_host || !q_host || !k_new_host || !v_new_host ||
                        !block_tables_host || !context_lens_host)) ||
      (num_pairs > 0 && !copy_pairs_host) || (shared && num_groups > 0 && !groups_host))
    return fail(PAGEDKV_EINVAL, "a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0)
    return fail(PAGEDKV_EINVAL, "staging must be 256-byte aligned");
  if (num_blocks <= 0) return fail(PAGEDKV_EINVAL, "num_blocks must be positive");
  StepLayout lay;
  int st = step_layout(&lay, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                       max_blocks_per_seq, max_context_len, partition_size, max_pairs, shared);
  if (st != PAGEDKV_OK) return st;
  if (staging_bytes < lay.total)
    return fail(PAGEDKV_EWORKSPACE, "staging of %zu bytes required, %zu given", lay.total,
                staging_bytes);
  // host-side checks of what the host already holds
  for (int b = 0; b < num_seqs; ++b) {
    const int L = context_lens_host[b];
    if (L < 1 || L > max_context_len)
      return fail(PAGEDKV_EINVAL, "context_lens[%d] = %d outside [1, max_context_len = %d]", b, L,
                  max_context_len);
  }
  st = check_pairs(copy_pairs_host, num_pairs, num_blocks);
  if (st != PAGEDKV_OK) return st;
  int max_prefix = 0, max_suffix = 0;
  if (shared) {
    if (num_groups < 0 || num_groups > (num_seqs / 2 > 0 ? num_seqs / 2 : 1))
      return fail(PAGEDKV_EINVAL, "num_groups %d outside [0, num_seqs / 2]", num_groups);
    for (int g = 0; g < num_groups; ++g) {
      const int pb = groups_host[(size_t)g * GROUP_WIDTH];
      if (pb > 0 && (long long)pb * block_size > max_prefix)
        max_prefix = (int)std::min<long long>((long long)pb * block_size, max_context_len);
    }
    // every sequence with a prefix must be a member of a group with that prefix length
    // (the device path cannot see a sequence that no group lists)
    std::vector<char> listed((size_t)num_seqs, 0);
    for (int g = 0; g < num_groups; ++g) {
      const int32_t* gd = groups_host + (size_t)g * GROUP_WIDTH;
      for (int i = 1; i < GROUP_WIDTH; ++i) {
        const int m = gd[i];
        if (m >= 0 && m < num_seqs && seq_prefix_tokens_host[m] == gd[0] * block_size)
          listed[(size_t)m] = 1;
      }
    }
    for (int b = 0; b < num_seqs; ++b) {
      const int P = seq_prefix_tokens_host[b];
      const int L = context_lens_host[b];
      if (P != 0 && !listed[(size_t)b])
        return fail(PAGEDKV_EINVAL, "sequence %d has %d prefix tokens but no group lists it", b,
                    P);
      // a prefix length the kernels reject counts as 0 (they flag it)
      const int rest = (P > 0 && P % block_size == 0 && P <= L - 1) ? L - P : L;
      max_suffix = rest > max_suffix ? rest : max_suffix;
    }
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(staging);
  const size_t B = (size_t)num_seqs, H = (size_t)num_heads, Hk = (size_t)num_kv_heads,
               D = (size_t)head_dim;
  const int nch = step_chunks(num_seqs, shared);
  if (nch > 1) {
    // Pipelined: the uploads run chunk by chunk, and each chunk's attention starts as
    // soon as its inputs have landed; each chunk's output is downloaded on a copy
    // stream while the next chunk computes.  The caller's stream waits for the last
    // download, so work it enqueues later (the next step overwriting this staging)
    // comes after all of it.
    StepAux* aux = nullptr;
    if ((st = step_aux(&aux)) != PAGEDKV_OK) return st;
    // On an error return after work was enqueued, the caller's stream still waits for
    // whatever the side streams hold (best effort), so that its next use of this
    // staging comes after it.
    struct SideJoin {
      cudaStream_t s;
      StepAux* aux;
      bool armed;
      ~SideJoin() {
        if (!armed) return;
        for (cudaStream_t side : {aux->up, aux->comp, aux->down}) {
          if (cudaEventRecord(aux->done, side) == cudaSuccess)
            cudaStreamWaitEvent(s, aux->done, 0);
        }
      }
    } side_join{s, aux, true};
    const size_t row_q = H * D * 2, row_kv = Hk * D * 2, row_t = (size_t)max_blocks_per_seq * 4;
    // Table rows go up with each chunk when every chunk's rows are a large copy of their
    // own; otherwise the whole table goes once, ahead of the first chunk.  (Copies below
    // STEP_SMALL_COPY bytes are staged by the host CPU, several microseconds each.)
    int min_count = num_seqs;
    for (int c = 0; c < nch; ++c) {
      int first = 0, count = 0;
      chunk_range(num_seqs, nch, c, &first, &count);
      min_count = count < min_count ? count : min_count;
    }
    const bool rows_per_chunk = (size_t)min_count * row_t >= STEP_SMALL_COPY;
    // uploads of chunk c: its table rows (when they go per chunk), q and new K/V rows
    auto upload = [&](int c, cudaStream_t us) -> int {
      int first = 0, count = 0, r = PAGEDKV_OK;
      chunk_range(num_seqs, nch, c, &first, &count);
      if ((rows_per_chunk &&
           (r = h2d(base + lay.tables + first * row_t,
                    reinterpret_cast<const char*>(block_tables_host) + first * row_t,
                    count * row_t, us, "block table upload")) != PAGEDKV_OK) ||
          (r = h2d(base + lay.q + first * row_q, static_cast<const char*>(q_host) + first * row_q,
                   count * row_q, us, "query upload")) != PAGEDKV_OK ||
          (r = h2d(base + lay.k + first * row_kv,
                   static_cast<const char*>(k_new_host) + first * row_kv, count * row_kv, us,
                   "new K upload")) != PAGEDKV_OK ||
          (r = h2d(base + lay.v + first * row_kv,
                   static_cast<const char*>(v_new_host) + first * row_kv, count * row_kv, us,
                   "new V upload")) != PAGEDKV_OK)
        return r;
      return PAGEDKV_OK;
    };
    // The pairs, the lengths, the table (unless it goes per chunk) and the first chunk's
    // inputs go up on the caller's stream, ahead of its kernels with no cross-stream wait
    // (and after the previous step on it, which read this staging); the copy stream
    // takes the other chunks once they have landed.
    if ((st = h2d(base + lay.pairs, copy_pairs_host, (size_t)num_pairs * 16, s,
                  "pair upload")) != PAGEDKV_OK ||
        (st = h2d(base + lay.lens, context_lens_host, B * 4, s, "context length upload")) !=
            PAGEDKV_OK ||
        (!rows_per_chunk && (st = h2d(base + lay.tables, block_tables_host, B * row_t, s,
                                      "block table upload")) != PAGEDKV_OK) ||
        (st = upload(0, s)) != PAGEDKV_OK)
      return st;
    PKV_CHECK_CUDA(cudaEventRecord(aux->start, s), "step start");
    PKV_CHECK_CUDA(cudaStreamWaitEvent(aux->up, aux->start, 0), "upload wait");
    for (int c = 1; c < nch; ++c) {
      if ((st = upload(c, aux->up)) != PAGEDKV_OK) return st;
      PKV_CHECK_CUDA(cudaEventRecord(aux->in[c], aux->up), "upload event");
    }
    if (num_pairs > 0) {
      void* kc[1] = {key_cache};
      void* vc[1] = {value_cache};
      st = copy_blocks(kc, vc, reinterpret_cast<const int64_t*>(base + lay.pairs), num_pairs, 1,
                       (size_t)num_kv_heads * block_size * head_dim, num_blocks, stream);
      if (st != PAGEDKV_OK) return st;
    }
    // the second compute stream starts after the copies (and after earlier work on s)
    PKV_CHECK_CUDA(cudaEventRecord(aux->copied, s), "copy event");
    PKV_CHECK_CUDA(cudaStreamWaitEvent(aux->comp, aux->copied, 0), "compute wait");
    for (int c = 0; c < nch; ++c) {
      int first = 0, count = 0;
      chunk_range(num_seqs, nch, c, &first, &count);
      // even chunks on the caller's stream, odd ones on the second, each with its workspace
      cudaStream_t cs = (c & 1) ? aux->comp : s;
      void* ws = lay.ws_bytes ? base + ((c & 1) ? lay.ws2 : lay.ws) : nullptr;
      if (c > 0) PKV_CHECK_CUDA(cudaStreamWaitEvent(cs, aux->in[c], 0), "compute wait");
      st = paged_attention_decode_append(
          base + lay.out + first * row_q, base + lay.q + first * row_q,
          base + lay.k + first * row_kv, base + lay.v + first * row_kv, key_cache, value_cache,
          reinterpret_cast<const int32_t*>(base + lay.tables + first * row_t),
          reinterpret_cast<const int32_t*>(base + lay.lens) + first, scale, block_size,
          num_kv_heads, count, num_heads, head_dim, max_blocks_per_seq, num_blocks,
          max_context_len, lay.chunk_part, ws, lay.ws_bytes, cs);
      if (st != PAGEDKV_OK) return st;
      PKV_CHECK_CUDA(cudaEventRecord(aux->out[c], cs), "compute event");
      PKV_CHECK_CUDA(cudaStreamWaitEvent(aux->down, aux->out[c], 0), "download wait");
      PKV_CHECK_CUDA(cudaMemcpyAsync(static_cast<char*>(out_host) + first * row_q,
                                     base + lay.out + first * row_q, count * row_q,
                                     cudaMemcpyDeviceToHost, aux->down),
                     "output download");
    }
    // the caller's stream joins the downloads (which follow every chunk's kernels)
    PKV_CHECK_CUDA(cudaEventRecord(aux->done, aux->down), "download event");
    PKV_CHECK_CUDA(cudaStreamWaitEvent(s, aux->done, 0), "step join");
    side_join.armed = false;
    return PAGEDKV_OK;
  }
  // 1. the step's inputs, host to device (small arrays first)
  if ((st = h2d(base + lay.tables, block_tables_host, B * max_blocks_per_seq * 4, s,
                "block table upload")) != PAGEDKV_OK ||
      (st = h2d(base + lay.lens, context_lens_host, B * 4, s, "context length upload")) !=
          PAGEDKV_OK ||
      (st = h2d(base + lay.pairs, copy_pairs_host, (size_t)num_pairs * 16, s, "pair upload")) !=
          PAGEDKV_OK)
    return st;
  if (shared &&
      ((st = h2d(base + lay.prefix, seq_prefix_tokens_host, B * 4, s, "prefix upload")) !=
           PAGEDKV_OK ||
       (st = h2d(base + lay.groups, groups_host, (size_t)num_groups * GROUP_WIDTH * 4, s,
                 "group upload")) != PAGEDKV_OK))
    return st;
  if ((st = h2d(base + lay.q, q_host, B * H * D * 2, s, "query upload")) != PAGEDKV_OK ||
      (st = h2d(base + lay.k, k_new_host, B * Hk * D * 2, s, "new K upload")) != PAGEDKV_OK ||
      (st = h2d(base + lay.v, v_new_host, B * Hk * D * 2, s, "new V upload")) != PAGEDKV_OK)
    return st;
  // 2. copy-on-write copies before any write into their destinations
  if (num_pairs > 0) {
    void* kc[1] = {key_cache};
    void* vc[1] = {value_cache};
    st = copy_blocks(kc, vc, reinterpret_cast<const int64_t*>(base + lay.pairs), num_pairs, 1,
                     (size_t)num_kv_heads * block_size * head_dim, num_blocks, stream);
    if (st != PAGEDKV_OK) return st;
  }
  if (num_seqs == 0) return PAGEDKV_OK;
  // 3. new rows written at position L - 1, then the attention over the updated cache
  void* ws = lay.ws_bytes ? base + lay.ws : nullptr;
  const int32_t* tables = reinterpret_cast<const int32_t*>(base + lay.tables);
  const int32_t* lens = reinterpret_cast<const int32_t*>(base + lay.lens);
  if (shared) {
    st = paged_attention_decode_shared_prefix(
        base + lay.out, base + lay.q, base + lay.k, base + lay.v, key_cache, value_cache, tables,
        lens, reinterpret_cast<const int32_t*>(base + lay.prefix),
        num_groups ? reinterpret_cast<const int32_t*>(base + lay.groups) : nullptr, num_groups,
        max_prefix, max_suffix, scale, block_size, num_kv_heads, num_seqs, num_heads, head_dim,
        max_blocks_per_seq, num_blocks, max_context_len, partition_size, ws, lay.ws_bytes, stream);
  } else {
    st = paged_attention_decode_append(base + lay.out, base + lay.q, base + lay.k, base + lay.v,
                                       key_cache, value_cache, tables, lens, scale, block_size,
                                       num_kv_heads, num_seqs, num_heads, head_dim,
                                       max_blocks_per_seq, num_blocks, max_context_len,
                                       partition_size, ws, lay.ws_bytes, stream);
  }
  if (st != PAGEDKV_OK) return st;
  // 4. the output back to the host
  const cudaError_t e =
      cudaMemcpyAsync(out_host, base + lay.out, B * H * D * 2, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "output download");
  return PAGEDKV_OK;
}

}  // extern "C"
