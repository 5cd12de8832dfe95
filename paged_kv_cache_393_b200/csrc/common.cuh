// Device helpers shared by the paged-KV kernels (sm_100a).
//
// Thin inline-PTX wrappers for the Blackwell/Hopper asynchronous copy engine
// (1-D bulk copies and tiled tensor copies, both completing on an mbarrier),
// the mbarrier itself, and the warp-level tensor-core instructions used by the
// grouped-query kernel (ldmatrix, movmatrix, mma.m16n8k16).
//
// Every wait is bounded: after WAIT_TIMEOUT_NS the caller gets `false`, sets
// ERR_TIMEOUT in the error word and winds down instead of spinning forever.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace pkv {

// Bits of the per-device error word (mirrors PAGEDKV_DEVERR_* in pagedkv.h).
constexpr unsigned ERR_BLOCK_ID = 1u;
constexpr unsigned ERR_CONTEXT_LEN = 2u;
constexpr unsigned ERR_SLOT = 4u;
constexpr unsigned ERR_TIMEOUT = 8u;
constexpr unsigned ERR_INTERNAL = 16u;
constexpr unsigned ERR_PREFIX = 32u;

constexpr unsigned long long WAIT_TIMEOUT_NS = 2000000000ull;  // 2 s

__device__ __forceinline__ void flag_error(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// Tokens of a sequence that its shared-prefix group covers (0 = none): a whole
// number of blocks that leaves at least the last token to the sequence itself.
// Any other value is reported through *bad and treated as 0 by every kernel.
// The shared-prefix tokens of a sequence of length L, given its entry P of
// seq_prefix_tokens: 0 when it has none or when P is not a whole number of blocks
// below L (then *bad is set).
__device__ __forceinline__ int prefix_tokens_checked(int P, int L, int bs, bool* bad) {
  if (P == 0) return 0;
  if (P < 0 || P % bs != 0 || P > L - 1) {
    *bad = true;
    return 0;
  }
  return P;
}

__device__ __forceinline__ int prefix_tokens_of(const int32_t* seq_prefix_tokens, int b, int L,
                                                int bs, bool* bad) {
  if (!seq_prefix_tokens) return 0;
  return prefix_tokens_checked(seq_prefix_tokens[b], L, bs, bad);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier -----------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the other threads and to the async proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) accesses of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete; false after the timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          unsigned long long timeout_ns = WAIT_TIMEOUT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// ---- asynchronous copies (TMA) -------------------------------------------------

// L2 policy for data streamed exactly once (K/V tiles): evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned)
// from global memory into this CTA's shared memory; completes tx on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// Tiled 2-D tensor copy (box given by the tensor map) into shared memory.
// x is the innermost coordinate (must be a multiple of 16 bytes / element size).
__device__ __forceinline__ void tensor_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                               uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---- fused append -----------------------------------------------------------------
//
// The attention kernels can write the step's new K/V row themselves (the
// scatter of the new token into its block, then the gather that reads it back:
// lpnh.cn/news/1824136 §3.1).  The producer warp stores the row with ordinary
// (generic-proxy) stores, orders them before its own later copies with a proxy
// fence, and only then issues the copy of the stage that holds the row, so the
// consumers read it like any other row.

// 16-byte relaxed store at gpu scope.  Several CTAs may store the same new row
// (query groups split over CTAs); relaxed stores of identical bytes do not race.
__device__ __forceinline__ void st_relaxed_gpu_v4(void* ptr, uint4 v) {
  asm volatile("st.relaxed.gpu.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Orders this thread's earlier generic-proxy global writes before its later
// async-proxy (bulk / tensor copy) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// The new K and V rows of NH consecutive kv heads (kv0 ..), spread as 16-byte
// vectors over the 32 lanes of a warp: vectors [0, NH*D/8) are K, the rest V.
template <int D, int NH>
struct NewRows {
  static constexpr int VPH = D / 8;             // vectors per head row
  static constexpr int NV = 2 * NH * VPH;
  static constexpr int PER_LANE = (NV + 31) / 32;
  uint4 v[PER_LANE];

  // k_new / v_new are [num_seqs][num_kv_heads][D]; the NH rows are contiguous.
  __device__ __forceinline__ void load(const __half* k_new, const __half* v_new, int b,
                                       int num_kv_heads, int kv0, int lane) {
    const size_t row0 = ((size_t)b * num_kv_heads + kv0) * D;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
      const int idx = lane + 32 * i;
      if (idx < NV) {
        const bool is_v = idx >= NH * VPH;
        const int off = is_v ? idx - NH * VPH : idx;
        v[i] = __ldg(reinterpret_cast<const uint4*>((is_v ? v_new : k_new) + row0) + off);
      }
    }
  }

  // Stores the rows into row r of physical block phys of the pools
  // ([N][Hk][bs][D]) and fences them before this warp's later copies.
  // Called by all 32 lanes.
  __device__ __forceinline__ void store(__half* k_cache, __half* v_cache, int num_kv_heads,
                                        int bs, int kv0, int phys, int r, int lane) const {
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
      const int idx = lane + 32 * i;
      if (idx < NV) {
        const bool is_v = idx >= NH * VPH;
        const int off = is_v ? idx - NH * VPH : idx;
        const int h = off / VPH;
        __half* dst = (is_v ? v_cache : k_cache) +
                      (((size_t)phys * num_kv_heads + kv0 + h) * bs + r) * D + (off % VPH) * 8;
        st_relaxed_gpu_v4(dst, v[i]);
      }
    }
    fence_proxy_async_global();
    __syncwarp();
  }
};

// ---- warp-level tensor-core helpers --------------------------------------------

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of an 8x8 b16 matrix held one 32-bit fragment per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D = A(16x16, row) * B(16x8, col) + D, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t x) {
  __half2 h = *reinterpret_cast<__half2*>(&x);
  return __half22float2(h);
}

// Online-softmax rescale factor 2^(m_old - m_new) for running maxima in log2
// units; a running max that is still -inf (nothing accumulated) gives 0.
__device__ __forceinline__ float rescale_factor(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
}

}  // namespace pkv
