// Merge of split-K partitions into the attention output (sm_100a).
//
// With partition maxima m_i (log2 units), sums l_i and unnormalised outputs
// o_i of one (sequence, head), the softmax over the whole context is
//     out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i,   M = max_i m_i,
// the same online-softmax rescaling the partition kernels use inside a
// partition.  Contexts that fit in one partition were written by the
// partition kernel itself and are skipped here.  With shared prefixes the
// slots of a (sequence, head) are its prefix partitions, then the partitions
// of the rest of its context.
//
// One CTA per (sequence, head): warp 0 turns the partition maxima into
// normalised weights in shared memory, then the threads split into groups
// over the partitions (each thread one float4 of D, every 4th-or-so
// partition), and the groups' sums are added through shared memory.  Many
// small CTAs keep enough loads in flight for the longest contexts.  The
// kernel is launched as a programmatic dependent of the partition pass: its
// CTAs can be resident before that pass ends and wait (griddepcontrol.wait)
// for its results.
#include "common.cuh"
#include "kernels.h"

namespace pkv {
namespace {

constexpr int MERGE_THREADS = 128;

template <int D>
__global__ void __launch_bounds__(MERGE_THREADS) split_merge_kernel(const DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the partition pass
  constexpr int V4 = D / 4;                           // float4 columns of one output row
  constexpr int NG = MERGE_THREADS / V4;              // partition groups
  extern __shared__ float s_w[];                      // [num_parts] normalised weights
  __shared__ float4 s_sum[NG][V4];
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  int L = p.context_lens[b];
  if (L > p.max_context_len) L = p.max_context_len;  // flagged by the partition pass
  // partial slots: a shared prefix's partitions (if any), then the rest of the context's
  bool bad = false;
  const int pre = L <= 0 ? 0 : prefix_tokens_of(p.seq_prefix_tokens, b, L, p.block_size, &bad);
  const int np = (pre + p.part_tokens - 1) / p.part_tokens;
  const int ns = L <= 0 ? 0 : (L - pre + p.part_tokens - 1) / p.part_tokens;
  const int P = np + ns;
  if (ns == 1) return;  // one partition after any prefix: finished by the partition pass
  __half* out = p.out + ((size_t)b * p.num_heads + h) * D;
  if (P == 0) {
    if (threadIdx.x < V4) *reinterpret_cast<uint2*>(out + threadIdx.x * 4) = make_uint2(0u, 0u);
    return;
  }
  const size_t base = ((size_t)b * p.num_heads + h) * p.num_parts;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const float* ml = p.ws_ml + base * 2;
    float M = -INFINITY;
    for (int i = lane; i < P; i += 32) M = fmaxf(M, ml[2 * i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int i = lane; i < P; i += 32) {
      const float w = rescale_factor(ml[2 * i], M);
      s_w[i] = w;
      den = fmaf(w, ml[2 * i + 1], den);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = 1.f / den;
    __syncwarp();
    for (int i = lane; i < P; i += 32) s_w[i] *= inv;
  }
  __syncthreads();
  const int col = threadIdx.x % V4;
  const int grp = threadIdx.x / V4;
  const float4* src = reinterpret_cast<const float4*>(p.ws_o + base * D) + col;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int i = grp;
  for (; i + 3 * NG < P; i += 4 * NG) {
    float4 x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) x[j] = src[(size_t)(i + j * NG) * V4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float w = s_w[i + j * NG];
      acc.x = fmaf(w, x[j].x, acc.x);
      acc.y = fmaf(w, x[j].y, acc.y);
      acc.z = fmaf(w, x[j].z, acc.z);
      acc.w = fmaf(w, x[j].w, acc.w);
    }
  }
  for (; i < P; i += NG) {
    const float4 x = src[(size_t)i * V4];
    const float w = s_w[i];
    acc.x = fmaf(w, x.x, acc.x);
    acc.y = fmaf(w, x.y, acc.y);
    acc.z = fmaf(w, x.z, acc.z);
    acc.w = fmaf(w, x.w, acc.w);
  }
  s_sum[grp][col] = acc;
  __syncthreads();
  if (grp == 0) {
#pragma unroll
    for (int g2 = 1; g2 < NG; ++g2) {
      const float4 y = s_sum[g2][col];
      acc.x += y.x;
      acc.y += y.y;
      acc.z += y.z;
      acc.w += y.w;
    }
    uint2 packed;
    packed.x = pack_half2(acc.x, acc.y);
    packed.y = pack_half2(acc.z, acc.w);
    *reinterpret_cast<uint2*>(out + col * 4) = packed;
  }
}

}  // namespace

size_t split_merge_smem_bytes(int num_parts) { return (size_t)num_parts * sizeof(float); }

cudaError_t launch_split_reduce(const DecodeParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_heads, p.num_seqs, 1);
  cfg.blockDim = dim3(MERGE_THREADS, 1, 1);
  cfg.dynamicSmemBytes = split_merge_smem_bytes(p.num_parts);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.head_dim == 64) {
    if (cfg.dynamicSmemBytes > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(split_merge_kernel<64>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)cfg.dynamicSmemBytes);
      if (e != cudaSuccess) return e;
    }
    return cudaLaunchKernelEx(&cfg, split_merge_kernel<64>, p);
  }
  if (p.head_dim == 128) {
    if (cfg.dynamicSmemBytes > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(split_merge_kernel<128>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)cfg.dynamicSmemBytes);
      if (e != cudaSuccess) return e;
    }
    return cudaLaunchKernelEx(&cfg, split_merge_kernel<128>, p);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pkv
