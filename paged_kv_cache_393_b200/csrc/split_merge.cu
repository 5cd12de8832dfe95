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
// One warp per (sequence, head), four per CTA.  The warp splits into four
// groups of eight lanes; group g folds partitions g, g+4, g+8, ... online
// (running maximum, rescaled sum and columns), each lane D/32 float4 columns of
// them, and a partition's (max, sum) and columns are loaded together, so a long
// context (tens of partitions) is a short chain of independent loads with many
// in flight.  Shuffles bring the four groups to the overall maximum and add
// them up.
// No shared memory and no CTA barrier, and the grid fits the GPU in about one
// wave.  The kernel is launched as a programmatic dependent of the partition
// pass: its CTAs can be resident before that pass ends and wait
// (griddepcontrol.wait) for its results.
#include "common.cuh"
#include "kernels.h"

namespace pkv {
namespace {

constexpr int MERGE_WARPS = 4;
constexpr int MERGE_GROUPS = 4;  // lane groups per warp, each over every 4th partition

template <int D>
__global__ void __launch_bounds__(MERGE_WARPS * 32) split_merge_kernel(const DecodeParams p) {
  constexpr int V4 = D / 4;                           // float4 columns of one output row
  constexpr int GL = 32 / MERGE_GROUPS;               // lanes per group
  constexpr int CPL = V4 / GL;                        // float4 columns per lane
  static_assert(V4 % GL == 0, "columns must split evenly over a group");
  const int lane = threadIdx.x & 31;
  const int grp = lane / GL;
  const int sub = lane % GL;
  const long long row = (long long)blockIdx.x * MERGE_WARPS + (threadIdx.x >> 5);  // b * H + h
  if (row >= (long long)p.num_seqs * p.num_heads) return;
  const int b = (int)(row / p.num_heads);
  // the lengths and prefix lengths are inputs no earlier kernel of the step writes: read
  // them while the partition pass may still run, then wait for its partials
  int L = p.context_lens[b];
  if (L > p.max_context_len) L = p.max_context_len;  // flagged by the partition pass
  // partial slots: a shared prefix's partitions (if any), then the rest of the context's
  bool bad = false;
  const int pre = L <= 0 ? 0 : prefix_tokens_of(p.seq_prefix_tokens, b, L, p.block_size, &bad);
  asm volatile("griddepcontrol.wait;" ::: "memory");  // partials of the partition pass
  const int np = (pre + p.prefix_part_tokens - 1) / p.prefix_part_tokens;
  const int ns = L <= 0 ? 0 : (L - pre + p.part_tokens - 1) / p.part_tokens;
  const int P = np + ns;
  // one partition after any prefix: finished by the partition pass (prefix partials folded)
  if (ns == 1 && (np == 0 || p.fold_prefix)) return;
  __half* out = p.out + row * D;
  if (P == 0) {
    if (lane < V4) *reinterpret_cast<uint2*>(out + lane * 4) = make_uint2(0u, 0u);
    return;
  }
  const float* ml = p.ws_ml + row * p.num_parts * 2;
  const float4* src = reinterpret_cast<const float4*>(p.ws_o + row * p.num_parts * D);
  // Group g folds partitions g, g + 4, g + 8, ... online: each partition's (max, sum)
  // and output columns are loaded together, so a context's partials are one round of
  // independent loads.  Then the four groups are combined by shuffles.
  float M = -INFINITY;  // this group's running maximum
  float den = 0.f;      // this group's sum, scaled to 2^-M
  float4 acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int k = grp; k < P; k += MERGE_GROUPS) {
    const float mk = ml[2 * k], lk = ml[2 * k + 1];
    float4 x[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) x[c] = src[(size_t)k * V4 + c * GL + sub];
    const float Mn = fmaxf(M, mk);
    const float a = rescale_factor(M, Mn), w = rescale_factor(mk, Mn);
    den = fmaf(w, lk, den * a);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      acc[c].x = fmaf(w, x[c].x, acc[c].x * a);
      acc[c].y = fmaf(w, x[c].y, acc[c].y * a);
      acc[c].z = fmaf(w, x[c].z, acc[c].z * a);
      acc[c].w = fmaf(w, x[c].w, acc[c].w * a);
    }
    M = Mn;
  }
  // the groups' maxima, sums and columns brought to the overall maximum and added up
  // (lanes sub, sub + 8, sub + 16, sub + 24 hold the same columns)
  float Mall = M;
#pragma unroll
  for (int o = GL; o < 32; o <<= 1) Mall = fmaxf(Mall, __shfl_xor_sync(0xffffffffu, Mall, o));
  const float a = rescale_factor(M, Mall);
  den *= a;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    acc[c].x *= a;
    acc[c].y *= a;
    acc[c].z *= a;
    acc[c].w *= a;
  }
#pragma unroll
  for (int o = GL; o < 32; o <<= 1) {
    den += __shfl_xor_sync(0xffffffffu, den, o);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      acc[c].x += __shfl_xor_sync(0xffffffffu, acc[c].x, o);
      acc[c].y += __shfl_xor_sync(0xffffffffu, acc[c].y, o);
      acc[c].z += __shfl_xor_sync(0xffffffffu, acc[c].z, o);
      acc[c].w += __shfl_xor_sync(0xffffffffu, acc[c].w, o);
    }
  }
  if (grp == 0) {
    const float inv = 1.f / den;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int col = c * GL + sub;
      *reinterpret_cast<uint2*>(out + col * 4) =
          make_uint2(pack_half2(acc[c].x * inv, acc[c].y * inv),
                     pack_half2(acc[c].z * inv, acc[c].w * inv));
    }
  }
}

}  // namespace

size_t split_merge_smem_bytes(int num_parts) {
  (void)num_parts;  // the merge keeps everything in registers
  return 0;
}

cudaError_t launch_split_reduce(const DecodeParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.num_seqs * p.num_heads;
  const dim3 grid((unsigned)((rows + MERGE_WARPS - 1) / MERGE_WARPS));
  // A programmatic dependent of the partition pass, except after a shared-prefix
  // pass: then the merge also reads the prefix pass's partials, and a suffix
  // CTA that exits early never waits for that pass, so the merge is ordered
  // behind both the ordinary way (its griddepcontrol.wait then returns at once).
  const bool pdl = p.after_prefix == 0;
  if (p.head_dim == 64)
    return launch_kernel(pdl, split_merge_kernel<64>, grid, dim3(MERGE_WARPS * 32), 0, stream, p);
  if (p.head_dim == 128)
    return launch_kernel(pdl, split_merge_kernel<128>, grid, dim3(MERGE_WARPS * 32), 0, stream,
                         p);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
