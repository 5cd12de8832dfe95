// Paged decode attention on the CUDA cores (sm_100a).
//
// What it computes (per sequence b and query head h, kv head h / G):
//   out[b][h] = softmax_i(scale * q[b][h] . K_b[i]) . V_b,   i < L_b,
// with K_b[i], V_b[i] read from physical block block_tables[b][i / bs], row
// i % bs -- the block-table gather of PagedAttention (lpnh.cn/news/1824136 §2.2
// item 3, §3.2 step 4; 5688vip ch. 4 "PagedAttention：显存管理、分页机制、块大小选择",
// section "分页机制：块表与物理块的组织方式").
//
// Design (one query token per head is ~1 flop per byte, so this is HBM-bound):
//  * CTA = (sequence, group of HPC query heads, context partition).  The group
//    reads KVC consecutive kv heads, which are adjacent inside every block.
//  * A producer warp turns block-table entries into 1-D TMA bulk copies
//    (cp.async.bulk, evict-first in L2) into a ring of shared-memory stages of
//    16 tokens each, whatever the block size: a stage is one block's KVC heads
//    (bs 16, one contiguous copy), 16 rows of each head of one block (bs 32/64),
//    or the KVC heads of 16/bs consecutive blocks (bs 4/8).  Each stage
//    completes on an mbarrier with its byte count.  Table entries are read 32 at
//    a time by the producer's lanes and staged in shared memory.
//  * HPC consumer warps, one per query head, read the staged tile with 16-byte
//    shared loads: D/8 lanes cover one K/V row, so a warp covers 32/(D/8) rows
//    per instruction.  Scores are reduced over the D/8 lanes of a row, the
//    online softmax runs in log2 units (scale*log2(e) folded into q) with fp32
//    accumulation, and rows beyond the context are never multiplied (their
//    slots may hold anything, NaN included).  Every consumer warp reads every
//    stage in order, so no warp can run a phase ahead of a stage's barrier.
//  * With a split, each CTA covers one partition and stores (max, sum,
//    unnormalised output) for split_merge_kernel; a context that fits in one
//    partition is finished here and written directly.
#include "common.cuh"
#include "kernels.h"

#include <atomic>

namespace pkv {
namespace {

__device__ __forceinline__ float dot8(const float (&q)[8], uint4 raw) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = unpack_half2(w[i]);
    acc = fmaf(q[2 * i], f.x, acc);
    acc = fmaf(q[2 * i + 1], f.y, acc);
  }
  return acc;
}

__device__ __forceinline__ void axpy8(float (&acc)[8], float a, uint4 raw) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = unpack_half2(w[i]);
    acc[2 * i] = fmaf(a, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(a, f.y, acc[2 * i + 1]);
  }
}

template <int D, int BS, int HPC, int KVC, bool SPLIT>
__global__ void __launch_bounds__((HPC + 1) * 32)
    simt_decode_kernel(const DecodeParams p) {
  constexpr int CHUNK = 16;                    // tokens per ring stage
  constexpr int CB = BS < CHUNK ? BS : CHUNK;  // rows per sub-tile: a whole block, or 16 rows of one
  constexpr int NB = CHUNK / CB;               // sub-tiles (blocks) per stage
  constexpr int LPR = D / 8;                   // lanes per K/V row (8 fp16 each)
  constexpr int RPW = 32 / LPR;                // rows per warp-wide 16-byte load
  constexpr int ITERS = CHUNK / RPW;           // row groups per stage
  constexpr int TILE = KVC * CHUNK * D;        // fp16 values of one K (or V) stage tile
  constexpr uint32_t TILE_BYTES = TILE * 2;
  constexpr uint32_t SUB_BYTES = KVC * CB * D * 2;  // one sub-tile: KVC heads x CB rows
  static_assert(CHUNK % RPW == 0 && CHUNK % CB == 0, "a stage must hold whole row groups");
  static_assert(32 % NB == 0, "stages must not straddle a window of 32 table entries");
  // A stage tile is laid out [NB sub-tiles][KVC heads][CB rows][D]: for bs <= 16
  // a sub-tile is one block's KVC adjacent heads (one contiguous copy), for
  // bs > 16 it is 16 rows of each of the KVC heads of one block.

  extern __shared__ __align__(128) unsigned char smem[];
  const int stages = p.stages;
  __half* tiles = reinterpret_cast<__half*>(smem);
  int* s_ids = reinterpret_cast<int*>(smem + (size_t)stages * 2 * TILE_BYTES);  // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_ids + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * stages);
  // bars[s]: stage s filled (1 arrival + tx bytes); bars[stages + s]: stage s drained (HPC arrivals)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int part = blockIdx.z;
  const int h0 = blockIdx.x * HPC;
  const int G = p.num_heads / p.num_kv_heads;
  const int kv0 = h0 / G;
  const bool reporter = threadIdx.x == 0 && blockIdx.x == 0 && part == 0;

  // the length and the shared-prefix entry are loaded together (one round trip)
  int L = p.context_lens[b];
  const int P_entry = p.seq_prefix_tokens ? p.seq_prefix_tokens[b] : 0;
  if (L > p.max_context_len) {
    if (reporter) flag_error(p.err, ERR_CONTEXT_LEN);
    L = p.max_context_len;
  }
  if (L <= 0) {
    if (reporter) flag_error(p.err, ERR_CONTEXT_LEN);
    if ((!SPLIT || p.seq_prefix_tokens) && warp < HPC && lane < LPR) {
      *reinterpret_cast<uint4*>(p.out + ((size_t)b * p.num_heads + h0 + warp) * D + lane * 8) =
          make_uint4(0, 0, 0, 0);
    }
    return;  // a plain split launch leaves the zeros to the merge kernel
  }
  // With a shared prefix, its group's pass covers tokens [0, P) and this kernel
  // the suffix [P, L): its partitions start at P, and their partial results go
  // after the prefix partitions' slots.
  bool bad_prefix = false;
  const int P = prefix_tokens_checked(P_entry, L, BS, &bad_prefix);
  if (bad_prefix && reporter) flag_error(p.err, ERR_PREFIX);
  const int tok0 = P + part * p.part_tokens;        // first token of this partition
  if (SPLIT && part == gridDim.z - 1 && tok0 + p.part_tokens < L && threadIdx.x == 0)
    flag_error(p.err, ERR_PREFIX);                  // the grid was sized below this suffix
  const int ntok = min(L, tok0 + p.part_tokens) - tok0;
  if (ntok <= 0) return;                            // partition beyond this context
  const int np = (P + p.prefix_part_tokens - 1) / p.prefix_part_tokens;  // prefix slots
  const int slot_part = np + part;
  // A CTA that covers a shared prefix's whole suffix finishes the output itself:
  // the prefix pass ran to completion before this launch, so its partial
  // results can be folded in here and no merge is needed.
  const bool merge_prefix = SPLIT && P > 0 && L - P <= p.part_tokens && p.fold_prefix;
  const bool direct = !SPLIT || (P == 0 && L <= p.part_tokens) || merge_prefix;
  const int nchunks = (ntok + CHUNK - 1) / CHUNK;
  const int blk0 = tok0 / BS;
  const int nblk = (ntok + BS - 1) / BS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[stages + s]), HPC);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == HPC) {
    // ---------------- producer warp ----------------
    const int32_t* row = p.block_tables + (size_t)b * p.max_blocks + blk0;
    const uint64_t policy = l2_evict_first_policy();
    const uint32_t ring = smem_u32(tiles);
    int issued = 0;
    // Fused append: the partition that ends the context writes the new rows of
    // its kv heads (token L-1) before it issues the stage that reads them.
    const int new_tok =
        (p.k_new && tok0 + ntok == L && p.context_lens[b] == L) ? ntok - 1 : -1;
    NewRows<D, KVC> fresh;
    if (new_tok >= 0) fresh.load(p.k_new, p.v_new, b, p.num_kv_heads, kv0, lane);

    // Issues stage c (lane 0 only); false when the wait for a free slot gave up.
    auto issue = [&](int c, int w0) -> bool {
      const int st = c % stages;
      const int round = c / stages;
      if (round > 0 && !mbar_wait(smem_u32(&bars[stages + st]), (round - 1) & 1)) {
        *abort_flag = 1;
        flag_error(p.err, ERR_TIMEOUT);
        return false;
      }
      const uint32_t full = smem_u32(&bars[st]);
      const uint32_t kdst = ring + (uint32_t)st * 2 * TILE_BYTES;
      const uint32_t vdst = kdst + TILE_BYTES;
      if (BS >= CHUNK) {
        const int tok = c * CHUNK;
        const int phys = s_ids[tok / BS - w0];
        const int r0 = tok % BS;
        // the partition's last stage copies only its rows in the context (the rest of
        // the tile is never read), each kv head's rows one contiguous copy
        const int rows = min(CHUNK, ntok - tok);
        if (BS == CHUNK && rows == CHUNK) {  // the KVC heads of one block: one contiguous tile
          const size_t off = ((size_t)phys * p.num_kv_heads + kv0) * (size_t)(BS * D);
          mbar_arrive_expect_tx(full, 2 * TILE_BYTES);
          bulk_load(kdst, p.k_cache + off, TILE_BYTES, full, policy);
          bulk_load(vdst, p.v_cache + off, TILE_BYTES, full, policy);
        } else {
          const uint32_t bytes = (uint32_t)rows * D * 2;
          mbar_arrive_expect_tx(full, 2u * KVC * bytes);
#pragma unroll
          for (int h = 0; h < KVC; ++h) {
            const size_t off = (((size_t)phys * p.num_kv_heads + kv0 + h) * BS + r0) * (size_t)D;
            bulk_load(kdst + h * CHUNK * D * 2, p.k_cache + off, bytes, full, policy);
            bulk_load(vdst + h * CHUNK * D * 2, p.v_cache + off, bytes, full, policy);
          }
        }
      } else {
        const int first = c * NB;                // first block of the stage
        const int nb = min(NB, nblk - first);
        // only the partition's last block can be partly in the context: its kv heads'
        // rows in the context are one copy each, the rest of the sub-tile is never read
        const int last_rows = ntok - (nblk - 1) * BS;
        const bool part_last = first + nb == nblk && last_rows < BS;
        const uint32_t last_bytes = (uint32_t)last_rows * D * 2;
        mbar_arrive_expect_tx(full, part_last ? 2u * ((nb - 1) * SUB_BYTES + KVC * last_bytes)
                                              : 2u * nb * SUB_BYTES);
        for (int k = 0; k < nb; ++k) {
          const size_t off =
              ((size_t)s_ids[first + k - w0] * p.num_kv_heads + kv0) * (size_t)(BS * D);
          if (part_last && k == nb - 1) {
#pragma unroll
            for (int h = 0; h < KVC; ++h) {
              const uint32_t hs = (uint32_t)h * CB * D * 2;
              bulk_load(kdst + k * SUB_BYTES + hs, p.k_cache + off + (size_t)h * BS * D,
                        last_bytes, full, policy);
              bulk_load(vdst + k * SUB_BYTES + hs, p.v_cache + off + (size_t)h * BS * D,
                        last_bytes, full, policy);
            }
          } else {
            bulk_load(kdst + k * SUB_BYTES, p.k_cache + off, SUB_BYTES, full, policy);
            bulk_load(vdst + k * SUB_BYTES, p.v_cache + off, SUB_BYTES, full, policy);
          }
        }
      }
      issued = c + 1;
      return true;
    };

    // table entries are read 32 at a time by the lanes and staged in shared memory
    for (int w0 = 0; w0 < nblk; w0 += 32) {
      if (w0 + lane < nblk) {
        int id = row[w0 + lane];
        if (id < 0 || id >= p.num_blocks) {
          flag_error(p.err, ERR_BLOCK_ID);
          id = 0;
        }
        s_ids[lane] = id;
      }
      __syncwarp();
      const int c_begin = w0 * BS / CHUNK;
      const int c_end = min(nchunks, (w0 + 32) * BS / CHUNK);
      // With an append, the rows are stored once the first ring fill is issued
      // (those copies are in flight meanwhile) and always before the last stage.
      const bool append_here = new_tok >= 0 && w0 == 0;
      const int c_split = append_here ? min(c_end, min(stages, nchunks - 1)) : c_end;
      if (lane == 0) {
        for (int c = c_begin; c < c_split && !*abort_flag; ++c)
          if (!issue(c, w0)) break;
      }
      if (append_here && !__shfl_sync(0xffffffffu, *abort_flag, 0)) {
        const int id = row[new_tok / BS];  // re-read: a bad id was replaced by 0 for reading only
        if (id >= 0 && id < p.num_blocks)
          fresh.store(const_cast<__half*>(p.k_cache), const_cast<__half*>(p.v_cache),
                      p.num_kv_heads, BS, kv0, id, new_tok % BS, lane);
      }
      if (lane == 0) {
        for (int c = c_split; c < c_end && !*abort_flag; ++c)
          if (!issue(c, w0)) break;
      }
      __syncwarp();  // s_ids is rewritten for the next window
    }
    if (lane == 0 && *abort_flag) {
      // Only the last `stages` fills can still be in flight: let them land
      // before this CTA's shared memory can be handed to another CTA.
      for (int c = max(0, issued - stages); c < issued; ++c)
        mbar_wait(smem_u32(&bars[c % stages]), (c / stages) & 1);
    }
    return;
  }

  // ---------------- consumer warps: one query head each ----------------
  const int h = h0 + warp;
  const int kvi = h / G - kv0;
  const int sub = lane / LPR;       // row inside a row group
  const int col = (lane % LPR) * 8; // first of this lane's 8 dims

  float qf[8];
  {
    const uint4 raw = *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.num_heads + h) * D + col);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = unpack_half2(w[i]);
      qf[2 * i] = f.x * p.scale_log2;
      qf[2 * i + 1] = f.y * p.scale_log2;
    }
  }

  float m = -INFINITY;  // running max of the scores (log2 units)
  float l = 0.f;        // running sum of 2^(s - m) over this lane's rows
  float acc[8];
#pragma unroll
  for (int d = 0; d < 8; ++d) acc[d] = 0.f;

  for (int c = 0; c < nchunks; ++c) {
    const int st = c % stages;
    if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
    const bool ready = mbar_wait(smem_u32(&bars[st]), (c / stages) & 1);
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, ERR_TIMEOUT);
      }
      break;
    }
    const __half* kt = tiles + (size_t)st * 2 * TILE;
    const __half* vt = kt + TILE;
    const int nvalid = min(CHUNK, ntok - c * CHUNK);

    float s[ITERS];
#pragma unroll
    for (int j = 0; j < ITERS; ++j) {
      const int t = j * RPW + sub;
      const int r = (((t / CB) * KVC + kvi) * CB + t % CB) * D + col;
      float d = dot8(qf, *reinterpret_cast<const uint4*>(kt + r));
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      s[j] = t < nvalid ? d : -INFINITY;
    }
    float mb = s[0];
#pragma unroll
    for (int j = 1; j < ITERS; ++j) mb = fmaxf(mb, s[j]);
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float m_new = fmaxf(m, mb);  // finite: the stage's first row is in the context
    const float alpha = rescale_factor(m, m_new);
    l *= alpha;
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[d] *= alpha;
#pragma unroll
    for (int j = 0; j < ITERS; ++j) {
      const int t = j * RPW + sub;
      if (t < nvalid) {
        const float pj = exp2f(s[j] - m_new);
        l += pj;
        const int r = (((t / CB) * KVC + kvi) * CB + t % CB) * D + col;
        axpy8(acc, pj, *reinterpret_cast<const uint4*>(vt + r));
      }
    }
    m = m_new;
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[stages + st]));
  }

  // Lanes with the same columns hold sums over different rows: add them up.
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
    l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
    for (int d = 0; d < 8; ++d) acc[d] += __shfl_xor_sync(0xffffffffu, acc[d], o);
  }
  // the merge kernel (if any) may be scheduled once every CTA got here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the shared-prefix pass this launch may overlap must be done before its
  // partials are read below (and before this grid counts as complete)
  if (p.after_prefix) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (sub == 0) {
    const size_t bh = (size_t)b * p.num_heads + h;
    if (direct) {
      if (merge_prefix) {
        // the prefix partials folded in online, one partition at a time: each
        // partition's loads are independent of the others', so they are in flight
        // together instead of a round of maxima before a round of outputs
        const float* ml = p.ws_ml + bh * p.num_parts * 2;
#pragma unroll 4
        for (int i = 0; i < np; ++i) {
          const float mi = ml[2 * i], li = ml[2 * i + 1];
          const float4* o =
              reinterpret_cast<const float4*>(p.ws_o + (bh * p.num_parts + i) * D + col);
          const float4 o0 = o[0], o1 = o[1];
          const float M = fmaxf(m, mi);
          const float a = rescale_factor(m, M), w = rescale_factor(mi, M);
          l = fmaf(w, li, l * a);
          acc[0] = fmaf(w, o0.x, acc[0] * a);
          acc[1] = fmaf(w, o0.y, acc[1] * a);
          acc[2] = fmaf(w, o0.z, acc[2] * a);
          acc[3] = fmaf(w, o0.w, acc[3] * a);
          acc[4] = fmaf(w, o1.x, acc[4] * a);
          acc[5] = fmaf(w, o1.y, acc[5] * a);
          acc[6] = fmaf(w, o1.z, acc[6] * a);
          acc[7] = fmaf(w, o1.w, acc[7] * a);
          m = M;
        }
      }
      uint4 packed;
      packed.x = pack_half2(acc[0] / l, acc[1] / l);
      packed.y = pack_half2(acc[2] / l, acc[3] / l);
      packed.z = pack_half2(acc[4] / l, acc[5] / l);
      packed.w = pack_half2(acc[6] / l, acc[7] / l);
      *reinterpret_cast<uint4*>(p.out + bh * D + col) = packed;
    } else {
      if (p.no_merge && lane == 0) flag_error(p.err, ERR_PREFIX);  // suffix bound too small
      const size_t slot = bh * p.num_parts + slot_part;
      float4* dst = reinterpret_cast<float4*>(p.ws_o + slot * D + col);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      if (lane == 0) {
        p.ws_ml[slot * 2] = m;
        p.ws_ml[slot * 2 + 1] = l;
      }
    }
  }
}

constexpr int MAX_DEVICES = 64;

// Raises a kernel's dynamic shared-memory limit once per device as needed.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, std::atomic<int>* granted) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  if (granted[dev].load(std::memory_order_relaxed) >= (int)bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) granted[dev].store((int)bytes, std::memory_order_relaxed);
  return e;
}

template <int D, int BS, int HPC, int KVC, bool SPLIT>
cudaError_t launch_simt_instance(const DecodeParams& p, cudaStream_t stream) {
  static std::atomic<int> granted[MAX_DEVICES];
  auto kernel = simt_decode_kernel<D, BS, HPC, KVC, SPLIT>;
  const size_t smem = simt_smem_bytes(D, BS, KVC, p.stages);
  cudaError_t e = allow_smem(kernel, smem, granted);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.num_heads / HPC, p.num_seqs, SPLIT ? p.grid_parts : 1);
  return launch_kernel(p.after_prefix != 0, kernel, grid, dim3((HPC + 1) * 32), smem, stream, p);
}

}  // namespace

size_t simt_stage_bytes(int head_dim, int block_size, int kvc) {
  (void)block_size;  // a stage is 16 tokens whatever the block size
  return 2ull * kvc * 16 * head_dim * sizeof(__half);
}

size_t simt_smem_bytes(int head_dim, int block_size, int kvc, int stages) {
  return (size_t)stages * simt_stage_bytes(head_dim, block_size, kvc) + 32 * sizeof(int) +
         2ull * stages * sizeof(uint64_t) + 16;
}

#define PKV_SIMT_CASE(D_, BS_, H_, K_)                                         \
  if (p.head_dim == D_ && p.block_size == BS_ && hpc == H_ && kvc == K_)       \
    return split ? launch_simt_instance<D_, BS_, H_, K_, true>(p, stream)      \
                 : launch_simt_instance<D_, BS_, H_, K_, false>(p, stream);
#define PKV_SIMT_BS(D_, H_, K_) \
  PKV_SIMT_CASE(D_, 4, H_, K_)  \
  PKV_SIMT_CASE(D_, 8, H_, K_)  \
  PKV_SIMT_CASE(D_, 16, H_, K_) \
  PKV_SIMT_CASE(D_, 32, H_, K_) \
  PKV_SIMT_CASE(D_, 64, H_, K_)
#define PKV_SIMT_GROUPS(D_) \
  PKV_SIMT_BS(D_, 1, 1)     \
  PKV_SIMT_BS(D_, 2, 2)     \
  PKV_SIMT_BS(D_, 4, 4)     \
  PKV_SIMT_BS(D_, 2, 1)     \
  PKV_SIMT_BS(D_, 4, 1)     \
  PKV_SIMT_BS(D_, 8, 1)

cudaError_t launch_simt_decode(const DecodeParams& p, int hpc, int kvc, bool split,
                               cudaStream_t stream) {
  PKV_SIMT_GROUPS(64)
  PKV_SIMT_GROUPS(128)
  return cudaErrorInvalidValue;
}

}  // namespace pkv
