// Paged decode attention for grouped-query heads on the tensor cores (sm_100a).
//
// Same result as the CUDA-core kernel (out[b][h] = softmax(scale q.K_b) V_b,
// gathered through the block table), for query groups of G = 2..8 heads that
// share one kv head.  Each K/V tile is then used by G queries, so QK^T and PV
// are small dense contractions worth the tensor cores (G flops per byte):
//
//   S^T[16 tokens][8 heads]  = K[16][D]  . Q^T[D][8]     (mma m16n8k16, D/16 steps)
//   O^T[D][8 heads]         += V^T[D][16] . P^T[16][8]    (D/16 mma, one k step)
//
// Rows are tokens, so the 16-token tile needs no padding; heads beyond G are
// zero queries.  The fp32 score fragment of S^T (thread: tokens g, g+8 x heads
// 2t, 2t+1) becomes the B operand of PV with two movmatrix transposes after the
// probabilities are rounded to fp16; the running sum l accumulates the same
// rounded values, so the weights used and the normaliser agree.
//
// Data movement: a producer warp issues tiled TMA tensor copies
// (cp.async.bulk.tensor.2d, 128-byte swizzle, evict-first) of [rows][64 cols]
// boxes of the pools viewed as a [N*Hk*bs][D] matrix into a ring of stages of
// 16 tokens: 16 rows of one block (bs >= 16) or two whole blocks (bs 8).
// ldmatrix reads the swizzled tiles without bank conflicts (K plain for the A
// operand of QK^T, V transposed for the A operand of PV).  Each stage has ONE
// owner warp, (stage index) mod 4, which consumes every fill of that stage in
// order; a warp therefore never waits on a barrier phase that a slower warp
// has not reached yet (parity waits cannot tell phase k from phase k+2).
// Four consumer warps, each with its own online softmax, merge through shared
// memory at the end, reusing the drained ring.  Rows past the context are
// masked out of the scores, and the matching V rows are zeroed in shared
// memory before PV (0 * NaN would poison the sum).
#include "common.cuh"
#include "kernels.h"

#include <atomic>

namespace pkv {
namespace {

constexpr int NW = MMA_CONSUMER_WARPS;

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier over `threads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// Shared-memory address of the 16-byte unit holding column `colh` (fp16 index)
// of token row `tok` in a stage tile laid out as [D/64 slices][CHUNK rows][128 B]
// with the 128-byte swizzle (unit index XOR row mod 8).
template <int CHUNK>
__device__ __forceinline__ uint32_t swz_addr(uint32_t tile, int tok, int colh) {
  const int sl = colh >> 6;
  const int unit = (colh & 63) >> 3;
  return tile + sl * (CHUNK * 128) + tok * 128 + ((unit ^ (tok & 7)) << 4);
}

template <int D, int BS, bool SPLIT>
__global__ void __launch_bounds__((NW + 1) * 32)
    mma_decode_kernel(const __grid_constant__ CUtensorMap k_map,
                      const __grid_constant__ CUtensorMap v_map, const DecodeParams p) {
  constexpr int CHUNK = 16;                    // tokens per stage
  constexpr int CB = BS < CHUNK ? BS : CHUNK;  // rows per TMA box
  constexpr int NB = CHUNK / CB;               // boxes (blocks) per stage and slice
  constexpr int NSL = D / 64;                  // 64-column slices (128 bytes)
  constexpr uint32_t SLICE_BYTES = CHUNK * 128;
  constexpr uint32_t TILE_BYTES = NSL * SLICE_BYTES;  // K (or V) of one stage
  constexpr uint32_t BOX_BYTES = CB * 128;
  constexpr int MT = D / 16;                   // 16-wide slices of D
  constexpr int OSTRIDE = D + 4;               // padded merge rows (fewer bank conflicts)
  static_assert(32 % NB == 0, "stages must not straddle a window of 32 table entries");

  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  const uint32_t ring = smem_u32(smem);  // [stages][K tile | V tile], 1024-aligned
  int* s_ids = reinterpret_cast<int*>(smem + (size_t)stages * 2 * TILE_BYTES);  // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_ids + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * stages);
  // merge buffers, placed over the ring once every stage has been consumed
  float* s_m = reinterpret_cast<float*>(smem);  // [NW][8]
  float* s_l = s_m + NW * 8;                    // [NW][8]
  float* s_o = s_l + NW * 8;                    // [NW][8][OSTRIDE]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  const int part = blockIdx.z;
  const int G = p.num_heads / p.num_kv_heads;
  const bool reporter = threadIdx.x == 0 && kvh == 0 && part == 0;

  int L = p.context_lens[b];
  if (L > p.max_context_len) {
    if (reporter) flag_error(p.err, ERR_CONTEXT_LEN);
    L = p.max_context_len;
  }
  if (L <= 0) {
    if (reporter) flag_error(p.err, ERR_CONTEXT_LEN);
    if (!SPLIT) {
      for (int i = threadIdx.x; i < G * D; i += blockDim.x)
        p.out[((size_t)b * p.num_heads + kvh * G) * D + i] = __float2half_rn(0.f);
    }
    return;
  }
  const int tok0 = part * p.part_tokens;
  const int ntok = min(L, tok0 + p.part_tokens) - tok0;
  if (ntok <= 0) return;
  const int nchunks = (ntok + CHUNK - 1) / CHUNK;
  const int blk0 = tok0 / BS;
  const int nblk = (ntok + BS - 1) / BS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[stages + s]), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      prefetch_tensor_map(&k_map);
      prefetch_tensor_map(&v_map);
    }
    const int32_t* row = p.block_tables + (size_t)b * p.max_blocks + blk0;
    const uint64_t policy = l2_evict_first_policy();
    int issued = 0;
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
      if (lane == 0) {
        const int c_end = min(nchunks, (w0 + 32) * BS / CHUNK);
        for (int c = w0 * BS / CHUNK; c < c_end && !*abort_flag; ++c) {
          const int st = c % stages;
          const int round = c / stages;
          if (round > 0 && !mbar_wait(smem_u32(&bars[stages + st]), (round - 1) & 1)) {
            *abort_flag = 1;
            flag_error(p.err, ERR_TIMEOUT);
            break;
          }
          const uint32_t full = smem_u32(&bars[st]);
          const uint32_t kdst = ring + (uint32_t)st * 2 * TILE_BYTES;
          const uint32_t vdst = kdst + TILE_BYTES;
          const int first = c * NB;  // first block of the stage (bs 8), or unused
          const int nb = BS >= CHUNK ? 1 : min(NB, nblk - first);
          mbar_arrive_expect_tx(full, 2u * nb * NSL * BOX_BYTES);
          for (int k = 0; k < nb; ++k) {
            int y;
            if (BS >= CHUNK) {
              const int tok = c * CHUNK;
              y = (s_ids[tok / BS - w0] * p.num_kv_heads + kvh) * BS + tok % BS;
            } else {
              y = (s_ids[first + k - w0] * p.num_kv_heads + kvh) * BS;
            }
#pragma unroll
            for (int sl = 0; sl < NSL; ++sl) {
              const uint32_t off = sl * SLICE_BYTES + k * BOX_BYTES;
              tensor_load_2d(kdst + off, &k_map, sl * 64, y, full, policy);
              tensor_load_2d(vdst + off, &v_map, sl * 64, y, full, policy);
            }
          }
          issued = c + 1;
        }
      }
      __syncwarp();
    }
    if (lane == 0 && *abort_flag) {
      for (int c = max(0, issued - stages); c < issued; ++c)
        mbar_wait(smem_u32(&bars[c % stages]), (c / stages) & 1);
    }
    return;
  }

  // ---------------- consumer warps ----------------
  const int g = lane >> 2;  // fragment row group
  const int t = lane & 3;   // fragment column pair
  // B operand of S^T = K . Q^T: Q[head g][16 dims of step ks], zero for g >= G.
  uint32_t qb[MT][2];
  {
    const __half* qrow = p.q + ((size_t)b * p.num_heads + kvh * G + g) * D;
#pragma unroll
    for (int ks = 0; ks < MT; ++ks) {
      qb[ks][0] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
      qb[ks][1] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t + 8) : 0u;
    }
  }
  float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2t, 2t+1 (log2 units)
  float l0 = 0.f, l1 = 0.f;              // this lane's part of the running sums
  float o[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

  const int mat = lane >> 3;  // ldmatrix: which 8x8 matrix this lane addresses
  const int r8 = lane & 7;    // ... and which of its rows
  bool gave_up = false;       // this warp stopped before consuming all its stages

  for (int c = 0; c < nchunks; ++c) {
    const int st = c % stages;
    if (st % NW != warp) continue;  // this stage belongs to another warp
    if (__shfl_sync(0xffffffffu, *abort_flag, 0)) {
      gave_up = true;
      break;
    }
    const bool ready = mbar_wait(smem_u32(&bars[st]), (c / stages) & 1);
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, ERR_TIMEOUT);
      }
      gave_up = true;
      break;
    }
    const uint32_t kt = ring + (uint32_t)st * 2 * TILE_BYTES;
    const uint32_t vt = kt + TILE_BYTES;
    const int valid = min(CHUNK, ntok - c * CHUNK);  // rows of this stage inside the context

    // ---- S^T = K . Q^T for 16 tokens ----
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < MT; ++ks) {
      const int tok = r8 + ((mat & 1) << 3);
      const int colh = ks * 16 + ((mat >> 1) << 3);
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(swz_addr<CHUNK>(kt, tok, colh), a0, a1, a2, a3);
      mma_16816(sc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
    }
    const float s0 = g < valid ? sc[0] * p.scale_log2 : -INFINITY;
    const float s1 = g < valid ? sc[1] * p.scale_log2 : -INFINITY;
    const float s2 = g + 8 < valid ? sc[2] * p.scale_log2 : -INFINITY;
    const float s3 = g + 8 < valid ? sc[3] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: row 0 is valid
    const float al0 = rescale_factor(m0, mn0), al1 = rescale_factor(m1, mn1);
    m0 = mn0;
    m1 = mn1;
    const uint32_t p01 = pack_half2(exp2f(s0 - mn0), exp2f(s1 - mn1));  // token g
    const uint32_t p23 = pack_half2(exp2f(s2 - mn0), exp2f(s3 - mn1));  // token g + 8
    const float2 f01 = unpack_half2(p01), f23 = unpack_half2(p23);
    l0 = fmaf(l0, al0, f01.x + f23.x);
    l1 = fmaf(l1, al1, f01.y + f23.y);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      o[mt][0] *= al0;
      o[mt][1] *= al1;
      o[mt][2] *= al0;
      o[mt][3] *= al1;
    }
    // P^T fragments: {P[token 2t][head g], P[token 2t+1][head g]} (+8 for pb1)
    const uint32_t pb0 = movmatrix_trans(p01);
    const uint32_t pb1 = movmatrix_trans(p23);
    const bool partial = valid < CHUNK;
    if (partial) {
      // Zero the V rows past the context (whole 128-byte rows, so the swizzle
      // does not matter).
      const int rows = CHUNK - valid;
      for (int idx = lane; idx < rows * NSL * 8; idx += 32) {
        const int r = valid + idx / (NSL * 8);
        const int rem = idx % (NSL * 8);
        const uint32_t addr = vt + (rem >> 3) * SLICE_BYTES + r * 128 + ((rem & 7) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
      }
      __syncwarp();
    }
    // ---- O^T += V^T . P^T ----
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int tok = r8 + ((mat >> 1) << 3);
      const int colh = mt * 16 + ((mat & 1) << 3);
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4_trans(swz_addr<CHUNK>(vt, tok, colh), a0, a1, a2, a3);
      mma_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
    }
    if (partial) fence_proxy_async_smem();  // generic writes before the next TMA fill
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[stages + st]));
  }

  // ---- merge the four warps' partial softmax states ----
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  // When every warp consumed all its stages, every copy has landed and the ring
  // can hold the merge buffers.  Otherwise copies may still be landing: give up
  // (the error word already says the output is invalid).
  if (named_barrier_or(1, NW * 32, gave_up)) return;
  if (g == 0) {
    s_m[warp * 8 + 2 * t] = m0;
    s_m[warp * 8 + 2 * t + 1] = m1;
    s_l[warp * 8 + 2 * t] = l0;
    s_l[warp * 8 + 2 * t + 1] = l1;
  }
  float* so = s_o + warp * 8 * OSTRIDE;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    so[(2 * t) * OSTRIDE + mt * 16 + g] = o[mt][0];
    so[(2 * t + 1) * OSTRIDE + mt * 16 + g] = o[mt][1];
    so[(2 * t) * OSTRIDE + mt * 16 + g + 8] = o[mt][2];
    so[(2 * t + 1) * OSTRIDE + mt * 16 + g + 8] = o[mt][3];
  }
  named_barrier_sync(1, NW * 32);
  for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
    const int head = idx / D;
    const int d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, s_m[w * 8 + head]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float a = rescale_factor(s_m[w * 8 + head], M);
      num = fmaf(a, s_o[(w * 8 + head) * OSTRIDE + d], num);
      den = fmaf(a, s_l[w * 8 + head], den);
    }
    const size_t bh = (size_t)b * p.num_heads + kvh * G + head;
    if (!SPLIT) {
      p.out[bh * D + d] = __float2half_rn(num / den);
    } else {
      const size_t slot = bh * p.num_parts + part;
      p.ws_o[slot * D + d] = num;
      if (d == 0) {
        p.ws_ml[slot * 2] = M;
        p.ws_ml[slot * 2 + 1] = den;
      }
    }
  }
}

constexpr int MAX_DEVICES = 64;

template <int D, int BS, bool SPLIT>
cudaError_t launch_mma_instance(const DecodeParams& p, const CUtensorMap& km,
                                const CUtensorMap& vm, cudaStream_t stream) {
  static std::atomic<int> granted[MAX_DEVICES];
  auto kernel = mma_decode_kernel<D, BS, SPLIT>;
  const size_t smem = mma_smem_bytes(D, BS, p.stages);
  if (smem > 48 * 1024) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    if (granted[dev].load(std::memory_order_relaxed) < (int)smem) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      granted[dev].store((int)smem, std::memory_order_relaxed);
    }
  }
  const dim3 grid(p.num_kv_heads, p.num_seqs, SPLIT ? p.num_parts : 1);
  kernel<<<grid, (NW + 1) * 32, smem, stream>>>(km, vm, p);
  return cudaGetLastError();
}

}  // namespace

size_t mma_stage_bytes(int head_dim, int block_size) {
  (void)block_size;  // a stage is 16 tokens whatever the block size
  return 2ull * 16 * head_dim * sizeof(__half);
}

size_t mma_merge_bytes(int head_dim) {
  return (size_t)NW * 8 * (2 + head_dim + 4) * sizeof(float);
}

size_t mma_smem_bytes(int head_dim, int block_size, int stages) {
  return 1024 /* alignment slack */ + (size_t)stages * mma_stage_bytes(head_dim, block_size) +
         32 * sizeof(int) + 2ull * stages * sizeof(uint64_t) + 16;
}

#define PKV_MMA_CASE(D_, BS_)                                                  \
  if (p.head_dim == D_ && p.block_size == BS_)                                 \
    return split ? launch_mma_instance<D_, BS_, true>(p, km, vm, stream)       \
                 : launch_mma_instance<D_, BS_, false>(p, km, vm, stream);

cudaError_t launch_mma_decode(const DecodeParams& p, const CUtensorMap& km, const CUtensorMap& vm,
                              bool split, cudaStream_t stream) {
  PKV_MMA_CASE(64, 8)
  PKV_MMA_CASE(64, 16)
  PKV_MMA_CASE(64, 32)
  PKV_MMA_CASE(64, 64)
  PKV_MMA_CASE(128, 8)
  PKV_MMA_CASE(128, 16)
  PKV_MMA_CASE(128, 32)
  PKV_MMA_CASE(128, 64)
  return cudaErrorInvalidValue;
}

}  // namespace pkv
